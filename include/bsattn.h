/*
 * bsattn.h — C ABI of the block-sparse attention library for 3D-tiled video
 * latent tokens (sm_100a).
 *
 * The method (sources named per entry point below):
 *   1. reorder the tokens of a T x H x W latent grid into (t, h, w) tiles
 *      ("video-aware block organisation", FVAttn summary page, Summary;
 *      "shared 3D tile granularity", FPSAttention page, Approach);
 *   2. mean-pool Q and K per tile and score tile pairs;
 *   3. keep, per query tile, a set of key tiles: top-k, top-p with a top-k
 *      floor (FVAttn summary page, Summary and Abstract), or a fixed 3D tile
 *      window (FPSAttention page, ablation rows on sparsity windows);
 *   4. run softmax attention over the kept tile pairs only (FPSAttention
 *      page, Approach; trainable sparse attention record, Research Type and
 *      Hardware Specification rows), optionally with Q/K quantised to e4m3
 *      per tile (FPSAttention page, Approach).
 *
 * Conventions for every entry point:
 *   - Device pointers are owned by the caller; the library never allocates
 *     on the hot path. A plan owns only host metadata plus a few small
 *     device buffers made at create time (window lists, error word).
 *   - All device pointers must be 16-byte aligned. Tensors are dense,
 *     row-major, with the layouts stated below.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Calls enqueue work and return; nothing synchronises except
 *     attn_check_device_status.
 *   - Argument errors are reported before anything is enqueued. A failed
 *     launch returns BSATTN_ERR_CUDA. Kernels never trap: an out-of-range
 *     list entry or an exhausted bounded wait sets the plan's device error
 *     word and the affected work is skipped; attn_check_device_status
 *     reports it.
 *   - A plan is bound to the device that was current at attn_plan_create
 *     (calls switch to that device while they run and give the caller its
 *     own current device back before returning) and is immutable
 *     afterwards, so it may be used from several streams at once (calls
 *     that share output buffers must still be ordered by the caller).
 *   - Block scores containing NaN give unspecified (but in-bounds) lists.
 *
 * Layouts (B batch, Hh heads, D head_dim, L = T*H*W, N = number of tiles,
 * V = rows per tile = tile_t*tile_h*tile_w, a multiple of 64, or 64 for a
 * tile of fewer than 64 tokens, whose extra rows are padding):
 *   natural   [B, L, Hh, D] bf16, token n = (t*H + h)*W + w
 *   tiled     [B, Hh, N, V, D] (bf16, or u8 e4m3 codes), tile id
 *             j = ((t/tile_t)*nH + h/tile_h)*nW + w/tile_w, in-tile row
 *             ((t%tile_t)*tile_h + h%tile_h)*tile_w + w%tile_w; padded
 *             slots (t>=T, h>=H or w>=W) are zero
 *   pooled    [B, Hh, N, D] fp32, mean over the tile's real tokens
 *   scores    [B, Hh, N, N] fp32, S[i][j] = softmax_scale * qbar_i . kbar_j
 *   idx       [B, Hh, N, kmax] int32, ascending kept key tiles of each query
 *             tile; entries at and beyond cnt are unspecified
 *   cnt       [B, Hh, N] int32
 *   tile scale [B, Hh, N] fp32 (e4m3 path)
 *   lse       natural [B, Hh, L] fp32 (attn_layer) or tiled [B, Hh, N, V]
 *             fp32 (attn_forward); natural-log sum of exp(scaled scores)
 */
#ifndef BSATTN_H
#define BSATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSATTN_OK = 0,
  BSATTN_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or rule */
  BSATTN_ERR_UNSUPPORTED = 2,  /* valid request outside the supported set   */
  BSATTN_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed      */
  BSATTN_ERR_TIMEOUT = 4,      /* a bounded device wait ran out             */
  BSATTN_ERR_INTERNAL = 5,     /* device error word: bad list entry etc.    */
  BSATTN_ERR_WORKSPACE = 6     /* workspace pointer null or too small       */
} bsattn_status;

typedef enum {
  BSATTN_RULE_TOPK = 0,   /* k largest scores, ties to the lower tile index */
  BSATTN_RULE_TOPP = 1,   /* smallest prefix with softmax mass >= p, >= k   */
  BSATTN_RULE_WINDOW = 2  /* |dt|<=win_t, |dh|<=win_h, |dw|<=win_w in tiles */
} bsattn_rule_kind;

typedef struct {
  int kind;              /* bsattn_rule_kind                                 */
  int k;                 /* top-k: count (1..N); top-p: floor (0..N)          */
  double p;              /* top-p: mass threshold in (0, 1]                   */
  int win_t, win_h, win_w; /* window half-widths in tiles (>= 0)             */
} bsattn_rule;

typedef struct {
  int B, heads, head_dim;       /* head_dim in {64, 128}                      */
  int T, H, W;                  /* latent grid, each >= 1                     */
  int tile_t, tile_h, tile_w;   /* tile shape; see attn_plan_create           */
  float softmax_scale;          /* <= 0 selects 1/sqrt(head_dim)              */
  int qk_fp8;                   /* 1: attn_forward takes per-tile e4m3 Q/K    */
} bsattn_desc;

typedef struct {
  int Tp, Hp, Wp;               /* padded grid                                */
  int nT, nH, nW;               /* tiles per axis                             */
  int n_blocks;                 /* N = nT*nH*nW                               */
  int tile_volume;              /* V = tile_t * tile_h * tile_w               */
  int kmax;                     /* idx row capacity                           */
  float softmax_scale;          /* resolved scale                             */
  size_t select_workspace_bytes;  /* attn_select                              */
  size_t forward_workspace_bytes; /* attn_forward                             */
  size_t layer_workspace_bytes;   /* attn_layer                               */
  size_t backward_workspace_bytes; /* attn_backward                           */
} bsattn_info;

typedef struct bsattn_plan bsattn_plan;

/* Validate a problem and rule and build a plan (host metadata; for the
 * window rule also the closed-form kept lists, copied once to the device;
 * a 4-byte device error word). The current CUDA device is bound to the plan.
 * Errors: INVALID_ARG (null, non-positive sizes, k outside its range,
 * p outside (0,1], negative half-widths), UNSUPPORTED (head_dim not 64/128,
 * unsupported tile shape, N above 2048 for top-k/top-p, more than 2^31
 * padded token rows over all batches and heads), CUDA.
 *
 * Tile shapes (the pages' "3D tile granularity"; FPSAttention's tile ablation
 * compares (3,4,4) with the hardware-friendly (6,8,8), and (3,4,4) with
 * (24,32,32)): either fewer than 64 tokens, e.g. (3,4,4), stored as one
 * 64-row chunk whose last 64 - V rows are padding (info.tile_volume is then
 * 64); or a volume V = 64 * c with 1 <= c <= 512, each side at most 1024, and
 * each run of 64 in-tile rows [64i, 64i + 64) a box of the tile: 64 /
 * (tile_h * tile_w) whole (h, w) frames when tile_h * tile_w divides 64, else
 * 64 / tile_w whole w rows when tile_w divides 64 (and 64 / tile_w divides
 * tile_h), else a 64-long run along w when 64 divides tile_w. (4,4,4),
 * (2,4,8), (6,8,8), (4,8,8), (8,8,8) and (24,32,32) qualify; (3,4,6) (V =
 * 72) does not. The attention works on these 64-row chunks. */
bsattn_status attn_plan_create(const bsattn_desc* desc, const bsattn_rule* rule,
                               bsattn_plan** out);
void attn_plan_destroy(bsattn_plan* plan);
bsattn_status attn_plan_info(const bsattn_plan* plan, bsattn_info* out);
const char* attn_status_string(bsattn_status s);

/* Step 1 (+2): gather natural bf16 tokens into the tiled layout with zero
 * pads; if `pooled` is non-NULL also write the fp32 tile means over real
 * tokens (pooling for the block scores; the pages leave the pooling function
 * open, the mean is this library's reading). */
bsattn_status attn_reorder(const bsattn_plan* plan, const void* x_nat, void* x_tiled,
                           float* pooled, void* stream);

/* Step 2 alone: fp32 tile means of natural bf16 tokens, no tiled copy. */
bsattn_status attn_pool(const bsattn_plan* plan, const void* x_nat, float* pooled,
                        void* stream);

/* Inverse of step 1: scatter tiled bf16 rows of real tokens back to the
 * natural layout (padded slots are dropped). */
bsattn_status attn_unreorder(const bsattn_plan* plan, const void* x_tiled, void* x_nat,
                             void* stream);

/* Step 2: block scores S = softmax_scale * pooled_q . pooled_k^T per
 * (batch, head), fp32 out. The routing frontend of the FVAttn summary page
 * (Summary and Abstract: Top-p routing with a Top-k safety floor over
 * video-aware blocks) ranks key blocks per query block; the pages do not
 * print the block score, and this library's reading is the scaled dot
 * product of the tiles' mean Q and mean K. Computed on the tensor cores as three TF32
 * products per term (each input split as hi + lo, hi exact in TF32; hi*hi +
 * hi*lo + lo*hi accumulated in fp32), within about 2^-20 of
 * sum_d |q_d k_d| of the exact dot product; the result is deterministic. A
 * bounded wait that gives up sets the device error word (TIMEOUT). */
bsattn_status attn_block_scores(const bsattn_plan* plan, const float* pooled_q,
                                const float* pooled_k, float* scores, void* stream);

/* Step 3 on a given score matrix: the plan's rule applied row by row
 * (top-p with a top-k floor: FVAttn summary page, Summary and Abstract;
 * top-k at a fixed density: "Faster Video Diffusion with Trainable Sparse
 * Attention" record, Dataset Splits row, final sparsity 0.9; the window:
 * FPSAttention page, ablation rows on the (6,6,1), (6,6,6) and (3,3,1)
 * sparsity windows).
 * Top-k: the k largest by (score descending, index ascending); -0.0 and
 * +0.0 tie. Top-p: in that order, the shortest prefix whose softmax mass
 * (fp64 exp, sum and scan) reaches p, then at least k and at most N tiles.
 * Window: the plan's closed-form lists (scores unused, may be NULL).
 * Lists come out ascending. */
bsattn_status attn_select_from_scores(const bsattn_plan* plan, const float* scores,
                                      int32_t* idx, int32_t* cnt, void* stream);

/* Steps 2-3 from natural Q and K: pool, score, select (the routing
 * frontend of the FVAttn summary page, Summary: video-aware blocks, Top-p
 * routing, Top-k floor; see attn_block_scores and attn_select_from_scores
 * for the readings). `ws` must hold info.select_workspace_bytes (pooled Q/K
 * and the score matrix); the window rule reads neither q/k nor ws. */
bsattn_status attn_select(const bsattn_plan* plan, const void* q_nat, const void* k_nat,
                          int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes,
                          void* stream);

/* attn_select with the scoring and the top-k selection fused (the same
 * routing frontend, FVAttn summary page, Summary, and the same top-k rule as
 * attn_select_from_scores): the score matrix is not written. The kernel
 * computes each 128-row block of S three times with the products and order
 * of attn_block_scores (every score bit-identical) and selects per row on
 * the fly; a row it cannot settle in three passes (more than 32 tiles in the
 * bin where its k-th largest score falls: runs of equal scores, a constant
 * or non-finite row) has its S row written to the workspace and is selected
 * by the row-wise kernel afterwards. Results equal attn_select's for the
 * same inputs. Top-k plans; the window rule as attn_select; top-p plans:
 * BSATTN_ERR_UNSUPPORTED. `ws` as for attn_select (info.select_workspace_bytes
 * also covers this call's list of rows to settle). scores_debug, if
 * non-NULL (16-byte aligned, [B, Hh, N, N] fp32), receives every row of S
 * as attn_block_scores writes it. */
bsattn_status attn_select_fused(const bsattn_plan* plan, const void* q_nat, const void* k_nat,
                                int32_t* idx, int32_t* cnt, float* scores_debug, void* ws,
                                size_t ws_bytes, void* stream);

/* Capacity of the library-owned scratch used by attn_select_static. */
#define BSATTN_STATIC_SELECT_SCRATCH_BYTES (16u << 20)

/* attn_select without a caller workspace (the method itself has no counterpart; this
 * is a convenience of this library). For callers that cannot allocate device
 * memory themselves, e.g. code that runs where cudaMalloc is not allowed or
 * whose allocator is owned by someone else. The pooled Q/K and the score
 * matrix live in one static device array of
 * BSATTN_STATIC_SELECT_SCRATCH_BYTES bytes. The call itself allocates nothing.
 * - The array is reserved on a device when attn_plan_create first runs there
 *   (it looks the array's device address up, once per device, with that
 *   device current, which loads the library module holding it); the device
 *   then holds it until the process exits. attn_plan_create does not fail if
 *   that memory is not available; attn_select_static then tries the lookup
 *   again and returns BSATTN_ERR_CUDA if it still fails.
 * - Problems whose select workspace (info.select_workspace_bytes) exceeds the
 *   capacity are rejected with BSATTN_ERR_UNSUPPORTED; the window rule needs
 *   no scratch.
 * - All calls share the one array: calls that may overlap on the GPU (other
 *   streams, other threads) race and must be serialised by the caller. No
 *   part of the array needs to start at zero: each call writes every byte it
 *   reads before reading it.
 * Results equal attn_select's for the same inputs. */
bsattn_status attn_select_static(const bsattn_plan* plan, const void* q_nat, const void* k_nat,
                                 int32_t* idx, int32_t* cnt, void* stream);

/* Per-tile e4m3 quantisation of a tiled bf16 tensor (FPSAttention page,
 * Approach: FP8 quantisation and block sparsity share one 3D tile
 * granularity): per (b, head, tile) scale = fp32(amax)/448 (amax 0 -> 1),
 * code = e4m3 of the IEEE fp32 quotient x/scale (computed without a division,
 * same bits), rounded to nearest even with finite saturation (OCP
 * E4M3; the page names FP8 without the format, this is the library's
 * reading). */
bsattn_status attn_quantize_e4m3(const bsattn_plan* plan, const void* x_tiled,
                                 uint8_t* codes, float* scales, void* stream);

/* Step 4: block-sparse attention on tiled inputs. q/k are bf16, or e4m3
 * codes with per-tile scales when the plan has qk_fp8 (q_scale/k_scale are
 * then required, else ignored). For every query tile i and j in
 * idx[..., i, :cnt]: S = scale * Q_i K_j^T (times q_scale_i * k_scale_j on
 * the e4m3 path), padded keys masked, fp32 online softmax, P rounded to
 * bf16, O += P V_j; O /= row sum. Writes tiled bf16 O (padded rows too) and,
 * if non-NULL, tiled fp32 lse. `ws`: info.forward_workspace_bytes (may be 0). */
bsattn_status attn_forward(const bsattn_plan* plan, const void* q, const void* k,
                           const float* q_scale, const float* k_scale, const void* v,
                           const int32_t* idx, const int32_t* cnt, void* o_tiled,
                           float* lse, void* ws, size_t ws_bytes, void* stream);

/* Step 4 on natural tensors: the same attention as attn_forward, reading
 * each (t, h, w) tile straight from natural [B, L, Hh, D] bf16 v (and q, k,
 * unless the plan has qk_fp8, in which case q/k are tiled e4m3 codes with
 * their tile scales as for attn_forward); tokens past the grid's edge read
 * as zero and are masked. Writes natural bf16 o_nat [B, L, Hh, D] and, if
 * non-NULL, natural fp32 lse [B, Hh, L]; padded slots are not written.
 * Pointers 16-byte aligned; `ws` as for attn_forward. */
bsattn_status attn_forward_natural(const bsattn_plan* plan, const void* q, const void* k,
                                   const float* q_scale, const float* k_scale, const void* v_nat,
                                   const int32_t* idx, const int32_t* cnt, void* o_nat,
                                   float* lse_nat, void* ws, size_t ws_bytes, void* stream);

/* The whole layer on natural tensors: pool (+ e4m3 quantisation of Q and K
 * into tile codes), block scores, selection, block-sparse attention. The
 * attention reads each 64-token chunk of Q straight from the natural layout
 * (the tile reorder happens in its loads; tokens past the grid's edge read
 * as zero and are masked) and writes natural bf16 O and, if non-NULL,
 * natural fp32 lse [B, Hh, L]. K and V are read the same way. Results
 * equal the step-by-step path (reorder, attn_forward, unreorder). If idx_out/cnt_out
 * are non-NULL the kept lists are also copied there. `ws` must hold
 * info.layer_workspace_bytes. */
bsattn_status attn_layer(const bsattn_plan* plan, const void* q_nat, const void* k_nat,
                         const void* v_nat, void* o_nat, float* lse_nat, int32_t* idx_out,
                         int32_t* cnt_out, void* ws, size_t ws_bytes, void* stream);

/* Backward of attn_forward (trainable block-sparse attention: "Faster Video
 * Diffusion with Trainable Sparse Attention", reproducibility record,
 * Research Type row). Tiled bf16 q, k, v, the forward's tiled bf16 o and fp32
 * lse [B, Hh, N, V], the incoming gradient d_o (tiled bf16) and the kept
 * lists the forward used; writes tiled bf16 dq, dk, dv. With P the masked
 * softmax recomputed from q, k and lse: dV = P^T dO, dS = P * (dO V^T -
 * rowsum(dO * O)), dQ = scale dS K, dK = scale dS^T Q, over kept tile pairs
 * and real (unpadded) tokens; rows of padded slots get zero gradients. P and
 * dS are rounded to bf16 for the products (fp32 accumulation). Any tile
 * shape attn_plan_create accepts; bf16 Q/K only (UNSUPPORTED for qk_fp8
 * plans). `ws` must hold
 * info.backward_workspace_bytes (rowsum, transposed lists). A list entry
 * outside [0, N) sets the device error word and is skipped. */
bsattn_status attn_backward(const bsattn_plan* plan, const void* q, const void* k, const void* v,
                            const void* o, const void* d_o, const float* lse, const int32_t* idx,
                            const int32_t* cnt, void* dq, void* dk, void* dv, void* ws,
                            size_t ws_bytes, void* stream);

/* Synchronise `stream`, read and clear the plan's device error word.
 * Returns OK, TIMEOUT or INTERNAL (bad list entry), or CUDA. */
bsattn_status attn_check_device_status(const bsattn_plan* plan, void* stream);

/* Denoising-step-aware schedule (FPSAttention page, Approach: the tile size,
 * the sparsity window and FP8 change between early, middle and late
 * denoising steps). Entry i is used for steps [first_step_i, first_step_{i+1})
 * and the last entry for every later step. Entries are ordered by strictly
 * increasing first_step starting at 0 and describe the same tensors (B,
 * heads, head_dim, T, H, W equal); tile shape, rule and qk_fp8 may differ.
 * At most BSATTN_MAX_SCHEDULE entries. */
#define BSATTN_MAX_SCHEDULE 64
typedef struct {
  int first_step;    /* first denoising step served by this entry          */
  bsattn_desc desc;
  bsattn_rule rule;
} bsattn_schedule_entry;
typedef struct bsattn_schedule bsattn_schedule;

/* Validate the entries (INVALID_ARG before any device call: null, n outside
 * [1, BSATTN_MAX_SCHEDULE], first_step not 0 then strictly increasing,
 * differing tensor shapes) and create one plan per entry (errors as
 * attn_plan_create; nothing is left allocated on failure). The schedule owns
 * its plans. */
bsattn_status attn_schedule_create(const bsattn_schedule_entry* entries, int n,
                                   bsattn_schedule** out);
void attn_schedule_destroy(bsattn_schedule* schedule);
/* The plan serving denoising step `step` (>= 0); owned by the schedule. */
bsattn_status attn_schedule_plan(const bsattn_schedule* schedule, int step,
                                 const bsattn_plan** plan);
/* Workspace for attn_schedule_layer at any step: the largest
 * info.layer_workspace_bytes of the schedule's plans. */
bsattn_status attn_schedule_workspace_bytes(const bsattn_schedule* schedule, size_t* bytes);
/* attn_layer with the plan serving `step`. idx_out/cnt_out (if non-NULL) are
 * sized for that plan ([B, Hh, N, kmax] and [B, Hh, N] of its tiles). */
bsattn_status attn_schedule_layer(const bsattn_schedule* schedule, int step, const void* q_nat,
                                  const void* k_nat, const void* v_nat, void* o_nat,
                                  float* lse_nat, int32_t* idx_out, int32_t* cnt_out, void* ws,
                                  size_t ws_bytes, void* stream);

/* Testing hooks. Neither is part of the method (the pages have no
 * counterpart); they let tests reach the failure paths without faulting a GPU.
 *
 * attn_testing_force_timeout(1): attention forward launches made afterwards
 * in this process (attn_forward, attn_forward_natural, attn_layer) cap the
 * kernel's abortable waits at about 1 ms and make each CTA's MMA-issuing
 * thread first wait on a barrier nothing arrives at, so every CTA takes its
 * bounded-wait timeout path: it records BSATTN_ERR_TIMEOUT in the plan's
 * device error word, lets its own copies and MMAs finish, frees its tensor
 * memory and returns; the outputs are then unspecified. (0) restores normal
 * launches. Process-wide; not for use while other threads launch work.
 *
 * attn_testing_set_error_word: writes `bits` (BSATTN_DEVERR_* bits: 1 = bad
 * list entry, 2 = timeout) into the plan's device error word with a
 * synchronous copy, so that attn_check_device_status's mapping can be tested
 * without a kernel. */
bsattn_status attn_testing_force_timeout(int on);
bsattn_status attn_testing_set_error_word(const bsattn_plan* plan, int bits);

#ifdef __cplusplus
}
#endif

#endif /* BSATTN_H */
