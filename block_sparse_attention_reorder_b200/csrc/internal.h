// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <stdint.h>
#include <stddef.h>

#include "bsattn.h"

// Device error word bits (plan->d_err).
enum : int {
  BSATTN_DEVERR_BAD_INDEX = 1,  // a kept-list entry or count outside [0, N]
  BSATTN_DEVERR_TIMEOUT = 2,    // a bounded wait gave up
};

struct bsattn_plan {
  bsattn_desc desc;
  bsattn_rule rule;
  int device;
  int Tp, Hp, Wp, nT, nH, nW, N, V, L, kmax;
  int nchunk;          // 64-row chunks per tile (V / 64)
  int ct, ch, cw;      // box of one chunk (t, h, w): ct * ch * cw = 64, or the whole tile of fewer tokens
  float scale;
  int* d_err;        // device error word
  int32_t* d_win_idx;  // window rule: [N, kmax]
  int32_t* d_win_cnt;  // window rule: [N]
};

// Geometry passed by value to kernels.
// Largest supported tile: 512 chunks of 64 tokens.
constexpr int kMaxChunks = 512;

// A tile holds V = 64 * nchunk tokens in (dt, dh, dw) row-major order; its
// rows [64c, 64c + 64) form chunk c, which is the box (ct, ch, cw) of the
// tile starting at in-tile coordinates chunk_origin(c).
struct Geom {
  int B, Hh, D;
  int T, H, W;
  int tt, th, tw;
  int nT, nH, nW, N, L;
  int V, nchunk, ct, ch, cw;
  int cr;  // rows of one chunk box, ct * ch * cw: 64, or fewer for a tile of fewer than 64 tokens
};

struct ChunkOrigin {
  int dt, dh, dw;
};
__host__ __device__ __forceinline__ ChunkOrigin chunk_origin(const Geom& g, int c) {
  const int r = 64 * c;
  return ChunkOrigin{r / (g.th * g.tw), (r / g.tw) % g.th, r % g.tw};
}

static inline Geom make_geom(const bsattn_plan* p) {
  Geom g;
  g.B = p->desc.B; g.Hh = p->desc.heads; g.D = p->desc.head_dim;
  g.T = p->desc.T; g.H = p->desc.H; g.W = p->desc.W;
  g.tt = p->desc.tile_t; g.th = p->desc.tile_h; g.tw = p->desc.tile_w;
  g.nT = p->nT; g.nH = p->nH; g.nW = p->nW; g.N = p->N; g.L = p->L;
  g.V = p->V; g.nchunk = p->nchunk; g.ct = p->ct; g.ch = p->ch; g.cw = p->cw;
  g.cr = p->ct * p->ch * p->cw;
  return g;
}

// Packed in-chunk offsets (t | h << 8 | w << 16) of chunk row r. Rows past
// the chunk box (rows cr..63 of a tile of fewer than 64 tokens, stored as 64
// rows) get 255 on every axis, which no real extent reaches.
__host__ __device__ __forceinline__ uint32_t chunk_row_code(const Geom& g, int r) {
  if (r >= g.cr) return 0xFFFFFFu;
  const int dt = r / (g.ch * g.cw), dh = (r / g.cw) % g.ch, dw = r % g.cw;
  return (uint32_t)dt | ((uint32_t)dh << 8) | ((uint32_t)dw << 16);
}

static inline bool aligned16(const void* ptr) { return (((uintptr_t)ptr) & 15u) == 0; }

// Makes `device` current for the lifetime of the object and gives the caller
// its own current device back when the object goes out of scope, so that no
// entry point changes the calling thread's current device. `status` is
// BSATTN_ERR_CUDA when either runtime call failed (then nothing is switched).
struct DeviceGuard {
  int prev = -1;
  bool switched = false;
  bsattn_status status = BSATTN_OK;
  explicit DeviceGuard(int device) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      status = BSATTN_ERR_CUDA;
      return;
    }
    if (prev != device) {
      if (cudaSetDevice(device) != cudaSuccess) {
        status = BSATTN_ERR_CUDA;
        return;
      }
      switched = true;
    }
  }
  ~DeviceGuard() {
    if (switched) cudaSetDevice(prev);
  }
  DeviceGuard(const DeviceGuard&) = delete;
  DeviceGuard& operator=(const DeviceGuard&) = delete;
};

// Testing hook (attn_testing_force_timeout): whether attention forward
// launches should take their timeout path.
bool bsattn_testing_timeout_forced();

// Looks up, with `device` current, the device address of the library-owned
// scratch array of attn_select_static and caches it; the lookup loads the
// module that holds the array (reserving its memory on that device).
bsattn_status bsattn_static_scratch_prepare(int device);

#define BSATTN_CUDA_TRY(expr)                         \
  do {                                                \
    cudaError_t e_ = (expr);                          \
    if (e_ != cudaSuccess) return BSATTN_ERR_CUDA;    \
  } while (0)

// Launch wrappers (each returns BSATTN_OK or BSATTN_ERR_CUDA).
// Natural -> tiled bf16 copy (padded slots zero).
bsattn_status launch_reorder(const Geom& g, const __nv_bfloat16* x_nat, __nv_bfloat16* x_tiled,
                             cudaStream_t st);
// e4m3 tile codes (tiled layout) and per-tile scales of natural Q and K, one launch.
bsattn_status launch_reorder_quant(const Geom& g, const __nv_bfloat16* q_nat, const __nv_bfloat16* k_nat,
                                   uint8_t* q_codes, uint8_t* k_codes, float* q_scales, float* k_scales,
                                   cudaStream_t st);
// fp32 tile means of one or two natural tensors (x1/p1 may be null).
bsattn_status launch_pool(const Geom& g, const __nv_bfloat16* x0, float* p0, const __nv_bfloat16* x1,
                          float* p1, cudaStream_t st);
bsattn_status launch_unreorder(const Geom& g, const __nv_bfloat16* x_tiled, __nv_bfloat16* x_nat,
                               const float* lse_tiled, float* lse_nat, cudaStream_t st);
bsattn_status launch_quant_tiled(const Geom& g, const __nv_bfloat16* x_tiled, uint8_t* codes,
                                 float* scales, cudaStream_t st);
// Block scores on the tensor cores (3xTF32); a bounded wait that gives up sets
// BSATTN_DEVERR_TIMEOUT in *err.
bsattn_status launch_block_scores(const Geom& g, const float* pq, const float* pk, float scale,
                                  float* S, int* err, cudaStream_t st);
bsattn_status launch_select_topk(int rows, int N, int k, const float* S, int32_t* idx,
                                 int32_t* cnt, int kmax, cudaStream_t st);
// Top-k of the rows listed in rlist[0, *rcount) only (rows <= total rows;
// the count is read on the device).
bsattn_status launch_select_topk_rows(int rows, int N, int k, const float* S, int32_t* idx, int32_t* cnt,
                                      int kmax, const int32_t* rlist, const int* rcount, cudaStream_t st);
// Fused block scores + top-k (S not materialised except for rows the fused
// kernel hands to the row-wise fallback, or every row when debug_s).
bsattn_status launch_fused_topk(const Geom& g, const float* pq, const float* pk, float scale, int k, int kmax,
                                int32_t* idx, int32_t* cnt, float* S, bool debug_s, int32_t* fb_rows, int* fb_count,
                                int* err, cudaStream_t st);
bsattn_status launch_select_topp(int rows, int N, int k, double p, const float* S, int32_t* idx,
                                 int32_t* cnt, int kmax, cudaStream_t st);
bsattn_status launch_broadcast_lists(int bh, int N, int kmax, const int32_t* src_idx,
                                     const int32_t* src_cnt, int32_t* idx, int32_t* cnt,
                                     cudaStream_t st);
// Where the attention's tensors live. Tiled: all tiled. Natural: Q, K, V, O
// and lse in the natural layout ([B, L, Hh, D], [B, Hh, L]). e4m3 Q/K are
// tile codes in both layouts.
enum class AttnLayout { Tiled, Natural };
bsattn_status launch_attention(const bsattn_plan* p, const void* q, const void* k,
                               const float* qs, const float* ks, const __nv_bfloat16* v,
                               const int32_t* idx, const int32_t* cnt, __nv_bfloat16* o,
                               float* lse, void* ws, size_t ws_bytes, cudaStream_t st,
                               AttnLayout lay);
// Tile axis (0 = t, 1 = h, 2 = w) along which two 64-token tiles are stacked
// into one 128-row block (attention: query tiles; dK/dV: key tiles). Top-k and
// top-p: t, whose neighbouring tiles keep the most key tiles in common on the
// blurred-field inputs (union efficiency 0.61 / 0.62 along t against 0.59 /
// 0.59 along w at the Wan-1.3B / Wan-14B sizes). Window: the axis the window
// reaches furthest along (t first on ties), so that the two lists overlap most.
static inline int pair_axis_of(const bsattn_plan* p) {
  if (p->rule.kind != BSATTN_RULE_WINDOW) return 0;
  const int w[3] = {p->rule.win_t, p->rule.win_h, p->rule.win_w};
  int a = 0;
  for (int x = 1; x < 3; ++x)
    if (w[x] > w[a]) a = x;
  return a;
}
size_t attention_workspace_bytes(const bsattn_plan* p);
// Scratch of the backward pass (carved from the caller's workspace).
struct BackwardWs {
  float* delta;    // [B, Hh, N, V] rowsum(dO * O)
  uint32_t* bm;    // [B, Hh, N, ceil(N/32)] transposed kept-list bitmaps
  int32_t* idxT;   // [B, Hh, N, N] query tiles keeping each key tile, ascending
  int32_t* cntT;   // [B, Hh, N]
};
bsattn_status launch_backward(const bsattn_plan* p, const void* q, const void* k, const void* v, const void* o,
                              const void* d_o, const float* lse, const int32_t* idx, const int32_t* cnt, void* dq,
                              void* dk, void* dv, const BackwardWs& w, cudaStream_t st);

// dQ of the backward on the tensor cores (tiled bf16 q, k, v, dO; lse and
// rowsum(dO * O) tiled fp32).
bsattn_status launch_backward_dq_tc(const bsattn_plan* p, const void* q, const void* k, const void* v,
                                    const void* d_o, const float* lse, const float* delta, const int32_t* idx,
                                    const int32_t* cnt, void* dq, cudaStream_t st);

// dK and dV of the backward on the tensor cores, over the transposed lists.
bsattn_status launch_backward_dkdv_tc(const bsattn_plan* p, const void* q, const void* k, const void* v,
                                      const void* d_o, const float* lse, const float* delta, const int32_t* idxT,
                                      const int32_t* cntT, void* dk, void* dv, cudaStream_t st);

// 2-D tiled tensor map over `rows` rows of `inner` elements of `esz` bytes.
bool bsattn_make_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esz, int inner,
                        uint64_t rows, int box_inner, int box_rows, CUtensorMapSwizzle sw);
