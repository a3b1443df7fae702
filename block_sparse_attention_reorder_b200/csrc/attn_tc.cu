// Block-sparse attention forward over kept tile pairs on the 5th-generation
// tensor cores (tcgen05, TMEM accumulators, TMA-fed shared memory).
//
// Work unit: a 128-row query block of two 64-row chunks, so that every QK^T
// and PV product is an M = 128 tcgen05.mma, and a step is one 64-key chunk.
// Tiles of 64 tokens (one chunk): the block stacks two adjacent query tiles
// i0, i1 of one (batch, head), next to each other along one axis of the tile
// grid (t for top-k / top-p, the window's widest axis for a window),
// and walks the union of their kept key-tile lists in ascending order; a key
// tile kept by only one of the two gives zero probabilities to the other
// tile's rows. Adjacent query tiles of a smooth video latent keep mostly the
// same key tiles, so little work is wasted. Larger tiles (64 * c tokens):
// the block holds chunks 2b and 2b + 1 of one query tile, which keep the
// same key tiles, and walks every chunk of each kept key tile that holds a
// real token; nothing is wasted.
//
// Roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r). Per key
//              tile: read S from TMEM, scale (and e4m3 tile scales), mask
//              padded keys, online softmax in fp32 with lazy rescaling
//              (the running max is only moved when it grows by more than
//              2^8, which keeps O and l exact up to rounding), write P as
//              bf16 into the TMEM columns S came from.
//   warp 4     TMA producer: Q block once, then K_j and V_j into two
//              separate two-stage rings (K released by its S MMA, V by its
//              PV MMA, so the next K loads while the current PV runs).
//   warp 5     MMA issuer (one thread): S_{n+2} = Q K^T is issued right
//              after PV_n so it overlaps softmax n+1; O += P_n V_n reads P
//              from TMEM (A operand) and V from shared memory (MN-major B).
// TMEM: columns [0,64) and [64,128) hold S/P double buffers, [128,128+D) O.
// Every mbarrier wait is bounded: on expiry the CTA sets the device error
// word, raises a CTA-wide abort flag, lets in-flight TMA copies land and
// frees its TMEM before returning.
#include <cudaTypedefs.h>
#include <math.h>


#include "internal.h"
#include "tc_common.cuh"

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on the driver library).
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

bool bsattn_make_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esz, int inner,
                        uint64_t rows, int box_inner, int box_rows, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)inner * esz};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 2;
static_assert(kStages == 2, "K/V slots are freed through the S / PV barriers of the same step parity");
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS0 = 0, kColS1 = 64, kColO = 128;
constexpr long long kWaitLimit = 4000000000LL;  // SM cycles (~2 s)
constexpr long long kTestWaitLimit = 2000000LL;  // ~1 ms, with the testing hook on
constexpr float kRescaleThreshold = 8.0f;        // log2 units

struct TcParams {
  Geom g;
  const float* qs;
  const float* ks;
  const int32_t* idx;
  const int32_t* cnt;
  int kmax;
  __nv_bfloat16* o;
  float* lse;
  float scale_log2;
  int* err;
  int umax;      // union list capacity (entries)
  int bm_words;  // bitmap words per list
  int pair_axis; // 0 = t, 1 = h, 2 = w
  int pdim[3];   // work items along t, h, w (pair axis halved)
  long long wait_limit;  // SM cycles a wait that can be aborted may take
  int stall;             // testing: the MMA thread first waits on a barrier nothing arrives at
};

template <int D, bool FP8>
struct Cfg {
  static constexpr int ESZ = FP8 ? 1 : 2;
  static constexpr int QRB = D * ESZ;                 // Q/K row bytes
  static constexpr int SWB = QRB >= 128 ? 128 : 64;   // swizzle span
  static constexpr uint32_t LAYOUT = SWB == 128 ? tc::kLayoutSW128 : tc::kLayoutSW64;
  static constexpr int QBLK = QRB / SWB;              // column blocks of Q/K
  static constexpr int NKS = QRB / 32;                // S MMAs (32 bytes of K each)
  static constexpr int KS_PER_BLK = SWB / 32;
  static constexpr int Q_BYTES = 128 * QRB;
  static constexpr int K_BYTES = 64 * QRB;
  static constexpr int V_BYTES = 64 * D * 2;
  static constexpr int VBLK = D / 64;                 // 64-column blocks of V
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + kStages * K_BYTES;
  static constexpr int OFF_BAR = OFF_V + kStages * V_BYTES;
  // barriers: q, kfull[S], vfull[S], sfull[2], pfull[2], pvdone[2], final
  static constexpr int NBAR = 1 + 2 * kStages + 7;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort, L, pad
  static constexpr int OFF_COL = OFF_MISC + 16;         // 64 packed column coords
  static constexpr int OFF_SCAN = OFF_COL + 256;        // block-scan scratch
  static constexpr int OFF_TOK = OFF_SCAN + 64;         // epilogue: natural token of each block row
  static constexpr int OFF_DYN = OFF_TOK + 512;         // bitmaps, union list
  static constexpr int O_PITCH = D * 2 + 16;            // epilogue staging row pitch
  static_assert(OFF_Q % 1024 == 0 && OFF_K % 1024 == 0 && OFF_V % 1024 == 0, "alignment");
  static_assert(128 * O_PITCH <= OFF_BAR - OFF_K, "epilogue staging fits in the ring");
};

__device__ __forceinline__ void record_timeout(volatile int* abort_flag, int* err) {
  *abort_flag = 1;
  atomicOr(err, BSATTN_DEVERR_TIMEOUT);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi, float& sum) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  float2 f = __bfloat1622float2(h);
  sum += f.x + f.y;
  return *reinterpret_cast<uint32_t*>(&h);
}

// NAT: Q, K and V are read from and O (and lse) written to the natural token
// layout [B, L, Hh, D] directly (else all tiled). Natural reads go
// through five-dimensional tensor maps whose box is one tile. e4m3 Q/K are
// always tile codes (tiled layout).
template <int D, bool FP8, bool NAT>
__global__ void __launch_bounds__(kThreads, 2)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, TcParams P) {
  using C = Cfg<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = tc::smem_addr(smem);
  const uint32_t bar_q = sb + C::OFF_BAR;
  // A K slot is free again when the S product that read it has completed,
  // a V slot when its PV product has: with kStages = 2 S buffers and ring
  // slots share the step parity, so the producer waits on sfull / pvdone
  // (their next phase needs its own next load first, so it cannot miss one).
  auto bar_kfull = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + s); };
  auto bar_vfull = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + kStages + s); };
  auto bar_sfull = [&](int b) { return sb + C::OFF_BAR + 8u * (1 + 2 * kStages + b); };
  auto bar_pfull = [&](int b) { return sb + C::OFF_BAR + 8u * (3 + 2 * kStages + b); };
  auto bar_pvdone = [&](int b) { return sb + C::OFF_BAR + 8u * (5 + 2 * kStages + b); };
  const uint32_t bar_final = sb + C::OFF_BAR + 8u * (7 + 2 * kStages);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* never = reinterpret_cast<volatile int*>(misc + 3);  // stays 0: waits that ignore abort
  uint32_t* colc = reinterpret_cast<uint32_t*>(smem + C::OFF_COL);
  int* scan = reinterpret_cast<int*>(smem + C::OFF_SCAN);
  uint32_t* bmA = reinterpret_cast<uint32_t*>(smem + C::OFF_DYN);
  uint32_t* bmB = bmA + P.bm_words;
  uint32_t* ulist = bmB + P.bm_words;
  uint32_t* uext = ulist + P.umax;  // real extent of each step's key chunk (see below)
  uint32_t* uorg = uext + P.umax;   // packed in-tile offsets of the steps' key chunks (several-chunk tiles)
  float* uks = reinterpret_cast<float*>(uorg + (P.g.nchunk > 1 ? P.umax : 0));  // e4m3: each step's key-tile scale

  const Geom& g = P.g;
  const int nchunk = g.nchunk;
  // Whether chunk c of tile j holds a real token (its first row, the box's
  // lowest corner, is inside the grid).
  auto chunk_real = [&](int j, int c) -> bool {
    const ChunkOrigin o = chunk_origin(g, c);
    const int bt = j / (g.nH * g.nW), bhh = (j / g.nW) % g.nH, bw = j % g.nW;
    return bt * g.tt + o.dt < g.T && bhh * g.th + o.dh < g.H && bw * g.tw + o.dw < g.W;
  };
  // Work item -> its two member (tile, chunk) halves; i1 = -1 when the
  // second half is absent (odd grid edge, odd chunk count; with natural
  // output also a chunk of padded rows only, which that output never holds).
  int i0, i1, c0 = 0, c1 = 0;
  if (nchunk > 1) {
    const int per = (nchunk + 1) / 2;
    i0 = i1 = blockIdx.x / per;
    c0 = 2 * (blockIdx.x % per);
    c1 = c0 + 1;
    if (c1 >= nchunk) i1 = -1;
    if (NAT) {
      if (i1 >= 0 && !chunk_real(i1, c1)) i1 = -1;
      if (!chunk_real(i0, c0)) {
        if (i1 < 0) return;  // uniform over the CTA, before any setup
        c0 = c1;
        i1 = -1;
      }
    }
  } else {
    const int nd[3] = {g.nT, g.nH, g.nW};
    int c[3], rem = blockIdx.x;
    c[2] = rem % P.pdim[2];
    rem /= P.pdim[2];
    c[1] = rem % P.pdim[1];
    c[0] = rem / P.pdim[1];
    c[P.pair_axis] *= 2;
    i0 = (c[0] * g.nH + c[1]) * g.nW + c[2];
    c[P.pair_axis] += 1;
    i1 = c[P.pair_axis] < nd[P.pair_axis] ? (c[0] * g.nH + c[1]) * g.nW + c[2] : -1;
  }
  const int head = blockIdx.y, b = blockIdx.z;
  const size_t bh = (size_t)b * g.Hh + head;
  const bool has1 = i1 >= 0;
  // Natural-layout coordinates (w, h, t) of a chunk's first token: the tile
  // origin plus the chunk's in-tile offset o. Computed once per chunk load
  // (and reused by a step's V load): the one producer thread issues every
  // load, so its integer divisions sit on the pipeline's path.
  struct NatXYZ {
    int x, y, z;
  };
  auto nat_xyz = [&](int tile, ChunkOrigin o) -> NatXYZ {
    const int bt = tile / (g.nH * g.nW), rem = tile - bt * (g.nH * g.nW);
    const int bhh = rem / g.nW, bw = rem - bhh * g.nW;
    return NatXYZ{bw * g.tw + o.dw, bhh * g.th + o.dh, bt * g.tt + o.dt};
  };
  // One chunk (64 tokens x 64 columns) of a natural-layout tensor: the box
  // {64 columns, cw, ch, ct, 1} at the chunk's first token, rows in (t, h, w)
  // order like the tiled layout; tokens past the grid's edge read as zero.
  auto load_nat = [&](uint32_t dst, const CUtensorMap* map, uint32_t bar, int col, NatXYZ p) {
    tc::tma_load_5d(dst, map, bar, col, p.x, p.y, p.z, b);
  };
  // In-tile offset of a step's key chunk (packed 10 bits per axis; zero for
  // one-chunk tiles).
  auto step_origin = [&](int n) -> ChunkOrigin {
    if (nchunk == 1) return ChunkOrigin{0, 0, 0};
    const uint32_t v = uorg[n];
    return ChunkOrigin{(int)(v & 0x3FFu), (int)((v >> 10) & 0x3FFu), (int)(v >> 20)};
  };
  // Real extent of a key chunk (tile j, in-tile offset o) from its first
  // token along t, h, w (capped at 255), bit 31 set when it is smaller than
  // the chunk box along some axis (padded keys to mask).
  auto chunk_ext = [&](int j, ChunkOrigin o) -> uint32_t {
    const int bt = j / (g.nH * g.nW), rem = j - bt * (g.nH * g.nW);
    const int bhh = rem / g.nW, bw = rem - bhh * g.nW;
    const int vt = min(g.T - bt * g.tt - o.dt, 255), vh = min(g.H - bhh * g.th - o.dh, 255),
              vw = min(g.W - bw * g.tw - o.dw, 255);
    const bool edge = vt < g.ct || vh < g.ch || vw < g.cw || g.cr < 64;
    return (uint32_t)vt | ((uint32_t)vh << 8) | ((uint32_t)vw << 16) | (edge ? 1u << 31 : 0u);
  };
  // First tiled-layout row of chunk c of tile j.
  auto tiled_row = [&](int j, int c) -> int { return (int)((bh * g.N + j) * g.V) + 64 * c; };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // The two kept-list counts and this thread's first entry of each list are
  // read first, so that their latency overlaps the set-up below: an entry's
  // address does not depend on the counts (entries at and beyond a count
  // are read but not used).
  const int32_t* lA = P.idx + (bh * g.N + i0) * (size_t)P.kmax;
  const int32_t* lB = has1 ? P.idx + (bh * g.N + i1) * (size_t)P.kmax : lA;
  int nA = P.cnt[bh * g.N + i0];
  int nB = has1 ? P.cnt[bh * g.N + i1] : 0;
  int jA = tid < P.kmax ? __ldg(lA + tid) : 0;
  int jB = has1 && tid < P.kmax ? __ldg(lB + tid) : 0;

  // ------------------------------------------------------------ setup
  if (tid == 0) {
    tc::mbar_init(bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(bar_kfull(s), 1);
      tc::mbar_init(bar_vfull(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(bar_sfull(x), 1);
      tc::mbar_init(bar_pfull(x), 128);
      tc::mbar_init(bar_pvdone(x), 1);
    }
    tc::mbar_init(bar_final, 1);
    misc[1] = 0;
    misc[3] = 0;
    tc::mbar_fence_init();
  }
  if (warp == 5) {
    tc::tmem_alloc(sb + C::OFF_MISC, kTmemCols);
    tc::tmem_relinquish();
  }
  if (tid < 64) colc[tid] = chunk_row_code(g, tid);  // in-chunk (t, h, w) offsets of each chunk row
  if (g.cr < 64) {
    // Tiles of fewer than 64 tokens: natural-layout loads fill only the
    // chunk box's rows; the rest of every V slot must hold finite values.
    for (int x = tid; x < kStages * C::V_BYTES / 16; x += kThreads)
      reinterpret_cast<uint4*>(smem + C::OFF_V)[x] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  for (int w = tid; w < 2 * P.bm_words; w += kThreads) bmA[w] = 0u;
  if (!has1) {
    // Rows 64..127 of the query block have no tile: zero them so no stale
    // bit pattern reaches the tensor cores.
    for (int x = tid; x < C::QBLK * 64 * C::SWB / 16; x += kThreads) {
      const int cb = x / (64 * C::SWB / 16), off = x % (64 * C::SWB / 16);
      reinterpret_cast<uint4*>(smem + C::OFF_Q + cb * 128 * C::SWB + 64 * C::SWB)[off] = make_uint4(0, 0, 0, 0);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  // Union of the two kept lists as a bitmap pair, then compacted ascending
  // into the step list: one entry per real 64-key chunk of each kept key
  // tile, key tile in bits 0-20, chunk in bits 21-29, bit 30 (31) set when
  // the first (second) query half keeps the tile.
  if (nA < 0 || nA > P.kmax || nB < 0 || nB > P.kmax) {
    if (tid == 0) atomicOr(P.err, BSATTN_DEVERR_BAD_INDEX);
    nA = min(max(nA, 0), P.kmax);
    nB = min(max(nB, 0), P.kmax);
  }
  for (int e = tid; e < max(nA, nB); e += kThreads) {
    if (e != tid) {
      jA = e < nA ? __ldg(lA + e) : 0;
      jB = e < nB ? __ldg(lB + e) : 0;
    }
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      if (e >= (x ? nB : nA)) continue;
      const int j = x ? jB : jA;
      if (j < 0 || j >= g.N) {
        atomicOr(P.err, BSATTN_DEVERR_BAD_INDEX);
        continue;
      }
      atomicOr(x ? &bmB[j >> 5] : &bmA[j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();
  {
    const int wpt = (P.bm_words + kThreads - 1) / kThreads;
    const int w0 = min(tid * wpt, P.bm_words), w1 = min(w0 + wpt, P.bm_words);
    auto real_chunks = [&](int j) -> int {
      int n = 0;
      for (int c = 0; c < nchunk; ++c) n += chunk_real(j, c) ? 1 : 0;
      return n;
    };
    int mine = 0;
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = bmA[w] | bmB[w];
      if (nchunk == 1) {
        mine += __popc(bits);
      } else {
        while (bits) {
          mine += real_chunks(w * 32 + __ffs(bits) - 1);
          bits &= bits - 1;
        }
      }
    }
    int x = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) scan[warp] = x;
    __syncthreads();
    int off = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) {
      off += i < warp ? scan[i] : 0;
      tot += scan[i];
    }
    int pos = off + x - mine;
    for (int w = w0; w < w1; ++w) {
      uint32_t a = bmA[w], bb = bmB[w], bits = a | bb;
      while (bits) {
        int bit = __ffs(bits) - 1;
        bits &= bits - 1;
        const int j = w * 32 + bit;
        const uint32_t e = (uint32_t)j | (((a >> bit) & 1u) << 30) | (((bb >> bit) & 1u) << 31);
        for (int c = 0; c < nchunk; ++c) {
          if (nchunk > 1 && !chunk_real(j, c)) continue;
          if (pos < P.umax) {
            ulist[pos] = e | ((uint32_t)c << 21);
            if (nchunk > 1) {
              const ChunkOrigin o = chunk_origin(g, c);
              uorg[pos] = (uint32_t)o.dt | ((uint32_t)o.dh << 10) | ((uint32_t)o.dw << 20);
              uext[pos] = chunk_ext(j, o);
            }
          }
          ++pos;
        }
      }
    }
    if (tid == 0) misc[2] = (uint32_t)min(tot, P.umax);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = misc[0];
  const int L = (int)misc[2];

  // ------------------------------------------------------------ roles
  if (warp == 4) {
    if (lane == 0 && L > 0) {
      tc::tma_prefetch_desc(&tmQ);
      tc::tma_prefetch_desc(&tmK);
      tc::tma_prefetch_desc(&tmV);
      // A natural-layout load fills the chunk box's rows (cr of them).
      const int qrows = NAT && !FP8 ? g.cr : 64, kvrows = NAT ? g.cr : 64;
      tc::mbar_arrive_expect_tx(bar_q, (has1 ? 2 : 1) * qrows * C::QRB);
      for (int x = 0; x < (has1 ? 2 : 1); ++x) {
        const int tile = x ? i1 : i0, chunk = x ? c1 : c0;
        const NatXYZ qp = NAT && !FP8 ? nat_xyz(tile, chunk_origin(g, chunk)) : NatXYZ{0, 0, 0};
#pragma unroll
        for (int cb = 0; cb < C::QBLK; ++cb) {
          const uint32_t dst = sb + C::OFF_Q + cb * 128 * C::SWB + x * 64 * C::SWB;
          if (NAT && !FP8)
            load_nat(dst, &tmQ, bar_q, head * D + cb * 64, qp);
          else
            tc::tma_load_2d(dst, &tmQ, bar_q, cb * C::SWB / C::ESZ, tiled_row(tile, chunk));
        }
      }
      // K_m is issued as soon as S_{m-2} has released its slot, V_{m-1} once
      // PV_{m-3} has: the two rings free up in MMA completion order, so K
      // runs one step ahead of V and its load latency hides behind softmax.
      int lastk[kStages], lastv[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) lastk[s] = lastv[s] = -1;
      NatXYZ kp{0, 0, 0};  // coordinates of the last natural K load, reused by its step's V load
      for (int m = 0; m <= L; ++m) {
        NatXYZ vp = kp;
        if (m < L) {
          const int s = m % kStages;
          if (m >= kStages &&
              !tc::mbar_wait(bar_sfull(s), ((m / kStages) - 1) & 1, abort_flag, P.wait_limit)) {
            record_timeout(abort_flag, P.err);
            break;
          }
          const int kt = (int)(ulist[m] & 0x1FFFFFu), kc = (int)((ulist[m] >> 21) & 0x1FFu);
          tc::mbar_arrive_expect_tx(bar_kfull(s), FP8 ? C::K_BYTES : kvrows * C::QRB);
          if (NAT && !FP8) kp = nat_xyz(kt, step_origin(m));
#pragma unroll
          for (int cb = 0; cb < C::QBLK; ++cb) {
            const uint32_t dst = sb + C::OFF_K + s * C::K_BYTES + cb * 64 * C::SWB;
            if (NAT && !FP8)
              load_nat(dst, &tmK, bar_kfull(s), head * D + cb * 64, kp);
            else
              tc::tma_load_2d(dst, &tmK, bar_kfull(s), cb * C::SWB / C::ESZ, tiled_row(kt, kc));
          }
          lastk[s] = m;
        }
        if (m >= 1) {
          const int v = m - 1, s = v % kStages;
          if (v >= kStages &&
              !tc::mbar_wait(bar_pvdone(s), ((v / kStages) - 1) & 1, abort_flag, P.wait_limit)) {
            record_timeout(abort_flag, P.err);
            break;
          }
          const int vt = (int)(ulist[v] & 0x1FFFFFu), vc = (int)((ulist[v] >> 21) & 0x1FFu);
          tc::mbar_arrive_expect_tx(bar_vfull(s), kvrows * D * 2);
          if (NAT && FP8) vp = nat_xyz(vt, step_origin(v));  // K came from tile codes: nothing to reuse
#pragma unroll
          for (int vb = 0; vb < C::VBLK; ++vb) {
            const uint32_t dst = sb + C::OFF_V + s * C::V_BYTES + vb * 8192;
            if (NAT)
              load_nat(dst, &tmV, bar_vfull(s), head * D + vb * 64, vp);
            else
              tc::tma_load_2d(dst, &tmV, bar_vfull(s), vb * 64, tiled_row(vt, vc));
          }
          lastv[s] = v;
        }
      }
      if (*abort_flag) {
        // Let copies already issued land before the CTA's memory goes away.
        tc::mbar_wait(bar_q, 0, never, kWaitLimit);
        for (int s = 0; s < kStages; ++s) {
          if (lastk[s] >= 0) tc::mbar_wait(bar_kfull(s), (lastk[s] / kStages) & 1, never, kWaitLimit);
          if (lastv[s] >= 0) tc::mbar_wait(bar_vfull(s), (lastv[s] / kStages) & 1, never, kWaitLimit);
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0 && L > 0) {
      constexpr uint32_t idS = FP8 ? tc::instr_desc(0, 0, 0, 0, 64, 128)
                                   : tc::instr_desc(1, 1, 0, 0, 64, 128);
      constexpr uint32_t idPV = tc::instr_desc(1, 1, 0, 1, D, 128);
      // Testing hook: bar_final gets its first arrival only from the final
      // commit below, so this wait runs out and the CTA takes the timeout path.
      bool ok = !P.stall || tc::mbar_wait(bar_final, 0, abort_flag, P.wait_limit);
      ok = ok && tc::mbar_wait(bar_q, 0, abort_flag, P.wait_limit);
      auto issue_S = [&](int m) -> bool {
        const int s = m % kStages;
        if (!tc::mbar_wait(bar_kfull(s), (m / kStages) & 1, abort_flag, P.wait_limit)) return false;
        tc::fence_after_sync();
        const uint32_t dS = tmem + ((m & 1) ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < C::NKS; ++kk) {
          const int cb = kk / C::KS_PER_BLK, within = kk % C::KS_PER_BLK;
          const uint64_t da = tc::smem_desc(sb + C::OFF_Q + cb * 128 * C::SWB + within * 32, 16,
                                            8 * C::SWB, C::LAYOUT);
          const uint64_t db = tc::smem_desc(sb + C::OFF_K + s * C::K_BYTES + cb * 64 * C::SWB + within * 32,
                                            16, 8 * C::SWB, C::LAYOUT);
          if (FP8)
            tc::mma_ss_f8(dS, da, db, idS, kk > 0 ? 1u : 0u);
          else
            tc::mma_ss_f16(dS, da, db, idS, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar_sfull(m & 1));
        return true;
      };
      if (ok) ok = issue_S(0);
      if (ok && L > 1) ok = issue_S(1);
      for (int n = 0; ok && n < L; ++n) {
        const int s = n % kStages;
        if (!tc::mbar_wait(bar_pfull(n & 1), (n >> 1) & 1, abort_flag, P.wait_limit) ||
            !tc::mbar_wait(bar_vfull(s), (n / kStages) & 1, abort_flag, P.wait_limit)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t pA = tmem + ((n & 1) ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t dv = tc::smem_desc(sb + C::OFF_V + s * C::V_BYTES + kk * 2048, 8192, 1024,
                                            tc::kLayoutSW128);
          tc::mma_ts_f16(tmem + kColO, pA + kk * 8, dv, idPV, (n > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(bar_pvdone(n & 1));
        if (n + 2 < L && !issue_S(n + 2)) {
          ok = false;
          break;
        }
      }
      if (!ok) record_timeout(abort_flag, P.err);
      // Every MMA issued so far has finished before TMEM is released.
      tc::mma_commit(bar_final);
      tc::mbar_wait(bar_final, 0, never, kWaitLimit);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- softmax
    const int r = tid;              // query row of the 128-row block
    const int half = r >> 6;        // 0: tile i0, 1: tile i1
    const bool row_exists = half == 0 || has1;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float qsc = (FP8 && row_exists) ? P.qs[bh * g.N + (half ? i1 : i0)] : 1.f;
    if (nchunk == 1 || FP8) {
      // Extents of one-chunk tiles, spread over the softmax threads (the
      // compaction above leaves them out: a dense bitmap word would put up
      // to 32 entries' divisions on one thread ahead of the CTA barrier),
      // and on the e4m3 path each step's key-tile scale, all fetched here
      // at once rather than one global load per step on the critical path.
      for (int n = r; n < L; n += 128) {
        const int jn = (int)(ulist[n] & 0x1FFFFFu);
        if (nchunk == 1) uext[n] = chunk_ext(jn, ChunkOrigin{0, 0, 0});
        if (FP8) uks[n] = __ldg(P.ks + bh * g.N + jn);
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
    }
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; n < L; ++n) {
      const uint32_t e = ulist[n];
      const bool keep = ((e >> (30 + half)) & 1u) != 0;  // uniform within the warp
      if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_sfull(n & 1), (n >> 1) & 1, abort_flag, P.wait_limit))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t sbuf = tmem + lane_base + ((n & 1) ? kColS1 : kColS0);
      uint32_t pk[32];
      bool need = false;
      float alpha = 1.f;
      if (keep) {
        uint32_t sr[64];
        tc::tmem_ld64_wait(sbuf, sr);
        const float c = P.scale_log2 * (FP8 ? qsc * uks[n] : 1.f);
        const uint32_t ext = uext[n];
        const bool edge = (ext >> 31) != 0;
        if (edge) {  // padded keys of an edge chunk
          const int vt = (int)(ext & 0xffu), vh = (int)((ext >> 8) & 0xffu), vw = (int)((ext >> 16) & 0xffu);
#pragma unroll
          for (int q = 0; q < 64; ++q) {
            const uint32_t cc = colc[q];
            if ((int)(cc & 0xffu) >= vt || (int)((cc >> 8) & 0xffu) >= vh || (int)((cc >> 16) & 0xffu) >= vw)
              sr[q] = 0xff800000u;  // -inf
          }
        }
        // Row max of the raw scores: three-input max, four chains. c > 0, so
        // the max of the scaled logits is c times the raw max.
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int q = 0; q < 32; ++q)
          mx4[q & 3] = tc::fmax3(mx4[q & 3], __uint_as_float(sr[2 * q]), __uint_as_float(sr[2 * q + 1]));
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * c;
        const float m_new = fmaxf(m, mx);
        if (m == -INFINITY) {
          m = m_new;  // first kept tile of this row: O row is still zero
        } else if (m_new - m > kRescaleThreshold) {
          alpha = tc::ex2(m - m_new);
          m = m_new;
          l *= alpha;
          need = true;
        }
        // p = 2^(s*c - m) on packed pairs. A quarter of the pairs of a full
        // tile take the FMA-pipe exponential so that the SFU, shared by both
        // CTAs' softmax warps, is not the bottleneck; edge tiles (with -inf
        // for padded keys) use the SFU throughout. The row sum uses the fp32
        // values, four packed chains.
        const float2 c2 = make_float2(c, c), nm2 = make_float2(-m, -m);
        float2 ls2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        auto emit = [&](int q, float2 pv) {
          ls2[q & 3] = __fadd2_rn(ls2[q & 3], pv);
          __nv_bfloat162 hv = __floats2bfloat162_rn(pv.x, pv.y);
          pk[q] = *reinterpret_cast<uint32_t*>(&hv);
        };
        if (edge) {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * q]), __uint_as_float(sr[2 * q + 1])), c2, nm2);
            emit(q, make_float2(tc::ex2(x.x), tc::ex2(x.y)));
          }
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * q]), __uint_as_float(sr[2 * q + 1])), c2, nm2);
            emit(q, (q & 3) == 3 ? tc::ex2_poly2(x) : make_float2(tc::ex2(x.x), tc::ex2(x.y)));
          }
        }
        const float2 lsa = __fadd2_rn(__fadd2_rn(ls2[0], ls2[1]), __fadd2_rn(ls2[2], ls2[3]));
        l += lsa.x + lsa.y;
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) pk[q] = 0u;
      }
      tc::tmem_st32(sbuf, pk);  // P_n over the first 32 columns of S_n
      if (__any_sync(0xffffffffu, need)) {
        // O holds PV_0..PV_{n-1} once PV_{n-1} has completed.
        if (!__all_sync(0xffffffffu,
                        tc::mbar_wait(bar_pvdone((n - 1) & 1), ((n - 1) >> 1) & 1, abort_flag, P.wait_limit))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
#pragma unroll
        for (int col = 0; col < D; col += 32) {
          uint32_t o[32];
          tc::tmem_ld32_wait(tmem + lane_base + kColO + col, o);
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
          tc::tmem_st32(tmem + lane_base + kColO + col, o);
        }
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(bar_pfull(n & 1));
    }
    if (!ok) record_timeout(abort_flag, P.err);
    // ---------------------------------------------------------- epilogue
    if (ok && L > 0) {
      if (!__all_sync(0xffffffffu,
                      tc::mbar_wait(bar_pvdone((L - 1) & 1), ((L - 1) >> 1) & 1, abort_flag, P.wait_limit))) {
        record_timeout(abort_flag, P.err);
        ok = false;
      }
      tc::fence_after_sync();
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    uint8_t* stage = smem + C::OFF_K + r * C::O_PITCH;
#pragma unroll
    for (int col = 0; col < D; col += 32) {
      uint32_t o[32];
      if (ok && L > 0) {
        tc::tmem_ld32_wait(tmem + lane_base + kColO + col, o);
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) o[q] = 0u;
      }
      uint32_t w[16];
      float dummy = 0.f;
#pragma unroll
      for (int q = 0; q < 16; ++q)
        w[q] = pack_bf16x2(__uint_as_float(o[2 * q]) * inv, __uint_as_float(o[2 * q + 1]) * inv, dummy);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        reinterpret_cast<uint4*>(stage + col * 2)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    }
    // Token of row rr of the block (natural layout), -1 for a padded slot.
    const ChunkOrigin qo0 = chunk_origin(g, c0), qo1 = chunk_origin(g, c1);
    auto token_of = [&](int rr) -> int {
      const int tile = rr >> 6 ? i1 : i0, q = rr & 63;
      if (q >= g.cr) return -1;
      const ChunkOrigin o = rr >> 6 ? qo1 : qo0;
      const int t = (tile / (g.nH * g.nW)) * g.tt + o.dt + q / (g.ch * g.cw);
      const int h = ((tile / g.nW) % g.nH) * g.th + o.dh + (q / g.cw) % g.ch;
      const int w = (tile % g.nW) * g.tw + o.dw + q % g.cw;
      return (t < g.T && h < g.H && w < g.W) ? (t * g.H + h) * g.W + w : -1;
    };
    const float lse_r = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
    // Each row's token once (its integer divisions would otherwise repeat
    // for every 16-byte piece of the row in the store loop below).
    int* tokrow = reinterpret_cast<int*>(smem + C::OFF_TOK);
    const int tok = NAT && row_exists ? token_of(r) : -1;
    if (NAT) tokrow[r] = tok;
    if (P.lse && row_exists) {
      if (NAT) {
        if (tok >= 0) P.lse[bh * (size_t)g.L + (size_t)tok] = lse_r;
      } else {
        P.lse[(size_t)tiled_row(half ? i1 : i0, half ? c1 : c0) + (r & 63)] = lse_r;
      }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    const int rows = has1 ? 128 : 64;
    for (int e2 = r; e2 < rows * CPR; e2 += 128) {
      const int rr = e2 / CPR, cc = e2 % CPR;
      const uint4 val = *reinterpret_cast<const uint4*>(smem + C::OFF_K + rr * C::O_PITCH + cc * 16);
      if (NAT) {
        const int n = tokrow[rr];
        if (n >= 0)
          reinterpret_cast<uint4*>(P.o + (((size_t)b * g.L + n) * g.Hh + head) * D)[cc] = val;
      } else {
        uint4* og = reinterpret_cast<uint4*>(P.o + (size_t)tiled_row(rr >> 6 ? i1 : i0, rr >> 6 ? c1 : c0) * D);
        og[(rr & 63) * CPR + cc] = val;
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
// Natural-layout tensor [B, T, H, W, Hh * D] as five dimensions, innermost
// first, with a one-chunk box of 64 columns (128 bytes, one swizzle span).
bool make_map_nat(CUtensorMap* map, const void* base, const bsattn_plan* p) {
  auto fn = encode_fn();
  if (!fn) return false;
  const bsattn_desc& d = p->desc;
  const cuuint64_t row = (cuuint64_t)d.heads * d.head_dim * 2;  // bytes per token
  cuuint64_t dims[5] = {(cuuint64_t)d.heads * d.head_dim, (cuuint64_t)d.W, (cuuint64_t)d.H, (cuuint64_t)d.T,
                        (cuuint64_t)d.B};
  cuuint64_t strides[4] = {row, row * d.W, row * d.W * d.H, row * d.W * d.H * d.T};
  cuuint32_t box[5] = {64, (cuuint32_t)p->cw, (cuuint32_t)p->ch, (cuuint32_t)p->ct, 1};  // one chunk
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool FP8, bool NAT>
bsattn_status run(const bsattn_plan* p, const void* q, const void* k, const __nv_bfloat16* v,
                  TcParams prm, cudaStream_t st) {
  using C = Cfg<D, FP8>;
  const uint64_t rows = (uint64_t)p->desc.B * p->desc.heads * p->N * p->V;
  if (rows + 128 >= (1ull << 31)) return BSATTN_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  const CUtensorMapDataType dqk = FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle sw = C::SWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (NAT && !FP8 ? !make_map_nat(&mq, q, p) : !bsattn_make_map_2d(&mq, q, dqk, C::ESZ, D, rows, C::SWB / C::ESZ, 64, sw))
    return BSATTN_ERR_CUDA;
  if (NAT && !FP8 ? !make_map_nat(&mk, k, p) : !bsattn_make_map_2d(&mk, k, dqk, C::ESZ, D, rows, C::SWB / C::ESZ, 64, sw))
    return BSATTN_ERR_CUDA;
  if (NAT ? !make_map_nat(&mv, v, p)
          : !bsattn_make_map_2d(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return BSATTN_ERR_CUDA;
  // Step list, extents and (tiles of several chunks) chunk offsets.
  size_t smem = 1024 + C::OFF_DYN + (size_t)prm.bm_words * 8 + (size_t)prm.umax * (p->nchunk > 1 ? 12 : 8) +
                (FP8 ? (size_t)prm.umax * 4 : 0);
  if (smem < 80 * 1024) smem = 80 * 1024;  // at most two CTAs (2 x 256 TMEM columns) per SM
  if (smem > 227 * 1024) return BSATTN_ERR_UNSUPPORTED;
  auto kern = attn_tc_kernel<D, FP8, NAT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return BSATTN_ERR_CUDA;
  const int items = p->nchunk > 1 ? p->N * ((p->nchunk + 1) / 2) : prm.pdim[0] * prm.pdim[1] * prm.pdim[2];
  dim3 grid(items, p->desc.heads, p->desc.B);
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

}  // namespace

size_t attention_workspace_bytes(const bsattn_plan*) { return 0; }

bsattn_status launch_attention(const bsattn_plan* p, const void* q, const void* k, const float* qs,
                               const float* ks, const __nv_bfloat16* v, const int32_t* idx,
                               const int32_t* cnt, __nv_bfloat16* o, float* lse, void*, size_t,
                               cudaStream_t st, AttnLayout lay) {
  if (p->N > 32768) return BSATTN_ERR_UNSUPPORTED;
  TcParams prm;
  prm.g = make_geom(p);
  prm.qs = qs;
  prm.ks = ks;
  prm.idx = idx;
  prm.cnt = cnt;
  prm.kmax = p->kmax;
  prm.o = o;
  prm.lse = lse;
  prm.scale_log2 = p->scale * 1.4426950408889634f;
  prm.err = p->d_err;
  // Step-list capacity: the union of two lists of one-chunk tiles, or one
  // list of tiles times their chunks.
  prm.umax = p->nchunk == 1 ? (p->N < 2 * p->kmax ? p->N : 2 * p->kmax)
                            : (p->N < p->kmax ? p->N : p->kmax) * p->nchunk;
  prm.bm_words = (p->N + 31) / 32;
  prm.pair_axis = pair_axis_of(p);
  prm.stall = bsattn_testing_timeout_forced() ? 1 : 0;
  prm.wait_limit = prm.stall ? kTestWaitLimit : kWaitLimit;
  const int nd[3] = {p->nT, p->nH, p->nW};
  for (int a = 0; a < 3; ++a) prm.pdim[a] = a == prm.pair_axis ? (nd[a] + 1) / 2 : nd[a];
  const bool fp8 = p->desc.qk_fp8 != 0, d128 = p->desc.head_dim == 128;
#define BSATTN_RUN(NATV)                                                                            \
  return d128 ? (fp8 ? run<128, true, NATV>(p, q, k, v, prm, st) : run<128, false, NATV>(p, q, k, v, prm, st)) \
              : (fp8 ? run<64, true, NATV>(p, q, k, v, prm, st) : run<64, false, NATV>(p, q, k, v, prm, st))
  if (lay == AttnLayout::Natural) BSATTN_RUN(true);
  BSATTN_RUN(false);
#undef BSATTN_RUN
}
