// dQ of the block-sparse attention backward on the 5th-generation tensor
// cores (tcgen05, TMEM accumulators, TMA-fed shared memory). The gradient of
// the trainable block-sparse attention ("Faster Video Diffusion with
// Trainable Sparse Attention", reproducibility record, Research Type row):
//   dQ_i = scale * sum_j dS_ij K_j,  dS_ij = P_ij * (dO_i V_j^T - Delta_i),
//   P_ij = 2^(scale log2(e) Q_i K_j^T - lse_i log2(e)),  Delta = rowsum(dO * O).
//
// Work unit, as in the forward kernel: a 128-row block of two 64-row chunks.
// With 64-token tiles, two adjacent query tiles (along t for top-k and top-p,
// the window's widest axis for a window) walking the union of their kept lists (a key tile
// kept by only one of the two gives zero dS to the other's rows); with tiles
// of several chunks, chunks 2b and 2b + 1 of one query tile walking every
// real chunk of each kept key tile.
//
// Roles (320 threads, one CTA per SM):
//   warps 0-7  warps w and w + 4 own query rows 32 (w % 4) .. (TMEM lanes);
//              warp w takes keys 0-31 of a step, warp w + 4 keys 32-63 (the
//              log-sum-exp is known, so the halves need no exchange). Each
//              reads its half of S and dP from TMEM, forms dS = P (dP - Delta)
//              in fp32 and writes it as bf16 over the first 16 columns of its
//              half of S.
//   warp 8     TMA producer: Q and dO blocks once, then K_j and V_j together
//              into a three-stage ring (a stage is released by the dQ MMA
//              that last reads K_j).
//   warp 9     MMA issuer (one thread): S_n = Q K_n^T and dP_n = dO V_n^T
//              (both SS, N = 64) into double buffers, two steps ahead of the
//              softmax side; dQ += dS_n K_n (dS from TMEM, K_n as an
//              MN-major shared-memory operand).
// TMEM (512 columns): S [0,64) and [64,128), dP [128,192) and [192,256),
// dQ [256, 256+D). Every mbarrier wait is bounded; on expiry the CTA sets
// the device error word, raises an abort flag, lets issued copies land,
// drains its MMAs and frees TMEM.
#include <cudaTypedefs.h>

#include "internal.h"
#include "tc_common.cuh"

namespace {

constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = 256;
constexpr int kStages = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256;
constexpr long long kWaitLimit = 4000000000LL;  // SM cycles (~2 s)

struct DqParams {
  Geom g;
  const int32_t* idx;
  const int32_t* cnt;
  const float* lse;    // tiled [B, Hh, N, 64], natural log
  const float* delta;  // tiled [B, Hh, N, 64]
  int kmax;
  __nv_bfloat16* dq;
  float scale;
  float scale_log2;
  int* err;
  int umax;
  int bm_words;
  int pair_axis;
  int pdim[3];
};

template <int D>
struct DqCfg {
  static constexpr int QRB = D * 2;                  // row bytes
  static constexpr int QBLK = QRB / 128;             // 128-byte column blocks
  static constexpr int NKS = QRB / 32;               // K = 16 MMAs per product
  static constexpr int BLK_BYTES = 128 * QRB;        // 128-row block (Q, dO)
  static constexpr int T_BYTES = 64 * QRB;           // one 64-row tile (K, V)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + BLK_BYTES;
  static constexpr int OFF_K = OFF_DO + BLK_BYTES;
  static constexpr int OFF_V = OFF_K + kStages * T_BYTES;
  static constexpr int OFF_BAR = OFF_V + kStages * T_BYTES;
  // barriers: q, full[S], empty[S], sfull[2], pfull[2], final
  static constexpr int NBAR = 1 + 2 * kStages + 5;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort, L, zero
  static constexpr int OFF_COL = OFF_MISC + 16;        // 64 packed in-tile coordinates
  static constexpr int OFF_SCAN = OFF_COL + 256;
  static constexpr int OFF_DYN = OFF_SCAN + 64;        // bitmaps, step list, extents
  static constexpr int O_PITCH = D * 2 + 16;           // epilogue staging pitch
  static_assert(128 * O_PITCH <= OFF_BAR - OFF_K, "epilogue staging fits in the rings");
};

// Work item -> its two (tile, chunk) halves; i1 = -1 when the second half is
// absent. 64-token tiles: adjacent tiles along the pair axis. Tiles of several
// chunks: chunks 2b and 2b + 1 of one tile (padding-only chunks included, so
// that their rows of the tiled gradients are written, as zeros).
__device__ __forceinline__ void block_halves(const Geom& g, int pair_axis, const int* pdim, int item, int* i0,
                                             int* i1, int* c0, int* c1) {
  if (g.nchunk > 1) {
    const int per = (g.nchunk + 1) / 2;
    *i0 = *i1 = item / per;
    *c0 = 2 * (item % per);
    *c1 = *c0 + 1;
    if (*c1 >= g.nchunk) *i1 = -1;
    return;
  }
  const int nd[3] = {g.nT, g.nH, g.nW};
  int c[3], rem = item;
  c[2] = rem % pdim[2];
  rem /= pdim[2];
  c[1] = rem % pdim[1];
  c[0] = rem / pdim[1];
  c[pair_axis] *= 2;
  *i0 = (c[0] * g.nH + c[1]) * g.nW + c[2];
  c[pair_axis] += 1;
  *i1 = c[pair_axis] < nd[pair_axis] ? (c[0] * g.nH + c[1]) * g.nW + c[2] : -1;
  *c0 = *c1 = 0;
}

// Whether chunk c of tile j holds a real token (its first row is in the grid).
__device__ __forceinline__ bool chunk_is_real(const Geom& g, int j, int c) {
  const ChunkOrigin o = chunk_origin(g, c);
  const int bt = j / (g.nH * g.nW), bhh = (j / g.nW) % g.nH, bw = j % g.nW;
  return bt * g.tt + o.dt < g.T && bhh * g.th + o.dh < g.H && bw * g.tw + o.dw < g.W;
}

// Compacts the union of two tile bitmaps into the ascending step list, one
// step per real 64-row chunk of each listed tile: tile in bits 0-20, chunk in
// bits 21-29, bit 30 (31) from the first (second) bitmap; ext gets the
// chunk's real extent from its first token (t, h, w bytes, capped at 255) and
// bit 31 when the chunk has padded rows. *count = steps (capped at cap). All
// threads of the CTA take part; the block-scan scratch holds one int per warp.
template <int NT>
__device__ __forceinline__ void compact_steps(const Geom& g, const uint32_t* bmA, const uint32_t* bmB, int words,
                                              uint32_t* list, uint32_t* ext, int cap, int* scan, uint32_t* count) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wpt = (words + NT - 1) / NT;
  const int w0 = min(tid * wpt, words), w1 = min(w0 + wpt, words);
  int mine = 0;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = bmA[w] | bmB[w];
    if (g.nchunk == 1) {
      mine += __popc(bits);
    } else {
      while (bits) {
        const int j = w * 32 + __ffs(bits) - 1;
        for (int c = 0; c < g.nchunk; ++c) mine += chunk_is_real(g, j, c) ? 1 : 0;
        bits &= bits - 1;
      }
    }
  }
  int x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scan[warp] = x;
  __syncthreads();
  int off = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) {
    off += i < warp ? scan[i] : 0;
    tot += scan[i];
  }
  int pos = off + x - mine;
  for (int w = w0; w < w1; ++w) {
    const uint32_t a = bmA[w], bb = bmB[w];
    uint32_t bits = a | bb;
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      const int j = w * 32 + bit;
      const uint32_t e = (uint32_t)j | (((a >> bit) & 1u) << 30) | (((bb >> bit) & 1u) << 31);
      const int bt = j / (g.nH * g.nW), bhh = (j / g.nW) % g.nH, bw = j % g.nW;
      for (int c = 0; c < g.nchunk; ++c) {
        if (g.nchunk > 1 && !chunk_is_real(g, j, c)) continue;
        if (pos < cap) {
          const ChunkOrigin o = chunk_origin(g, c);
          const int vt = min(g.T - bt * g.tt - o.dt, 255), vh = min(g.H - bhh * g.th - o.dh, 255),
                    vw = min(g.W - bw * g.tw - o.dw, 255);
          const bool edge = vt < g.ct || vh < g.ch || vw < g.cw || g.cr < 64;
          list[pos] = e | ((uint32_t)c << 21);
          ext[pos] = (uint32_t)vt | ((uint32_t)vh << 8) | ((uint32_t)vw << 16) | (edge ? 1u << 31 : 0u);
        }
        ++pos;
      }
    }
  }
  if (tid == 0) *count = (uint32_t)min(tot, cap);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, DqParams P) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = tc::smem_addr(smem);
  const uint32_t bar_q = sb + C::OFF_BAR;
  auto bar_full = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + s); };
  auto bar_empty = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + kStages + s); };
  auto bar_sfull = [&](int b) { return sb + C::OFF_BAR + 8u * (1 + 2 * kStages + b); };
  auto bar_pfull = [&](int b) { return sb + C::OFF_BAR + 8u * (3 + 2 * kStages + b); };
  const uint32_t bar_final = sb + C::OFF_BAR + 8u * (5 + 2 * kStages);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* never = reinterpret_cast<volatile int*>(misc + 3);
  uint32_t* colc = reinterpret_cast<uint32_t*>(smem + C::OFF_COL);
  int* scan = reinterpret_cast<int*>(smem + C::OFF_SCAN);
  uint32_t* bmA = reinterpret_cast<uint32_t*>(smem + C::OFF_DYN);
  uint32_t* bmB = bmA + P.bm_words;
  uint32_t* ulist = bmB + P.bm_words;
  uint32_t* uext = ulist + P.umax;

  const Geom& g = P.g;
  int i0, i1, c0 = 0, c1 = 0;
  block_halves(g, P.pair_axis, P.pdim, blockIdx.x, &i0, &i1, &c0, &c1);
  const int head = blockIdx.y, b = blockIdx.z;
  const size_t bh = (size_t)b * g.Hh + head;
  const bool has1 = i1 >= 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // First tiled-layout row of chunk c of tile j.
  auto tile_row = [&](int j, int c) -> int { return (int)((bh * g.N + j) * g.V) + 64 * c; };

  // ------------------------------------------------------------ setup
  if (tid == 0) {
    tc::mbar_init(bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(bar_full(s), 1);
      tc::mbar_init(bar_empty(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(bar_sfull(x), 1);
      tc::mbar_init(bar_pfull(x), kSoftmaxThreads);
    }
    tc::mbar_init(bar_final, 1);
    misc[1] = 0;
    misc[3] = 0;
    tc::mbar_fence_init();
  }
  if (warp == 9) {
    tc::tmem_alloc(sb + C::OFF_MISC, kTmemCols);
    tc::tmem_relinquish();
  }
  if (tid < 64) colc[tid] = chunk_row_code(g, tid);  // in-chunk (t, h, w) offsets of each chunk row
  for (int w = tid; w < 2 * P.bm_words; w += kThreads) bmA[w] = 0u;
  if (!has1) {  // rows 64..127 have no tile: zero their Q and dO
    for (int x = tid; x < C::QBLK * 64 * 128 / 16; x += kThreads) {
      const int cb = x / (64 * 128 / 16), off = x % (64 * 128 / 16);
      reinterpret_cast<uint4*>(smem + C::OFF_Q + cb * 128 * 128 + 64 * 128)[off] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(smem + C::OFF_DO + cb * 128 * 128 + 64 * 128)[off] = make_uint4(0, 0, 0, 0);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  // Union of the two kept lists, ascending, one step per real 64-key chunk:
  // key tile in bits 0-20, chunk in bits 21-29, bit 30 (31) when the first
  // (second) query half keeps the tile; uext holds the key chunk's real
  // extent from its first token (t, h, w bytes) and bit 31 when it has
  // padded keys.
  int nA = P.cnt[bh * g.N + i0];
  int nB = has1 ? P.cnt[bh * g.N + i1] : 0;
  if (nA < 0 || nA > P.kmax || nB < 0 || nB > P.kmax) {
    if (tid == 0) atomicOr(P.err, BSATTN_DEVERR_BAD_INDEX);
    nA = min(max(nA, 0), P.kmax);
    nB = min(max(nB, 0), P.kmax);
  }
  {
    const int32_t* lA = P.idx + (bh * g.N + i0) * (size_t)P.kmax;
    const int32_t* lB = has1 ? P.idx + (bh * g.N + i1) * (size_t)P.kmax : lA;
    for (int e = tid; e < nA + nB; e += kThreads) {
      const int j = e < nA ? __ldg(lA + e) : __ldg(lB + (e - nA));
      if (j < 0 || j >= g.N) {
        atomicOr(P.err, BSATTN_DEVERR_BAD_INDEX);
        continue;
      }
      atomicOr(e < nA ? &bmA[j >> 5] : &bmB[j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();
  compact_steps<kThreads>(g, bmA, bmB, P.bm_words, ulist, uext, P.umax, scan, misc + 2);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = misc[0];
  const int L = (int)misc[2];

  // ------------------------------------------------------------ roles
  if (warp == 8) {
    if (lane == 0 && L > 0) {
      tc::tma_prefetch_desc(&tmQ);
      tc::tma_prefetch_desc(&tmDO);
      tc::tma_prefetch_desc(&tmK);
      tc::tma_prefetch_desc(&tmV);
      tc::mbar_arrive_expect_tx(bar_q, (has1 ? 2 : 1) * 2 * 64 * C::QRB);
      for (int x = 0; x < (has1 ? 2 : 1); ++x) {
        const int row = x ? tile_row(i1, c1) : tile_row(i0, c0);
#pragma unroll
        for (int cb = 0; cb < C::QBLK; ++cb) {
          const uint32_t d = cb * 128 * 128 + x * 64 * 128;
          tc::tma_load_2d(sb + C::OFF_Q + d, &tmQ, bar_q, cb * 64, row);
          tc::tma_load_2d(sb + C::OFF_DO + d, &tmDO, bar_q, cb * 64, row);
        }
      }
      int last[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) last[s] = -1;
      for (int m = 0; m < L; ++m) {
        const int s = m % kStages;
        if (m >= kStages && !tc::mbar_wait(bar_empty(s), ((m / kStages) - 1) & 1, abort_flag, kWaitLimit)) {
          *abort_flag = 1;
          atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
          break;
        }
        const int krow = tile_row((int)(ulist[m] & 0x1FFFFFu), (int)((ulist[m] >> 21) & 0x1FFu));
        tc::mbar_arrive_expect_tx(bar_full(s), 2 * C::T_BYTES);
#pragma unroll
        for (int cb = 0; cb < C::QBLK; ++cb) {
          tc::tma_load_2d(sb + C::OFF_K + s * C::T_BYTES + cb * 64 * 128, &tmK, bar_full(s), cb * 64, krow);
          tc::tma_load_2d(sb + C::OFF_V + s * C::T_BYTES + cb * 64 * 128, &tmV, bar_full(s), cb * 64, krow);
        }
        last[s] = m;
      }
      if (*abort_flag) {
        tc::mbar_wait(bar_q, 0, never, kWaitLimit);
        for (int s = 0; s < kStages; ++s)
          if (last[s] >= 0) tc::mbar_wait(bar_full(s), (last[s] / kStages) & 1, never, kWaitLimit);
      }
    }
  } else if (warp == 9) {
    if (lane == 0 && L > 0) {
      constexpr uint32_t idS = tc::instr_desc(1, 1, 0, 0, 64, 128);   // bf16, K-major A and B, N = 64
      constexpr uint32_t idQ = tc::instr_desc(1, 1, 0, 1, D, 128);    // B (K tile) MN-major, N = D
      bool ok = tc::mbar_wait(bar_q, 0, abort_flag, kWaitLimit);
      // S_m = Q K_m^T and dP_m = dO V_m^T into buffer m & 1.
      auto issue_sdp = [&](int m) -> bool {
        const int s = m % kStages;
        if (!tc::mbar_wait(bar_full(s), (m / kStages) & 1, abort_flag, kWaitLimit)) return false;
        tc::fence_after_sync();
        const uint32_t dS = tmem + kColS + (m & 1) * 64, dP = tmem + kColDP + (m & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < C::NKS; ++kk) {
          const int cb = kk / 4, within = kk % 4;
          const uint32_t aoff = cb * 128 * 128 + within * 32, boff = s * C::T_BYTES + cb * 64 * 128 + within * 32;
          tc::mma_ss_f16(dS, tc::smem_desc(sb + C::OFF_Q + aoff, 16, 1024, tc::kLayoutSW128),
                         tc::smem_desc(sb + C::OFF_K + boff, 16, 1024, tc::kLayoutSW128), idS, kk > 0 ? 1u : 0u);
          tc::mma_ss_f16(dP, tc::smem_desc(sb + C::OFF_DO + aoff, 16, 1024, tc::kLayoutSW128),
                         tc::smem_desc(sb + C::OFF_V + boff, 16, 1024, tc::kLayoutSW128), idS, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar_sfull(m & 1));
        return true;
      };
      if (ok) ok = issue_sdp(0);
      if (ok && L > 1) ok = issue_sdp(1);
      for (int n = 0; ok && n < L; ++n) {
        const int s = n % kStages;
        if (!tc::mbar_wait(bar_pfull(n & 1), (n >> 1) & 1, abort_flag, kWaitLimit)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        // dS_n (bf16): keys 0-31 in S_n's columns 0-15, keys 32-63 in 32-47.
        const uint32_t dsA = tmem + kColS + (n & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 keys per MMA: 2048 bytes of the K tile
          const uint64_t dk = tc::smem_desc(sb + C::OFF_K + s * C::T_BYTES + kk * 2048, 8192, 1024, tc::kLayoutSW128);
          tc::mma_ts_f16(tmem + kColDQ, dsA + (kk < 2 ? kk * 8 : 32 + (kk - 2) * 8), dk, idQ,
                         (n > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(bar_empty(s));
        if (n + 2 < L && !issue_sdp(n + 2)) {
          ok = false;
          break;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
      }
      tc::mma_commit(bar_final);
      tc::mbar_wait(bar_final, 0, never, kWaitLimit);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- dS
    const int quad = warp & 3, part = warp >> 2;  // lane quadrant, key half
    const int r = quad * 32 + lane;
    const int half = r >> 6;
    const bool row_exists = half == 0 || has1;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const size_t lrow = row_exists ? (size_t)(half ? tile_row(i1, c1) : tile_row(i0, c0)) + (r & 63) : 0;
    const float lse2 = row_exists ? P.lse[lrow] * 1.4426950408889634f : 0.f;
    const float dlt = row_exists ? P.delta[lrow] : 0.f;
    const float c = P.scale_log2;
    bool ok = true;
    for (int n = 0; n < L; ++n) {
      const uint32_t e = ulist[n];
      const bool keep = row_exists && ((e >> (30 + half)) & 1u) != 0;  // uniform within the warp
      if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_sfull(n & 1), (n >> 1) & 1, abort_flag, kWaitLimit))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t sbuf = tmem + lane_base + kColS + (n & 1) * 64 + 32 * part;
      const uint32_t pbuf = tmem + lane_base + kColDP + (n & 1) * 64 + 32 * part;
      uint32_t dsw[16];
      if (keep) {
        const uint32_t ext = uext[n];
        const bool edge = (ext >> 31) != 0;
        const int vt = (int)(ext & 0xffu), vh = (int)((ext >> 8) & 0xffu), vw = (int)((ext >> 16) & 0xffu);
        uint32_t sr[32], pr[32];
        tc::tmem_ld32_wait(sbuf, sr);
        tc::tmem_ld32_wait(pbuf, pr);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float d2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            bool real = true;
            if (edge) {
              const uint32_t cc = colc[32 * part + 2 * q + u];
              real = (int)(cc & 0xffu) < vt && (int)((cc >> 8) & 0xffu) < vh && (int)((cc >> 16) & 0xffu) < vw;
            }
            const float p = real ? tc::ex2(__uint_as_float(sr[2 * q + u]) * c - lse2) : 0.f;
            d2[u] = p * (__uint_as_float(pr[2 * q + u]) - dlt);
          }
          __nv_bfloat162 hv = __floats2bfloat162_rn(d2[0], d2[1]);
          dsw[q] = *reinterpret_cast<uint32_t*>(&hv);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) dsw[q] = 0u;
      }
      tc::tmem_st16(sbuf, dsw);  // dS of this half over the first 16 columns of its S
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(bar_pfull(n & 1));
    }
    if (!ok) {
      *abort_flag = 1;
      atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && L > 0) {
      if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_final, 0, abort_flag, kWaitLimit))) {
        *abort_flag = 1;
        atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
        ok = false;
      }
      tc::fence_after_sync();
    }
    uint8_t* stage = smem + C::OFF_K + r * C::O_PITCH;
    constexpr int OC = D / 2;  // dQ columns this warp writes
#pragma unroll
    for (int col = part * OC; col < part * OC + OC; col += 32) {
      uint32_t o[32];
      if (ok && L > 0) {
        tc::tmem_ld32_wait(tmem + lane_base + kColDQ + col, o);
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) o[q] = 0u;
      }
      uint32_t w[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(o[2 * q]) * P.scale,
                                                  __uint_as_float(o[2 * q + 1]) * P.scale);
        w[q] = *reinterpret_cast<uint32_t*>(&hv);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        reinterpret_cast<uint4*>(stage + col * 2)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory");
    constexpr int CPR = D / 8;
    const int rows = has1 ? 128 : 64;
    for (int e2 = tid; e2 < rows * CPR; e2 += kSoftmaxThreads) {
      const int rr = e2 / CPR, cc = e2 % CPR;
      const uint4 val = *reinterpret_cast<const uint4*>(smem + C::OFF_K + rr * C::O_PITCH + cc * 16);
      uint4* og = reinterpret_cast<uint4*>(P.dq + (size_t)(rr >> 6 ? tile_row(i1, c1) : tile_row(i0, c0)) * D);
      og[(rr & 63) * CPR + cc] = val;
    }
  }

  // ------------------------------------------------------------ teardown
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
bsattn_status run_dq(const bsattn_plan* p, const void* q, const void* k, const void* v, const void* d_o,
                     DqParams prm, cudaStream_t st) {
  using C = DqCfg<D>;
  const uint64_t rows = (uint64_t)p->desc.B * p->desc.heads * p->N * p->V;
  if (rows + 128 >= (1ull << 31)) return BSATTN_ERR_UNSUPPORTED;
  CUtensorMap mq, mdo, mk, mv;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!bsattn_make_map_2d(&mq, q, bf, 2, D, rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bsattn_make_map_2d(&mdo, d_o, bf, 2, D, rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bsattn_make_map_2d(&mk, k, bf, 2, D, rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bsattn_make_map_2d(&mv, v, bf, 2, D, rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return BSATTN_ERR_CUDA;
  const size_t smem = 1024 + C::OFF_DYN + (size_t)prm.bm_words * 8 + (size_t)prm.umax * 8;
  if (smem > 227 * 1024) return BSATTN_ERR_UNSUPPORTED;
  auto kern = bwd_dq_tc_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return BSATTN_ERR_CUDA;
  const int items = p->nchunk > 1 ? p->N * ((p->nchunk + 1) / 2) : prm.pdim[0] * prm.pdim[1] * prm.pdim[2];
  dim3 grid(items, p->desc.heads, p->desc.B);
  kern<<<grid, kThreads, smem, st>>>(mq, mdo, mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

// ---------------------------------------------------------------- dK, dV
// Two adjacent key tiles j0, j1 stacked into one 128-row block walk the union
// of their transposed lists (the query tiles that keep them), on the same
// pattern with rows and columns exchanged:
//   S^T = K Q_i^T and dP^T = V dO_i^T (SS, N = 64) into TMEM double buffers;
//   P^T = 2^(S^T scale log2(e) - lse_i log2(e)) per query column,
//   dS^T = P^T (dP^T - Delta_i), both written back as bf16 over the first 16
//   columns of each key half of their buffers by eight warps;
//   dV += P^T dO_i and dK += dS^T Q_i (A from TMEM, dO_i and Q_i as MN-major
//   shared-memory operands), accumulated in TMEM; dK is scaled at the end.
// Per step the TMA warp brings Q_i, dO_i and the 64 lse and Delta values of
// query tile i into a three-stage ring.
struct KvParams {
  Geom g;
  const int32_t* idxT;  // [B, Hh, N, N] query tiles keeping each key tile, ascending
  const int32_t* cntT;  // [B, Hh, N]
  const float* lse;
  const float* delta;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float scale;
  float scale_log2;
  int* err;
  int umax;
  int bm_words;
  int pair_axis;
  int pdim[3];
};

template <int D>
struct KvCfg {
  static constexpr int QRB = D * 2;
  static constexpr int QBLK = QRB / 128;
  static constexpr int NKS = QRB / 32;
  static constexpr int BLK_BYTES = 128 * QRB;   // K or V block (two key tiles)
  static constexpr int T_BYTES = 64 * QRB;      // Q or dO tile
  static constexpr int STAGE = 2 * T_BYTES + 1024;  // Q, dO, lse (256 B), Delta (256 B), pad
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + BLK_BYTES;
  static constexpr int OFF_RING = OFF_V + BLK_BYTES;
  static constexpr int OFF_BAR = OFF_RING + kStages * STAGE;
  static constexpr int NBAR = 1 + 2 * kStages + 5;  // kv, full[S], empty[S], sfull[2], pfull[2], final
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_COL = OFF_MISC + 16;
  static constexpr int OFF_SCAN = OFF_COL + 256;
  static constexpr int OFF_DYN = OFF_SCAN + 64;
  static constexpr int O_PITCH = D * 2 + 16;
  static_assert(STAGE % 1024 == 0, "stage alignment");
  static_assert(2 * 128 * O_PITCH <= OFF_BAR - OFF_RING, "epilogue staging fits in the ring");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, KvParams P) {
  using C = KvCfg<D>;
  constexpr uint32_t kColST = 0, kColDPT = 128, kColDV = 256, kColDK = 256 + D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = tc::smem_addr(smem);
  const uint32_t bar_kv = sb + C::OFF_BAR;
  auto bar_full = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + s); };
  auto bar_empty = [&](int s) { return sb + C::OFF_BAR + 8u * (1 + kStages + s); };
  auto bar_sfull = [&](int b) { return sb + C::OFF_BAR + 8u * (1 + 2 * kStages + b); };
  auto bar_pfull = [&](int b) { return sb + C::OFF_BAR + 8u * (3 + 2 * kStages + b); };
  const uint32_t bar_final = sb + C::OFF_BAR + 8u * (5 + 2 * kStages);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* never = reinterpret_cast<volatile int*>(misc + 3);
  uint32_t* colc = reinterpret_cast<uint32_t*>(smem + C::OFF_COL);
  int* scan = reinterpret_cast<int*>(smem + C::OFF_SCAN);
  uint32_t* bmA = reinterpret_cast<uint32_t*>(smem + C::OFF_DYN);
  uint32_t* bmB = bmA + P.bm_words;
  uint32_t* ulist = bmB + P.bm_words;
  uint32_t* uext = ulist + P.umax;

  const Geom& g = P.g;
  int j0, j1, kc0 = 0, kc1 = 0;
  block_halves(g, P.pair_axis, P.pdim, blockIdx.x, &j0, &j1, &kc0, &kc1);
  const int head = blockIdx.y, b = blockIdx.z;
  const size_t bh = (size_t)b * g.Hh + head;
  const bool has1 = j1 >= 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // First tiled-layout row of chunk c of tile j.
  auto tile_row = [&](int j, int c) -> int { return (int)((bh * g.N + j) * g.V) + 64 * c; };
  // Whether row q of chunk c of tile j is a real token.
  auto row_is_real = [&](int j, int c, int q) -> bool {
    const ChunkOrigin o = chunk_origin(g, c);
    const int bt = j / (g.nH * g.nW), bhh = (j / g.nW) % g.nH, bw = j % g.nW;
    const uint32_t cc = colc[q];
    return bt * g.tt + o.dt + (int)(cc & 0xffu) < g.T && bhh * g.th + o.dh + (int)((cc >> 8) & 0xffu) < g.H &&
           bw * g.tw + o.dw + (int)((cc >> 16) & 0xffu) < g.W;
  };

  // ------------------------------------------------------------ setup
  if (tid == 0) {
    tc::mbar_init(bar_kv, 1);
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(bar_full(s), 1);
      tc::mbar_init(bar_empty(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(bar_sfull(x), 1);
      tc::mbar_init(bar_pfull(x), kSoftmaxThreads);
    }
    tc::mbar_init(bar_final, 1);
    misc[1] = 0;
    misc[3] = 0;
    tc::mbar_fence_init();
  }
  if (warp == 9) {
    tc::tmem_alloc(sb + C::OFF_MISC, kTmemCols);
    tc::tmem_relinquish();
  }
  if (tid < 64) colc[tid] = chunk_row_code(g, tid);  // in-chunk (t, h, w) offsets of each chunk row
  for (int w = tid; w < 2 * P.bm_words; w += kThreads) bmA[w] = 0u;
  if (!has1) {  // rows 64..127 have no key tile: zero their K and V
    for (int x = tid; x < C::QBLK * 64 * 128 / 16; x += kThreads) {
      const int cb = x / (64 * 128 / 16), off = x % (64 * 128 / 16);
      reinterpret_cast<uint4*>(smem + C::OFF_K + cb * 128 * 128 + 64 * 128)[off] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(smem + C::OFF_V + cb * 128 * 128 + 64 * 128)[off] = make_uint4(0, 0, 0, 0);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  // Union of the two transposed lists, ascending, one step per real chunk of
  // each listed query tile: query tile in bits 0-20, chunk in bits 21-29, bit
  // 30 (31) when it keeps j0 (j1); uext holds the query chunk's real extent
  // and bit 31 when it has padded rows.
  {
    const int nA = min(max(P.cntT[bh * g.N + j0], 0), g.N);
    const int nB = has1 ? min(max(P.cntT[bh * g.N + j1], 0), g.N) : 0;
    const int32_t* lA = P.idxT + (bh * g.N + j0) * (size_t)g.N;
    const int32_t* lB = has1 ? P.idxT + (bh * g.N + j1) * (size_t)g.N : lA;
    for (int e = tid; e < nA + nB; e += kThreads) {
      const int i = e < nA ? __ldg(lA + e) : __ldg(lB + (e - nA));
      if (i < 0 || i >= g.N) continue;  // the transposed lists are built in range
      atomicOr(e < nA ? &bmA[i >> 5] : &bmB[i >> 5], 1u << (i & 31));
    }
  }
  __syncthreads();
  compact_steps<kThreads>(g, bmA, bmB, P.bm_words, ulist, uext, P.umax, scan, misc + 2);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = misc[0];
  const int L = (int)misc[2];

  // ------------------------------------------------------------ roles
  if (warp == 8) {
    if (lane == 0 && L > 0) {
      tc::tma_prefetch_desc(&tmQ);
      tc::tma_prefetch_desc(&tmDO);
      tc::tma_prefetch_desc(&tmK);
      tc::tma_prefetch_desc(&tmV);
      tc::mbar_arrive_expect_tx(bar_kv, (has1 ? 2 : 1) * 2 * 64 * C::QRB);
      for (int x = 0; x < (has1 ? 2 : 1); ++x) {
        const int row = x ? tile_row(j1, kc1) : tile_row(j0, kc0);
#pragma unroll
        for (int cb = 0; cb < C::QBLK; ++cb) {
          const uint32_t d = cb * 128 * 128 + x * 64 * 128;
          tc::tma_load_2d(sb + C::OFF_K + d, &tmK, bar_kv, cb * 64, row);
          tc::tma_load_2d(sb + C::OFF_V + d, &tmV, bar_kv, cb * 64, row);
        }
      }
      int last[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) last[s] = -1;
      for (int m = 0; m < L; ++m) {
        const int s = m % kStages;
        if (m >= kStages && !tc::mbar_wait(bar_empty(s), ((m / kStages) - 1) & 1, abort_flag, kWaitLimit)) {
          *abort_flag = 1;
          atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
          break;
        }
        const int qrow = tile_row((int)(ulist[m] & 0x1FFFFFu), (int)((ulist[m] >> 21) & 0x1FFu));
        const uint32_t st = sb + C::OFF_RING + s * C::STAGE;
        tc::mbar_arrive_expect_tx(bar_full(s), 2 * C::T_BYTES + 512);
#pragma unroll
        for (int cb = 0; cb < C::QBLK; ++cb) {
          tc::tma_load_2d(st + cb * 64 * 128, &tmQ, bar_full(s), cb * 64, qrow);
          tc::tma_load_2d(st + C::T_BYTES + cb * 64 * 128, &tmDO, bar_full(s), cb * 64, qrow);
        }
        tc::bulk_load(st + 2 * C::T_BYTES, P.lse + qrow, 256, bar_full(s));
        tc::bulk_load(st + 2 * C::T_BYTES + 256, P.delta + qrow, 256, bar_full(s));
        last[s] = m;
      }
      if (*abort_flag) {
        tc::mbar_wait(bar_kv, 0, never, kWaitLimit);
        for (int s = 0; s < kStages; ++s)
          if (last[s] >= 0) tc::mbar_wait(bar_full(s), (last[s] / kStages) & 1, never, kWaitLimit);
      }
    }
  } else if (warp == 9) {
    if (lane == 0 && L > 0) {
      constexpr uint32_t idS = tc::instr_desc(1, 1, 0, 0, 64, 128);  // K-major A and B, N = 64
      constexpr uint32_t idG = tc::instr_desc(1, 1, 0, 1, D, 128);   // B MN-major, N = D
      bool ok = tc::mbar_wait(bar_kv, 0, abort_flag, kWaitLimit);
      auto issue_sdp = [&](int m) -> bool {
        const int s = m % kStages;
        if (!tc::mbar_wait(bar_full(s), (m / kStages) & 1, abort_flag, kWaitLimit)) return false;
        tc::fence_after_sync();
        const uint32_t st = sb + C::OFF_RING + s * C::STAGE;
        const uint32_t dS = tmem + kColST + (m & 1) * 64, dP = tmem + kColDPT + (m & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < C::NKS; ++kk) {
          const int cb = kk / 4, within = kk % 4;
          const uint32_t aoff = cb * 128 * 128 + within * 32, boff = cb * 64 * 128 + within * 32;
          tc::mma_ss_f16(dS, tc::smem_desc(sb + C::OFF_K + aoff, 16, 1024, tc::kLayoutSW128),
                         tc::smem_desc(st + boff, 16, 1024, tc::kLayoutSW128), idS, kk > 0 ? 1u : 0u);
          tc::mma_ss_f16(dP, tc::smem_desc(sb + C::OFF_V + aoff, 16, 1024, tc::kLayoutSW128),
                         tc::smem_desc(st + C::T_BYTES + boff, 16, 1024, tc::kLayoutSW128), idS, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar_sfull(m & 1));
        return true;
      };
      if (ok) ok = issue_sdp(0);
      if (ok && L > 1) ok = issue_sdp(1);
      for (int n = 0; ok && n < L; ++n) {
        const int s = n % kStages;
        if (!tc::mbar_wait(bar_pfull(n & 1), (n >> 1) & 1, abort_flag, kWaitLimit)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t st = sb + C::OFF_RING + s * C::STAGE;
        // P^T and dS^T (bf16): queries 0-31 in columns 0-15, 32-63 in 32-47.
        const uint32_t pA = tmem + kColST + (n & 1) * 64, dsA = tmem + kColDPT + (n & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 queries per MMA: 2048 bytes of the dO / Q tile
          const uint32_t acol = kk < 2 ? kk * 8 : 32 + (kk - 2) * 8;
          const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
          tc::mma_ts_f16(tmem + kColDV, pA + acol,
                         tc::smem_desc(st + C::T_BYTES + kk * 2048, 8192, 1024, tc::kLayoutSW128), idG, acc);
          tc::mma_ts_f16(tmem + kColDK, dsA + acol, tc::smem_desc(st + kk * 2048, 8192, 1024, tc::kLayoutSW128),
                         idG, acc);
        }
        tc::mma_commit(bar_empty(s));
        if (n + 2 < L && !issue_sdp(n + 2)) {
          ok = false;
          break;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
      }
      tc::mma_commit(bar_final);
      tc::mbar_wait(bar_final, 0, never, kWaitLimit);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- P^T, dS^T
    const int quad = warp & 3, part = warp >> 2;  // lane quadrant, query half
    const int r = quad * 32 + lane;                // key row of the block
    const int half = r >> 6;                       // 0: tile j0, 1: tile j1
    const bool row_exists = half == 0 || has1;
    const bool key_real = row_exists && (half ? row_is_real(j1, kc1, r & 63) : row_is_real(j0, kc0, r & 63));
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const float c = P.scale_log2;
    bool ok = true;
    for (int n = 0; n < L; ++n) {
      const uint32_t e = ulist[n];
      const bool keep = row_exists && ((e >> (30 + half)) & 1u) != 0;  // uniform within the warp
      if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_sfull(n & 1), (n >> 1) & 1, abort_flag, kWaitLimit))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t sbuf = tmem + lane_base + kColST + (n & 1) * 64 + 32 * part;
      const uint32_t pbuf = tmem + lane_base + kColDPT + (n & 1) * 64 + 32 * part;
      // lse and Delta of this step's query tile came with its TMA copies:
      // observe their barrier before reading them.
      if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_full(n % kStages), (n / kStages) & 1, abort_flag, kWaitLimit))) {
        ok = false;
        break;
      }
      uint32_t pw[16], dw[16];
      if (keep) {
        const float* ld = reinterpret_cast<const float*>(smem + C::OFF_RING + (n % kStages) * C::STAGE + 2 * C::T_BYTES);
        const uint32_t ext = uext[n];
        const bool edge = (ext >> 31) != 0;
        const int vt = (int)(ext & 0xffu), vh = (int)((ext >> 8) & 0xffu), vw = (int)((ext >> 16) & 0xffu);
        uint32_t sr[32], pr[32];
        tc::tmem_ld32_wait(sbuf, sr);
        tc::tmem_ld32_wait(pbuf, pr);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float pp[2], d2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int qc = 32 * part + 2 * q + u;  // query column
            bool real = key_real;
            if (edge) {
              const uint32_t cc = colc[qc];
              real = real && (int)(cc & 0xffu) < vt && (int)((cc >> 8) & 0xffu) < vh && (int)((cc >> 16) & 0xffu) < vw;
            }
            const float p = real ? tc::ex2(__uint_as_float(sr[2 * q + u]) * c - ld[qc] * 1.4426950408889634f) : 0.f;
            pp[u] = p;
            d2[u] = p * (__uint_as_float(pr[2 * q + u]) - ld[64 + qc]);
          }
          __nv_bfloat162 hp = __floats2bfloat162_rn(pp[0], pp[1]), hd = __floats2bfloat162_rn(d2[0], d2[1]);
          pw[q] = *reinterpret_cast<uint32_t*>(&hp);
          dw[q] = *reinterpret_cast<uint32_t*>(&hd);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) pw[q] = dw[q] = 0u;
      }
      tc::tmem_st16(sbuf, pw);  // P^T over the first 16 columns of this half of S^T
      tc::tmem_st16(pbuf, dw);  // dS^T over the first 16 columns of this half of dP^T
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(bar_pfull(n & 1));
    }
    if (!ok) {
      *abort_flag = 1;
      atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && L > 0) {
      if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_final, 0, abort_flag, kWaitLimit))) {
        *abort_flag = 1;
        atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
        ok = false;
      }
      tc::fence_after_sync();
    }
    // dK (scaled) and dV rows staged in the ring: dK at rows 0-127, dV at 128-255.
    constexpr int OC = D / 2;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      uint8_t* stage = smem + C::OFF_RING + (which * 128 + r) * C::O_PITCH;
      const float mul = which == 0 ? P.scale : 1.f;
      const uint32_t base = which == 0 ? kColDK : kColDV;
#pragma unroll
      for (int col = part * OC; col < part * OC + OC; col += 32) {
        uint32_t o[32];
        if (ok && L > 0) {
          tc::tmem_ld32_wait(tmem + lane_base + base + col, o);
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(o[2 * q]) * mul, __uint_as_float(o[2 * q + 1]) * mul);
          w[q] = *reinterpret_cast<uint32_t*>(&hv);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          reinterpret_cast<uint4*>(stage + col * 2)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory");
    constexpr int CPR = D / 8;
    const int rows = has1 ? 128 : 64;
    for (int e2 = tid; e2 < 2 * rows * CPR; e2 += kSoftmaxThreads) {
      const int which = e2 / (rows * CPR), rem = e2 % (rows * CPR);
      const int rr = rem / CPR, cc = rem % CPR;
      const uint4 val = *reinterpret_cast<const uint4*>(smem + C::OFF_RING + (which * 128 + rr) * C::O_PITCH + cc * 16);
      __nv_bfloat16* dst = which == 0 ? P.dk : P.dv;
      uint4* og = reinterpret_cast<uint4*>(dst + (size_t)(rr >> 6 ? tile_row(j1, kc1) : tile_row(j0, kc0)) * D);
      og[(rr & 63) * CPR + cc] = val;
    }
  }

  // ------------------------------------------------------------ teardown
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
bsattn_status run_dkdv(const bsattn_plan* p, const void* q, const void* k, const void* v, const void* d_o,
                       KvParams prm, cudaStream_t st) {
  using C = KvCfg<D>;
  const uint64_t rows = (uint64_t)p->desc.B * p->desc.heads * p->N * p->V;
  if (rows + 128 >= (1ull << 31)) return BSATTN_ERR_UNSUPPORTED;
  CUtensorMap mq, mdo, mk, mv;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!bsattn_make_map_2d(&mq, q, bf, 2, D, rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bsattn_make_map_2d(&mdo, d_o, bf, 2, D, rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bsattn_make_map_2d(&mk, k, bf, 2, D, rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bsattn_make_map_2d(&mv, v, bf, 2, D, rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return BSATTN_ERR_CUDA;
  const size_t smem = 1024 + C::OFF_DYN + (size_t)prm.bm_words * 8 + (size_t)prm.umax * 8;
  if (smem > 227 * 1024) return BSATTN_ERR_UNSUPPORTED;
  auto kern = bwd_dkdv_tc_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return BSATTN_ERR_CUDA;
  const int items = p->nchunk > 1 ? p->N * ((p->nchunk + 1) / 2) : prm.pdim[0] * prm.pdim[1] * prm.pdim[2];
  dim3 grid(items, p->desc.heads, p->desc.B);
  kern<<<grid, kThreads, smem, st>>>(mq, mdo, mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

}  // namespace

bsattn_status launch_backward_dq_tc(const bsattn_plan* p, const void* q, const void* k, const void* v,
                                    const void* d_o, const float* lse, const float* delta, const int32_t* idx,
                                    const int32_t* cnt, void* dq, cudaStream_t st) {
  DqParams prm;
  prm.g = make_geom(p);
  prm.idx = idx;
  prm.cnt = cnt;
  prm.lse = lse;
  prm.delta = delta;
  prm.kmax = p->kmax;
  prm.dq = (__nv_bfloat16*)dq;
  prm.scale = p->scale;
  prm.scale_log2 = p->scale * 1.4426950408889634f;
  prm.err = p->d_err;
  // Steps: the union of two kept lists (one list for tiles of several chunks), times the chunks.
  prm.umax = p->nchunk == 1 ? (p->N < 2 * p->kmax ? p->N : 2 * p->kmax) : (p->N < p->kmax ? p->N : p->kmax) * p->nchunk;
  prm.bm_words = (p->N + 31) / 32;
  prm.pair_axis = pair_axis_of(p);
  const int nd[3] = {p->nT, p->nH, p->nW};
  for (int a = 0; a < 3; ++a) prm.pdim[a] = a == prm.pair_axis ? (nd[a] + 1) / 2 : nd[a];
  return p->desc.head_dim == 128 ? run_dq<128>(p, q, k, v, d_o, prm, st) : run_dq<64>(p, q, k, v, d_o, prm, st);
}

bsattn_status launch_backward_dkdv_tc(const bsattn_plan* p, const void* q, const void* k, const void* v,
                                      const void* d_o, const float* lse, const float* delta, const int32_t* idxT,
                                      const int32_t* cntT, void* dk, void* dv, cudaStream_t st) {
  KvParams prm;
  prm.g = make_geom(p);
  prm.idxT = idxT;
  prm.cntT = cntT;
  prm.lse = lse;
  prm.delta = delta;
  prm.dk = (__nv_bfloat16*)dk;
  prm.dv = (__nv_bfloat16*)dv;
  prm.scale = p->scale;
  prm.scale_log2 = p->scale * 1.4426950408889634f;
  prm.err = p->d_err;
  // Steps: at most N query tiles in the union of two transposed lists, times their chunks.
  prm.umax = p->N * p->nchunk;
  prm.bm_words = (p->N + 31) / 32;
  prm.pair_axis = pair_axis_of(p);
  const int nd[3] = {p->nT, p->nH, p->nW};
  for (int a = 0; a < 3; ++a) prm.pdim[a] = a == prm.pair_axis ? (nd[a] + 1) / 2 : nd[a];
  return p->desc.head_dim == 128 ? run_dkdv<128>(p, q, k, v, d_o, prm, st)
                                 : run_dkdv<64>(p, q, k, v, d_o, prm, st);
}
