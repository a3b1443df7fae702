// Coarse block scores S = scale * Pq Pk^T per (batch, head) on the tensor
// cores: tcgen05.mma kind::tf32 with three products per term. Each pooled
// fp32 value is split as x = hi + lo, hi keeping sign, exponent and the top
// 10 mantissa bits (exact in TF32) and lo = x - hi (exact in fp32); S
// accumulates hi*hi + hi*lo + lo*hi in fp32 in TMEM. What is left out (lo*lo
// and the TF32 rounding of lo) stays below 2^-20 of |a||b| per product.
//
// The output is cut into 128 x 128 blocks; a persistent CTA (one per SM)
// takes a contiguous run of blocks, so that consecutive blocks share their
// query rows (bh, bi). Roles:
//   warp 8    TMA: the Pq block (all of D) into a staging buffer when the row
//             block changes, and Pk row slices of 32 columns (128 rows x 128
//             bytes, 128-byte swizzle) into a ring;
//   warps 4-7 split: the Pq block goes to TMEM as hi and lo columns (TMEM
//             lane = row; the MMAs take A from TMEM, so it costs no shared
//             memory bandwidth per block), each Pk slice is split in place
//             into hi and a lo copy;
//   warp 9    one thread issues the twelve MMAs per slice into one of two TMEM
//             accumulators;
//   warps 0-3 read a finished accumulator with tcgen05.ld (lane = output row),
//             scale it, transpose 32 x 32 pieces through shared memory and
//             store whole 128-byte row segments, while the next block runs.
// Every block is accumulated in the same order (slices ascending, then the
// 8-wide K steps, hi*hi, hi*lo, lo*hi), so the result does not depend on how
// blocks are shared among CTAs.
//
// Fused score + top-k (FUSED): S is never written. A CTA takes whole 128-row
// blocks of S and computes every block of the row three times, with the same
// products in the same order as above (so every score is bit-identical to
// the materialised S); the epilogue threads (thread = row) select on the
// fly: pass 0 the row's exact min and max, pass 1 a 128-bin histogram over
// that range, pass 2 a bit mask of the tiles above the bin where the count
// from the top reaches k and the tiles of that bin as 64-bit keys, ranked
// exactly at the end; their bits join the mask, written out ascending. A
// row whose boundary bin holds more than 32 tiles (runs of equal scores, a
// constant or non-finite row) writes its S row in pass 2 instead and is
// handed, through a row list, to the row-wise top-k kernel.
#include "internal.h"
#include "tc_common.cuh"

namespace {

constexpr int kRows = 128;                       // output block edge (M = N = 128)
constexpr int kSlice = 32;                       // fp32 columns of D per slice (128 bytes)
constexpr int kSliceBytes = kRows * kSlice * 4;  // 16 KB per operand slice
constexpr int kThreads = 320;
constexpr int kSplitThreads = 128;
constexpr int kEpiBytes = 32 * 128;              // one warp's 32 x 32 transpose buffer
constexpr long long kWaitLimit = 4000000000LL;   // SM cycles (~2 s)

constexpr int kFusedPasses = 3;                  // min/max, histogram, collect
constexpr int kFusedBins = 128;
constexpr int kFusedCand = 32;                   // boundary-bin tiles ranked in the kernel
// Per-row state words (one row per epilogue thread): the 128 16-bit bin
// counts of pass 1, then the 64 kept-tile mask words of pass 2 (N <= 2048),
// plus one word of padding so that the rows fall on different banks.
constexpr int kStateWords = 65;

template <int D, bool FUSED>
struct ScoresCfg {
  static constexpr int STAGES = FUSED ? 3 : 4;            // Pk slice ring
  static constexpr int KS = D / kSlice;                   // slices per block
  static constexpr int OFF_ASTG = 0;                      // Pq block staging, KS slices
  static constexpr int OFF_RING = KS * kSliceBytes;       // stage s: Pk hi, then Pk lo
  static constexpr int STAGE = 2 * kSliceBytes;
  static constexpr int OFF_EPI = OFF_RING + STAGES * STAGE;
  // Epilogue: the transpose buffers, or (fused) per-row state words and the
  // boundary-bin keys [slot][row].
  static constexpr int EPI_BYTES = FUSED ? kRows * kStateWords * 4 + kFusedCand * kRows * 8 : 4 * kEpiBytes;
  static constexpr int OFF_BAR = OFF_EPI + EPI_BYTES;
  // a_full, a_stage_free, a_split, a_free, b_full[S], b_split[S], b_empty[S], acc_full[2],
  // acc_empty[2], final
  static constexpr int NBAR = 4 + 3 * STAGES + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;     // TMEM base, abort flag, a word that stays 0
  static constexpr int SMEM = OFF_MISC + 16 + 1024;       // + alignment slack
  // TMEM columns: Pq hi [0, D), Pq lo [D, 2D), accumulators at 2D and 2D + 128.
  static constexpr uint32_t COL_LO = D, COL_ACC = 2 * D;
  static_assert(SMEM <= 232448, "block scores shared memory");
  static_assert(2 * D + 2 * kRows <= 512, "TMEM columns");
};

struct ScoresParams {
  int N;              // tiles per (batch, head)
  int nb;             // 128-row blocks per (batch, head)
  long long blocks;   // B * Hh * nb * nb
  float scale;
  float* S;           // fused: rows handed to the fallback (every row when debug_s)
  int* err;
  // fused top-k only
  long long rblocks;  // B * Hh * nb row blocks
  int k, kmax;
  int32_t* idx;
  int32_t* cnt;
  int debug_s;        // 1: every row's S is written as well
  int32_t* fb_rows;   // rows for the row-wise fallback, *fb_count of them
  int* fb_count;
};

__device__ __forceinline__ uint32_t fused_order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;  // -0.0 ties with +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// D[tmem] (+)= A[tmem] * B[smem desc], TF32 operands.
__device__ __forceinline__ void mma_ts_tf32(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                            uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ uint32_t hi_bits(uint32_t x) { return x & 0xFFFFE000u; }

// Split one Pk slice in place: hi over the loaded values, lo = x - hi into
// the slice after it. Thread t takes 16-byte pieces t, t + 128, ...
__device__ __forceinline__ void split_slice(uint8_t* hi, int t) {
  float4 x[kSliceBytes / 16 / kSplitThreads];
#pragma unroll
  for (int u = 0; u < kSliceBytes / 16 / kSplitThreads; ++u)
    x[u] = reinterpret_cast<const float4*>(hi)[t + u * kSplitThreads];
#pragma unroll
  for (int u = 0; u < kSliceBytes / 16 / kSplitThreads; ++u) {
    const float4 h = make_float4(__uint_as_float(hi_bits(__float_as_uint(x[u].x))),
                                 __uint_as_float(hi_bits(__float_as_uint(x[u].y))),
                                 __uint_as_float(hi_bits(__float_as_uint(x[u].z))),
                                 __uint_as_float(hi_bits(__float_as_uint(x[u].w))));
    reinterpret_cast<float4*>(hi)[t + u * kSplitThreads] = h;
    reinterpret_cast<float4*>(hi + kSliceBytes)[t + u * kSplitThreads] =
        make_float4(x[u].x - h.x, x[u].y - h.y, x[u].z - h.z, x[u].w - h.w);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int D, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
block_scores_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       ScoresParams P) {
  using C = ScoresCfg<D, FUSED>;
  constexpr int kStages = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = tc::smem_addr(smem);
  const uint32_t bar_afull = sb + C::OFF_BAR, bar_astg = bar_afull + 8, bar_asplit = bar_afull + 16,
                 bar_afree = bar_afull + 24;
  auto bar_bfull = [&](int s) { return sb + C::OFF_BAR + 8u * (4 + s); };
  auto bar_bsplit = [&](int s) { return sb + C::OFF_BAR + 8u * (4 + kStages + s); };
  auto bar_bempty = [&](int s) { return sb + C::OFF_BAR + 8u * (4 + 2 * kStages + s); };
  auto bar_accfull = [&](int a) { return sb + C::OFF_BAR + 8u * (4 + 3 * kStages + a); };
  auto bar_accempty = [&](int a) { return sb + C::OFF_BAR + 8u * (6 + 3 * kStages + a); };
  const uint32_t bar_final = sb + C::OFF_BAR + 8u * (8 + 3 * kStages);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* never = reinterpret_cast<volatile int*>(misc + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // This CTA's contiguous run of blocks; block = ((bh * nb) + bi) * PN + pass * nb + bj
  // (fused: whole row blocks, each computed in kFusedPasses passes; else one pass).
  const int nb = P.nb;
  const int PN = (FUSED ? kFusedPasses : 1) * nb;
  const long long blk0 = FUSED ? P.rblocks * blockIdx.x / gridDim.x * PN : P.blocks * blockIdx.x / gridDim.x;
  const long long blk1 =
      FUSED ? P.rblocks * (blockIdx.x + 1) / gridDim.x * PN : P.blocks * (blockIdx.x + 1) / gridDim.x;

  if (tid == 0) {
    tc::mbar_init(bar_afull, 1);
    tc::mbar_init(bar_astg, kSplitThreads);
    tc::mbar_init(bar_asplit, kSplitThreads);
    tc::mbar_init(bar_afree, 1);
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(bar_bfull(s), 1);
      tc::mbar_init(bar_bsplit(s), kSplitThreads);
      tc::mbar_init(bar_bempty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(bar_accfull(a), 1);
      tc::mbar_init(bar_accempty(a), 128);
    }
    tc::mbar_init(bar_final, 1);
    misc[1] = 0;
    misc[2] = 0;
    tc::mbar_fence_init();
  }
  if (warp == 9) {
    tc::tmem_alloc(sb + C::OFF_MISC, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = misc[0];

  if (warp == 8) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      tc::tma_prefetch_desc(&tmA);
      tc::tma_prefetch_desc(&tmB);
      long long m = 0, prev = -1, last_b[kStages];
      int arow = 0;
      for (int s = 0; s < kStages; ++s) last_b[s] = -1;
      bool ok = true;
      for (long long blk = blk0; ok && blk < blk1; ++blk) {
        const long long rk = blk / PN, bh = rk / nb;
        const int bi = (int)(rk % nb), bj = (int)(blk % nb);
        if (rk != prev) {
          // The split warps must have read the previous Pq block out of staging.
          if (arow > 0 && !tc::mbar_wait(bar_astg, (arow - 1) & 1, abort_flag, kWaitLimit)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(bar_afull, C::KS * kSliceBytes);
          for (int kc = 0; kc < C::KS; ++kc)
            tc::tma_load_2d(sb + C::OFF_ASTG + kc * kSliceBytes, &tmA, bar_afull, kc * kSlice,
                            (int)(bh * P.N + (long long)bi * kRows));
          ++arow;
          prev = rk;
        }
        for (int kc = 0; kc < C::KS; ++kc, ++m) {
          const int s = (int)(m % kStages);
          if (m >= kStages && !tc::mbar_wait(bar_bempty(s), (int)((m / kStages) - 1) & 1, abort_flag, kWaitLimit)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(bar_bfull(s), kSliceBytes);
          tc::tma_load_2d(sb + C::OFF_RING + s * C::STAGE, &tmB, bar_bfull(s), kc * kSlice,
                          (int)(bh * P.N + (long long)bj * kRows));
          last_b[s] = m;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
      }
      if (*abort_flag) {  // let this thread's copies land before the CTA goes away
        if (arow > 0) tc::mbar_wait(bar_afull, (arow - 1) & 1, never, kWaitLimit);
        for (int s = 0; s < kStages; ++s)
          if (last_b[s] >= 0) tc::mbar_wait(bar_bfull(s), (int)(last_b[s] / kStages) & 1, never, kWaitLimit);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      // TF32 inputs, fp32 accumulator, A (TMEM) and B K-major, M = N = 128.
      constexpr uint32_t idesc = tc::instr_desc(2, 2, 0, 0, kRows, kRows);
      long long m = 0, prev = -1;
      int arow = 0, t = 0;
      bool ok = true;
      for (long long blk = blk0; ok && blk < blk1; ++blk, ++t) {
        const long long rk = blk / PN;
        if (rk != prev) {
          if (!tc::mbar_wait(bar_asplit, arow & 1, abort_flag, kWaitLimit)) {
            ok = false;
            break;
          }
          ++arow;
          prev = rk;
        }
        const int a = t & 1;
        if (t >= 2 && !tc::mbar_wait(bar_accempty(a), ((t >> 1) - 1) & 1, abort_flag, kWaitLimit)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t d = tmem + C::COL_ACC + (uint32_t)(a * kRows);
        for (int kc = 0; kc < C::KS; ++kc, ++m) {
          const int s = (int)(m % kStages);
          if (!tc::mbar_wait(bar_bsplit(s), (int)(m / kStages) & 1, abort_flag, kWaitLimit)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t stg = sb + C::OFF_RING + s * C::STAGE;
#pragma unroll
          for (int kk = 0; kk < kSlice / 8; ++kk) {  // 8 fp32 of K per MMA
            const uint32_t ah = tmem + (uint32_t)(kc * kSlice + kk * 8), al = ah + C::COL_LO;
            const uint64_t bhi = tc::smem_desc(stg + kk * 32, 16, 1024, tc::kLayoutSW128);
            const uint64_t blo = tc::smem_desc(stg + kSliceBytes + kk * 32, 16, 1024, tc::kLayoutSW128);
            mma_ts_tf32(d, ah, bhi, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
            mma_ts_tf32(d, ah, blo, idesc, 1u);
            mma_ts_tf32(d, al, bhi, idesc, 1u);
          }
          tc::mma_commit(bar_bempty(s));
        }
        if (!ok) break;
        tc::mma_commit(bar_accfull(a));
        // Pq columns of TMEM are rewritten for the next row block only after
        // this one's MMAs are done.
        if (blk + 1 < blk1 && (blk + 1) / PN != rk) tc::mma_commit(bar_afree);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
      }
      tc::mma_commit(bar_final);  // drain every issued MMA before TMEM and shared memory go away
      tc::mbar_wait(bar_final, 0, never, kWaitLimit);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ split
    const int t = tid - 128, r = t;  // thread t owns row r of the Pq block (TMEM lane r)
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    long long m = 0, prev = -1;
    int arow = 0;
    bool ok = true;
    for (long long blk = blk0; ok && blk < blk1; ++blk) {
      const long long rk = blk / PN;
      if (rk != prev) {
        if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_afull, arow & 1, abort_flag, kWaitLimit)) ||
            (arow > 0 && !__all_sync(0xffffffffu, tc::mbar_wait(bar_afree, (arow - 1) & 1, abort_flag, kWaitLimit)))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
#pragma unroll 1
        for (int kc = 0; kc < C::KS; ++kc) {
          // Row r of a 128-byte-swizzled slice: 16-byte piece c sits at c ^ (r & 7).
          const uint8_t* row = smem + C::OFF_ASTG + kc * kSliceBytes + r * 128;
          uint32_t h[32], l[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 x = *reinterpret_cast<const float4*>(row + ((c ^ (r & 7)) << 4));
            const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t hb = hi_bits(__float_as_uint(xv[e]));
              h[4 * c + e] = hb;
              l[4 * c + e] = __float_as_uint(xv[e] - __uint_as_float(hb));
            }
          }
          tc::tmem_st32(tmem + lane_base + (uint32_t)(kc * kSlice), h);
          tc::tmem_st32(tmem + lane_base + C::COL_LO + (uint32_t)(kc * kSlice), l);
        }
        tc::tmem_wait_st();
        tc::mbar_arrive(bar_astg);
        tc::fence_before_sync();
        tc::mbar_arrive(bar_asplit);
        ++arow;
        prev = rk;
      }
      for (int kc = 0; kc < C::KS; ++kc, ++m) {
        const int s = (int)(m % kStages);
        if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_bfull(s), (int)(m / kStages) & 1, abort_flag, kWaitLimit))) {
          ok = false;
          break;
        }
        split_slice(smem + C::OFF_RING + s * C::STAGE, t);
        tc::mbar_arrive(bar_bsplit(s));
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
    }
  } else if constexpr (FUSED) {
    // ------------------------------------------------------------ fused top-k epilogue
    // Thread r owns row r of the current 128-row block (TMEM lane r).
    const int r = tid;
    // This row's state: bin counts in pass 1, then its kept-tile mask (one
    // bit per tile, ascending) in pass 2; only this thread touches it.
    uint32_t* rowstate = reinterpret_cast<uint32_t*>(smem + C::OFF_EPI) + r * kStateWords;
    uint16_t* hist = reinterpret_cast<uint16_t*>(rowstate);
    uint32_t* bmask = rowstate;
    uint64_t* cand = reinterpret_cast<uint64_t*>(smem + C::OFF_EPI + kRows * kStateWords * 4);  // [slot][row]
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: bin index in the low mantissa bits
    const float qnan = __int_as_float(0x7fc00000);
    const int rr = min(P.k, P.N);
    float mn = qnan, mx = qnan, sc = 0.f, offm = kMagic;
    int bstar = -1, need = 0, ncand = 0;
    bool crowded = false;
    // Equal-width bins over [mn, mx], monotone in the score (one FMA; NaN and
    // a range that overflows land in bin 0).
    auto bin_of = [&](float x) -> int {
      const float u = fminf(fmaxf(fmaf(x, sc, offm), kMagic), kMagic + (float)(kFusedBins - 1));
      return __float_as_int(u) - __float_as_int(kMagic);
    };
    int t = 0;
    bool ok = true;
    for (long long blk = blk0; blk < blk1; ++blk, ++t) {
      const int a = t & 1;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_accfull(a), (t >> 1) & 1, abort_flag, kWaitLimit))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const long long rk = blk / PN, bh = rk / nb;
      const int pass = (int)((blk / nb) % kFusedPasses), bj = (int)(blk % nb);
      const int i = (int)(rk % nb) * kRows + r;  // this thread's row within its (batch, head)
      const bool row_ok = i < P.N;
      const size_t grow = (size_t)bh * P.N + i;  // row of the whole score matrix
      if (bj == 0 && pass == 0) {
        mn = mx = qnan;
        crowded = false;
      }
      if (bj == 0 && pass == 1) {
        // A constant or non-finite row has no range to bin: fallback.
        crowded = !(mn < mx) || !(mx - mn <= 3.0e38f);
        sc = crowded ? 0.f : (float)kFusedBins / (mx - mn);
        if (!(sc <= 3.0e38f)) crowded = true;
        if (crowded) sc = 0.f;
        offm = crowded ? kMagic : fmaf(-mn, sc, kMagic);
        for (int q = 0; q < kFusedBins / 2; ++q) rowstate[q] = 0u;
      }
      if (bj == 0 && pass == 2) {
        // The bin in which the count, taken from the top bin down, reaches rr.
        int run = 0;
        bstar = -1;
        for (int q = kFusedBins - 1; q >= 0; --q) {
          const int c = hist[q];
          if (run + c >= rr) {
            bstar = q;
            need = rr - run;
            crowded = crowded || c > kFusedCand;
            break;
          }
          run += c;
        }
        if (bstar < 0) crowded = true;
        ncand = 0;
      }
      int32_t* out = P.idx + grow * P.kmax;
      float* srow = P.S + grow * P.N;
      // One straight-line loop per pass over 32 columns at a time (the
      // columns past N are masked, not branched out of).
#pragma unroll 1
      for (int c0 = 0; c0 < kRows; c0 += 32) {
        uint32_t v[32];
        tc::tmem_ld32_wait(tmem + lane_base + C::COL_ACC + (uint32_t)(a * kRows + c0), v);
        const int j0 = bj * kRows + c0;
        const int jn = row_ok ? min(32, P.N - j0) : 0;  // valid columns of this piece
        if (pass == 0) {
          float lo = mn, hi = mx;
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const float x = q < jn ? __uint_as_float(v[q]) * P.scale : qnan;
            lo = fminf(lo, x);
            hi = fmaxf(hi, x);
          }
          mn = lo;
          mx = hi;
        } else if (pass == 1) {
          if (!crowded) {
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (q < jn) {
                // 16-bit counts, two to a word (at most 2,048 each): an atomic
                // add that returns nothing, so the thread does not wait for
                // its previous increment to land.
                const int bx = bin_of(__uint_as_float(v[q]) * P.scale);
                atomicAdd(rowstate + (bx >> 1), 1u << (16 * (bx & 1)));
              }
          }
        } else if (jn > 0) {
          if (crowded || P.debug_s) {
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (q < jn) srow[j0 + q] = __uint_as_float(v[q]) * P.scale;
          }
          if (!crowded) {
            // Tiles above the boundary bin as one 32-bit mask word per piece;
            // the boundary bin's tiles as keys.
            uint32_t above_bits = 0;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const float x = __uint_as_float(v[q]) * P.scale;
              const int bx = q < jn ? bin_of(x) : -1;
              above_bits |= (bx > bstar ? 1u : 0u) << q;
              if (bx == bstar) {
                if (ncand < kFusedCand)
                  cand[ncand * kRows + r] =
                      ((uint64_t)fused_order_key(x) << 32) | (uint64_t)(0xffffffffu - (uint32_t)(j0 + q));
                ++ncand;
              }
            }
            bmask[j0 >> 5] = above_bits;
          }
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(bar_accempty(a));
      if (pass == kFusedPasses - 1 && bj == nb - 1 && row_ok) {
        if (crowded) {
          P.fb_rows[atomicAdd(P.fb_count, 1)] = (int32_t)grow;
        } else {
          // The boundary bin's keys are unique; the `need` largest are kept:
          // their bits join the mask, which is then written out ascending.
          const int nc = min(ncand, kFusedCand);
          for (int x1 = 0; x1 < nc; ++x1) {
            const uint64_t kx = cand[x1 * kRows + r];
            int rank = 0;
            for (int x2 = 0; x2 < nc; ++x2) rank += cand[x2 * kRows + r] > kx ? 1 : 0;
            if (rank < need) {
              const uint32_t jj = 0xffffffffu - (uint32_t)kx;
              bmask[jj >> 5] |= 1u << (jj & 31);
            }
          }
          int total = 0;
          const int nwords = (P.N + 31) >> 5;
          for (int wd = 0; wd < nwords; ++wd) {
            uint32_t bits = bmask[wd];
            while (bits) {
              if (total < P.kmax) out[total] = wd * 32 + __ffs(bits) - 1;
              ++total;
              bits &= bits - 1;
            }
          }
          P.cnt[grow] = min(total, P.kmax);
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    uint8_t* epi = smem + C::OFF_EPI + warp * kEpiBytes;  // 32 rows x 128 bytes, swizzled
    int t = 0;
    bool ok = true;
    const bool vec = (P.N & 3) == 0;
    for (long long blk = blk0; blk < blk1; ++blk, ++t) {
      const int a = t & 1;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_accfull(a), (t >> 1) & 1, abort_flag, kWaitLimit))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const long long rk = blk / nb, bh = rk / nb;
      const int i0 = (int)(rk % nb) * kRows + warp * 32;  // first output row of this warp
      const int j0 = (int)(blk % nb) * kRows;
#pragma unroll 1
      for (int c = 0; c < kRows; c += 32) {
        uint32_t v[32];
        tc::tmem_ld32_wait(tmem + ((uint32_t)(warp * 32) << 16) + C::COL_ACC + (uint32_t)(a * kRows + c), v);
        // This lane's row, 32 columns, into the transpose buffer (piece q at q ^ (lane & 7)).
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<float4*>(epi + lane * 128 + ((q ^ (lane & 7)) << 4)) =
              make_float4(__uint_as_float(v[4 * q]) * P.scale, __uint_as_float(v[4 * q + 1]) * P.scale,
                          __uint_as_float(v[4 * q + 2]) * P.scale, __uint_as_float(v[4 * q + 3]) * P.scale);
        __syncwarp();
        // Four rows of 128 bytes per store instruction.
        const int q = lane & 7, j = j0 + c + 4 * q;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int rr = it * 4 + (lane >> 3), i = i0 + rr;
          const float4 x = *reinterpret_cast<const float4*>(epi + rr * 128 + ((q ^ (rr & 7)) << 4));
          if (i < P.N) {
            float* dst = P.S + ((size_t)bh * P.N + (size_t)i) * P.N + j;
            if (vec && j + 4 <= P.N) {
              *reinterpret_cast<float4*>(dst) = x;
            } else {
              if (j < P.N) dst[0] = x.x;
              if (j + 1 < P.N) dst[1] = x.y;
              if (j + 2 < P.N) dst[2] = x.z;
              if (j + 3 < P.N) dst[3] = x.w;
            }
          }
        }
        __syncwarp();
      }
      tc::fence_before_sync();
      tc::mbar_arrive(bar_accempty(a));
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(P.err, BSATTN_DEVERR_TIMEOUT);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// The fused top-k's outputs (FUSED kernels only).
struct FusedArgs {
  int k, kmax;
  int32_t* idx;
  int32_t* cnt;
  int debug_s;
  int32_t* fb_rows;
  int* fb_count;
};

template <int D, bool FUSED>
bsattn_status run_scores(const Geom& g, const float* pq, const float* pk, float scale, float* S, int* err,
                         const FusedArgs* fa, cudaStream_t st) {
  using C = ScoresCfg<D, FUSED>;
  const uint64_t rows = (uint64_t)g.B * g.Hh * g.N;
  CUtensorMap ma, mb;
  if (!bsattn_make_map_2d(&ma, pq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, rows, kSlice, kRows,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bsattn_make_map_2d(&mb, pk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, rows, kSlice, kRows,
                          CU_TENSOR_MAP_SWIZZLE_128B))
    return BSATTN_ERR_CUDA;
  auto kern = block_scores_tc_kernel<D, FUSED>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
    return BSATTN_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return BSATTN_ERR_CUDA;
  ScoresParams prm{};
  prm.N = g.N;
  prm.nb = (g.N + kRows - 1) / kRows;
  prm.blocks = (long long)g.B * g.Hh * prm.nb * prm.nb;
  prm.rblocks = (long long)g.B * g.Hh * prm.nb;
  prm.scale = scale;
  prm.S = S;
  prm.err = err;
  if (FUSED) {
    prm.k = fa->k;
    prm.kmax = fa->kmax;
    prm.idx = fa->idx;
    prm.cnt = fa->cnt;
    prm.debug_s = fa->debug_s;
    prm.fb_rows = fa->fb_rows;
    prm.fb_count = fa->fb_count;
  }
  const long long units = FUSED ? prm.rblocks : prm.blocks;  // fused CTAs take whole row blocks
  const int grid = (int)(units < sms ? units : sms);
  kern<<<grid, kThreads, C::SMEM, st>>>(ma, mb, prm);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

}  // namespace

bsattn_status launch_block_scores(const Geom& g, const float* pq, const float* pk, float scale,
                                  float* S, int* err, cudaStream_t st) {
  // Row coordinates of the tensor maps (B * Hh * N rows, plus a block) stay in int32.
  if ((uint64_t)g.B * g.Hh * g.N + kRows >= (1ull << 31)) return BSATTN_ERR_UNSUPPORTED;
  if (g.B <= 0 || g.Hh <= 0 || g.N <= 0) return BSATTN_OK;
  return g.D == 128 ? run_scores<128, false>(g, pq, pk, scale, S, err, nullptr, st)
                    : run_scores<64, false>(g, pq, pk, scale, S, err, nullptr, st);
}

bsattn_status launch_fused_topk(const Geom& g, const float* pq, const float* pk, float scale, int k, int kmax,
                                int32_t* idx, int32_t* cnt, float* S, bool debug_s, int32_t* fb_rows, int* fb_count,
                                int* err, cudaStream_t st) {
  if ((uint64_t)g.B * g.Hh * g.N + kRows >= (1ull << 31)) return BSATTN_ERR_UNSUPPORTED;
  if (g.B <= 0 || g.Hh <= 0 || g.N <= 0) return BSATTN_OK;
  if (cudaMemsetAsync(fb_count, 0, sizeof(int), st) != cudaSuccess) return BSATTN_ERR_CUDA;
  const FusedArgs fa{k, kmax, idx, cnt, debug_s ? 1 : 0, fb_rows, fb_count};
  bsattn_status s = g.D == 128 ? run_scores<128, true>(g, pq, pk, scale, S, err, &fa, st)
                               : run_scores<64, true>(g, pq, pk, scale, S, err, &fa, st);
  if (s != BSATTN_OK) return s;
  // Rows the kernel could not settle: the row-wise top-k over their S rows.
  return launch_select_topk_rows((int)((uint64_t)g.B * g.Hh * g.N), g.N, k, S, idx, cnt, kmax, fb_rows, fb_count, st);
}
