// Coarse block scores S = scale * Pq Pk^T per (batch, head) on the tensor
// cores: tcgen05.mma kind::tf32 with three products per term. Each pooled
// fp32 value is split as x = hi + lo, hi keeping sign, exponent and the top
// 10 mantissa bits (exact in TF32) and lo = x - hi (exact in fp32); S
// accumulates hi*hi + hi*lo + lo*hi in fp32 in TMEM. What is left out (lo*lo
// and the TF32 rounding of lo) stays below 2^-20 of |a||b| per product.
//
// One CTA computes a 128 x 128 block of S: for each 32-column slice of D, TMA
// brings the Pq and Pk row slices (128 rows x 128 bytes, 128-byte swizzle)
// into shared memory, the CTA splits them in place into hi and a lo copy (an
// element-wise pass keeps the swizzled layout), one thread issues the twelve
// MMAs, and at the end the accumulator is read back with tcgen05.ld, scaled
// and stored. Three CTAs per SM overlap one another's loads, splits and MMAs.
#include "internal.h"
#include "tc_common.cuh"

namespace {

constexpr int kRows = 128;                       // output block edge (M = N = 128)
constexpr int kSlice = 32;                       // fp32 columns of D per slice (128 bytes)
constexpr int kSliceBytes = kRows * kSlice * 4;  // 16 KB per operand slice
constexpr int OFF_AHI = 0, OFF_BHI = kSliceBytes, OFF_ALO = 2 * kSliceBytes, OFF_BLO = 3 * kSliceBytes;
constexpr int OFF_BAR = 4 * kSliceBytes;         // load barrier, MMA barrier
constexpr int OFF_TMEM = OFF_BAR + 16;           // TMEM base address, then a word that stays 0
constexpr int kSmem = OFF_TMEM + 16 + 1024;      // + alignment slack
constexpr long long kWaitLimit = 4000000000LL;   // SM cycles (~2 s)

__device__ __forceinline__ void mma_tf32(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(128)
block_scores_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int N,
                       float scale, float* __restrict__ S, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = tc::smem_addr(smem);
  const uint32_t bar_ld = sb + OFF_BAR, bar_mma = sb + OFF_BAR + 8;
  volatile int* never = reinterpret_cast<volatile int*>(smem + OFF_TMEM + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.z, i0 = blockIdx.y * kRows, j0 = blockIdx.x * kRows;
  if (tid == 0) {
    tc::mbar_init(bar_ld, 1);
    tc::mbar_init(bar_mma, 1);
    *never = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(sb + OFF_TMEM, kRows);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM);
  // TF32 inputs, fp32 accumulator, both operands K-major, M = N = 128.
  constexpr uint32_t idesc = tc::instr_desc(2, 2, 0, 0, kRows, kRows);
  bool ok = true;
  int ld_pending = -1, mma_pending = -1;  // phase of a wait that gave up
  for (int kc = 0; kc < D / kSlice; ++kc) {
    if (tid == 0) {
      tc::mbar_arrive_expect_tx(bar_ld, 2 * kSliceBytes);
      tc::tma_load_2d(sb + OFF_AHI, &tmA, bar_ld, kc * kSlice, bh * N + i0);
      tc::tma_load_2d(sb + OFF_BHI, &tmB, bar_ld, kc * kSlice, bh * N + j0);
    }
    if (!tc::mbar_wait(bar_ld, kc & 1, never, kWaitLimit)) ok = false;
    if (!__syncthreads_and(ok)) {
      ok = false;
      ld_pending = kc & 1;
      break;
    }
    // Split in place: hi keeps sign, exponent and the top 10 mantissa bits.
    for (int q = tid; q < 2 * kSliceBytes / 16; q += 128) {
      float4* hp = reinterpret_cast<float4*>(smem + OFF_AHI + q * 16);  // A slice, then B slice
      float4* lp = reinterpret_cast<float4*>(smem + OFF_ALO + q * 16);
      const float4 x = *hp;
      const float4 h = make_float4(__uint_as_float(__float_as_uint(x.x) & 0xFFFFE000u),
                                   __uint_as_float(__float_as_uint(x.y) & 0xFFFFE000u),
                                   __uint_as_float(__float_as_uint(x.z) & 0xFFFFE000u),
                                   __uint_as_float(__float_as_uint(x.w) & 0xFFFFE000u));
      *hp = h;
      *lp = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < kSlice / 8; ++kk) {  // 8 fp32 (32 bytes) of K per MMA
        const uint64_t ah = tc::smem_desc(sb + OFF_AHI + kk * 32, 16, 1024, tc::kLayoutSW128);
        const uint64_t bhi = tc::smem_desc(sb + OFF_BHI + kk * 32, 16, 1024, tc::kLayoutSW128);
        const uint64_t al = tc::smem_desc(sb + OFF_ALO + kk * 32, 16, 1024, tc::kLayoutSW128);
        const uint64_t bl = tc::smem_desc(sb + OFF_BLO + kk * 32, 16, 1024, tc::kLayoutSW128);
        mma_tf32(tmem, ah, bhi, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        mma_tf32(tmem, ah, bl, idesc, 1u);
        mma_tf32(tmem, al, bhi, idesc, 1u);
      }
      tc::mma_commit(bar_mma);
    }
    // The slice buffers are refilled only after the MMAs have read them.
    if (!tc::mbar_wait(bar_mma, kc & 1, never, kWaitLimit)) ok = false;
    tc::fence_after_sync();
    if (!__syncthreads_and(ok)) {
      ok = false;
      mma_pending = kc & 1;
      break;
    }
  }
  if (!ok) {
    // Let the copies and MMAs already issued finish (bounded) before the
    // shared memory and TMEM go away.
    if (tid == 0) {
      atomicOr(err, BSATTN_DEVERR_TIMEOUT);
      if (ld_pending >= 0) tc::mbar_wait(bar_ld, ld_pending, never, kWaitLimit);
      if (mma_pending >= 0) tc::mbar_wait(bar_mma, mma_pending, never, kWaitLimit);
    }
  } else {
    // Row i0 + 32 warp + lane of the block, 32 columns at a time.
    const int i = i0 + warp * 32 + lane;
    float* row = S + ((size_t)bh * N + i) * N;
    const bool vec = (N & 3) == 0;
#pragma unroll
    for (int c = 0; c < kRows; c += 32) {
      uint32_t v[32];
      tc::tmem_ld32_wait(tmem + ((uint32_t)(warp * 32) << 16) + c, v);
      if (i >= N) continue;
      const int j = j0 + c;
      if (vec && j + 32 <= N) {
#pragma unroll
        for (int q = 0; q < 32; q += 4)
          *reinterpret_cast<float4*>(row + j + q) =
              make_float4(__uint_as_float(v[q]) * scale, __uint_as_float(v[q + 1]) * scale,
                          __uint_as_float(v[q + 2]) * scale, __uint_as_float(v[q + 3]) * scale);
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (j + q < N) row[j + q] = __uint_as_float(v[q]) * scale;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kRows);
  }
}

template <int D>
bsattn_status run_scores(const Geom& g, const float* pq, const float* pk, float scale, float* S, int* err,
                         cudaStream_t st) {
  const uint64_t rows = (uint64_t)g.B * g.Hh * g.N;
  CUtensorMap ma, mb;
  if (!bsattn_make_map_2d(&ma, pq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, rows, kSlice, kRows,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bsattn_make_map_2d(&mb, pk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, rows, kSlice, kRows,
                          CU_TENSOR_MAP_SWIZZLE_128B))
    return BSATTN_ERR_CUDA;
  auto kern = block_scores_tc_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
    return BSATTN_ERR_CUDA;
  const int nb = (g.N + kRows - 1) / kRows;
  dim3 grid(nb, nb, g.B * g.Hh);
  kern<<<grid, 128, kSmem, st>>>(ma, mb, g.N, scale, S, err);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

}  // namespace

bsattn_status launch_block_scores(const Geom& g, const float* pq, const float* pk, float scale,
                                  float* S, int* err, cudaStream_t st) {
  // Row coordinates of the tensor maps (B * Hh * N rows, plus a block) stay in int32.
  if ((uint64_t)g.B * g.Hh * g.N + kRows >= (1ull << 31)) return BSATTN_ERR_UNSUPPORTED;
  return g.D == 128 ? run_scores<128>(g, pq, pk, scale, S, err, st)
                    : run_scores<64>(g, pq, pk, scale, S, err, st);
}
