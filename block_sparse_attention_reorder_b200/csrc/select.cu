// Key-tile selection on a block-score matrix: exact top-k, top-p with a
// top-k floor, and the broadcast of the fixed window lists.
//
// Ordering: a score maps to a 32-bit unsigned key that orders like the
// float (-0.0 is folded into +0.0 first, so they tie); ties are broken by
// the lower tile index. Lists are written ascending.
#include "internal.h"

namespace {

__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;  // -0.0 ties with +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

// ---------------------------------------------------------------------------
// Top-k: one warp per row, the row's keys in registers (lane l holds columns
// l, l+32, ...). The k-th largest key v is found by a bitwise search from the
// most significant bit (count of keys >= candidate, warp-reduced). Keys > v
// are kept, and of the keys == v the lowest-index (k - #{> v}) ones.
// ---------------------------------------------------------------------------
template <int VPT>
__global__ void __launch_bounds__(256)
topk_kernel(int rows, int N, int k, const float* __restrict__ S, int32_t* __restrict__ idx,
            int32_t* __restrict__ cnt, int kmax) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* s = S + (size_t)row * N;
  uint32_t key[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    int j = lane + 32 * i;
    key[i] = j < N ? order_key(__ldg(s + j)) : 0u;  // 0 is below every real key
  }
  uint32_t v = 0;
  for (int bit = 31; bit >= 0; --bit) {
    uint32_t c = v | (1u << bit);
    uint32_t n = 0;
#pragma unroll
    for (int i = 0; i < VPT; ++i) n += key[i] >= c;
    if (__reduce_add_sync(0xffffffffu, n) >= (uint32_t)k) v = c;
  }
  uint32_t gt = 0;
#pragma unroll
  for (int i = 0; i < VPT; ++i) gt += key[i] > v;
  const int need_eq = k - (int)__reduce_add_sync(0xffffffffu, gt);
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base = 0, eq_seen = 0;
  int32_t* out = idx + (size_t)row * kmax;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    int j = lane + 32 * i;
    bool eq = (j < N) && key[i] == v;
    uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    bool keep = key[i] > v || (eq && eq_seen + __popc(eqm & lt_mask) < need_eq);
    eq_seen += __popc(eqm);
    uint32_t km = __ballot_sync(0xffffffffu, keep);
    if (keep) out[base + __popc(km & lt_mask)] = j;
    base += __popc(km);
  }
  if (lane == 0) cnt[row] = base;
}

// ---------------------------------------------------------------------------
// Top-p with a top-k floor: one CTA per row. The row's 64-bit keys
// (order key << 32 | ~index) are bitonic-sorted descending in shared memory,
// which orders by (score desc, index asc). Then, in fp64: pi_m =
// exp(s_m - s_max) / sum, inclusive prefix sums c_m, m* = first m with
// c_m >= p, kept = min(N, max(m*, k)). The kept indices are flagged and
// compacted in ascending order.
// ---------------------------------------------------------------------------
constexpr int kTopPThreads = 256;

__device__ __forceinline__ double block_sum_f64(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < kTopPThreads / 32; ++w) t += red[w];
  __syncthreads();
  return t;
}

// Exclusive prefix over threads of a per-thread value (fp64 or int), in
// thread order; also returns the total.
template <typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T* red, T* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  T x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[w] = x;
  __syncthreads();
  T off = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kTopPThreads / 32; ++i) {
    if (i < w) off += red[i];
    tot += red[i];
  }
  __syncthreads();
  *total = tot;
  return off + x - v;
}

template <int NP>
__global__ void __launch_bounds__(kTopPThreads)
topp_kernel(int N, int k, double p, const float* __restrict__ S, int32_t* __restrict__ idx,
            int32_t* __restrict__ cnt, int kmax) {
  constexpr int PER = NP / kTopPThreads > 0 ? NP / kTopPThreads : 1;
  __shared__ unsigned long long keys[NP];
  __shared__ unsigned char flag[NP];
  __shared__ double redd[kTopPThreads / 32];
  __shared__ int redi[kTopPThreads / 32];
  __shared__ int mstar_s;
  const size_t row = blockIdx.x;
  const float* s = S + row * N;
  for (int j = threadIdx.x; j < NP; j += kTopPThreads) {
    keys[j] = j < N ? ((unsigned long long)order_key(__ldg(s + j)) << 32) |
                          (unsigned long long)(0xffffffffu - (uint32_t)j)
                    : 0ull;
    flag[j] = 0;
  }
  if (threadIdx.x == 0) mstar_s = N;
  __syncthreads();
  // Bitonic sort, descending.
  for (int size = 2; size <= NP; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < NP / 2; t += kTopPThreads) {
        int a = 2 * t - (t & (stride - 1));
        int b = a + stride;
        bool desc = (a & size) == 0;
        unsigned long long x = keys[a], y = keys[b];
        if (desc ? (x < y) : (x > y)) {
          keys[a] = y;
          keys[b] = x;
        }
      }
      __syncthreads();
    }
  }
  const double smax = (double)key_to_float((uint32_t)(keys[0] >> 32));
  // Thread t owns sorted positions [t*PER, (t+1)*PER).
  double e[PER];
  double local = 0.0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    int m = threadIdx.x * PER + i;
    e[i] = m < N ? exp((double)key_to_float((uint32_t)(keys[m] >> 32)) - smax) : 0.0;
    local += e[i];
  }
  // Total mass: sum of the per-thread sums (fixed order), then pi = e / total.
  const double total = block_sum_f64(local, redd);
  double run = 0.0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    e[i] = e[i] / total;
    run += e[i];
  }
  double all;
  double c = block_exclusive_scan<double>(run, redd, &all);
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    int m = threadIdx.x * PER + i;
    c += e[i];
    if (m < N && c >= p) {
      atomicMin(&mstar_s, m + 1);
      break;
    }
  }
  __syncthreads();
  int kept = max(mstar_s, k);
  kept = min(kept, N);
  for (int m = threadIdx.x; m < kept; m += kTopPThreads)
    flag[0xffffffffu - (uint32_t)(keys[m] & 0xffffffffull)] = 1;
  __syncthreads();
  // Ascending compaction: thread t owns indices [t*PER, (t+1)*PER).
  int mine = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) mine += flag[threadIdx.x * PER + i];
  int tot;
  int pos = block_exclusive_scan<int>(mine, redi, &tot);
  int32_t* out = idx + row * kmax;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    int j = threadIdx.x * PER + i;
    if (flag[j]) out[pos++] = j;
  }
  if (threadIdx.x == 0) cnt[row] = kept;
}

__global__ void broadcast_lists_kernel(int N, int kmax, const int32_t* __restrict__ src_idx,
                                       const int32_t* __restrict__ src_cnt, int32_t* __restrict__ idx,
                                       int32_t* __restrict__ cnt) {
  const size_t bh = blockIdx.y;
  const int per = N * kmax;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < per; e += gridDim.x * blockDim.x)
    idx[bh * per + e] = src_idx[e];
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < N; e += gridDim.x * blockDim.x)
    cnt[bh * N + e] = src_cnt[e];
}

template <int VPT>
bsattn_status run_topk(int rows, int N, int k, const float* S, int32_t* idx, int32_t* cnt,
                       int kmax, cudaStream_t st) {
  topk_kernel<VPT><<<(rows + 7) / 8, 256, 0, st>>>(rows, N, k, S, idx, cnt, kmax);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

template <int NP>
bsattn_status run_topp(int rows, int N, int k, double p, const float* S, int32_t* idx,
                       int32_t* cnt, int kmax, cudaStream_t st) {
  topp_kernel<NP><<<rows, kTopPThreads, 0, st>>>(N, k, p, S, idx, cnt, kmax);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

}  // namespace

bsattn_status launch_select_topk(int rows, int N, int k, const float* S, int32_t* idx,
                                 int32_t* cnt, int kmax, cudaStream_t st) {
  int vpt = (N + 31) / 32;
  if (vpt <= 1) return run_topk<1>(rows, N, k, S, idx, cnt, kmax, st);
  if (vpt <= 2) return run_topk<2>(rows, N, k, S, idx, cnt, kmax, st);
  if (vpt <= 4) return run_topk<4>(rows, N, k, S, idx, cnt, kmax, st);
  if (vpt <= 8) return run_topk<8>(rows, N, k, S, idx, cnt, kmax, st);
  if (vpt <= 16) return run_topk<16>(rows, N, k, S, idx, cnt, kmax, st);
  if (vpt <= 32) return run_topk<32>(rows, N, k, S, idx, cnt, kmax, st);
  if (vpt <= 48) return run_topk<48>(rows, N, k, S, idx, cnt, kmax, st);
  if (vpt <= 64) return run_topk<64>(rows, N, k, S, idx, cnt, kmax, st);
  return BSATTN_ERR_UNSUPPORTED;
}

bsattn_status launch_select_topp(int rows, int N, int k, double p, const float* S, int32_t* idx,
                                 int32_t* cnt, int kmax, cudaStream_t st) {
  if (N <= 256) return run_topp<256>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (N <= 512) return run_topp<512>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (N <= 1024) return run_topp<1024>(rows, N, k, p, S, idx, cnt, kmax, st);
  if (N <= 2048) return run_topp<2048>(rows, N, k, p, S, idx, cnt, kmax, st);
  return BSATTN_ERR_UNSUPPORTED;
}

bsattn_status launch_broadcast_lists(int bh, int N, int kmax, const int32_t* src_idx,
                                     const int32_t* src_cnt, int32_t* idx, int32_t* cnt,
                                     cudaStream_t st) {
  int per = N * kmax;
  dim3 grid((per + 255) / 256 < 64 ? (per + 255) / 256 : 64, bh);
  broadcast_lists_kernel<<<grid, 256, 0, st>>>(N, kmax, src_idx, src_cnt, idx, cnt);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}
