// Coarse block scores S = scale * Pq Pk^T per (batch, head), fp32.
//
// Each output is one fp32 dot product of length D accumulated with FMA in
// order d = 0..D-1, then multiplied by the softmax scale. A CTA computes a
// 64 x 64 block of S from smem-staged 32-wide slices of Pq and Pk; each
// thread owns a 4 x 4 register block and stores rows as float4 when N % 4 == 0.
#include "internal.h"

namespace {

constexpr int BT = 64;   // output block edge
constexpr int BK = 32;   // d slice

__global__ void __launch_bounds__(256)
block_scores_kernel(int N, int D, const float* __restrict__ pq, const float* __restrict__ pk,
                    float scale, float* __restrict__ S) {
  __shared__ __align__(16) float As[BK][BT + 4];
  __shared__ __align__(16) float Bs[BK][BT + 4];
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * BT, j0 = blockIdx.x * BT;
  const float* A = pq + (size_t)bh * N * D;
  const float* Bm = pk + (size_t)bh * N * D;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < D; k0 += BK) {
    // 64 rows x 32 d per operand: 8 values per thread, transposed into smem.
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int lin = threadIdx.x + 256 * e;
      int r = lin / BK, d = lin % BK;
      As[d][r] = (i0 + r < N) ? A[(size_t)(i0 + r) * D + k0 + d] : 0.f;
      Bs[d][r] = (j0 + r < N) ? Bm[(size_t)(j0 + r) * D + k0 + d] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int d = 0; d < BK; ++d) {
      float4 a = *reinterpret_cast<const float4*>(&As[d][ty * 4]);
      float4 b = *reinterpret_cast<const float4*>(&Bs[d][tx * 4]);
      float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
    __syncthreads();
  }
  float* out = S + (size_t)bh * N * N;
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    int i = i0 + ty * 4 + x;
    if (i >= N) continue;
    int j = j0 + tx * 4;
    float4 v = make_float4(acc[x][0] * scale, acc[x][1] * scale, acc[x][2] * scale, acc[x][3] * scale);
    if ((N & 3) == 0 && j + 3 < N) {
      *reinterpret_cast<float4*>(out + (size_t)i * N + j) = v;
    } else {
      float vv[4] = {v.x, v.y, v.z, v.w};
      for (int y = 0; y < 4; ++y)
        if (j + y < N) out[(size_t)i * N + j + y] = vv[y];
    }
  }
}

}  // namespace

bsattn_status launch_block_scores(const Geom& g, const float* pq, const float* pk, float scale,
                                  float* S, cudaStream_t st) {
  dim3 grid((g.N + BT - 1) / BT, (g.N + BT - 1) / BT, g.B * g.Hh);
  block_scores_kernel<<<grid, 256, 0, st>>>(g.N, g.D, pq, pk, scale, S);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}
