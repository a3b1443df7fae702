// Coarse block scores S = scale * Pq Pk^T per (batch, head), fp32.
//
// Each output is one fp32 dot product of length D accumulated with FMA in
// order d = 0..D-1, then multiplied by the softmax scale. A CTA computes a
// 64 x 64 (small N) or 128 x 128 block of S from smem-staged 32-wide slices
// of Pq and Pk; each thread owns a 4 x 4 or 8 x 8 register block and stores
// rows as float4 when N % 4 == 0.
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

// Large rows: 128 x 128 output blocks, 8 x 8 per thread as two 4 x 4
// quadrants 64 apart (conflict-free float4 shared loads), same per-output
// accumulation order d = 0..D-1.
constexpr int BT2 = 128;

__global__ void __launch_bounds__(256, 2)
block_scores_128_kernel(int N, int D, const float* __restrict__ pq, const float* __restrict__ pk,
                        float scale, float* __restrict__ S) {
  __shared__ __align__(16) float As[BK][BT2 + 4];
  __shared__ __align__(16) float Bs[BK][BT2 + 4];
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * BT2, j0 = blockIdx.x * BT2;
  const float* A = pq + (size_t)bh * N * D;
  const float* Bm = pk + (size_t)bh * N * D;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[8][8] = {};
  for (int k0 = 0; k0 < D; k0 += BK) {
    // 128 rows x 32 d per operand: four float4 per thread, transposed into smem.
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int lin = threadIdx.x + 256 * e;  // 0..1023: row lin / 8, d chunk lin % 8
      const int r = lin >> 3, d4 = (lin & 7) * 4;
      const float4 a = (i0 + r < N) ? *reinterpret_cast<const float4*>(A + (size_t)(i0 + r) * D + k0 + d4)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 b = (j0 + r < N) ? *reinterpret_cast<const float4*>(Bm + (size_t)(j0 + r) * D + k0 + d4)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
      As[d4][r] = a.x; As[d4 + 1][r] = a.y; As[d4 + 2][r] = a.z; As[d4 + 3][r] = a.w;
      Bs[d4][r] = b.x; Bs[d4 + 1][r] = b.y; Bs[d4 + 2][r] = b.z; Bs[d4 + 3][r] = b.w;
    }
    __syncthreads();
#pragma unroll 4
    for (int d = 0; d < BK; ++d) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[d][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[d][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[d][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[d][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int y = 0; y < 8; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
    __syncthreads();
  }
  float* out = S + (size_t)bh * N * N;
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    const int i = i0 + (x < 4 ? ty * 4 + x : 64 + ty * 4 + x - 4);
    if (i >= N) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = j0 + h * 64 + tx * 4;
      const float4 v = make_float4(acc[x][4 * h] * scale, acc[x][4 * h + 1] * scale, acc[x][4 * h + 2] * scale,
                                   acc[x][4 * h + 3] * scale);
      if ((N & 3) == 0 && j + 3 < N) {
        *reinterpret_cast<float4*>(out + (size_t)i * N + j) = v;
      } else {
        const float vv[4] = {v.x, v.y, v.z, v.w};
        for (int y = 0; y < 4; ++y)
          if (j + y < N) out[(size_t)i * N + j + y] = vv[y];
      }
    }
  }
}

}  // namespace

bsattn_status launch_block_scores(const Geom& g, const float* pq, const float* pk, float scale,
                                  float* S, cudaStream_t st) {
  // 128-wide blocks once they fill the GPU (about 4 per SM), 64-wide below.
  const long long blocks128 = (long long)((g.N + BT2 - 1) / BT2) * ((g.N + BT2 - 1) / BT2) * g.B * g.Hh;
  if (blocks128 >= 4 * 148) {
    dim3 grid((g.N + BT2 - 1) / BT2, (g.N + BT2 - 1) / BT2, g.B * g.Hh);
    block_scores_128_kernel<<<grid, 256, 0, st>>>(g.N, g.D, pq, pk, scale, S);
  } else {
    dim3 grid((g.N + BT - 1) / BT, (g.N + BT - 1) / BT, g.B * g.Hh);
    block_scores_kernel<<<grid, 256, 0, st>>>(g.N, g.D, pq, pk, scale, S);
  }
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}
