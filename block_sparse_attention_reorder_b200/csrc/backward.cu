// Backward pass of block-sparse attention (the trainable block-sparse
// attention of "Faster Video Diffusion with Trainable Sparse Attention",
// reproducibility record, Research Type row: models are trained through it).
//
// With P the masked softmax of the forward pass (recomputed from Q, K and the
// forward's log-sum-exp), dO the incoming gradient and Delta = rowsum(dO * O):
//   dV_j += P_ij^T dO_i,  dP_ij = dO_i V_j^T,  dS_ij = P_ij * (dP_ij - Delta_i),
//   dK_j += scale dS_ij^T Q_i,  dQ_i += scale dS_ij K_j
// over the kept tile pairs (i, j). No atomics: this file computes Delta and
// transposes the kept lists (bitmaps, then ascending lists of the query tiles
// that keep each key tile); the tensor-core kernels in csrc/bwd_tc.cu then
// accumulate dK and dV per pair of key tiles over the transposed lists, and
// dQ per pair of query tiles over the kept lists. P and dS are rounded to
// bf16 for the products, as the forward rounds P.
//
// Tiled layout [B, Hh, N, V, D] (D in {64, 128}); the kernels work on 64-row
// chunks of the tiles as the forward does; padded key and query slots are
// masked from their chunk's real extent.
#include "internal.h"

namespace {

// Delta = rowsum(dO * O) per query row (fp32 of the bf16 values).
template <int D>
__global__ void __launch_bounds__(256)
bwd_delta_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ d_o, float* __restrict__ delta,
                 size_t rows) {
  const size_t row = (size_t)blockIdx.x * 64 + threadIdx.x / 4;
  const int part = threadIdx.x % 4;  // D/4 columns each
  float s = 0.f;
  if (row < rows) {
    const __nv_bfloat16* a = o + row * D + part * (D / 4);
    const __nv_bfloat16* b = d_o + row * D + part * (D / 4);
#pragma unroll
    for (int c = 0; c < D / 4; c += 8) {
      const uint4 x = *reinterpret_cast<const uint4*>(a + c), y = *reinterpret_cast<const uint4*>(b + c);
      const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&x);
      const __nv_bfloat162* yh = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 xf = __bfloat1622float2(xh[e]), yf = __bfloat1622float2(yh[e]);
        s = fmaf(xf.x, yf.x, s);
        s = fmaf(xf.y, yf.y, s);
      }
    }
  }
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  if (row < rows && part == 0) delta[row] = s;
}

// Transposed kept lists: bit i of row (bh, j) set when query tile i keeps j.
__global__ void bwd_bitmap_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int N, int kmax,
                                  int words, uint32_t* __restrict__ bm, int* err) {
  const size_t r = blockIdx.x;  // (bh, i)
  const size_t bh = r / N;
  const int i = (int)(r % N);
  const int c = min(max(cnt[r], 0), kmax);
  for (int e = threadIdx.x; e < c; e += blockDim.x) {
    const int j = idx[r * kmax + e];
    if (j < 0 || j >= N) {
      atomicOr(err, BSATTN_DEVERR_BAD_INDEX);
      continue;
    }
    atomicOr(&bm[(bh * N + j) * words + (i >> 5)], 1u << (i & 31));
  }
}

// Bitmap rows -> ascending lists (one warp per row).
__global__ void bwd_compact_kernel(const uint32_t* __restrict__ bm, int N, int words, size_t rows,
                                   int32_t* __restrict__ idxT, int32_t* __restrict__ cntT) {
  const size_t r = (size_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  int base = 0;
  for (int w0 = 0; w0 < words; w0 += 32) {
    const uint32_t v = w0 + lane < words ? bm[r * words + w0 + lane] : 0u;
    const int pc = __popc(v);
    int x = pc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    int pos = base + x - pc;
    uint32_t m = v;
    while (m) {
      idxT[r * N + pos++] = (w0 + lane) * 32 + __ffs(m) - 1;
      m &= m - 1;
    }
    base += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) cntT[r] = base;
}

template <int D>
bsattn_status run_backward(const bsattn_plan* p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const __nv_bfloat16* o, const __nv_bfloat16* d_o, const float* lse,
                           const int32_t* idx, const int32_t* cnt, __nv_bfloat16* dq, __nv_bfloat16* dk,
                           __nv_bfloat16* dv, const BackwardWs& w, cudaStream_t st) {
  const Geom g = make_geom(p);
  const size_t rows = (size_t)g.B * g.Hh * g.N;  // tile rows of the lists
  const int words = (g.N + 31) / 32;
  const size_t qrows = rows * g.V;  // query rows of the tiled layout
  bwd_delta_kernel<D><<<(unsigned)((qrows + 63) / 64), 256, 0, st>>>(o, d_o, w.delta, qrows);
  BSATTN_CUDA_TRY(cudaMemsetAsync(w.bm, 0, rows * words * sizeof(uint32_t), st));
  bwd_bitmap_kernel<<<(unsigned)rows, 64, 0, st>>>(idx, cnt, g.N, p->kmax, words, w.bm, p->d_err);
  bwd_compact_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(w.bm, g.N, words, rows, w.idxT, w.cntT);
  if (cudaGetLastError() != cudaSuccess) return BSATTN_ERR_CUDA;
  bsattn_status s = launch_backward_dkdv_tc(p, q, k, v, d_o, lse, w.delta, w.idxT, w.cntT, dk, dv, st);
  if (s) return s;
  return launch_backward_dq_tc(p, q, k, v, d_o, lse, w.delta, idx, cnt, dq, st);
}

}  // namespace

bsattn_status launch_backward(const bsattn_plan* p, const void* q, const void* k, const void* v, const void* o,
                              const void* d_o, const float* lse, const int32_t* idx, const int32_t* cnt, void* dq,
                              void* dk, void* dv, const BackwardWs& w, cudaStream_t st) {
  using B16 = __nv_bfloat16;
  if (p->desc.head_dim == 128)
    return run_backward<128>(p, (const B16*)q, (const B16*)k, (const B16*)v, (const B16*)o, (const B16*)d_o, lse,
                             idx, cnt, (B16*)dq, (B16*)dk, (B16*)dv, w, st);
  return run_backward<64>(p, (const B16*)q, (const B16*)k, (const B16*)v, (const B16*)o, (const B16*)d_o, lse, idx,
                          cnt, (B16*)dq, (B16*)dk, (B16*)dv, w, st);
}
