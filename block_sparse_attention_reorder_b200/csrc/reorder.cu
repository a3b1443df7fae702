// Tile reorder (natural -> tiled) with fused per-tile e4m3 quantisation, the
// inverse scatter, standalone tile quantisation, and tile-mean pooling.
//
// These steps move bytes: one CTA per (batch, head, 64-row chunk of a tile)
// moves the chunk's 64 rows of D bf16 with 16-byte vector accesses. Reads are
// 64 row segments of 2*D bytes (the natural layout interleaves heads), writes
// are one contiguous 64*D*2-byte block, so both sides use full 32-byte
// sectors. e4m3 quantisation needs the whole tile's amax: with one chunk per
// tile the values stay in registers, with several a CTA takes the tile and
// reads it twice (the second time mostly from L2). Q and K are quantised by
// one launch (the grid's z covers both tensors).
#include <cuda_fp8.h>

#include "internal.h"

namespace {

constexpr int kThreads = 256;

struct TileCoord {
  int t0, h0, w0;     // first token coordinate of the tile
  int vt, vh, vw;     // real extent along each axis (<= tile)
};

__device__ __forceinline__ TileCoord tile_coord(const Geom& g, int j) {
  TileCoord c;
  int bt = j / (g.nH * g.nW), bh = (j / g.nW) % g.nH, bw = j % g.nW;
  c.t0 = bt * g.tt; c.h0 = bh * g.th; c.w0 = bw * g.tw;
  c.vt = min(g.tt, g.T - c.t0); c.vh = min(g.th, g.H - c.h0); c.vw = min(g.tw, g.W - c.w0);
  return c;
}

// Natural token index of in-tile row r, or -1 for a padded slot.
__device__ __forceinline__ int row_token(const Geom& g, const TileCoord& c, int r) {
  int dt = r / (g.th * g.tw), dh = (r / g.tw) % g.th, dw = r % g.tw;
  if (dt >= c.vt || dh >= c.vh || dw >= c.vw) return -1;
  return ((c.t0 + dt) * g.H + (c.h0 + dh)) * g.W + (c.w0 + dw);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 x = __bfloat1622float2(h[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}

// max(|x|) of 8 bf16 values, taken on bf16 pairs (exact: the maximum of bf16
// magnitudes is one of them; a NaN is passed over, as fmaxf does).
__device__ __forceinline__ __nv_bfloat162 absmax8(__nv_bfloat162 m, const uint4& u) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) m = __hmax2(m, __habs2(h[i]));
  return m;
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; ++i) m = fmaxf(m, red[i]);
  return m;
}

// x / scale as the e4m3 conversion sees it: the IEEE fp32 quotient
// fl(x / scale), computed without a division by Markstein's FMA correction.
// With y = rscale the correctly rounded 1/scale and p = fl(x * y), p is
// within an ulp of x / scale, the residual x - p * scale is exact in fp32 and
// fl(p + r * y) is the correctly rounded quotient. The residual is exact when
// ulp(p) * ulp(scale) >= 2^-149; for codes that can be nonzero (|p| >= 2^-11)
// that holds once scale >= 2^-92. Tiles with a smaller scale, or with one
// above 2^126 (reciprocal subnormal or zero, e.g. an infinite amax), divide
// instead; the test is per tile, hence uniform across the CTA. The kernels
// form t = p * scale - x (exact, t = -r) and q = p + t * (-y), so that x = -0
// gives -0, on packed pairs of values.
constexpr float kFmaQuotientMinScale = 0x1p-92f, kFmaQuotientMaxScale = 0x1p126f;

__device__ __forceinline__ bool fma_quotient_ok(float scale) {
  return scale >= kFmaQuotientMinScale && scale <= kFmaQuotientMaxScale;
}

// e4m3 codes of 8 values divided by `scale` (as the IEEE fp32 division), RNE,
// satfinite; FMA: by the correction above (the tile passed fma_quotient_ok),
// else by division.
template <bool FMA>
__device__ __forceinline__ uint2 quant8(const float* f, float scale, float rscale) {
  uint32_t w[2];
  if constexpr (FMA) {
    const float2 y2 = make_float2(rscale, rscale), s2 = make_float2(scale, scale),
                 ny2 = make_float2(-rscale, -rscale);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t acc = 0;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 x = make_float2(f[4 * h + 2 * i], f[4 * h + 2 * i + 1]);
        const float2 p = __fmul2_rn(x, y2);
        const float2 t = __ffma2_rn(p, s2, make_float2(-x.x, -x.y));
        const float2 q = __ffma2_rn(t, ny2, p);
        acc |= (uint32_t)__nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3) << (16 * i);
      }
      w[h] = acc;
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t acc = 0;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 q = make_float2(__fdiv_rn(f[4 * h + 2 * i], scale), __fdiv_rn(f[4 * h + 2 * i + 1], scale));
        acc |= (uint32_t)__nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3) << (16 * i);
      }
      w[h] = acc;
    }
  }
  return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ float tile_scale_from_amax(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
}

template <int D>
__global__ void __launch_bounds__(kThreads)
reorder_kernel(Geom g, const __nv_bfloat16* __restrict__ x_nat, __nv_bfloat16* __restrict__ x_tiled) {
  constexpr int CH = D / 8;                 // 16-byte chunks per row
  constexpr int ITER = 64 * CH / kThreads;  // chunks per thread
  constexpr int RSTEP = kThreads / CH;      // row stride between a thread's chunks
  __shared__ int rowtok[64];  // token of each row of the chunk, -1 for a padded slot

  const int j = blockIdx.x / g.nchunk, head = blockIdx.y, b = blockIdx.z;
  const int c = threadIdx.x % CH;
  const int r0 = threadIdx.x / CH;
  const TileCoord tc = tile_coord(g, j);
  const int row0 = 64 * (blockIdx.x % g.nchunk);  // first in-tile row of the chunk
  const size_t tile_off = (((size_t)b * g.Hh + head) * g.N + j) * g.V + row0;
  // Each row's token once per CTA: the CH threads of a row would otherwise
  // all repeat its integer divisions.
  if (threadIdx.x < 64) rowtok[threadIdx.x] = row_token(g, tc, row0 + threadIdx.x);
  __syncthreads();

  uint4 v[ITER];
#pragma unroll
  for (int i = 0; i < ITER; ++i) {
    int n = rowtok[r0 + RSTEP * i];
    v[i] = n >= 0 ? __ldg(reinterpret_cast<const uint4*>(x_nat + (((size_t)b * g.L + n) * g.Hh + head) * D) + c)
                  : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < ITER; ++i)
    reinterpret_cast<uint4*>(x_tiled + (tile_off + r0 + RSTEP * i) * D)[c] = v[i];
}

// Source and destination of the e4m3 quantisation of one or two tensors
// (Q and K); blockIdx.z = batch * ntensor + tensor.
struct QuantPair {
  const __nv_bfloat16* src[2];
  uint8_t* codes[2];
  float* scales[2];
};

// e4m3 codes and tile scales of one-chunk tiles straight from the natural
// layout: one CTA per (tile, head, tensor, batch) holds the tile's 64 rows in
// registers, takes their amax, and writes the codes as one contiguous block.
// Capped at 40 registers so six CTAs share an SM and keep loads in flight
// across each CTA's amax barrier.
template <int D>
__global__ void __launch_bounds__(kThreads, 6)
reorder_quant_kernel(Geom g, QuantPair qp) {
  constexpr int CH = D / 8;
  constexpr int ITER = 64 * CH / kThreads;
  constexpr int RSTEP = kThreads / CH;
  __shared__ float wred[kThreads / 32];
  __shared__ int rowtok[64];
  const int nt = gridDim.z / g.B;
  const int tensor = blockIdx.z % nt, b = blockIdx.z / nt;
  const int j = blockIdx.x, head = blockIdx.y;
  const int c = threadIdx.x % CH;
  const int r0 = threadIdx.x / CH;
  const size_t tile = ((size_t)b * g.Hh + head) * g.N + j;
  if (threadIdx.x < 64) rowtok[threadIdx.x] = row_token(g, tile_coord(g, j), threadIdx.x);
  __syncthreads();
  const __nv_bfloat16* x_nat = qp.src[tensor];
  uint4 v[ITER];
#pragma unroll
  for (int i = 0; i < ITER; ++i) {
    int n = rowtok[r0 + RSTEP * i];
    v[i] = n >= 0 ? __ldg(reinterpret_cast<const uint4*>(x_nat + (((size_t)b * g.L + n) * g.Hh + head) * D) + c)
                  : make_uint4(0, 0, 0, 0);
  }
  __nv_bfloat162 m2 = __float2bfloat162_rn(0.f);
#pragma unroll
  for (int i = 0; i < ITER; ++i) m2 = absmax8(m2, v[i]);
  const float m = fmaxf(__low2float(m2), __high2float(m2));
  const float scale = tile_scale_from_amax(block_max(m, wred)), rscale = __frcp_rn(scale);
  uint2* dst = reinterpret_cast<uint2*>(qp.codes[tensor] + tile * 64 * D);
  const bool fma = fma_quotient_ok(scale);
#pragma unroll
  for (int i = 0; i < ITER; ++i) {
    float f[8];
    bf16x8_to_f32(v[i], f);
    dst[(r0 + RSTEP * i) * CH + c] = fma ? quant8<true>(f, scale, rscale) : quant8<false>(f, scale, rscale);
  }
  if (threadIdx.x == 0) qp.scales[tensor][tile] = scale;
}

template <int D>
__global__ void __launch_bounds__(kThreads)
unreorder_kernel(Geom g, const __nv_bfloat16* __restrict__ x_tiled, __nv_bfloat16* __restrict__ x_nat,
                 const float* __restrict__ lse_tiled, float* __restrict__ lse_nat) {
  constexpr int CH = D / 8;
  constexpr int ITER = 64 * CH / kThreads;
  constexpr int RSTEP = kThreads / CH;
  __shared__ int rowtok[64];  // token of each row of the chunk, -1 for a padded slot
  const int j = blockIdx.x / g.nchunk, head = blockIdx.y, b = blockIdx.z;
  const int c = threadIdx.x % CH;
  const int r0 = threadIdx.x / CH;
  const TileCoord tc = tile_coord(g, j);
  const int row0 = 64 * (blockIdx.x % g.nchunk);
  const size_t tile_off = (((size_t)b * g.Hh + head) * g.N + j) * g.V + row0;
  if (threadIdx.x < 64) rowtok[threadIdx.x] = row_token(g, tc, row0 + threadIdx.x);
  __syncthreads();
#pragma unroll
  for (int i = 0; i < ITER; ++i) {
    int r = r0 + RSTEP * i;
    int n = rowtok[r];
    if (n < 0) continue;
    uint4 v = __ldg(reinterpret_cast<const uint4*>(x_tiled + (tile_off + r) * D) + c);
    reinterpret_cast<uint4*>(x_nat + (((size_t)b * g.L + n) * g.Hh + head) * D)[c] = v;
  }
  if (lse_tiled && threadIdx.x < 64) {
    int n = rowtok[threadIdx.x];
    if (n >= 0) lse_nat[((size_t)b * g.Hh + head) * g.L + n] = lse_tiled[tile_off + threadIdx.x];
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads)
quant_tiled_kernel(Geom g, const __nv_bfloat16* __restrict__ x_tiled, uint8_t* __restrict__ codes,
                   float* __restrict__ scales) {
  constexpr int CH = D / 8;
  constexpr int ITER = 64 * CH / kThreads;
  __shared__ float wred[kThreads / 32];
  const size_t tile = ((size_t)blockIdx.z * g.Hh + blockIdx.y) * g.N + blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(x_tiled + tile * 64 * D);
  uint4 v[ITER];
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < ITER; ++i) {
    v[i] = __ldg(src + threadIdx.x + kThreads * i);
    float f[8];
    bf16x8_to_f32(v[i], f);
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
  }
  const float scale = tile_scale_from_amax(block_max(m, wred)), rscale = __frcp_rn(scale);
  uint2* dst = reinterpret_cast<uint2*>(codes + tile * 64 * D);
  const bool fma = fma_quotient_ok(scale);
#pragma unroll
  for (int i = 0; i < ITER; ++i) {
    float f[8];
    bf16x8_to_f32(v[i], f);
    dst[threadIdx.x + kThreads * i] = fma ? quant8<true>(f, scale, rscale) : quant8<false>(f, scale, rscale);
  }
  if (threadIdx.x == 0) scales[tile] = scale;
}

// e4m3 codes of tiles of several chunks: pass 1 takes the tile's amax, pass 2
// reads the tile again (mostly from L2) and writes the codes. NAT: the
// sources are natural-layout tensors (padded rows read as zero); else tiled
// bf16 tensors.
template <int D, bool NAT>
__global__ void __launch_bounds__(kThreads)
quant_multi_kernel(Geom g, QuantPair qp) {
  constexpr int CH = D / 8;
  constexpr int ITER = 64 * CH / kThreads;
  constexpr int RSTEP = kThreads / CH;
  __shared__ float wred[kThreads / 32];
  const int nt = gridDim.z / g.B;
  const int tensor = blockIdx.z % nt, b = blockIdx.z / nt;
  const int j = blockIdx.x, head = blockIdx.y;
  const int c = threadIdx.x % CH;
  const int r0 = threadIdx.x / CH;
  const TileCoord tc = tile_coord(g, j);
  const size_t tile = ((size_t)b * g.Hh + head) * g.N + j;
  const __nv_bfloat16* src = qp.src[tensor];
  auto load = [&](int r) -> uint4 {
    if (NAT) {
      const int n = row_token(g, tc, r);
      if (n < 0) return make_uint4(0, 0, 0, 0);
      return __ldg(reinterpret_cast<const uint4*>(src + (((size_t)b * g.L + n) * g.Hh + head) * D) + c);
    }
    return __ldg(reinterpret_cast<const uint4*>(src + (tile * g.V + r) * D) + c);
  };
  __nv_bfloat162 m2 = __float2bfloat162_rn(0.f);
  for (int row0 = 0; row0 < g.V; row0 += 64) {
    uint4 v[ITER];
#pragma unroll
    for (int i = 0; i < ITER; ++i) v[i] = load(row0 + r0 + RSTEP * i);
#pragma unroll
    for (int i = 0; i < ITER; ++i) m2 = absmax8(m2, v[i]);
  }
  const float m = fmaxf(__low2float(m2), __high2float(m2));
  const float scale = tile_scale_from_amax(block_max(m, wred)), rscale = __frcp_rn(scale);
  uint8_t* codes = qp.codes[tensor];
  const bool fma = fma_quotient_ok(scale);
  for (int row0 = 0; row0 < g.V; row0 += 64) {
    uint4 v[ITER];
#pragma unroll
    for (int i = 0; i < ITER; ++i) v[i] = load(row0 + r0 + RSTEP * i);
#pragma unroll
    for (int i = 0; i < ITER; ++i) {
      const size_t row = tile * g.V + row0 + r0 + RSTEP * i;
      float f[8];
      bf16x8_to_f32(v[i], f);
      reinterpret_cast<uint2*>(codes + row * D)[c] =
          fma ? quant8<true>(f, scale, rscale) : quant8<false>(f, scale, rscale);
    }
  }
  if (threadIdx.x == 0) qp.scales[tensor][tile] = scale;
}

// Tile means of natural bf16 tokens. A token row holds all heads
// (Hh*D*2 contiguous bytes); a CTA takes one tile of one batch and tensor and
// a block of kPoolCols 16-byte column chunks of those rows, thread c owning
// chunk c: it sums the chunk over the tile's rows in (t, h, w) order, so rows
// are read coalesced, no cross-thread reduction is needed and the sum order
// is fixed. Loads go out sixteen at a time and unconditionally (a padded row
// reloads the tile's first row, which is cached, and adds zero), which keeps
// all sixteen in flight.
constexpr int kPoolCols = 128;

template <int D>
__global__ void __launch_bounds__(kPoolCols)
pool_kernel(Geom g, const __nv_bfloat16* __restrict__ x0, const __nv_bfloat16* __restrict__ x1,
            float* __restrict__ p0, float* __restrict__ p1, int ncblk) {
  constexpr int CH = D / 8;   // 16-byte chunks per head row
  __shared__ int rowoff[64];  // token offset of each row of a 64-row chunk from the tile's first token, -1 if padded
  const int tensor = blockIdx.z / ncblk, cblk = blockIdx.z % ncblk;
  const __nv_bfloat16* x = tensor ? x1 : x0;
  float* pooled = tensor ? p1 : p0;
  const int j = blockIdx.x, b = blockIdx.y;
  const TileCoord tc = tile_coord(g, j);
  const int n0 = (tc.t0 * g.H + tc.h0) * g.W + tc.w0;
  const int cpt = g.Hh * CH;  // chunks per token (all heads)
  const int c = cblk * kPoolCols + threadIdx.x;
  const bool active = c < cpt;
  const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)b * g.L + n0) * g.Hh * D) + c;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int row0 = 0; row0 < g.V; row0 += 64) {
    if (row0 > 0) __syncthreads();  // every thread is done with the previous offsets
    if (threadIdx.x < 64) {
      const int n = row_token(g, tc, row0 + threadIdx.x);
      rowoff[threadIdx.x] = n >= 0 ? n - n0 : -1;
    }
    __syncthreads();
    if (!active) continue;
#pragma unroll 1
    for (int r0 = 0; r0 < 64; r0 += 16) {
      uint4 v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = __ldg(src + (size_t)max(rowoff[r0 + i], 0) * cpt);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (rowoff[r0 + i] < 0) continue;
        float f[8];
        bf16x8_to_f32(v[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += f[e];
      }
    }
  }
  if (!active) return;
  const float nvalid = (float)(tc.vt * tc.vh * tc.vw);
  const int head = c / CH, d0 = (c % CH) * 8;
  float4* out = reinterpret_cast<float4*>(pooled + (((size_t)b * g.Hh + head) * g.N + j) * D + d0);
  out[0] = make_float4(__fdiv_rn(acc[0], nvalid), __fdiv_rn(acc[1], nvalid), __fdiv_rn(acc[2], nvalid),
                       __fdiv_rn(acc[3], nvalid));
  out[1] = make_float4(__fdiv_rn(acc[4], nvalid), __fdiv_rn(acc[5], nvalid), __fdiv_rn(acc[6], nvalid),
                       __fdiv_rn(acc[7], nvalid));
}

}  // namespace

bsattn_status launch_pool(const Geom& g, const __nv_bfloat16* x0, float* p0, const __nv_bfloat16* x1,
                          float* p1, cudaStream_t st) {
  const int cpt = g.Hh * g.D / 8, ncblk = (cpt + kPoolCols - 1) / kPoolCols;
  dim3 grid(g.N, g.B, (x1 ? 2 : 1) * ncblk);
  if (g.D == 128)
    pool_kernel<128><<<grid, kPoolCols, 0, st>>>(g, x0, x1, p0, p1, ncblk);
  else
    pool_kernel<64><<<grid, kPoolCols, 0, st>>>(g, x0, x1, p0, p1, ncblk);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

bsattn_status launch_reorder(const Geom& g, const __nv_bfloat16* x_nat, __nv_bfloat16* x_tiled,
                             cudaStream_t st) {
  dim3 grid(g.N * g.nchunk, g.Hh, g.B);
  if (g.D == 128)
    reorder_kernel<128><<<grid, kThreads, 0, st>>>(g, x_nat, x_tiled);
  else
    reorder_kernel<64><<<grid, kThreads, 0, st>>>(g, x_nat, x_tiled);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

bsattn_status launch_reorder_quant(const Geom& g, const __nv_bfloat16* q_nat, const __nv_bfloat16* k_nat,
                                   uint8_t* q_codes, uint8_t* k_codes, float* q_scales, float* k_scales,
                                   cudaStream_t st) {
  const QuantPair qp{{q_nat, k_nat}, {q_codes, k_codes}, {q_scales, k_scales}};
  dim3 grid(g.N, g.Hh, 2 * g.B);
  if (g.nchunk > 1) {
    if (g.D == 128)
      quant_multi_kernel<128, true><<<grid, kThreads, 0, st>>>(g, qp);
    else
      quant_multi_kernel<64, true><<<grid, kThreads, 0, st>>>(g, qp);
  } else if (g.D == 128) {
    reorder_quant_kernel<128><<<grid, kThreads, 0, st>>>(g, qp);
  } else {
    reorder_quant_kernel<64><<<grid, kThreads, 0, st>>>(g, qp);
  }
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

bsattn_status launch_unreorder(const Geom& g, const __nv_bfloat16* x_tiled, __nv_bfloat16* x_nat,
                               const float* lse_tiled, float* lse_nat, cudaStream_t st) {
  dim3 grid(g.N * g.nchunk, g.Hh, g.B);
  if (g.D == 128)
    unreorder_kernel<128><<<grid, kThreads, 0, st>>>(g, x_tiled, x_nat, lse_tiled, lse_nat);
  else
    unreorder_kernel<64><<<grid, kThreads, 0, st>>>(g, x_tiled, x_nat, lse_tiled, lse_nat);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

bsattn_status launch_quant_tiled(const Geom& g, const __nv_bfloat16* x_tiled, uint8_t* codes,
                                 float* scales, cudaStream_t st) {
  dim3 grid(g.N, g.Hh, g.B);
  if (g.nchunk > 1) {
    const QuantPair qp{{x_tiled, x_tiled}, {codes, codes}, {scales, scales}};
    if (g.D == 128)
      quant_multi_kernel<128, false><<<grid, kThreads, 0, st>>>(g, qp);
    else
      quant_multi_kernel<64, false><<<grid, kThreads, 0, st>>>(g, qp);
    return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
  }
  if (g.D == 128)
    quant_tiled_kernel<128><<<grid, kThreads, 0, st>>>(g, x_tiled, codes, scales);
  else
    quant_tiled_kernel<64><<<grid, kThreads, 0, st>>>(g, x_tiled, codes, scales);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}
