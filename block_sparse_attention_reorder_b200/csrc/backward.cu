// Backward pass of block-sparse attention (the trainable block-sparse
// attention of "Faster Video Diffusion with Trainable Sparse Attention",
// reproducibility record, Research Type row: models are trained through it).
//
// With P the masked softmax of the forward pass (recomputed from Q, K and the
// forward's log-sum-exp), dO the incoming gradient and Delta = rowsum(dO * O):
//   dV_j += P_ij^T dO_i,  dP_ij = dO_i V_j^T,  dS_ij = P_ij * (dP_ij - Delta_i),
//   dK_j += scale dS_ij^T Q_i,  dQ_i += scale dS_ij K_j
// over the kept tile pairs (i, j). Two kernels avoid atomics: one per key
// tile walks the query tiles that keep it (a transposed list built from
// bitmaps, ascending) and accumulates dK_j and dV_j (here, on the warp-level
// bf16 tensor core instruction mma.sync m16n8k16 with fp32 accumulation;
// each of four warps owns 16 rows of the tile, so no cross-warp reduction is
// needed); one per pair of query tiles walks their kept lists and
// accumulates dQ_i on tcgen05 (csrc/bwd_tc.cu). P and dS are rounded to bf16
// for the products, as the forward rounds P.
//
// Tiles of 64 tokens (tiled layout [B, Hh, N, 64, D], D in {64, 128}); padded
// key and query slots are masked from their tile's real extent.
#include "internal.h"

namespace {

constexpr int kRowsT = 64;   // tile rows
constexpr int kThreadsB = 128;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared-memory tile: 64 rows of D bf16 with a 16-byte pad per row, so the
// eight rows an ldmatrix reads fall in different banks.
template <int D>
struct TileS {
  static constexpr int PITCH = D * 2 + 16;  // bytes
  static constexpr int BYTES = kRowsT * PITCH;
};

// Copy tile rows [0, 64) x D (contiguous in global memory) into a padded tile.
template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const __nv_bfloat16* src) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  for (int c = threadIdx.x; c < kRowsT * CPR; c += kThreadsB) {
    const int r = c / CPR, k = c % CPR;
    cp_async16(dst + r * TileS<D>::PITCH + k * 16, src + (size_t)r * D + k * 8);
  }
}

// Bit r set when in-tile row r of tile j is a real token.
__device__ __forceinline__ uint64_t real_rows(const Geom& g, int j) {
  const int bt = j / (g.nH * g.nW), bhh = (j / g.nW) % g.nH, bw = j % g.nW;
  const int vt = g.T - bt * g.tt, vh = g.H - bhh * g.th, vw = g.W - bw * g.tw;
  if (vt >= g.tt && vh >= g.th && vw >= g.tw) return ~0ull;  // interior tile
  uint64_t m = 0;
  for (int r = 0; r < kRowsT; ++r) {
    const int dt = r / (g.th * g.tw), dh = (r / g.tw) % g.th, dw = r % g.tw;
    if (dt < vt && dh < vh && dw < vw) m |= 1ull << r;
  }
  return m;
}

// X (16 rows of this warp) x Y^T over D: acc[t][0..3] for 8 column tiles of
// 8 (64 columns of Y's rows). X rows at xs (tile rows w*16..), Y rows at ys.
template <int D>
__device__ __forceinline__ void xyt(const uint8_t* xs, const uint8_t* ys, int w, int lane, float (&acc)[8][4]) {
  constexpr int P = TileS<D>::PITCH;
#pragma unroll
  for (int t = 0; t < 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(smem_u32(xs + (w * 16 + (lane & 15)) * P + kk * 32 + (lane >> 4) * 16), a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int t2 = 0; t2 < 4; ++t2) {  // two column tiles per ldmatrix.x4
      uint32_t b0, b1, b2, b3;
      const int row = t2 * 16 + (lane & 7) + (lane >> 4) * 8;
      ldsm_x4(smem_u32(ys + row * P + kk * 32 + ((lane >> 3) & 1) * 16), b0, b1, b2, b3);
      mma_bf16(acc[2 * t2], a, b0, b1);
      mma_bf16(acc[2 * t2 + 1], a, b2, b3);
    }
  }
}

// acc (16 x D, this warp) += A (16 x 64, bf16 fragments from a 16 x 64 fp32
// accumulator) x Z (64 rows x D at zs, row-major: Z[k][n]).
template <int D>
__device__ __forceinline__ void az(const uint32_t (&af)[4][4], const uint8_t* zs, int lane, float (&acc)[D / 8][4]) {
  constexpr int P = TileS<D>::PITCH;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {  // 16 rows of Z per step
#pragma unroll
    for (int n2 = 0; n2 < D / 16; ++n2) {  // two 8-column tiles per ldmatrix.x4.trans
      uint32_t b0, b1, b2, b3;
      const int row = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      ldsm_x4_t(smem_u32(zs + row * P + n2 * 32 + (lane >> 4) * 16), b0, b1, b2, b3);
      mma_bf16(acc[2 * n2], af[kk], b0, b1);
      mma_bf16(acc[2 * n2 + 1], af[kk], b2, b3);
    }
  }
}

// bf16 A fragments (k = 64 columns) from a 16 x 64 fp32 accumulator.
__device__ __forceinline__ void to_afrag(const float (&c)[8][4], uint32_t (&af)[4][4]) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    af[kk][0] = pack_bf16(c[2 * kk][0], c[2 * kk][1]);
    af[kk][1] = pack_bf16(c[2 * kk][2], c[2 * kk][3]);
    af[kk][2] = pack_bf16(c[2 * kk + 1][0], c[2 * kk + 1][1]);
    af[kk][3] = pack_bf16(c[2 * kk + 1][2], c[2 * kk + 1][3]);
  }
}

// Store a warp's 16 x D fp32 accumulator (times `mul`) as bf16 rows.
template <int D>
__device__ __forceinline__ void store_rows(__nv_bfloat16* dst, const float (&acc)[D / 8][4], int w, int lane,
                                           float mul) {
  const int r0 = w * 16 + (lane >> 2), c0 = (lane & 3) * 2;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    *reinterpret_cast<uint32_t*>(dst + (size_t)r0 * D + n * 8 + c0) = pack_bf16(acc[n][0] * mul, acc[n][1] * mul);
    *reinterpret_cast<uint32_t*>(dst + (size_t)(r0 + 8) * D + n * 8 + c0) =
        pack_bf16(acc[n][2] * mul, acc[n][3] * mul);
  }
}

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

// dK_j, dV_j: one CTA per (key tile j, head, batch); warp w owns key rows
// 16w .. 16w + 15 and walks the query tiles that keep j.
template <int D>
__global__ void __launch_bounds__(kThreadsB)
bwd_dkdv_kernel(Geom g, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ d_o,
                const float* __restrict__ lse, const float* __restrict__ delta, const int32_t* __restrict__ idxT,
                const int32_t* __restrict__ cntT, float c_log2, float scale, __nv_bfloat16* __restrict__ dk,
                __nv_bfloat16* __restrict__ dv) {
  // K_j, V_j, then two stages of (Q_i, dO_i, lse_i, Delta_i): the next query
  // tile loads while the current one is used.
  extern __shared__ __align__(16) uint8_t sm[];
  constexpr int STAGE = 2 * TileS<D>::BYTES + 2 * kRowsT * 4;
  uint8_t* Ks = sm;
  uint8_t* Vs = Ks + TileS<D>::BYTES;
  uint8_t* stage0 = Vs + TileS<D>::BYTES;
  const int j = blockIdx.x, head = blockIdx.y, b = blockIdx.z;
  const size_t bh = (size_t)b * g.Hh + head;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t tj = (bh * g.N + j) * kRowsT;
  const int nq = cntT[bh * g.N + j];
  const int32_t* qlist = idxT + (bh * g.N + j) * g.N;
  auto load_query = [&](int e) {
    uint8_t* st = stage0 + (e & 1) * STAGE;
    const size_t ti = (bh * g.N + qlist[e]) * kRowsT;
    load_tile<D>(st, q + ti * D);
    load_tile<D>(st + TileS<D>::BYTES, d_o + ti * D);
    if (threadIdx.x < 32) {  // 64 lse then 64 Delta values, 16 bytes per thread
      const float* src = threadIdx.x < 16 ? lse + ti + threadIdx.x * 4 : delta + ti + (threadIdx.x - 16) * 4;
      cp_async16(st + 2 * TileS<D>::BYTES + threadIdx.x * 16, src);
    }
  };
  load_tile<D>(Ks, k + tj * D);
  load_tile<D>(Vs, v + tj * D);
  if (nq > 0) load_query(0);
  cp_async_commit();
  const uint64_t kreal = real_rows(g, j);
  // This thread's key rows: w*16 + lane/4 and +8.
  const int kr0 = w * 16 + (lane >> 2);
  const bool kv0 = (kreal >> kr0) & 1, kv1 = (kreal >> (kr0 + 8)) & 1;
  float dka[D / 8][4], dva[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) dka[n][0] = dka[n][1] = dka[n][2] = dka[n][3] = dva[n][0] = dva[n][1] = dva[n][2] = dva[n][3] = 0.f;
  for (int e = 0; e < nq; ++e) {
    const int i = qlist[e];
    // Stage e&1 was last read in iteration e-2, behind the barrier ending
    // iteration e-1, so the prefetch of e+1 into the other stage is safe.
    if (e + 1 < nq) load_query(e + 1);
    cp_async_commit();
    cp_async_wait<1>();  // everything but the newest group has landed
    __syncthreads();
    uint8_t* Qs = stage0 + (e & 1) * STAGE;
    uint8_t* Os = Qs + TileS<D>::BYTES;
    const float* lse_s = reinterpret_cast<const float*>(Os + TileS<D>::BYTES);
    const float* del_s = lse_s + kRowsT;
    const uint64_t qreal = real_rows(g, i);
    // S^T = K Q^T (16 keys x 64 queries), then P^T = 2^(S^T c - lse[q]).
    float st[8][4];
    xyt<D>(Ks, Qs, w, lane, st);
    float dpt[8][4];
    xyt<D>(Vs, Os, w, lane, dpt);  // dP^T = V dO^T
#pragma unroll
    for (int t = 0; t < 8; ++t) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int qc = t * 8 + (lane & 3) * 2 + h;  // query column
        const bool qv = (qreal >> qc) & 1;
        const float l2 = lse_s[qc] * 1.4426950408889634f, dl = del_s[qc];
        const float p0 = (qv && kv0) ? ex2(st[t][h] * c_log2 - l2) : 0.f;
        const float p1 = (qv && kv1) ? ex2(st[t][2 + h] * c_log2 - l2) : 0.f;
        st[t][h] = p0;
        st[t][2 + h] = p1;
        dpt[t][h] = p0 * (dpt[t][h] - dl);       // dS^T
        dpt[t][2 + h] = p1 * (dpt[t][2 + h] - dl);
      }
    }
    uint32_t pf[4][4], sf[4][4];
    to_afrag(st, pf);
    to_afrag(dpt, sf);
    az<D>(pf, Os, lane, dva);  // dV += P^T dO
    az<D>(sf, Qs, lane, dka);  // dK += dS^T Q
    __syncthreads();  // this stage is refilled two iterations on
  }
  store_rows<D>(dk + tj * D, dka, w, lane, scale);
  store_rows<D>(dv + tj * D, dva, w, lane, 1.f);
}

template <int D>
bsattn_status run_backward(const bsattn_plan* p, const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const __nv_bfloat16* o, const __nv_bfloat16* d_o, const float* lse,
                           const int32_t* idx, const int32_t* cnt, __nv_bfloat16* dq, __nv_bfloat16* dk,
                           __nv_bfloat16* dv, const BackwardWs& w, cudaStream_t st) {
  const Geom g = make_geom(p);
  const size_t rows = (size_t)g.B * g.Hh * g.N;  // tile rows of the lists
  const int words = (g.N + 31) / 32;
  const float scale = p->scale, c_log2 = p->scale * 1.4426950408889634f;
  bwd_delta_kernel<D><<<(unsigned)((rows * kRowsT + 63) / 64), 256, 0, st>>>(o, d_o, w.delta, rows * kRowsT);
  BSATTN_CUDA_TRY(cudaMemsetAsync(w.bm, 0, rows * words * sizeof(uint32_t), st));
  bwd_bitmap_kernel<<<(unsigned)rows, 64, 0, st>>>(idx, cnt, g.N, p->kmax, words, w.bm, p->d_err);
  bwd_compact_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(w.bm, g.N, words, rows, w.idxT, w.cntT);
  const size_t smem_kv = 2 * (size_t)TileS<D>::BYTES + 2 * (2 * (size_t)TileS<D>::BYTES + 2 * kRowsT * 4);
  auto kkv = bwd_dkdv_kernel<D>;
  if (cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_kv) != cudaSuccess)
    return BSATTN_ERR_CUDA;
  dim3 grid(g.N, g.Hh, g.B);
  kkv<<<grid, kThreadsB, smem_kv, st>>>(g, q, k, v, d_o, lse, w.delta, w.idxT, w.cntT, c_log2, scale, dk, dv);
  if (cudaGetLastError() != cudaSuccess) return BSATTN_ERR_CUDA;
  // dQ on the tensor cores (csrc/bwd_tc.cu).
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
