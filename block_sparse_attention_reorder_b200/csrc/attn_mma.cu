// Block-sparse attention forward over kept tile pairs, warp-level MMA form.
//
// One CTA (4 warps) per (query tile, head, batch); warp w owns query rows
// 16w..16w+15 of the 64-row tile. For every kept key tile j (ascending, from
// the caller's lists) the K_j and V_j tiles are staged in shared memory by
// cp.async (two stages), then per warp
//   S = Q K_j^T            (bf16 m16n8k16, or e4m3 m16n8k32 with tile scales)
//   padded keys -> -inf, online softmax in fp32 (log2 domain),
//   P rounded to bf16,  O += P V_j   (bf16 m16n8k16, fp32 accumulators).
// Finally O /= l and O (bf16) and lse (fp32, natural log) are written for all
// 64 rows of the tile.
//
// List entries outside [0, N) and counts outside [0, kmax] set the plan's
// device error word; bad entries are skipped and counts clamped.
#include <math.h>

#include "internal.h"

namespace {

struct AttnParams {
  Geom g;
  const uint8_t* q;   // bf16 or e4m3 tiled
  const uint8_t* k;
  const float* qs;    // e4m3 tile scales (or null)
  const float* ks;
  const __nv_bfloat16* v;
  const int32_t* idx;
  const int32_t* cnt;
  int kmax;
  __nv_bfloat16* o;
  float* lse;
  float scale_log2;   // softmax scale * log2(e)
  int* err;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_e4m3(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Byte offset of 16-byte chunk c of row r in a swizzled tile whose rows hold
// CPR chunks (CPR >= 4). Eight consecutive rows read at one logical chunk hit
// eight distinct bank groups.
template <int CPR>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  int pc = CPR >= 8 ? (c ^ (r & 7)) : (c ^ ((r >> 1) & 3));
  return (uint32_t)(r * CPR + pc) * 16u;
}

// Copy a 64-row tile of RB bytes per row from global to swizzled smem.
template <int RB>
__device__ __forceinline__ void load_tile(uint32_t sbase, const uint8_t* gsrc) {
  constexpr int CPR = RB / 16;
  constexpr int TOTAL = 64 * CPR;
#pragma unroll
  for (int i = 0; i < TOTAL / 128; ++i) {
    int lin = threadIdx.x + 128 * i;
    int r = lin / CPR, c = lin % CPR;
    cp_async16(sbase + swz<CPR>(r, c), gsrc + (size_t)lin * 16);
  }
}

__device__ __forceinline__ bool key_col_valid(const Geom& g, int t0, int h0, int w0, int r) {
  int dt = r / (g.th * g.tw), dh = (r / g.tw) % g.th, dw = r % g.tw;
  return (t0 + dt < g.T) && (h0 + dh < g.H) && (w0 + dw < g.W);
}

template <int D, bool FP8>
__global__ void __launch_bounds__(128)
attn_mma_kernel(AttnParams P) {
  constexpr int QB = FP8 ? 1 : 2;        // bytes per Q/K element
  constexpr int QRB = D * QB;            // Q/K row bytes
  constexpr int VRB = D * 2;             // V row bytes
  constexpr int QCPR = QRB / 16, VCPR = VRB / 16;
  constexpr int KSTEP = FP8 ? 32 : 16;   // MMA k for S
  constexpr int NKS = D / KSTEP;         // k-steps for S
  constexpr int QTILE = 64 * QRB, VTILE = 64 * VRB;
  constexpr int NDT = D / 8;             // O n-tiles

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + QTILE;                  // 2 stages
  uint8_t* sV = sK + 2 * QTILE;              // 2 stages

  const Geom& g = P.g;
  const int i = blockIdx.x, head = blockIdx.y, b = blockIdx.z;
  const size_t bh = (size_t)b * g.Hh + head;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, qd = lane & 3;

  int n = P.cnt[bh * g.N + i];
  if (n < 0 || n > P.kmax) {
    if (threadIdx.x == 0) atomicOr(P.err, BSATTN_DEVERR_BAD_INDEX);
    n = n < 0 ? 0 : P.kmax;
  }
  const int32_t* list = P.idx + (bh * g.N + i) * P.kmax;

  const uint8_t* qg = P.q + (bh * g.N + i) * (size_t)QTILE;
  load_tile<QRB>(smem_u32(sQ), qg);
  auto fetch = [&](int it, int stage) -> bool {
    int j = __ldg(list + it);
    if (j < 0 || j >= g.N) return false;
    load_tile<QRB>(smem_u32(sK + stage * QTILE), P.k + (bh * g.N + j) * (size_t)QTILE);
    load_tile<VRB>(smem_u32(sV + stage * VTILE),
                   reinterpret_cast<const uint8_t*>(P.v) + (bh * g.N + j) * (size_t)VTILE);
    return true;
  };
  if (n > 0) fetch(0, 0);
  cp_async_commit();

  float o_acc[NDT][4];
#pragma unroll
  for (int d = 0; d < NDT; ++d) o_acc[d][0] = o_acc[d][1] = o_acc[d][2] = o_acc[d][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY};
  float l_r[2] = {0.f, 0.f};
  uint32_t qf[NKS][4];
  const float q_scale = FP8 ? P.qs[bh * g.N + i] : 1.f;

  for (int it = 0; it < n; ++it) {
    const int stage = it & 1;
    if (it + 1 < n) fetch(it + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (it == 0) {
      // Q fragments once (rows 16*warp.., every k-step).
#pragma unroll
      for (int ks = 0; ks < NKS; ++ks) {
        int r = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        int c = ks * 2 + (lane >> 4);
        ldsm_x4(smem_u32(sQ) + swz<QCPR>(r, c), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
      }
    }
    const int j = __ldg(list + it);
    if (j < 0 || j >= g.N) {
      if (threadIdx.x == 0) atomicOr(P.err, BSATTN_DEVERR_BAD_INDEX);
      __syncthreads();
      continue;
    }
    const uint32_t kb = smem_u32(sK + stage * QTILE);
    const uint32_t vb = smem_u32(sV + stage * VTILE);

    // S = Q K_j^T: 16 rows x 64 keys per warp.
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        int r = 8 * (nt + (lane >> 4)) + (lane & 7);
        int c = ks * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz<QCPR>(r, c), b0, b1, b2, b3);
        if (FP8) {
          mma_e4m3(s[nt], qf[ks], b0, b1);
          mma_e4m3(s[nt + 1], qf[ks], b2, b3);
        } else {
          mma_bf16(s[nt], qf[ks], b0, b1);
          mma_bf16(s[nt + 1], qf[ks], b2, b3);
        }
      }
    }
    // Logits in the log2 domain, padded keys masked.
    const float f = P.scale_log2 * (FP8 ? q_scale * P.ks[bh * g.N + j] : 1.f);
    const int bt = j / (g.nH * g.nW), bhh = (j / g.nW) % g.nH, bw = j % g.nW;
    const int t0 = bt * g.tt, h0 = bhh * g.th, w0 = bw * g.tw;
    const bool partial = (t0 + g.tt > g.T) || (h0 + g.th > g.H) || (w0 + g.tw > g.W);
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int col = nt * 8 + qd * 2 + (e & 1);
        float x = s[nt][e] * f;
        if (partial && !key_col_valid(g, t0, h0, w0, col)) x = -INFINITY;
        s[nt][e] = x;
        mx[e >> 1] = fmaxf(mx[e >> 1], x);
      }
    }
    float alpha[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
      float m_new = fmaxf(m_r[h], mx[h]);
      alpha[h] = exp2f(m_r[h] - m_new);  // m_r = -inf on the first kept tile -> 0
      m_r[h] = m_new;
      l_r[h] *= alpha[h];
    }
#pragma unroll
    for (int d = 0; d < NDT; ++d) {
      o_acc[d][0] *= alpha[0]; o_acc[d][1] *= alpha[0];
      o_acc[d][2] *= alpha[1]; o_acc[d][3] *= alpha[1];
    }
    // P = exp2(x - m), rounded to bf16 for the PV product; l sums the rounded P.
    uint32_t pf[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float p0 = exp2f(s[nt][0] - m_r[0]);
      float p1 = exp2f(s[nt][1] - m_r[0]);
      float p2 = exp2f(s[nt][2] - m_r[1]);
      float p3 = exp2f(s[nt][3] - m_r[1]);
      uint32_t lo = pack_bf16(p0, p1), hi = pack_bf16(p2, p3);
      __nv_bfloat162 blo = *reinterpret_cast<__nv_bfloat162*>(&lo);
      __nv_bfloat162 bhi = *reinterpret_cast<__nv_bfloat162*>(&hi);
      float2 flo = __bfloat1622float2(blo), fhi = __bfloat1622float2(bhi);
      l_r[0] += flo.x + flo.y;
      l_r[1] += fhi.x + fhi.y;
      pf[nt >> 1][(nt & 1) * 2 + 0] = lo;
      pf[nt >> 1][(nt & 1) * 2 + 1] = hi;
    }
    // O += P V_j.
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4] = {pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3]};
#pragma unroll
      for (int dt = 0; dt < NDT; dt += 2) {
        int r = 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1);
        int c = dt + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + swz<VCPR>(r, c), b0, b1, b2, b3);
        mma_bf16(o_acc[dt], a, b0, b1);
        mma_bf16(o_acc[dt + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // Finalise: row sums across the quad, normalise, stage O in smem, store.
  float inv[2], lse2[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float l = l_r[h];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    inv[h] = l > 0.f ? 1.f / l : 0.f;
    lse2[h] = l > 0.f ? m_r[h] + log2f(l) : -INFINITY;
  }
  __syncthreads();
  uint8_t* sO = sK;  // reuse stage memory: 64 x D bf16
#pragma unroll
  for (int dt = 0; dt < NDT; ++dt) {
    int r0 = warp * 16 + gq;
    int col = dt * 8 + qd * 2;
    uint32_t lo = pack_bf16(o_acc[dt][0] * inv[0], o_acc[dt][1] * inv[0]);
    uint32_t hi = pack_bf16(o_acc[dt][2] * inv[1], o_acc[dt][3] * inv[1]);
    *reinterpret_cast<uint32_t*>(sO + swz<VCPR>(r0, col / 8) + (col % 8) * 2) = lo;
    *reinterpret_cast<uint32_t*>(sO + swz<VCPR>(r0 + 8, col / 8) + (col % 8) * 2) = hi;
  }
  if (P.lse && qd == 0) {
    float* lse = P.lse + (bh * g.N + i) * 64;
    lse[warp * 16 + gq] = lse2[0] * 0.69314718055994531f;
    lse[warp * 16 + gq + 8] = lse2[1] * 0.69314718055994531f;
  }
  __syncthreads();
  uint4* og = reinterpret_cast<uint4*>(P.o + (bh * g.N + i) * 64 * D);
#pragma unroll
  for (int e = 0; e < 64 * VCPR / 128; ++e) {
    int lin = threadIdx.x + 128 * e;
    int r = lin / VCPR, c = lin % VCPR;
    og[lin] = *reinterpret_cast<const uint4*>(sO + swz<VCPR>(r, c));
  }
}

template <int D, bool FP8>
bsattn_status run(const AttnParams& prm, cudaStream_t st) {
  constexpr int QB = FP8 ? 1 : 2;
  constexpr int smem = 64 * D * QB * 3 + 64 * D * 2 * 2;
  auto kern = attn_mma_kernel<D, FP8>;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return BSATTN_ERR_CUDA;
  }
  dim3 grid(prm.g.N, prm.g.Hh, prm.g.B);
  kern<<<grid, 128, smem, st>>>(prm);
  return cudaGetLastError() == cudaSuccess ? BSATTN_OK : BSATTN_ERR_CUDA;
}

}  // namespace

size_t attention_workspace_bytes(const bsattn_plan*) { return 0; }

bsattn_status launch_attention(const bsattn_plan* p, const void* q, const void* k, const float* qs,
                               const float* ks, const __nv_bfloat16* v, const int32_t* idx,
                               const int32_t* cnt, __nv_bfloat16* o, float* lse, void*, size_t,
                               cudaStream_t st) {
  AttnParams prm;
  prm.g = make_geom(p);
  prm.q = static_cast<const uint8_t*>(q);
  prm.k = static_cast<const uint8_t*>(k);
  prm.qs = qs;
  prm.ks = ks;
  prm.v = v;
  prm.idx = idx;
  prm.cnt = cnt;
  prm.kmax = p->kmax;
  prm.o = o;
  prm.lse = lse;
  prm.scale_log2 = p->scale * 1.4426950408889634f;
  prm.err = p->d_err;
  const bool fp8 = p->desc.qk_fp8 != 0;
  if (p->desc.head_dim == 128) return fp8 ? run<128, true>(prm, st) : run<128, false>(prm, st);
  return fp8 ? run<64, true>(prm, st) : run<64, false>(prm, st);
}
