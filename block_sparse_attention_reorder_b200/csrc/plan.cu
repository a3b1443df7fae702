// Plans, argument checking and the C ABI entry points. Host code only: every
// step of the computation runs in the kernels of the other translation units.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <new>
#include <vector>

#include "internal.h"

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Carves sub-buffers out of a caller-provided workspace, 256-byte aligned.
struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* b) : base(static_cast<char*>(b)) {}
  void* take(size_t bytes) {
    off = align_up(off, 256);
    void* p = base ? base + off : nullptr;
    off += bytes;
    return p;
  }
};

struct SelectWs {
  float* pq;
  float* pk;
  float* S;
  int32_t* fb_rows;  // top-k: rows attn_select_fused hands to the row-wise selection
  int* fb_count;
};

SelectWs carve_select(const bsattn_plan* p, Carve& c) {
  size_t bh = (size_t)p->desc.B * p->desc.heads;
  SelectWs w;
  w.pq = (float*)c.take(bh * p->N * p->desc.head_dim * sizeof(float));
  w.pk = (float*)c.take(bh * p->N * p->desc.head_dim * sizeof(float));
  w.S = (float*)c.take(bh * p->N * p->N * sizeof(float));
  const bool topk = p->rule.kind == BSATTN_RULE_TOPK;
  w.fb_rows = (int32_t*)c.take(topk ? bh * p->N * sizeof(int32_t) : 0);
  w.fb_count = (int*)c.take(topk ? sizeof(int) : 0);
  return w;
}

// The layer reads Q, K, V and writes O in the natural layout; e4m3 Q/K codes
// (with their tile scales) are tiled.
struct LayerWs {
  uint8_t* qt;  // e4m3 tile codes (qk_fp8 only)
  uint8_t* kt;
  float* qs;
  float* ks;
  SelectWs sel;
  int32_t* idx;
  int32_t* cnt;
  void* attn_ws;
};

LayerWs carve_layer(const bsattn_plan* p, Carve& c) {
  size_t bh = (size_t)p->desc.B * p->desc.heads;
  size_t elems = bh * p->N * p->V * p->desc.head_dim;
  LayerWs w;
  w.qt = (uint8_t*)c.take(p->desc.qk_fp8 ? elems : 0);
  w.kt = (uint8_t*)c.take(p->desc.qk_fp8 ? elems : 0);
  w.qs = (float*)c.take(p->desc.qk_fp8 ? bh * p->N * sizeof(float) : 0);
  w.ks = (float*)c.take(p->desc.qk_fp8 ? bh * p->N * sizeof(float) : 0);
  if (p->rule.kind == BSATTN_RULE_WINDOW) {
    w.sel.pq = w.sel.pk = w.sel.S = nullptr;
  } else {
    w.sel = carve_select(p, c);
  }
  w.idx = (int32_t*)c.take(bh * p->N * p->kmax * sizeof(int32_t));
  w.cnt = (int32_t*)c.take(bh * p->N * sizeof(int32_t));
  w.attn_ws = c.take(attention_workspace_bytes(p));
  return w;
}

BackwardWs carve_backward(const bsattn_plan* p, Carve& c) {
  const size_t rows = (size_t)p->desc.B * p->desc.heads * p->N;
  BackwardWs w;
  w.delta = (float*)c.take(rows * p->V * sizeof(float));
  w.bm = (uint32_t*)c.take(rows * ((p->N + 31) / 32) * sizeof(uint32_t));
  w.idxT = (int32_t*)c.take(rows * p->N * sizeof(int32_t));
  w.cntT = (int32_t*)c.take(rows * sizeof(int32_t));
  return w;
}

bool ok_ptr(const void* x) { return x != nullptr && aligned16(x); }


std::atomic<int> g_force_timeout{0};

}  // namespace

bool bsattn_testing_timeout_forced() { return g_force_timeout.load(std::memory_order_relaxed) != 0; }

extern "C" {

bsattn_status attn_testing_force_timeout(int on) {
  g_force_timeout.store(on ? 1 : 0, std::memory_order_relaxed);
  return BSATTN_OK;
}

bsattn_status attn_testing_set_error_word(const bsattn_plan* p, int bits) {
  if (!p) return BSATTN_ERR_INVALID_ARG;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  BSATTN_CUDA_TRY(cudaMemcpy(p->d_err, &bits, sizeof(int), cudaMemcpyHostToDevice));
  return BSATTN_OK;
}

const char* attn_status_string(bsattn_status s) {
  switch (s) {
    case BSATTN_OK: return "ok";
    case BSATTN_ERR_INVALID_ARG: return "invalid argument";
    case BSATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case BSATTN_ERR_CUDA: return "CUDA error";
    case BSATTN_ERR_TIMEOUT: return "device wait timed out";
    case BSATTN_ERR_INTERNAL: return "device reported a bad kept-list entry";
    case BSATTN_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

// Box (ct, ch, cw) of 64 tokens covering in-tile rows [64c, 64c + 64) of a
// (tt, th, tw) tile in (dt, dh, dw) row-major order, if those rows form a box
// for every c: whole (dh, dw) planes, whole dw rows, or 64-wide dw runs.
static bool chunk_box(int tt, int th, int tw, int* ct, int* ch, int* cw) {
  if (th * tw <= 64) {
    if (64 % (th * tw) != 0 || tt % (64 / (th * tw)) != 0) return false;
    *ct = 64 / (th * tw); *ch = th; *cw = tw;
    return true;
  }
  if (tw <= 64) {
    if (64 % tw != 0 || th % (64 / tw) != 0) return false;
    *ct = 1; *ch = 64 / tw; *cw = tw;
    return true;
  }
  if (tw % 64 != 0) return false;
  *ct = 1; *ch = 1; *cw = 64;
  return true;
}

bsattn_status attn_plan_create(const bsattn_desc* d, const bsattn_rule* r, bsattn_plan** out) {
  if (!d || !r || !out) return BSATTN_ERR_INVALID_ARG;
  *out = nullptr;
  if (d->B < 1 || d->heads < 1 || d->T < 1 || d->H < 1 || d->W < 1 || d->tile_t < 1 ||
      d->tile_h < 1 || d->tile_w < 1 || d->head_dim < 1)
    return BSATTN_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return BSATTN_ERR_UNSUPPORTED;
  // Tiles of 64 * nchunk tokens whose 64-row chunks are boxes of the tile.
  // Tiles of fewer than 64 tokens are one chunk box, stored as 64 rows of
  // which the last 64 - V are padding.
  int ct, ch, cw;
  const long long vol = (long long)d->tile_t * d->tile_h * d->tile_w;
  if (vol < 64) {
    ct = d->tile_t; ch = d->tile_h; cw = d->tile_w;
  } else {
    if (vol % 64 != 0 || vol > 64LL * kMaxChunks) return BSATTN_ERR_UNSUPPORTED;
    if (d->tile_t > 1024 || d->tile_h > 1024 || d->tile_w > 1024) return BSATTN_ERR_UNSUPPORTED;
    if (!chunk_box(d->tile_t, d->tile_h, d->tile_w, &ct, &ch, &cw)) return BSATTN_ERR_UNSUPPORTED;
  }
  if (d->qk_fp8 != 0 && d->qk_fp8 != 1) return BSATTN_ERR_INVALID_ARG;
  long long Tp = (d->T + d->tile_t - 1) / d->tile_t * (long long)d->tile_t;
  long long Hp = (d->H + d->tile_h - 1) / d->tile_h * (long long)d->tile_h;
  long long Wp = (d->W + d->tile_w - 1) / d->tile_w * (long long)d->tile_w;
  long long N = (Tp / d->tile_t) * (Hp / d->tile_h) * (Wp / d->tile_w);
  long long L = (long long)d->T * d->H * d->W;
  if (N > (1 << 20) || L > (1LL << 30) / d->heads) return BSATTN_ERR_UNSUPPORTED;
  // Tiled row coordinates (B * heads * Tp * Hp * Wp rows) stay within int32.
  if ((long long)d->B * d->heads * Tp * Hp * Wp >= (1LL << 31)) return BSATTN_ERR_UNSUPPORTED;

  int kmax = 0;
  switch (r->kind) {
    case BSATTN_RULE_TOPK:
      if (r->k < 1 || r->k > N) return BSATTN_ERR_INVALID_ARG;
      if (N > 2048) return BSATTN_ERR_UNSUPPORTED;
      kmax = r->k;
      break;
    case BSATTN_RULE_TOPP:
      if (r->k < 0 || r->k > N || !(r->p > 0.0 && r->p <= 1.0)) return BSATTN_ERR_INVALID_ARG;
      if (N > 2048) return BSATTN_ERR_UNSUPPORTED;
      kmax = (int)N;
      break;
    case BSATTN_RULE_WINDOW: {
      if (r->win_t < 0 || r->win_h < 0 || r->win_w < 0) return BSATTN_ERR_INVALID_ARG;
      long long a = 2LL * r->win_t + 1, b = 2LL * r->win_h + 1, c = 2LL * r->win_w + 1;
      long long nt = Tp / d->tile_t, nh = Hp / d->tile_h, nw = Wp / d->tile_w;
      kmax = (int)((a < nt ? a : nt) * (b < nh ? b : nh) * (c < nw ? c : nw));
      break;
    }
    default:
      return BSATTN_ERR_INVALID_ARG;
  }

  bsattn_plan* p = new (std::nothrow) bsattn_plan();
  if (!p) return BSATTN_ERR_INTERNAL;
  p->desc = *d;
  p->rule = *r;
  p->Tp = (int)Tp; p->Hp = (int)Hp; p->Wp = (int)Wp;
  p->nT = (int)(Tp / d->tile_t); p->nH = (int)(Hp / d->tile_h); p->nW = (int)(Wp / d->tile_w);
  p->N = (int)N; p->L = (int)L; p->kmax = kmax;
  p->V = vol < 64 ? 64 : (int)vol;  // rows per tile in the tiled layout
  p->nchunk = p->V / 64;
  p->ct = ct; p->ch = ch; p->cw = cw;
  p->scale = d->softmax_scale > 0.f ? d->softmax_scale : (float)(1.0 / sqrt((double)d->head_dim));
  if (cudaGetDevice(&p->device) != cudaSuccess) { delete p; return BSATTN_ERR_CUDA; }
  if (cudaMalloc(&p->d_err, sizeof(int)) != cudaSuccess) { delete p; return BSATTN_ERR_CUDA; }
  if (cudaMemset(p->d_err, 0, sizeof(int)) != cudaSuccess) {
    attn_plan_destroy(p);
    return BSATTN_ERR_CUDA;
  }
  // Load attn_select_static's scratch array here, where the caller can
  // allocate, so that the selection call itself reserves nothing. A failure
  // is not the plan's: attn_select_static retries and reports it.
  bsattn_static_scratch_prepare(p->device);
  if (r->kind == BSATTN_RULE_WINDOW) {
    // Closed-form clipped window lists, ascending because j grows with
    // (t, h, w) in row-major tile order.
    std::vector<int32_t> idx((size_t)N * kmax, -1), cnt((size_t)N, 0);
    for (int i = 0; i < N; ++i) {
      int ti = i / (p->nH * p->nW), hi = (i / p->nW) % p->nH, wi = i % p->nW;
      int c = 0;
      for (int t = ti - r->win_t; t <= ti + r->win_t; ++t)
        for (int h = hi - r->win_h; h <= hi + r->win_h; ++h)
          for (int w = wi - r->win_w; w <= wi + r->win_w; ++w) {
            if (t < 0 || h < 0 || w < 0 || t >= p->nT || h >= p->nH || w >= p->nW) continue;
            idx[(size_t)i * kmax + c++] = (t * p->nH + h) * p->nW + w;
          }
      cnt[i] = c;
    }
    if (cudaMalloc(&p->d_win_idx, idx.size() * 4) != cudaSuccess ||
        cudaMalloc(&p->d_win_cnt, cnt.size() * 4) != cudaSuccess ||
        cudaMemcpy(p->d_win_idx, idx.data(), idx.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(p->d_win_cnt, cnt.data(), cnt.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess) {
      attn_plan_destroy(p);
      return BSATTN_ERR_CUDA;
    }
  }
  *out = p;
  return BSATTN_OK;
}

void attn_plan_destroy(bsattn_plan* p) {
  if (!p) return;
  int cur = -1;
  cudaGetDevice(&cur);
  if (cur != p->device) cudaSetDevice(p->device);
  if (p->d_err) cudaFree(p->d_err);
  if (p->d_win_idx) cudaFree(p->d_win_idx);
  if (p->d_win_cnt) cudaFree(p->d_win_cnt);
  if (cur >= 0 && cur != p->device) cudaSetDevice(cur);
  delete p;
}

bsattn_status attn_plan_info(const bsattn_plan* p, bsattn_info* o) {
  if (!p || !o) return BSATTN_ERR_INVALID_ARG;
  memset(o, 0, sizeof(*o));
  o->Tp = p->Tp; o->Hp = p->Hp; o->Wp = p->Wp;
  o->nT = p->nT; o->nH = p->nH; o->nW = p->nW;
  o->n_blocks = p->N; o->tile_volume = p->V; o->kmax = p->kmax;
  o->softmax_scale = p->scale;
  {
    Carve c(nullptr);
    if (p->rule.kind != BSATTN_RULE_WINDOW) carve_select(p, c);
    o->select_workspace_bytes = align_up(c.off, 256);
  }
  o->forward_workspace_bytes = attention_workspace_bytes(p);
  {
    Carve c(nullptr);
    carve_layer(p, c);
    o->layer_workspace_bytes = align_up(c.off, 256);
  }
  {
    Carve c(nullptr);
    carve_backward(p, c);
    o->backward_workspace_bytes = align_up(c.off, 256);
  }
  return BSATTN_OK;
}

bsattn_status attn_reorder(const bsattn_plan* p, const void* x_nat, void* x_tiled, float* pooled,
                           void* stream) {
  if (!p || !ok_ptr(x_nat) || !ok_ptr(x_tiled) || (pooled && !aligned16(pooled)))
    return BSATTN_ERR_INVALID_ARG;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  Geom g = make_geom(p);
  if ((s = launch_reorder(g, (const __nv_bfloat16*)x_nat, (__nv_bfloat16*)x_tiled, (cudaStream_t)stream)))
    return s;
  return pooled ? launch_pool(g, (const __nv_bfloat16*)x_nat, pooled, nullptr, nullptr, (cudaStream_t)stream)
                : BSATTN_OK;
}

bsattn_status attn_pool(const bsattn_plan* p, const void* x_nat, float* pooled, void* stream) {
  if (!p || !ok_ptr(x_nat) || !ok_ptr(pooled)) return BSATTN_ERR_INVALID_ARG;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  return launch_pool(make_geom(p), (const __nv_bfloat16*)x_nat, pooled, nullptr, nullptr,
                     (cudaStream_t)stream);
}

bsattn_status attn_unreorder(const bsattn_plan* p, const void* x_tiled, void* x_nat,
                             void* stream) {
  if (!p || !ok_ptr(x_tiled) || !ok_ptr(x_nat)) return BSATTN_ERR_INVALID_ARG;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  return launch_unreorder(make_geom(p), (const __nv_bfloat16*)x_tiled, (__nv_bfloat16*)x_nat,
                          nullptr, nullptr, (cudaStream_t)stream);
}

bsattn_status attn_block_scores(const bsattn_plan* p, const float* pq, const float* pk,
                                float* S, void* stream) {
  if (!p || !ok_ptr(pq) || !ok_ptr(pk) || !ok_ptr(S)) return BSATTN_ERR_INVALID_ARG;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  return launch_block_scores(make_geom(p), pq, pk, p->scale, S, p->d_err, (cudaStream_t)stream);
}

static bsattn_status select_core(const bsattn_plan* p, const float* S, int32_t* idx,
                                 int32_t* cnt, cudaStream_t st) {
  int rows = p->desc.B * p->desc.heads * p->N;
  switch (p->rule.kind) {
    case BSATTN_RULE_TOPK:
      return launch_select_topk(rows, p->N, p->rule.k, S, idx, cnt, p->kmax, st);
    case BSATTN_RULE_TOPP:
      return launch_select_topp(rows, p->N, p->rule.k, p->rule.p, S, idx, cnt, p->kmax, st);
    default:
      return launch_broadcast_lists(p->desc.B * p->desc.heads, p->N, p->kmax, p->d_win_idx,
                                    p->d_win_cnt, idx, cnt, st);
  }
}

bsattn_status attn_select_from_scores(const bsattn_plan* p, const float* S, int32_t* idx,
                                      int32_t* cnt, void* stream) {
  if (!p || !ok_ptr(idx) || !ok_ptr(cnt)) return BSATTN_ERR_INVALID_ARG;
  if (p->rule.kind != BSATTN_RULE_WINDOW && !ok_ptr(S)) return BSATTN_ERR_INVALID_ARG;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  return select_core(p, S, idx, cnt, (cudaStream_t)stream);
}

bsattn_status attn_select(const bsattn_plan* p, const void* q_nat, const void* k_nat,
                          int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
  if (!p || !ok_ptr(idx) || !ok_ptr(cnt)) return BSATTN_ERR_INVALID_ARG;
  bsattn_info info;
  attn_plan_info(p, &info);
  cudaStream_t st = (cudaStream_t)stream;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  if (p->rule.kind == BSATTN_RULE_WINDOW) return select_core(p, nullptr, idx, cnt, st);
  if (!ok_ptr(q_nat) || !ok_ptr(k_nat)) return BSATTN_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws) || ws_bytes < info.select_workspace_bytes) return BSATTN_ERR_WORKSPACE;
  Carve c(ws);
  SelectWs w = carve_select(p, c);
  Geom g = make_geom(p);
  if ((s = launch_pool(g, (const __nv_bfloat16*)q_nat, w.pq, (const __nv_bfloat16*)k_nat, w.pk, st))) return s;
  if ((s = launch_block_scores(g, w.pq, w.pk, p->scale, w.S, p->d_err, st))) return s;
  return select_core(p, w.S, idx, cnt, st);
}

bsattn_status attn_select_fused(const bsattn_plan* p, const void* q_nat, const void* k_nat, int32_t* idx,
                                int32_t* cnt, float* scores_debug, void* ws, size_t ws_bytes, void* stream) {
  if (!p || !ok_ptr(idx) || !ok_ptr(cnt) || (scores_debug && !aligned16(scores_debug)))
    return BSATTN_ERR_INVALID_ARG;
  if (p->rule.kind == BSATTN_RULE_TOPP) return BSATTN_ERR_UNSUPPORTED;
  bsattn_info info;
  attn_plan_info(p, &info);
  cudaStream_t st = (cudaStream_t)stream;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  if (p->rule.kind == BSATTN_RULE_WINDOW) return select_core(p, nullptr, idx, cnt, st);
  if (!ok_ptr(q_nat) || !ok_ptr(k_nat)) return BSATTN_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws) || ws_bytes < info.select_workspace_bytes) return BSATTN_ERR_WORKSPACE;
  Carve c(ws);
  SelectWs w = carve_select(p, c);
  Geom g = make_geom(p);
  if ((s = launch_pool(g, (const __nv_bfloat16*)q_nat, w.pq, (const __nv_bfloat16*)k_nat, w.pk, st))) return s;
  return launch_fused_topk(g, w.pq, w.pk, p->scale, p->rule.k, p->kmax, idx, cnt,
                           scores_debug ? scores_debug : w.S, scores_debug != nullptr, w.fb_rows, w.fb_count,
                           p->d_err, st);
}

bsattn_status attn_quantize_e4m3(const bsattn_plan* p, const void* x_tiled, uint8_t* codes,
                                 float* scales, void* stream) {
  if (!p || !ok_ptr(x_tiled) || !ok_ptr(codes) || !ok_ptr(scales)) return BSATTN_ERR_INVALID_ARG;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  return launch_quant_tiled(make_geom(p), (const __nv_bfloat16*)x_tiled, codes, scales,
                            (cudaStream_t)stream);
}

bsattn_status attn_forward(const bsattn_plan* p, const void* q, const void* k, const float* qs,
                           const float* ks, const void* v, const int32_t* idx, const int32_t* cnt,
                           void* o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!p || !ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(idx) || !ok_ptr(cnt) || !ok_ptr(o) ||
      (lse && !aligned16(lse)))
    return BSATTN_ERR_INVALID_ARG;
  if (p->desc.qk_fp8 && (!ok_ptr(qs) || !ok_ptr(ks))) return BSATTN_ERR_INVALID_ARG;
  size_t need = attention_workspace_bytes(p);
  if (need && (!ws || !aligned16(ws) || ws_bytes < need)) return BSATTN_ERR_WORKSPACE;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  return launch_attention(p, q, k, qs, ks, (const __nv_bfloat16*)v, idx, cnt, (__nv_bfloat16*)o,
                          lse, ws, ws_bytes, (cudaStream_t)stream, AttnLayout::Tiled);
}

bsattn_status attn_backward(const bsattn_plan* p, const void* q, const void* k, const void* v, const void* o,
                            const void* d_o, const float* lse, const int32_t* idx, const int32_t* cnt, void* dq,
                            void* dk, void* dv, void* ws, size_t ws_bytes, void* stream) {
  if (!p || !ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(o) || !ok_ptr(d_o) || !ok_ptr(lse) ||
      !ok_ptr(idx) || !ok_ptr(cnt) || !ok_ptr(dq) || !ok_ptr(dk) || !ok_ptr(dv))
    return BSATTN_ERR_INVALID_ARG;
  if (p->desc.qk_fp8) return BSATTN_ERR_UNSUPPORTED;
  bsattn_info info;
  attn_plan_info(p, &info);
  if (!ws || !aligned16(ws) || ws_bytes < info.backward_workspace_bytes) return BSATTN_ERR_WORKSPACE;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  Carve c(ws);
  const BackwardWs w = carve_backward(p, c);
  return launch_backward(p, q, k, v, o, d_o, lse, idx, cnt, dq, dk, dv, w, (cudaStream_t)stream);
}

bsattn_status attn_forward_natural(const bsattn_plan* p, const void* q, const void* k, const float* qs,
                                   const float* ks, const void* v_nat, const int32_t* idx,
                                   const int32_t* cnt, void* o_nat, float* lse_nat, void* ws,
                                   size_t ws_bytes, void* stream) {
  if (!p || !ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v_nat) || !ok_ptr(idx) || !ok_ptr(cnt) ||
      !ok_ptr(o_nat) || (lse_nat && !aligned16(lse_nat)))
    return BSATTN_ERR_INVALID_ARG;
  if (p->desc.qk_fp8 && (!ok_ptr(qs) || !ok_ptr(ks))) return BSATTN_ERR_INVALID_ARG;
  size_t need = attention_workspace_bytes(p);
  if (need && (!ws || !aligned16(ws) || ws_bytes < need)) return BSATTN_ERR_WORKSPACE;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  return launch_attention(p, q, k, qs, ks, (const __nv_bfloat16*)v_nat, idx, cnt, (__nv_bfloat16*)o_nat,
                          lse_nat, ws, ws_bytes, (cudaStream_t)stream, AttnLayout::Natural);
}

bsattn_status attn_layer(const bsattn_plan* p, const void* q_nat, const void* k_nat,
                         const void* v_nat, void* o_nat, float* lse_nat, int32_t* idx_out,
                         int32_t* cnt_out, void* ws, size_t ws_bytes, void* stream) {
  if (!p || !ok_ptr(q_nat) || !ok_ptr(k_nat) || !ok_ptr(v_nat) || !ok_ptr(o_nat) ||
      (lse_nat && !aligned16(lse_nat)) || (idx_out && !aligned16(idx_out)) ||
      (cnt_out && !aligned16(cnt_out)) || ((idx_out == nullptr) != (cnt_out == nullptr)))
    return BSATTN_ERR_INVALID_ARG;
  bsattn_info info;
  attn_plan_info(p, &info);
  if (!ws || !aligned16(ws) || ws_bytes < info.layer_workspace_bytes) return BSATTN_ERR_WORKSPACE;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  cudaStream_t st = (cudaStream_t)stream;
  Carve c(ws);
  LayerWs w = carve_layer(p, c);
  Geom g = make_geom(p);
  int32_t* idx = idx_out ? idx_out : w.idx;
  int32_t* cnt = cnt_out ? cnt_out : w.cnt;
  bool pool = p->rule.kind != BSATTN_RULE_WINDOW;
  const void* q = q_nat;
  const void* k = k_nat;
  if (p->desc.qk_fp8) {
    // e4m3 tile codes and scales.
    if ((s = launch_reorder_quant(g, (const __nv_bfloat16*)q_nat, (const __nv_bfloat16*)k_nat, w.qt, w.kt, w.qs,
                                  w.ks, st)))
      return s;
    q = w.qt;
    k = w.kt;
  }
  // Tile means for the scores; the attention reads natural tensors tile by tile.
  if (pool && (s = launch_pool(g, (const __nv_bfloat16*)q_nat, w.sel.pq, (const __nv_bfloat16*)k_nat, w.sel.pk, st)))
    return s;
  if (pool && (s = launch_block_scores(g, w.sel.pq, w.sel.pk, p->scale, w.sel.S, p->d_err, st))) return s;
  if ((s = select_core(p, w.sel.S, idx, cnt, st))) return s;
  return launch_attention(p, q, k, w.qs, w.ks, (const __nv_bfloat16*)v_nat, idx, cnt, (__nv_bfloat16*)o_nat,
                          lse_nat, w.attn_ws, attention_workspace_bytes(p), st, AttnLayout::Natural);
}

bsattn_status attn_check_device_status(const bsattn_plan* p, void* stream) {
  if (!p) return BSATTN_ERR_INVALID_ARG;
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  bsattn_status s = BSATTN_OK;
  BSATTN_CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
  int h = 0;
  BSATTN_CUDA_TRY(cudaMemcpy(&h, p->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  if (h) BSATTN_CUDA_TRY(cudaMemset(p->d_err, 0, sizeof(int)));
  if (h & BSATTN_DEVERR_TIMEOUT) return BSATTN_ERR_TIMEOUT;
  if (h & BSATTN_DEVERR_BAD_INDEX) return BSATTN_ERR_INTERNAL;
  return BSATTN_OK;
}

}  // extern "C"
