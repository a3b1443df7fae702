// Denoising-step-aware plan schedule (FPSAttention page, Approach: the
// quantisation tile size and the sparsity window change between the early,
// middle and late denoising steps). A schedule is an ordered list of plans
// over the same tensors; entry i serves the steps [first_step_i,
// first_step_{i+1}) and the last entry every later step. Host code only: it
// picks a plan and hands the call to attn_layer.
#include <new>
#include <vector>

#include "internal.h"

struct bsattn_schedule {
  std::vector<int> first;            // first step of each entry, ascending, first[0] = 0
  std::vector<bsattn_plan*> plans;   // owned
  size_t layer_ws;                   // max over plans of info.layer_workspace_bytes
};

static bool same_tensors(const bsattn_desc& a, const bsattn_desc& b) {
  return a.B == b.B && a.heads == b.heads && a.head_dim == b.head_dim && a.T == b.T && a.H == b.H &&
         a.W == b.W;
}

bsattn_status attn_schedule_create(const bsattn_schedule_entry* e, int n, bsattn_schedule** out) {
  if (!e || !out || n < 1 || n > BSATTN_MAX_SCHEDULE) return BSATTN_ERR_INVALID_ARG;
  *out = nullptr;
  if (e[0].first_step != 0) return BSATTN_ERR_INVALID_ARG;
  for (int i = 1; i < n; ++i)
    if (e[i].first_step <= e[i - 1].first_step || !same_tensors(e[i].desc, e[0].desc))
      return BSATTN_ERR_INVALID_ARG;
  bsattn_schedule* s = new (std::nothrow) bsattn_schedule();
  if (!s) return BSATTN_ERR_INTERNAL;
  s->layer_ws = 0;
  for (int i = 0; i < n; ++i) {
    bsattn_plan* p = nullptr;
    const bsattn_status st = attn_plan_create(&e[i].desc, &e[i].rule, &p);
    if (st != BSATTN_OK) {
      attn_schedule_destroy(s);
      return st;
    }
    s->plans.push_back(p);
    s->first.push_back(e[i].first_step);
    bsattn_info info;
    attn_plan_info(p, &info);
    if (info.layer_workspace_bytes > s->layer_ws) s->layer_ws = info.layer_workspace_bytes;
  }
  *out = s;
  return BSATTN_OK;
}

void attn_schedule_destroy(bsattn_schedule* s) {
  if (!s) return;
  for (bsattn_plan* p : s->plans) attn_plan_destroy(p);
  delete s;
}

bsattn_status attn_schedule_plan(const bsattn_schedule* s, int step, const bsattn_plan** plan) {
  if (!s || !plan || step < 0) return BSATTN_ERR_INVALID_ARG;
  size_t i = s->first.size() - 1;
  while (s->first[i] > step) --i;  // first[0] = 0 <= step ends the walk
  *plan = s->plans[i];
  return BSATTN_OK;
}

bsattn_status attn_schedule_workspace_bytes(const bsattn_schedule* s, size_t* bytes) {
  if (!s || !bytes) return BSATTN_ERR_INVALID_ARG;
  *bytes = s->layer_ws;
  return BSATTN_OK;
}

bsattn_status attn_schedule_layer(const bsattn_schedule* s, int step, const void* q_nat,
                                  const void* k_nat, const void* v_nat, void* o_nat, float* lse_nat,
                                  int32_t* idx_out, int32_t* cnt_out, void* ws, size_t ws_bytes,
                                  void* stream) {
  const bsattn_plan* p = nullptr;
  const bsattn_status st = attn_schedule_plan(s, step, &p);
  if (st != BSATTN_OK) return st;
  return attn_layer(p, q_nat, k_nat, v_nat, o_nat, lse_nat, idx_out, cnt_out, ws, ws_bytes, stream);
}
