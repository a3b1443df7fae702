// attn_select with library-owned scratch, for callers that cannot allocate
// device memory. The scratch is one file-scope device array; host code must
// not pass the array's name to a kernel (on the host it names a shadow, not
// device memory), so its device address is looked up per device with
// cudaGetSymbolAddress and cached.
//
// This file holds no kernel, so with lazy module loading (the CUDA 12 default)
// the array is reserved on a device only when the first lookup there loads
// the module. attn_plan_create makes that lookup, with the plan's device
// current, so a call of attn_select_static never loads modules or reserves
// memory itself.
#include <mutex>

#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_select_scratch[BSATTN_STATIC_SELECT_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_select_scratch on `device`, which must be current.
bsattn_status scratch_address(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return BSATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[device]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || !p) return BSATTN_ERR_CUDA;
    g_addr[device] = p;
  }
  *out = g_addr[device];
  return BSATTN_OK;
}

}  // namespace

bsattn_status bsattn_static_scratch_prepare(int device) {
  void* p = nullptr;
  return scratch_address(device, &p);
}

extern "C" bsattn_status attn_select_static(const bsattn_plan* p, const void* q_nat,
                                            const void* k_nat, int32_t* idx, int32_t* cnt,
                                            void* stream) {
  if (!p) return BSATTN_ERR_INVALID_ARG;
  bsattn_info info;
  bsattn_status s = attn_plan_info(p, &info);
  if (s) return s;
  if (info.select_workspace_bytes > BSATTN_STATIC_SELECT_SCRATCH_BYTES) return BSATTN_ERR_UNSUPPORTED;
  // The window rule reads no scratch: its lists come from the plan.
  if (info.select_workspace_bytes == 0) return attn_select(p, q_nat, k_nat, idx, cnt, nullptr, 0, stream);
  DeviceGuard dev(p->device);
  if (dev.status) return dev.status;
  void* ws = nullptr;
  if ((s = scratch_address(p->device, &ws))) return s;
  return attn_select(p, q_nat, k_nat, idx, cnt, ws, BSATTN_STATIC_SELECT_SCRATCH_BYTES, stream);
}
