// The whole layer with its scratch in a fixed, load-time device array, for
// callers that must not allocate device memory on their call path.
//
// Who needs it: inference servers that reserve device memory once at start-up
// and forbid allocation while serving (cudaMalloc can synchronise the device,
// stalling every stream, and fragments a tuned pool); real-time pipelines
// with a fixed latency budget per frame; hosts where another component owns
// all device memory.  Such a caller creates its plan during set-up
// (ug_plan_create allocates then) and afterwards calls
// ug_layer_fwd_static_scratch, which allocates nothing: the window-first
// intermediates live in g_layer_scratch below, which every GPU that loads
// this library holds until the process exits.
#include <cstdint>

#include "ug_internal.h"
#include "ug_per_device.h"

namespace {

constexpr int64_t kScratchBytes = UG_STATIC_SCRATCH_BYTES;

// Device-side scratch.  In host code this name is only a host-side stand-in
// for the symbol, not a device address; the device address comes from
// cudaGetSymbolAddress below, per device.
__device__ __align__(256) unsigned char g_layer_scratch[kScratchBytes];

// Device address of g_layer_scratch, per device.
ug::PerDevice<void*> g_scratch_ptr;

}  // namespace

namespace ug {

// Looks up the scratch's device address with `device` current and caches it.
// ug_plan_create calls this during set-up: under lazy module loading the
// lookup is what loads this module (and places the array), so it happens
// there, not on the allocation-free call path.
int prepare_static_scratch(int device) {
  return g_scratch_ptr.get(device, [](void*& ptr) {
    if (cudaGetSymbolAddress(&ptr, g_layer_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return (int)UG_ERR_CUDA;
    }
    return (int)UG_OK;
  });
}

}  // namespace ug

extern "C" int ug_layer_fwd_static_scratch(const ug_plan* p, const void* q_hr, const void* k_hr,
                                           const void* v_hr, const void* q_lr, const void* k_lr,
                                           const void* v_lr, void* o_hr, void* o_lr, float* lse,
                                           void* stream) {
  if (!p) return UG_ERR_INVALID_ARG;
  const int64_t need = ug_layer_workspace_bytes(p);
  if (need > kScratchBytes) return UG_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return UG_ERR_CUDA;
  if (dev != p->device) return UG_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int st = g_scratch_ptr.get(dev, [](void*&) { return (int)UG_ERR_CUDA; }, &scratch);
  if (st != UG_OK) return st;  // set-up (ug_plan_create on this device) has not succeeded
  // Every byte of the scratch that the layer reads it first writes in the
  // same call, so nothing needs clearing between calls.
  return ug_layer_fwd(p, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse, scratch, need,
                      stream);
}
