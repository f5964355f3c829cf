// Forward entry point whose workspace is a fixed device array inside the
// library, for callers that cannot allocate device memory themselves.
//
// Such callers exist: plugin code run by a host framework that owns every
// device allocation and forbids cudaMalloc inside its execution callback, or
// code that must not risk the implicit device-wide synchronisation cudaMalloc
// and cudaFree may perform.  They still pass their own inputs and outputs; only
// the scratch the forward needs (block map, lists, fixed-m bound) comes from
// here.
#include <mutex>

#include "internal.h"

namespace {

// Upper bound of the forward workspace this entry point serves.  Every GPU that
// loads the library holds this much device memory until the process exits.
constexpr size_t kStaticScratchBytes = size_t{32} << 20;
constexpr int kMaxDevices = 64;

}  // namespace

static __device__ __align__(256) uint8_t g_bsa_static_scratch[kStaticScratchBytes];

namespace {

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the array for the current device.  The host-side name
// g_bsa_static_scratch is only a stand-in symbol, never a device address, so it
// is resolved once per device with that device current.  The first lookup on a
// device may load this library's device code there (lazy module loading),
// which is when the driver places the array in device memory.
bsa_status scratch_for_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return BSA_ERR_NO_DEVICE;
  if (dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bsa_static_scratch) != cudaSuccess || p == nullptr)
      return BSA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return BSA_OK;
}

}  // namespace

extern "C" bsa_status bsa_attn_fwd_static_scratch(const bsa_problem *prob,
                                                  const bsa_mask_spec *mask,
                                                  const bsa_options *opt, const void *q,
                                                  const void *k, const void *v, void *out,
                                                  float *lse, bsa_stream_t stream) {
  const bool empty = bsa::problem_is_empty(prob);
  if (!empty && (q == nullptr || k == nullptr || v == nullptr || out == nullptr || lse == nullptr))
    return BSA_ERR_INVALID_ARG;
  size_t need = 0;
  bsa_status st = bsa_workspace_size(prob, mask, 0, &need);
  if (st != BSA_OK) return st;
  // an empty problem still has its options checked, then does nothing
  if (empty) return bsa::attn_fwd_impl(prob, mask, opt, q, k, v, out, lse, nullptr, 0, stream, false);
  if (need > kStaticScratchBytes) return BSA_ERR_WORKSPACE_TOO_SMALL;
  void *ws = nullptr;
  if ((st = scratch_for_current_device(&ws)) != BSA_OK) return st;
  // the array keeps whatever the previous call left: always rebuild the plan
  // and the fixed-m bound (the planner clears the status word and counters)
  bsa_options o{};
  if (opt != nullptr) o = *opt;
  o.plan_ready = 0;
  o.bound_ready = 0;
  o.o_residual = BSA_O_RESIDUAL_DROP;  // no backward shares this scratch
  // plan and bound one after the other on `stream`: no side stream, no events
  return bsa::attn_fwd_impl(prob, mask, &o, q, k, v, out, lse, ws, kStaticScratchBytes, stream,
                            false);
}

extern "C" bsa_status bsa_static_scratch_init(void) {
  void *ws = nullptr;
  return scratch_for_current_device(&ws);
}

extern "C" bsa_status bsa_static_scratch_status(bsa_stream_t stream, int32_t clear) {
  void *ws = nullptr;
  const bsa_status st = scratch_for_current_device(&ws);
  if (st != BSA_OK) return st;
  // the array's first bytes are the workspace header: the sticky status word,
  // then the fixed-m gate-warning count (read into the caller's stack: no
  // allocation)
  return bsa_get_device_status(ws, kStaticScratchBytes, stream, clear);
}
