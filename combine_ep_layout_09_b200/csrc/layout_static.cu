// layout_static.cu -- ep_layout_static: the layout entry point for callers
// that cannot allocate device memory.
//
// ep_layout needs a few kilobytes to a few megabytes of scratch (look-back
// descriptors and counters) that its caller normally allocates and passes
// in. Some callers cannot do that: a plugin running inside a host framework
// that owns every device allocation and hands the plugin none, a serving
// runtime that plans all device memory up front and treats an allocation on
// the request path as a fault, or code that runs while a CUDA graph is being
// captured in global mode, where cudaMalloc is an error. For them this file
// keeps the scratch in a fixed device array that the library itself holds,
// so the call allocates nothing.
//
// The array lives in the library's device image: every GPU on which the
// library is used holds EP_LAYOUT_STATIC_SCRATCH_BYTES of it until the
// process exits. All calls on a device share it, so two calls that may run
// on the GPU at the same time (different streams, or several host threads
// without ordering) corrupt each other; issue them in order on one stream.
// Each call clears what must start at zero itself: ep_layout zeroes the
// counters with an async memset and its first kernel zeroes the look-back
// flags, so whatever the previous call left behind does not matter.
//
// Size: ep_layout needs 256 + align256(4E) + ceil(N*K/4096) * 4E bytes, so
// the 1 MiB array holds E=256 up to 1022 tiles of 4096 entries, that is
// N*K <= 4,186,112; E=64 up to 16,366,592 entries.
#include <cuda.h>  // CUcontext / CUresult types only: the two driver calls
                   // below are reached through cudaGetDriverEntryPoint
#include <mutex>

#include "../../include/eplayout.h"
#include "ep_launch.h"

namespace {

constexpr int kMaxDevices = 128;

// The scratch itself. In host code this name is only a stand-in for the
// device symbol: its host address must never reach a kernel. The device
// address is looked up with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char
    g_layout_scratch[EP_LAYOUT_STATIC_SCRATCH_BYTES];

// Per device: the array's device address and the unique id of the context
// it was looked up in. A context that replaces the device's primary context
// (after cudaDeviceReset, say) has a new id, so the address is looked up
// again in it; a stale address is never handed to a kernel.
struct Cached {
  unsigned long long ctx_id;
  void* addr;
};
std::mutex g_mu;
Cached g_scratch_dev[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context, 0 when there is none
// or the driver cannot tell (the caller then looks the address up anew).
// Called with g_mu held.
unsigned long long current_context_id() {
  static bool looked_up = false;
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!looked_up) {
    looked_up = true;
    cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound;
    cudaDriverEntryPointQueryResult q2 = cudaDriverEntryPointSymbolNotFound;
    void* f1 = nullptr;
    void* f2 = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) ==
            cudaSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) ==
            cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess && q2 == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
      get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
  }
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_layout_scratch on the current device, looked up with
// that device current once per (device, context) and cached.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return EP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  Cached& c = g_scratch_dev[dev];
  const unsigned long long id = current_context_id();
  if (c.addr == nullptr || id == 0 || c.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || !p)
      return EP_ERR_CUDA;
    c.addr = p;
    // the lookup makes the primary context current if none was
    c.ctx_id = current_context_id();
  }
  *out = c.addr;
  return EP_OK;
}

}  // namespace

extern "C" int ep_layout_static(const int32_t* topk_experts, int R, int S,
                                int K, int E, int token_padding,
                                int32_t* tokens_per_expert,
                                int32_t* expert_offsets, int32_t* pos,
                                int32_t* row_src, int64_t cap, int32_t* status,
                                void* stream) {
  // Problems whose scratch would not fit are refused before any CUDA call.
  const size_t need =
      ep_layout_workspace_bytes(int64_t(R) * int64_t(S), K, E);
  if (need > size_t(EP_LAYOUT_STATIC_SCRATCH_BYTES)) return EP_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != EP_OK) return rc;
  return ep_layout(topk_experts, R, S, K, E, token_padding, tokens_per_expert,
                   expert_offsets, pos, row_src, cap, scratch,
                   size_t(EP_LAYOUT_STATIC_SCRATCH_BYTES), status, stream);
}
