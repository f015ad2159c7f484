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

std::mutex g_mu;
void* g_scratch_dev[kMaxDevices] = {nullptr};

// Device address of g_layout_scratch on the current device; looked up once
// per device (with that device current) and cached.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return EP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_dev[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || !p)
      return EP_ERR_CUDA;
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
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
