// api.cu -- the extern "C" entry points of libeplayout.so (include/eplayout.h):
// argument validation on the host, then the kernel launchers.
#include <climits>
#include <cstdint>

#include "../../include/eplayout.h"
#include "ep_launch.h"

namespace {

constexpr int kAbiVersion = 5;  // 5: ep_debug_stream_read
constexpr int kMaxK = 32;
constexpr int kMaxH = 32768;
constexpr int64_t kMaxEntries = (int64_t(1) << 30) - 1;

bool aligned16(const void* p) {
  return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}
bool status_ok(const int32_t* s) {
  return s == nullptr || (reinterpret_cast<uintptr_t>(s) & 3u) == 0;
}
cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
int sms_or_all(int num_sms) {
  const int all = ep::device_sm_count();
  if (num_sms <= 0 || num_sms > all) return all;
  return num_sms;
}
int cuda_rc(cudaError_t e) { return e == cudaSuccess ? EP_OK : EP_ERR_CUDA; }

}  // namespace

namespace ep {

int device_sm_count() {
  static int cache[128] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess ||
        n <= 0)
      return 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace ep

extern "C" {

int ep_abi_version(void) { return kAbiVersion; }

const char* ep_strerror(int code) {
  switch (code) {
    case EP_OK: return "ok";
    case EP_ERR_INVALID_ARG: return "invalid argument";
    case EP_ERR_ALIGNMENT: return "pointer NULL or not 16-byte aligned";
    case EP_ERR_WORKSPACE: return "workspace too small";
    case EP_ERR_CAPACITY: return "capacity below the static bound or above INT32_MAX";
    case EP_ERR_CUDA: return "CUDA launch failed";
    case EP_DEV_BAD_EXPERT: return "device: expert id outside [0, E)";
    case EP_DEV_CAPACITY: return "device: row index outside [0, cap)";
    case EP_DEV_TIMEOUT: return "device: bounded wait gave up";
    case EP_DEV_SLOTS: return "device: balanced plan ran out of prefetch slots";
    case EP_DEV_PLAN_TOTAL: return "device: tokens_per_expert does not sum to R*S*K";
    default: return "unknown code";
  }
}

int64_t ep_capacity_bound(int64_t num_tokens, int K, int E, int token_padding) {
  if (num_tokens < 0 || K < 1 || E < 1 || token_padding < 1) return -1;
  return num_tokens * K + int64_t(E) * (token_padding - 1);
}

size_t ep_layout_workspace_bytes(int64_t num_tokens, int K, int E) {
  if (num_tokens < 0 || K < 1 || K > kMaxK || E < 1 || E > ep::kMaxExperts)
    return 0;
  return ep::layout_workspace_bytes(num_tokens * K, E);
}

int ep_layout(const int32_t* topk_experts, int R, int S, int K, int E,
              int token_padding, int32_t* tokens_per_expert,
              int32_t* expert_offsets, int32_t* pos, int32_t* row_src,
              int64_t cap, void* workspace, size_t workspace_bytes,
              int32_t* status, void* stream) {
  if (R < 1 || S < 0 || K < 1 || K > kMaxK || E < 1 || E > ep::kMaxExperts ||
      E % R != 0 || token_padding < 1)
    return EP_ERR_INVALID_ARG;
  const int64_t N = int64_t(R) * S;
  const int64_t M = N * K;
  if (M > kMaxEntries) return EP_ERR_INVALID_ARG;
  const int64_t bound = ep_capacity_bound(N, K, E, token_padding);
  if (cap < bound || cap > INT32_MAX) return EP_ERR_CAPACITY;
  if (!aligned16(tokens_per_expert) || !aligned16(expert_offsets) ||
      !aligned16(workspace) || !status_ok(status))
    return EP_ERR_ALIGNMENT;
  if (M > 0 && (!aligned16(topk_experts) || !aligned16(pos)))
    return EP_ERR_ALIGNMENT;
  if (cap > 0 && !aligned16(row_src)) return EP_ERR_ALIGNMENT;
  if (workspace_bytes < ep::layout_workspace_bytes(M, E)) return EP_ERR_WORKSPACE;
  const int sms = sms_or_all(0);
  if (ep::small_layout_fits(N, K, E, 8, 0, sms))
    return cuda_rc(ep::launch_layout_small(topk_experts, N, K, E, token_padding,
                                           tokens_per_expert, expert_offsets,
                                           pos, row_src, cap, sms, status,
                                           as_stream(stream)));
  return cuda_rc(ep::launch_layout(topk_experts, M, E, token_padding,
                                   tokens_per_expert, expert_offsets, pos,
                                   row_src, cap, workspace, status, sms,
                                   as_stream(stream)));
}

int ep_layout_dispatch(const int32_t* topk_experts, const void* hidden,
                       const float* route_weights, int R, int S, int K, int E,
                       int H, int token_padding, int fp8,
                       int32_t* tokens_per_expert, int32_t* expert_offsets,
                       int32_t* pos, int32_t* row_src, int64_t cap, void* recv,
                       float* recv_scales, float* recv_weights,
                       void* workspace, size_t workspace_bytes, int num_sms,
                       int32_t* status, void* stream) {
  if (R < 1 || S < 0 || K < 1 || K > kMaxK || E < 1 || E > ep::kMaxExperts ||
      E % R != 0 || token_padding < 1 || H < 8 || H > kMaxH || H % 8 != 0 ||
      (fp8 != 0 && fp8 != 1) || (fp8 && H % 128 != 0) || num_sms < 0)
    return EP_ERR_INVALID_ARG;
  const int64_t N = int64_t(R) * S;
  const int64_t M = N * K;
  if (M > kMaxEntries) return EP_ERR_INVALID_ARG;
  const int64_t bound = ep_capacity_bound(N, K, E, token_padding);
  if (cap < bound || cap > INT32_MAX) return EP_ERR_CAPACITY;
  if (!aligned16(tokens_per_expert) || !aligned16(expert_offsets) ||
      !aligned16(workspace) || !status_ok(status))
    return EP_ERR_ALIGNMENT;
  if (M > 0 && (!aligned16(topk_experts) || !aligned16(pos) ||
                !aligned16(hidden) || !aligned16(route_weights)))
    return EP_ERR_ALIGNMENT;
  if (cap > 0 && (!aligned16(row_src) || !aligned16(recv))) return EP_ERR_ALIGNMENT;
  if (cap > 0 && fp8 && !aligned16(recv_scales)) return EP_ERR_ALIGNMENT;
  if (recv_weights && !aligned16(recv_weights)) return EP_ERR_ALIGNMENT;
  if (workspace_bytes < ep::layout_workspace_bytes(M, E)) return EP_ERR_WORKSPACE;
  const int sms = sms_or_all(num_sms);
  cudaStream_t st = as_stream(stream);
  if (ep::small_layout_fits(N, K, E, H, fp8 ? 2 : 1, sms))
    return cuda_rc(ep::launch_layout_dispatch_small(
        topk_experts, N, K, E, token_padding, H, fp8 != 0, tokens_per_expert,
        expert_offsets, pos, row_src, cap, hidden, route_weights, recv,
        fp8 ? recv_scales : nullptr, recv_weights, sms, status, st));
  cudaError_t err = ep::launch_layout(topk_experts, M, E, token_padding,
                                      tokens_per_expert, expert_offsets, pos,
                                      row_src, cap, workspace, status,
                                      sms_or_all(0), st);
  if (err != cudaSuccess) return EP_ERR_CUDA;
  if (N == 0 && cap == 0) return EP_OK;
  return cuda_rc(ep::launch_dispatch(hidden, route_weights, pos, row_src,
                                     expert_offsets, N, K, E, H, cap, fp8 != 0,
                                     recv, fp8 ? recv_scales : nullptr,
                                     recv_weights, sms, status, st, true));
}

int ep_dispatch(const void* hidden, const float* route_weights,
                const int32_t* pos, const int32_t* row_src,
                const int32_t* expert_offsets, int64_t num_tokens, int K,
                int E, int H, int64_t cap, int fp8, void* recv,
                float* recv_scales, float* recv_weights, int num_sms,
                int32_t* status, void* stream) {
  if (num_tokens < 0 || K < 1 || K > kMaxK || E < 1 || H < 8 || H > kMaxH ||
      H % 8 != 0 || (fp8 != 0 && fp8 != 1) || (fp8 && H % 128 != 0) ||
      cap < 0 || cap > INT32_MAX || num_sms < 0 ||
      num_tokens * K > kMaxEntries)
    return EP_ERR_INVALID_ARG;
  if (!aligned16(expert_offsets) || !status_ok(status)) return EP_ERR_ALIGNMENT;
  if (num_tokens > 0 && (!aligned16(hidden) || !aligned16(route_weights) ||
                         !aligned16(pos)))
    return EP_ERR_ALIGNMENT;
  if (cap > 0 && (!aligned16(row_src) || !aligned16(recv))) return EP_ERR_ALIGNMENT;
  if (cap > 0 && fp8 && !aligned16(recv_scales)) return EP_ERR_ALIGNMENT;
  if (recv_weights && !aligned16(recv_weights)) return EP_ERR_ALIGNMENT;
  if (num_tokens == 0 && cap == 0) return EP_OK;
  return cuda_rc(ep::launch_dispatch(hidden, route_weights, pos, row_src,
                                     expert_offsets, num_tokens, K, E, H, cap,
                                     fp8 != 0, recv, fp8 ? recv_scales : nullptr,
                                     recv_weights, sms_or_all(num_sms), status,
                                     as_stream(stream)));
}

int ep_combine(const void* expert_out, const int32_t* pos,
               const float* route_weights, int64_t num_tokens, int K, int H,
               int64_t cap, void* out, int num_sms, int32_t* status,
               void* stream) {
  if (num_tokens < 0 || K < 1 || K > kMaxK || H < 8 || H > kMaxH ||
      H % 8 != 0 || cap < 0 || cap > INT32_MAX || num_sms < 0 ||
      num_tokens * K > kMaxEntries)
    return EP_ERR_INVALID_ARG;
  if (!status_ok(status)) return EP_ERR_ALIGNMENT;
  if (num_tokens == 0) return EP_OK;
  if (!aligned16(pos) || !aligned16(route_weights) || !aligned16(out))
    return EP_ERR_ALIGNMENT;
  if (cap > 0 && !aligned16(expert_out)) return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_combine(expert_out, pos, route_weights, nullptr,
                                    nullptr, num_tokens, K, H, cap, out,
                                    sms_or_all(num_sms), status,
                                    as_stream(stream)));
}

int ep_combine_recv_weights(const void* expert_out, const int32_t* pos,
                            const float* recv_weights, int64_t num_tokens,
                            int K, int H, int64_t cap, void* out,
                            float* gathered_route_weights, int num_sms,
                            int32_t* status, void* stream) {
  if (num_tokens < 0 || K < 1 || K > kMaxK || H < 8 || H > kMaxH ||
      H % 8 != 0 || cap < 0 || cap > INT32_MAX || num_sms < 0 ||
      num_tokens * K > kMaxEntries)
    return EP_ERR_INVALID_ARG;
  if (!status_ok(status)) return EP_ERR_ALIGNMENT;
  if (num_tokens == 0) return EP_OK;
  if (!aligned16(pos) || !aligned16(out) || !aligned16(recv_weights))
    return EP_ERR_ALIGNMENT;
  if (gathered_route_weights && !aligned16(gathered_route_weights))
    return EP_ERR_ALIGNMENT;
  if (cap > 0 && !aligned16(expert_out)) return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_combine(expert_out, pos, nullptr, recv_weights,
                                    gathered_route_weights, num_tokens, K, H,
                                    cap, out, sms_or_all(num_sms), status,
                                    as_stream(stream)));
}

int ep_dispatch_backward(const void* grad_recv, const int32_t* pos,
                         int64_t num_tokens, int K, int H, int64_t cap,
                         void* grad_hidden, int num_sms, int32_t* status,
                         void* stream) {
  if (num_tokens < 0 || K < 1 || K > kMaxK || H < 8 || H > kMaxH ||
      H % 8 != 0 || cap < 0 || cap > INT32_MAX || num_sms < 0 ||
      num_tokens * K > kMaxEntries)
    return EP_ERR_INVALID_ARG;
  if (!status_ok(status)) return EP_ERR_ALIGNMENT;
  if (num_tokens == 0) return EP_OK;
  if (!aligned16(pos) || !aligned16(grad_hidden)) return EP_ERR_ALIGNMENT;
  if (cap > 0 && !aligned16(grad_recv)) return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_combine(grad_recv, pos, nullptr, nullptr, nullptr,
                                    num_tokens, K, H, cap, grad_hidden,
                                    sms_or_all(num_sms), status,
                                    as_stream(stream)));
}

int ep_combine_backward(const void* grad_out, const void* expert_out,
                        const int32_t* pos, const int32_t* row_src,
                        const int32_t* expert_offsets,
                        const float* route_weights, int64_t num_tokens, int K,
                        int E, int H, int64_t cap, void* grad_expert_out,
                        float* grad_route_weights, int num_sms,
                        int32_t* status, void* stream) {
  if (num_tokens < 0 || K < 1 || K > kMaxK || E < 1 || H < 8 || H > kMaxH ||
      H % 8 != 0 || cap < 0 || cap > INT32_MAX || num_sms < 0 ||
      num_tokens * K > kMaxEntries)
    return EP_ERR_INVALID_ARG;
  if (!aligned16(expert_offsets) || !status_ok(status)) return EP_ERR_ALIGNMENT;
  if (num_tokens > 0 && (!aligned16(grad_out) || !aligned16(pos) ||
                         !aligned16(route_weights) ||
                         !aligned16(grad_route_weights)))
    return EP_ERR_ALIGNMENT;
  if (cap > 0 && (!aligned16(expert_out) || !aligned16(row_src) ||
                  !aligned16(grad_expert_out)))
    return EP_ERR_ALIGNMENT;
  if (num_tokens == 0 && cap == 0) return EP_OK;
  return cuda_rc(ep::launch_combine_backward(
      grad_out, expert_out, pos, row_src, expert_offsets, route_weights,
      num_tokens, K, E, H, cap, grad_expert_out, grad_route_weights,
      sms_or_all(num_sms), status, as_stream(stream)));
}

int ep_gather_route_weights(const float* row_values, const int32_t* pos,
                            int64_t num_tokens, int K, int64_t cap, float* out,
                            void* stream) {
  if (num_tokens < 0 || K < 1 || K > kMaxK || cap < 0 || cap > INT32_MAX ||
      num_tokens * K > kMaxEntries)
    return EP_ERR_INVALID_ARG;
  if (num_tokens == 0) return EP_OK;
  if (!aligned16(pos) || !aligned16(out)) return EP_ERR_ALIGNMENT;
  if (cap > 0 && !aligned16(row_values)) return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_gather_row_values(row_values, pos, num_tokens * K,
                                              cap, out, as_stream(stream)));
}

int ep_plan_balanced(const int32_t* tokens_per_expert, int R, int S, int K,
                     int E, int B, int32_t* plan_cu, int32_t* plan_expert,
                     int32_t* plan_wrow, int32_t* plan_nseg,
                     int32_t* slot_expert, int32_t* status, void* stream) {
  if (R < 1 || S < 0 || K < 1 || K > kMaxK || E < 1 || E > ep::kMaxExperts ||
      B < 0 || int64_t(R) * S * K > kMaxEntries || int64_t(R) * B > INT32_MAX)
    return EP_ERR_INVALID_ARG;
  if (!aligned16(tokens_per_expert) || !aligned16(plan_cu) ||
      !aligned16(plan_expert) || !aligned16(plan_wrow) || !aligned16(plan_nseg) ||
      !status_ok(status))
    return EP_ERR_ALIGNMENT;
  if (B > 0 && !aligned16(slot_expert)) return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_plan_balanced(tokens_per_expert, R, S, K, E, B,
                                          plan_cu, plan_expert, plan_wrow,
                                          plan_nseg, slot_expert, status,
                                          as_stream(stream)));
}

int ep_prefetch_weights(const int32_t* slot_expert, int R, int E, int B,
                        int64_t elems_per_expert, void* gate, void* up,
                        void* down, int num_sms, int32_t* status,
                        void* stream) {
  if (R < 1 || E < 1 || B < 0 || elems_per_expert < 0 ||
      (elems_per_expert * 2) % 16 != 0 || num_sms < 0)
    return EP_ERR_INVALID_ARG;
  if (!status_ok(status)) return EP_ERR_ALIGNMENT;
  if (B == 0 || elems_per_expert == 0) return EP_OK;
  if (!aligned16(slot_expert) || !aligned16(gate) || !aligned16(up) ||
      !aligned16(down))
    return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_prefetch(slot_expert, R, E, B, elems_per_expert,
                                     gate, up, down, sms_or_all(num_sms),
                                     status, as_stream(stream)));
}

int ep_reduce_slot_grads(const int32_t* slot_expert, int R, int E, int B,
                         int64_t elems_per_expert, float* grad_gate,
                         float* grad_up, float* grad_down, int num_sms,
                         void* stream) {
  if (R < 1 || E < 1 || B < 0 || elems_per_expert < 0 ||
      elems_per_expert % 4 != 0 || num_sms < 0 || int64_t(R) * B > 1024)
    return EP_ERR_INVALID_ARG;
  if (B == 0 || elems_per_expert == 0) return EP_OK;
  if (!aligned16(slot_expert) || !aligned16(grad_gate) || !aligned16(grad_up) ||
      !aligned16(grad_down))
    return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_reduce_slot_grads(slot_expert, R, E, B,
                                              elems_per_expert, grad_gate,
                                              grad_up, grad_down,
                                              sms_or_all(num_sms),
                                              as_stream(stream)));
}

int ep_debug_e4m3_encode(const float* x, uint8_t* out, int64_t n,
                         void* stream) {
  if (n < 0) return EP_ERR_INVALID_ARG;
  if (n == 0) return EP_OK;
  if (!aligned16(x) || !aligned16(out)) return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_debug_e4m3(x, out, n, as_stream(stream)));
}

int ep_debug_quantize(const float* x, const float* group_scale, uint8_t* out,
                      int64_t n, void* stream) {
  if (n < 0 || n % 16 != 0) return EP_ERR_INVALID_ARG;
  if (n == 0) return EP_OK;
  if (!aligned16(x) || !aligned16(group_scale) || !aligned16(out))
    return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_debug_quantize(x, group_scale, out, n,
                                           as_stream(stream)));
}

int ep_debug_bounded_wait(const int32_t* flag, int64_t max_polls,
                          int32_t* status, void* stream) {
  if (max_polls < 0) return EP_ERR_INVALID_ARG;
  if (!aligned16(flag) || status == nullptr || !status_ok(status))
    return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_debug_wait(flag, max_polls, status, as_stream(stream)));
}

int ep_debug_stream_read(const void* src, int64_t bytes, uint32_t* sink,
                         void* stream) {
  if (bytes < 0 || bytes % 32 != 0 || sink == nullptr) return EP_ERR_INVALID_ARG;
  if (bytes == 0) return EP_OK;
  if ((reinterpret_cast<uintptr_t>(src) & 31u) != 0 ||
      (reinterpret_cast<uintptr_t>(sink) & 3u) != 0)
    return EP_ERR_ALIGNMENT;
  return cuda_rc(ep::launch_debug_stream_read(src, bytes, sink, as_stream(stream)));
}

int ep_debug_force_timeouts(uint32_t sites, int64_t budget_ns) {
  if ((sites & ~uint32_t(EP_WAIT_SITE_ALL)) != 0u ||
      (sites != 0u && (budget_ns <= 0 || budget_ns > 2000000000)))
    return EP_ERR_INVALID_ARG;
  const uint64_t b = uint64_t(budget_ns);
  cudaError_t (*const setters[])(uint32_t, uint64_t) = {
      ep::set_wait_debug_layout, ep::set_wait_debug_layout_small,
      ep::set_wait_debug_dispatch, ep::set_wait_debug_combine,
      ep::set_wait_debug_plan};
  for (auto set : setters)
    if (set(sites, b) != cudaSuccess) return EP_ERR_CUDA;
  return EP_OK;
}

}  // extern "C"
