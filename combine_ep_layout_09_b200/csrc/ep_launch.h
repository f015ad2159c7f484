// ep_launch.h -- host-side launchers of the kernels, called by api.cu after
// argument validation. Every launcher enqueues on `stream` and returns the
// launch's cudaError_t.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ep {

// ---- layout ---------------------------------------------------------------

// Entries handled by one CTA of the position scan (its look-back tile).
constexpr int kScanTile = 4096;
// Largest E the layout kernels keep in shared memory.
constexpr int kMaxExperts = 1024;

size_t layout_workspace_bytes(int64_t entries, int E);

cudaError_t launch_layout(const int32_t* topk, int64_t entries, int E, int pad,
                          int32_t* tokens_per_expert, int32_t* expert_offsets,
                          int32_t* pos, int32_t* row_src, int64_t cap,
                          void* workspace, int32_t* status, int num_sms,
                          cudaStream_t stream);

// Small batches: one launch, every CTA counts all entries itself and places
// its own chunk of tokens (layout_small.cu). Taken up to kSmallMaxEntries
// entries N*K, with at most kSmallMaxChunkEntries entries ranked per CTA and
// the CTA's shared-memory plan within kSmallMaxSmem bytes.
constexpr int64_t kSmallMaxEntries = 32768;
constexpr int64_t kSmallMaxChunkEntries = 1024;
constexpr int kSmallMaxSmem = 227 * 1024;

// copy: 0 layout only, 1 bf16 rows, 2 FP8 rows
bool small_layout_fits(int64_t N, int K, int E, int H, int copy, int num_sms);

cudaError_t launch_layout_small(const int32_t* topk, int64_t N, int K, int E,
                                int pad, int32_t* tokens_per_expert,
                                int32_t* expert_offsets, int32_t* pos,
                                int32_t* row_src, int64_t cap, int num_sms,
                                int32_t* status, cudaStream_t stream);

// ep_layout followed by ep_dispatch, in one launch
cudaError_t launch_layout_dispatch_small(
    const int32_t* topk, int64_t N, int K, int E, int pad, int H, bool fp8,
    int32_t* tokens_per_expert, int32_t* expert_offsets, int32_t* pos,
    int32_t* row_src, int64_t cap, const void* hidden, const float* w,
    void* recv, float* scales, float* recv_w, int num_sms, int32_t* status,
    cudaStream_t stream);

// ---- dispatch / combine ---------------------------------------------------

cudaError_t launch_dispatch(const void* hidden, const float* w,
                            const int32_t* pos, const int32_t* row_src,
                            const int32_t* expert_offsets, int64_t N, int K,
                            int E, int H, int64_t cap, bool fp8, void* recv,
                            float* recv_scales, float* recv_w, int num_sms,
                            int32_t* status, cudaStream_t stream,
                            bool pdl = false);

// Weights: w_rows (per receive row, [cap]) when non-NULL, with each entry's
// weight also written to `gathered` [N,K] when that is non-NULL; else w_tok
// (per entry, [N,K]); both NULL: unit weights (dispatch backward).
cudaError_t launch_combine(const void* y, const int32_t* pos,
                           const float* w_tok, const float* w_rows,
                           float* gathered, int64_t N, int K, int H,
                           int64_t cap, void* out, int num_sms,
                           int32_t* status, cudaStream_t stream);

// ---- backward pair ---------------------------------------------------------

cudaError_t launch_combine_backward(const void* grad_out, const void* y,
                                    const int32_t* pos, const int32_t* row_src,
                                    const int32_t* expert_offsets,
                                    const float* w, int64_t N, int K, int E,
                                    int H, int64_t cap, void* grad_rows,
                                    float* grad_w, int num_sms,
                                    int32_t* status, cudaStream_t stream);

cudaError_t launch_gather_row_values(const float* vals, const int32_t* pos,
                                     int64_t n, int64_t cap, float* out,
                                     cudaStream_t stream);

// ---- balanced plan / prefetch ---------------------------------------------

cudaError_t launch_plan_balanced(const int32_t* counts, int R, int S, int K,
                                 int E, int B, int32_t* plan_cu,
                                 int32_t* plan_expert, int32_t* plan_wrow,
                                 int32_t* plan_nseg, int32_t* slot_expert,
                                 int32_t* status, cudaStream_t stream);

cudaError_t launch_prefetch(const int32_t* slot_expert, int R, int E, int B,
                            int64_t elems, void* gate, void* up, void* down,
                            int num_sms, int32_t* status, cudaStream_t stream);

cudaError_t launch_reduce_slot_grads(const int32_t* slot_expert, int R, int E,
                                     int B, int64_t elems, float* g0, float* g1,
                                     float* g2, int num_sms,
                                     cudaStream_t stream);

// ---- diagnostics ----------------------------------------------------------

cudaError_t launch_debug_e4m3(const float* x, uint8_t* out, int64_t n,
                             cudaStream_t stream);
cudaError_t launch_debug_quantize(const float* x, const float* scale,
                                  uint8_t* out, int64_t n, cudaStream_t stream);
cudaError_t launch_debug_wait(const int32_t* flag, int64_t max_polls,
                              int32_t* status, cudaStream_t stream);
cudaError_t launch_debug_stream_read(const void* src, int64_t bytes,
                                     uint32_t* sink, cudaStream_t stream);

// Forced give-ups of the listed wait sites (EP_WAIT_SITE_* bits) on the
// current device, one setter per translation unit that holds wait sites.
cudaError_t set_wait_debug_layout(uint32_t sites, uint64_t budget_ns);
cudaError_t set_wait_debug_layout_small(uint32_t sites, uint64_t budget_ns);
cudaError_t set_wait_debug_dispatch(uint32_t sites, uint64_t budget_ns);
cudaError_t set_wait_debug_combine(uint32_t sites, uint64_t budget_ns);
cudaError_t set_wait_debug_plan(uint32_t sites, uint64_t budget_ns);

// SM count of the current device (cached per device).
int device_sm_count();

}  // namespace ep
