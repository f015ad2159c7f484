/*
 * eplayout.h -- C ABI of libeplayout.so: MoE token dispatch / combine with an
 * expert-grouped receive layout, on one NVIDIA B200 (sm_100a).
 *
 * Expert-parallel ranks are logical: the receive regions of all R ranks live
 * in one device buffer, rank-major, experts in order inside each rank
 * ("Экспертный параллелизм (EP)" glossary, "Что подтверждено": E experts over
 * ep_size ranks, E divisible by ep_size, E/ep_size local experts per rank;
 * rank r owns experts [r*E/R, (r+1)*E/R)).
 *
 * Conventions shared by every entry point
 *   - Every data pointer is a DEVICE pointer owned by the caller. The library
 *     allocates no memory, never synchronises the device or the stream, and
 *     enqueues all of its work on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Output buffers are fully overwritten over the ranges
 *     stated below; nothing is read from them.
 *   - Arrays are dense and row-major. bf16 is IEEE bfloat16, e4m3 is the OCP
 *     FP8 E4M3 ("fn") format, weights are IEEE fp32.
 *   - Token t of logical rank r has global index t = r*S + s. Entry (t,k) has
 *     flat index t*K + k.
 *   - Return value: EP_OK (0) or a negative EP_ERR_* code; on error nothing
 *     has been enqueued. Arguments are checked on the host before any CUDA
 *     call. Conditions only the device can see are OR-ed into `*status`, a
 *     device int32 the caller zeroes beforehand and reads when it wishes
 *     (EP_DEV_* bits). No kernel traps; every device-side wait is bounded.
 *   - Every array pointer must be non-NULL and 16-byte aligned unless stated
 *     otherwise; `status` may be NULL (no reporting) or 4-byte aligned
 *     (EP_ERR_ALIGNMENT otherwise).
 */
#ifndef EPLAYOUT_H_
#define EPLAYOUT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define EP_OK 0
#define EP_ERR_INVALID_ARG (-1) /* a size or flag outside its stated range */
#define EP_ERR_ALIGNMENT (-2)   /* a pointer that is NULL or not 16-B aligned */
#define EP_ERR_WORKSPACE (-3)   /* workspace smaller than ep_layout_workspace_bytes */
#define EP_ERR_CAPACITY (-4)    /* cap below ep_capacity_bound, or above INT32_MAX */
#define EP_ERR_CUDA (-5)        /* a CUDA launch or attribute call failed */

/* device status bits (OR-ed into *status) */
#define EP_DEV_BAD_EXPERT 1  /* an expert id outside [0, E); that entry skipped */
#define EP_DEV_CAPACITY 2    /* a row index outside [0, cap); that access skipped */
#define EP_DEV_TIMEOUT 4     /* a bounded device-side wait gave up */
#define EP_DEV_SLOTS 8       /* the balanced plan needed more than B slots on a rank */
#define EP_DEV_PLAN_TOTAL 16 /* sum(tokens_per_expert) != R*S*K; plan not written */

/* Version of this ABI (bumped when an entry point is added or changed). */
EP_API int ep_abi_version(void);

/* Static text for a return code or a single status bit. */
EP_API const char* ep_strerror(int code);

/* Rows any routing of N tokens can need once each expert's group is padded
 * to a multiple of token_padding: N*K + E*(token_padding-1). Negative on
 * invalid arguments. ("MoonEP核心功能深度剖析", "2. 高效通信机制": static
 * shapes, so the receive buffer is sized without a host sync.) */
EP_API int64_t ep_capacity_bound(int64_t num_tokens, int K, int E, int token_padding);

/* Bytes of scratch ep_layout needs for N tokens, K, E (0 on invalid input). */
EP_API size_t ep_layout_workspace_bytes(int64_t num_tokens, int K, int E);

/*
 * ep_layout -- steps 1-3 of dispatch: count tokens per expert, pad each
 * expert's group, and give every (token, k) entry its final row in the
 * expert-grouped receive buffer ("MoonEP核心功能深度剖析", "2. 高效通信机制":
 * tokens are written straight to their final expert-grouped position;
 * "快速上手": tokens_per_expert [E], token_padding; search results for
 * "EP Moe": padding instead of dropping).
 *
 * in   topk_experts      int32 [N, K], N = R*S; ids in [0, E)
 *      R, S, K, E        logical ranks, tokens per rank, experts per token,
 *                        experts; E % R == 0, 1 <= K <= 32, 1 <= E <= 1024,
 *                        N*K < 2^30
 *      token_padding     >= 1; each expert's group is rounded up to a
 *                        multiple of it
 * out  tokens_per_expert int32 [E]
 *      expert_offsets    int32 [E+1]: expert e owns rows
 *                        [off[e], off[e+1]); off[E] = rows used; rank r's
 *                        region is [off[r*E/R], off[(r+1)*E/R])
 *      pos               int32 [N, K]: row of entry (t,k); -1 for a bad id.
 *                        Inside an expert's group rows follow (t, k) order.
 *      row_src           int32 [cap]: t*K+k for every used row, -1 for
 *                        padding rows in [0, off[E]); rows >= off[E] untouched
 *      cap               rows of row_src; ep_capacity_bound(...) <= cap
 *                        <= INT32_MAX
 *      workspace         scratch of >= ep_layout_workspace_bytes(N, K, E)
 *                        bytes, contents ignored and overwritten; must not be
 *                        shared by two calls in flight at the same time
 *      status            device int32, EP_DEV_BAD_EXPERT / EP_DEV_TIMEOUT /
 *                        EP_DEV_CAPACITY may be OR-ed in
 * Launches on `stream`: for N*K <= 32768 (and at most 1024 entries per
 * SM) one kernel in which every CTA counts all entries and places its own
 * tokens, workspace unused; above that a memset and one cooperative kernel
 * (tiles that sum each other's published counts), or a memset and two
 * kernels (a histogram, then a decoupled look-back scan) when the tiles
 * cannot all be resident.
 */
EP_API int ep_layout(const int32_t* topk_experts, int R, int S, int K, int E,
              int token_padding, int32_t* tokens_per_expert,
              int32_t* expert_offsets, int32_t* pos, int32_t* row_src,
              int64_t cap, void* workspace, size_t workspace_bytes,
              int32_t* status, void* stream);

/*
 * ep_layout_static -- ep_layout for callers that cannot allocate device
 * memory. The pages have no counterpart to this entry point; it exists for
 * users of this library whose code may not call cudaMalloc: a plugin inside
 * a host framework that owns all device memory, a serving runtime that plans
 * every byte up front and forbids allocation on its request path, or code
 * running while a CUDA graph is captured in global mode.
 *
 * Same arguments, results and errors as ep_layout, minus the workspace: the
 * scratch is a fixed array inside the library's device image, of
 * EP_LAYOUT_STATIC_SCRATCH_BYTES per GPU, held from the library's first use
 * on a GPU until the process exits. Nothing is allocated by the call.
 *   - Limit: problems with ep_layout_workspace_bytes(R*S, K, E) larger than
 *     EP_LAYOUT_STATIC_SCRATCH_BYTES are refused with EP_ERR_WORKSPACE
 *     before any CUDA call. That size is 256 + align256(4E) +
 *     ceil(N*K/4096) * 4E bytes: E=256 fits up to N*K = 4,186,112 entries
 *     (1022 tiles of 4096), E=64 up to 16,366,592.
 *   - The first call on each GPU looks up the array's device address
 *     (cudaGetSymbolAddress, with that GPU current) and caches it together
 *     with the unique id of the context it was found in; a call in another
 *     context (after cudaDeviceReset, for instance) looks it up again. Make
 *     the first call on a GPU, and the first after its context changed,
 *     before any stream capture.
 *   - All calls on a GPU share the array and it keeps the last call's
 *     contents. Each call clears what must start at zero, but two calls that
 *     overlap on the GPU (different streams, unordered host threads) race
 *     and corrupt each other: order them on one stream.
 */
#define EP_LAYOUT_STATIC_SCRATCH_BYTES (1u << 20)
EP_API int ep_layout_static(const int32_t* topk_experts, int R, int S, int K,
                            int E, int token_padding,
                            int32_t* tokens_per_expert,
                            int32_t* expert_offsets, int32_t* pos,
                            int32_t* row_src, int64_t cap, int32_t* status,
                            void* stream);

/*
 * ep_dispatch -- step 4: copy every token row to its K receive rows
 * ("Экспертный параллелизм (EP)", "Что подтверждено": token activations are
 * sent to the experts; "DeepSeek开源周第二天：DeepEP深度分析", "性能": FP8
 * dispatch; "MoonEP核心功能深度剖析", "快速上手": dispatch(hidden_sh,
 * route_weights_sk, topk_experts_sk, ...) -> hidden_nvsh, route_weights_nvs).
 *
 * in   hidden            bf16 [N, H]
 *      route_weights     fp32 [N, K]
 *      pos, row_src,
 *      expert_offsets    as written by ep_layout for the same topk
 *      N, K, E, H        H % 8 == 0 (bf16), H % 128 == 0 (fp8), H <= 32768
 *      cap               rows of recv / recv_scales / recv_weights
 *      fp8               0: recv is bf16 [cap, H], a bit copy of the row.
 *                        1: recv is e4m3 [cap, H]; per row and 128-channel
 *                        group g: amax = max|x|, scale = amax / 448 (fp32,
 *                        round to nearest), code = e4m3(x / scale) with the
 *                        quotient in fp32 and the encoding round-to-nearest-
 *                        even, saturating to +-448; scale 0 gives code 0.
 * out  recv              rows pos[t,k] <- token t; padding rows (row_src ==
 *                        -1 below off[E]) <- zeros; rows >= off[E] untouched
 *      recv_scales       fp32 [cap, H/128] when fp8 (padding rows 0), else
 *                        ignored (may be NULL)
 *      recv_weights      fp32 [cap]: w[t,k] at pos[t,k], 0 on padding rows;
 *                        may be NULL
 *      num_sms           SMs to use, 0 = all. With all SMs (0, or at least
 *                        the device's count) the copy runs one CTA per
 *                        token; with fewer it runs persistent CTAs on that
 *                        many SMs. The results are the same bits either way.
 *                        hidden and recv 32-byte aligned (and H % 16 == 0
 *                        for bf16) let the per-token kernels use 32-byte
 *                        accesses; 16-byte alignment is enough.
 *      status            EP_DEV_CAPACITY, EP_DEV_TIMEOUT may be OR-ed in
 */
EP_API int ep_dispatch(const void* hidden, const float* route_weights,
                const int32_t* pos, const int32_t* row_src,
                const int32_t* expert_offsets, int64_t num_tokens, int K,
                int E, int H, int64_t cap, int fp8, void* recv,
                float* recv_scales, float* recv_weights, int num_sms,
                int32_t* status, void* stream);

/*
 * ep_layout_dispatch -- ep_layout then ep_dispatch, in ONE launch for small
 * (decode-sized) batches ("DeepSeek开源周第二天：DeepEP深度分析", "DeepEP介绍":
 * low-latency kernels for latency-sensitive decoding). Every CTA counts all
 * N*K entries in shared memory, places its own contiguous chunk of tokens
 * and copies their rows, with no workspace and no wait on another CTA.
 * Taken when N*K <= 32768, at most 1024 entries fall to one CTA and the
 * CTA's staged rows fit in shared memory; otherwise the call runs ep_layout
 * and ep_dispatch as separate launches, the dispatch kernel launched as a
 * programmatic dependent of the layout kernel (its CTAs start loading token
 * rows while the layout finishes). Either way the results are those of the
 * two calls, bit for bit.
 *
 * in   topk_experts, R, S, K, E, token_padding, cap, workspace,
 *      workspace_bytes   as for ep_layout (the workspace is needed only when
 *                        the batch is too large for the single launch)
 *      hidden, route_weights, H, fp8, num_sms
 *                        as for ep_dispatch
 * out  tokens_per_expert, expert_offsets, pos, row_src
 *                        as for ep_layout
 *      recv, recv_scales, recv_weights
 *                        as for ep_dispatch
 *      status            any bit ep_layout or ep_dispatch may set
 * Errors: those of ep_layout and ep_dispatch, checked before any launch.
 */
EP_API int ep_layout_dispatch(const int32_t* topk_experts, const void* hidden,
                              const float* route_weights, int R, int S, int K,
                              int E, int H, int token_padding, int fp8,
                              int32_t* tokens_per_expert,
                              int32_t* expert_offsets, int32_t* pos,
                              int32_t* row_src, int64_t cap, void* recv,
                              float* recv_scales, float* recv_weights,
                              void* workspace, size_t workspace_bytes,
                              int num_sms, int32_t* status, void* stream);

/*
 * ep_combine -- gather each token's K expert outputs and reduce them with the
 * route weights, back in token order ("Экспертный параллелизм (EP)", "Что
 * подтверждено": the results come back through a second AllToAll and are
 * combined; "DeepSeek开源周第二天：DeepEP深度分析", "性能": BF16 combine;
 * "MoonEP核心功能深度剖析", "快速上手": combine(plan, expert_output_nvsh, ...)
 * -> output_sh).
 *
 * in   expert_out        bf16 [cap, H], row pos[t,k] holds expert output
 *      pos               int32 [N, K] (entries < 0 are skipped)
 *      route_weights     fp32 [N, K]
 * out  out               bf16 [N, H]:
 *                        out[t,h] = bf16_rne(acc), acc = +0 then for k = 0..K-1
 *                        acc = fma(w[t,k], float(y[pos[t,k], h]), acc) in fp32
 *      num_sms           SMs to use, 0 = all
 *      status            EP_DEV_CAPACITY may be OR-ed in
 */
EP_API int ep_combine(const void* expert_out, const int32_t* pos,
               const float* route_weights, int64_t num_tokens, int K, int H,
               int64_t cap, void* out, int num_sms, int32_t* status,
               void* stream);

/*
 * ep_combine_recv_weights -- ep_combine with the weights taken on the
 * receive side, as in the pages' combine(plan, expert_output_nvsh,
 * route_weights_nvs) -> output_sh, gathered_route_weights_sk
 * ("MoonEP核心功能深度剖析", "快速上手"): the weight of entry (t,k) is
 * recv_weights[pos[t,k]], the per-row weight ep_dispatch wrote, and the
 * call also hands those weights back in token order. One launch: the
 * gather rides on the combine's own reads of pos.
 *
 * in   expert_out        bf16 [cap, H]
 *      pos               int32 [N, K] (entries outside [0, cap) skipped)
 *      recv_weights      fp32 [cap]
 * out  out               bf16 [N, H], as ep_combine with
 *                        w[t,k] = recv_weights[pos[t,k]] (bit-identical to
 *                        ep_combine with the token-side weights dispatch
 *                        copied, since those are the same values)
 *      gathered_route_weights  fp32 [N, K] or NULL: recv_weights[pos[t,k]],
 *                        0 where pos[t,k] is outside [0, cap)
 *      num_sms, status   as for ep_combine
 */
EP_API int ep_combine_recv_weights(const void* expert_out, const int32_t* pos,
                                   const float* recv_weights,
                                   int64_t num_tokens, int K, int H,
                                   int64_t cap, void* out,
                                   float* gathered_route_weights, int num_sms,
                                   int32_t* status, void* stream);

/*
 * ep_dispatch_backward -- gradient of the bf16 dispatch with respect to the
 * token rows: each token's gradient is the sum of the gradients of its K
 * receive rows, grad_hidden[t,h] = bf16_rne(acc), acc = +0 then for
 * k = 0..K-1 acc += float(grad_recv[pos[t,k], h]) in fp32 (combine with
 * unit weights). ("DeepSeek开源周第二天：DeepEP深度分析", "DeepEP介绍":
 * kernels for training as well as inference.)
 *
 * in   grad_recv         bf16 [cap, H]: gradient of the receive buffer
 *      pos               int32 [N, K] from ep_layout (entries < 0 skipped)
 * out  grad_hidden       bf16 [N, H]
 *      status            EP_DEV_CAPACITY may be OR-ed in
 */
EP_API int ep_dispatch_backward(const void* grad_recv, const int32_t* pos,
                                int64_t num_tokens, int K, int H, int64_t cap,
                                void* grad_hidden, int num_sms,
                                int32_t* status, void* stream);

/*
 * ep_combine_backward -- gradients of the combine with respect to the expert
 * outputs and to the route weights ("DeepSeek开源周第二天：DeepEP深度分析",
 * "DeepEP介绍": training kernels; "MoonEP核心功能深度剖析", "快速上手":
 * combine's outputs include what the backward pass needs).
 *
 * in   grad_out          bf16 [N, H]: gradient of the combined output
 *      expert_out        bf16 [cap, H]: the forward pass's expert outputs y
 *      pos, row_src,
 *      expert_offsets    from ep_layout
 *      route_weights     fp32 [N, K]
 * out  grad_expert_out   bf16 [cap, H]: row pos[t,k] <- bf16_rne(w[t,k] *
 *                        float(grad_out[t])) (fp32 product); padding rows
 *                        (row_src == -1 below off[E]) <- 0; rows >= off[E]
 *                        untouched
 *      grad_route_weights fp32 [N, K]: sum over h of float(y[pos[t,k], h]) *
 *                        float(grad_out[t, h]) in fp32; the summation order
 *                        is fixed by the implementation (deterministic), so
 *                        it matches the exact sum within the fp32 rounding
 *                        bound H * 2^-24 * sum|terms|; 0 where pos < 0
 *      status            EP_DEV_CAPACITY may be OR-ed in
 */
EP_API int ep_combine_backward(const void* grad_out, const void* expert_out,
                               const int32_t* pos, const int32_t* row_src,
                               const int32_t* expert_offsets,
                               const float* route_weights, int64_t num_tokens,
                               int K, int E, int H, int64_t cap,
                               void* grad_expert_out,
                               float* grad_route_weights, int num_sms,
                               int32_t* status, void* stream);

/*
 * ep_gather_route_weights -- per-row values of the receive side gathered
 * back into token order, out[t,k] = row_values[pos[t,k]] (0 where pos < 0):
 * the pages' gathered_route_weights_sk ("MoonEP核心功能深度剖析", "快速上手":
 * combine(...) -> output_sh, gathered_route_weights_sk).
 *
 * in   row_values        fp32 [cap] (e.g. recv_weights from ep_dispatch)
 *      pos               int32 [N, K]
 * out  out               fp32 [N, K]
 */
EP_API int ep_gather_route_weights(const float* row_values, const int32_t* pos,
                                   int64_t num_tokens, int K, int64_t cap,
                                   float* out, void* stream);

/*
 * ep_plan_balanced -- the perfectly balanced plan ("MoonEP核心功能深度剖析",
 * "1. 完美负载平衡": every rank receives exactly S*K rows however skewed the
 * routing, through a few redundant experts planned online; "3. 智能内存管理":
 * the weight buffer holds all experts in rows [0, E) and each rank's prefetch
 * slots after them).
 *
 * The unpadded expert-grouped rows (ep_layout with token_padding = 1) are cut
 * into R chunks of exactly T = S*K rows; chunk d is rank d's receive region.
 * A segment is one expert's rows inside one chunk. The chunk holding an
 * expert's first row reads its own weight row e; each later chunk the expert
 * reaches takes that rank's next free slot b and weight row E + d*B + b.
 *
 * in   tokens_per_expert int32 [E], must sum to R*S*K
 *      R, S, K, E, B     B = prefetch slots per rank (>= 0)
 * out  plan_cu           int32 [R, E+1]: segment j of rank d covers chunk
 *                        rows [cu[d,j], cu[d,j+1]); cu[d, nseg..E] = T
 *      plan_expert       int32 [R, E]: expert of segment j, -1 past nseg
 *      plan_wrow         int32 [R, E]: weight row of segment j, -1 past nseg
 *                        (and -1 with EP_DEV_SLOTS if no slot was free)
 *      plan_nseg         int32 [R]
 *      slot_expert       int32 [R, B]: expert to prefetch into slot b, -1 if
 *                        unused (may be NULL when B == 0)
 *      status            EP_DEV_PLAN_TOTAL (slot_expert all -1, the other
 *                        outputs left unwritten),
 *                        EP_DEV_SLOTS
 * One single-CTA kernel.
 */
EP_API int ep_plan_balanced(const int32_t* tokens_per_expert, int R, int S, int K,
                     int E, int B, int32_t* plan_cu, int32_t* plan_expert,
                     int32_t* plan_wrow, int32_t* plan_nseg,
                     int32_t* slot_expert, int32_t* status, void* stream);

/*
 * ep_prefetch_weights -- fill the redundant-expert slots before the expert
 * GEMMs ("MoonEP核心功能深度剖析", "快速上手": prefetch_weight(plan,
 * full_gate_weight, full_up_weight, full_down_weight); "3. 智能内存管理",
 * 图3: rows [E, E+B) are the local prefetch slots).
 *
 * in   slot_expert       int32 [R, B] from ep_plan_balanced
 *      elems_per_expert  16-bit elements per expert row of one projection
 *                        (H*I); elems_per_expert*2 % 16 == 0
 * in/out gate, up, down  16-bit [E + R*B, elems_per_expert] each: row
 *                        E + d*B + b <- row slot_expert[d,b] when that is
 *                        >= 0; every other row is left as it is
 *      num_sms           SMs to use, 0 = all
 *      status            EP_DEV_TIMEOUT may be OR-ed in
 */
EP_API int ep_prefetch_weights(const int32_t* slot_expert, int R, int E, int B,
                        int64_t elems_per_expert, void* gate, void* up,
                        void* down, int num_sms, int32_t* status,
                        void* stream);

/*
 * ep_reduce_slot_grads -- fold the gradients of the prefetched expert copies
 * back into the experts' own gradient rows ("MoonEP核心功能深度剖析",
 * "3. 智能内存管理", 图4: the gradient buffer mirrors the weight buffer, rows
 * [0, E) the owners' gradients, the slots' gradients reduced into them).
 *
 * in   slot_expert       int32 [R, B] from ep_plan_balanced; R*B <= 1024
 *      elems_per_expert  fp32 elements per expert row of one projection
 *                        (H*I), a multiple of 4
 * in/out grad_gate, grad_up, grad_down  fp32 [E + R*B, elems_per_expert]:
 *                        row e += row E + d*B + b for every slot with
 *                        slot_expert[d,b] == e, the slots added in (d, b)
 *                        order with one fp32 addition each; slot rows and
 *                        rows of experts without slots are left as they are
 *      num_sms           SMs to use, 0 = all
 */
EP_API int ep_reduce_slot_grads(const int32_t* slot_expert, int R, int E,
                                int B, int64_t elems_per_expert,
                                float* grad_gate, float* grad_up,
                                float* grad_down, int num_sms, void* stream);

/* ---- diagnostics (used by the test-suite) ------------------------------ */

/* out[i] = e4m3 code of x[i] through the same device conversion the FP8
 * dispatch uses (round to nearest even, saturate to +-448). */
EP_API int ep_debug_e4m3_encode(const float* x, uint8_t* out, int64_t n,
                         void* stream);

/* out[i] = e4m3(RN(x[i] / group_scale[i/16])) for n values (n % 16 == 0),
 * computed by the same device routine the FP8 dispatch quantises with
 * (bracketed reciprocal products, correctly rounded division on the rare
 * values near a rounding boundary); a zero scale gives code 0. */
EP_API int ep_debug_quantize(const float* x, const float* group_scale,
                             uint8_t* out, int64_t n, void* stream);

/* One thread polls *flag until it is non-zero, giving up after `max_polls`
 * polls with EP_DEV_TIMEOUT OR-ed into *status: the bounded wait every
 * device-side spin in this library uses, exposed so its give-up path can be
 * exercised with a flag that nothing sets. */
EP_API int ep_debug_bounded_wait(const int32_t* flag, int64_t max_polls,
                          int32_t* status, void* stream);

/* Read `bytes` bytes at src (32-byte aligned, bytes % 32 == 0) once with
 * 256-bit loads from four 512-thread CTAs per SM, and XOR every 32-bit word
 * into *sink (caller-zeroed, 4-byte aligned). A measuring stick for the
 * read side of the roofline: on the B200 it streams 4 GiB faster than a
 * framework reduction does. */
EP_API int ep_debug_stream_read(const void* src, int64_t bytes, uint32_t* sink,
                                void* stream);

/* Wait sites of the shipped kernels, for ep_debug_force_timeouts. */
#define EP_WAIT_SITE_LOOKBACK 1u    /* layout, two-kernel path: look-back over
                                       the earlier tiles' published counts */
#define EP_WAIT_SITE_TILE_REDUCE 2u /* layout, cooperative path: wait until
                                       every tile has published its counts */
#define EP_WAIT_SITE_DISPATCH 4u    /* dispatch kernels: token row landed in
                                       shared memory / stage free again */
#define EP_WAIT_SITE_COMBINE 8u     /* large-batch combine: gathered part-rows
                                       landed / stage free again */
#define EP_WAIT_SITE_SMALL 16u      /* one-launch layout + dispatch: row
                                       landed / quantised / output read */
#define EP_WAIT_SITE_PREFETCH 32u   /* weight prefetch: chunk landed */
#define EP_WAIT_SITE_ALL 63u

/* Make every wait at the listed sites give up, on the current device, for
 * the launches that follow: such a wait ignores its condition, as if nothing
 * ever set it, spins for budget_ns (0 < budget_ns <= 2e9) and then takes the
 * kernel's give-up path (EP_DEV_TIMEOUT OR-ed into *status, the kernel
 * returns; outputs are then undefined but every access stays in bounds).
 * Waits for copies already in flight, which a CTA drains before it exits,
 * are never forced. sites = 0 restores normal operation (budget_ns is then
 * ignored). The setting is
 * written with synchronous copies to the device, so call it outside stream
 * capture and with no launch of this library in flight. For tests of the
 * give-up paths: a stall is made without any GPU fault or hang. */
EP_API int ep_debug_force_timeouts(uint32_t sites, int64_t budget_ns);

#ifdef __cplusplus
}
#endif

#endif /* EPLAYOUT_H_ */
