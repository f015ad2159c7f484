/*
 * oracle.c -- plain, slow, obviously correct CPU oracle for MoE token
 * dispatch / combine with expert-grouped layout.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test-suite, the package smoke check and
 * the CPU-baseline leg of the benchmark may load this library. It shares no
 * code, header, table or constant with the CUDA library, and the CUDA library
 * never calls it.
 *
 * Every loop below runs in the order the definition states, one element at a
 * time, single-threaded. Built with -O2 -ffp-contract=off and without
 * fast-math, so float arithmetic is IEEE-754 single precision with
 * round-to-nearest-even, and fmaf is the correctly rounded fused multiply-add.
 *
 * Notation: N tokens (token t = r*S + s for logical rank r), K experts per
 * token, E experts, H channels per row, pad = token_padding, entry (t,k) has
 * flat index t*K + k.
 *
 * Sources (page title, section):
 *   [EP]  "Экспертный параллелизм (EP)" glossary, "Что подтверждено":
 *         E must divide by ep_size, E/ep_size local experts per rank; the MoE
 *         forward sends token activations to experts (AllToAll), returns the
 *         results (second AllToAll) and combines them.
 *   [DEP] "DeepSeek开源周第二天：DeepEP深度分析", "DeepEP介绍" and "性能":
 *         dispatch / combine, FP8 dispatch with BF16 combine.
 *   [MEP] "MoonEP核心功能深度剖析", "1. 完美负载平衡" (each rank receives exactly
 *         S*K rows), "2. 高效通信机制" (tokens written straight to their final
 *         expert-grouped position; static shapes), "3. 智能内存管理" (weight
 *         buffer: rows [0,E) all experts, rows after E local prefetch slots),
 *         "快速上手" (Buffer(...token_padding), dispatch / prefetch_weight /
 *         combine argument shapes).
 *   [OCP] OCP 8-bit Floating Point Specification (OFP8), E4M3 format: bias 7,
 *         3 mantissa bits, no infinities, S.1111.111 is NaN, max 448, smallest
 *         subnormal 2^-9.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* oracle status bits (the oracle's own; tests compare meanings, not values) */
#define ORC_BAD_EXPERT 1
#define ORC_CAPACITY 2
#define ORC_SLOTS 8
#define ORC_PLAN_TOTAL 16

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32                                                            */
/* ------------------------------------------------------------------------ */

/* bf16 is the upper half of an fp32 bit pattern: widening is exact. */
float oracle_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even, on the dropped 16 bits.
 * Inputs are finite here; a carry into the exponent gives the correctly
 * rounded overflow to infinity. */
uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t upper = u >> 16;
    uint32_t lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;
    return (uint16_t)upper;
}

/* ------------------------------------------------------------------------ */
/* FP8 E4M3 encoder [OCP], round to nearest even, saturate to +-448          */
/* ------------------------------------------------------------------------ */

/* Round a non-negative double to the nearest integer, ties to even. */
static double round_half_even(double v) {
    double fl = floor(v);
    double diff = v - fl;
    if (diff > 0.5) return fl + 1.0;
    if (diff < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* Encode one fp32 value. The sign bit is kept (so -0 and negative values
 * that round to zero give 0x80). Finite inputs only; a NaN gives 0x7F. */
uint8_t oracle_e4m3_encode(float x) {
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    if (isnan(x)) return (uint8_t)(sign | 0x7F);
    double a = fabs((double)x); /* exact */
    if (a >= 448.0) return (uint8_t)(sign | 0x7E); /* satfinite */
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: value = m * 2^-9, m in [0,7]; m = 8 is the
         * smallest normal 2^-6, whose code is also 8 (exponent 1, mantissa 0) */
        double m = round_half_even(a / ldexp(1.0, -9));
        return (uint8_t)(sign | (uint8_t)m);
    }
    int ex;
    double f = frexp(a, &ex);  /* a = f * 2^ex, f in [0.5, 1) */
    int e_unb = ex - 1;        /* a = (2f) * 2^e_unb, 2f in [1, 2) */
    double m = round_half_even(2.0 * f * 8.0); /* in [8, 16] */
    if (m == 16.0) {
        m = 8.0;
        e_unb += 1;
    }
    /* largest finite: exponent field 15, mantissa 6 -> 1.75 * 2^8 = 448 */
    if (e_unb > 8 || (e_unb == 8 && m > 14.0)) return (uint8_t)(sign | 0x7E);
    int efield = e_unb + 7;
    return (uint8_t)(sign | (uint8_t)(efield << 3) | (uint8_t)((int)m - 8));
}

/* Decode one code to its exact value (NaN codes give NaN). */
double oracle_e4m3_decode(uint8_t c) {
    int s = (c >> 7) & 1;
    int ef = (c >> 3) & 0xF;
    int mf = c & 7;
    double v;
    if (ef == 15 && mf == 7) return NAN;
    if (ef == 0)
        v = ldexp((double)mf, -9);
    else
        v = ldexp(1.0 + mf / 8.0, ef - 7);
    return s ? -v : v;
}

void oracle_e4m3_encode_array(const float* x, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Layout: histogram, padded expert offsets, stable positions                */
/* ------------------------------------------------------------------------ */

/* tokens_per_expert[e] = number of entries (t,k) with topk[t,k] == e.
 * Ids outside [0, E) are not counted; they raise ORC_BAD_EXPERT. */
int oracle_histogram(const int32_t* topk, int64_t N, int K, int E,
                     int32_t* counts) {
    int st = 0;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t t = 0; t < N; ++t)
        for (int k = 0; k < K; ++k) {
            int32_t e = topk[t * K + k];
            if (e < 0 || e >= E) {
                st |= ORC_BAD_EXPERT;
                continue;
            }
            counts[e] += 1;
        }
    return st;
}

/* expert_offsets[0] = 0, expert_offsets[e+1] = expert_offsets[e] +
 * ceil(counts[e] / pad) * pad: each expert's group is padded up to a
 * multiple of token_padding [MEP "快速上手" token_padding]. Experts are laid
 * out in global order, which is rank-major when rank r owns experts
 * [r*E/R, (r+1)*E/R) [EP]. */
void oracle_expert_offsets(const int32_t* counts, int E, int pad,
                           int32_t* offsets) {
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        int32_t padded = ((counts[e] + pad - 1) / pad) * pad;
        offsets[e + 1] = offsets[e] + padded;
    }
}

/* Stable positions: entries are visited in (t,k) order and each takes the
 * next free row of its expert's group, so rows inside a group are ordered by
 * (token, k). row_src is the inverse map (row -> t*K+k); padding rows inside
 * [0, offsets[E]) hold -1; rows at and above offsets[E] are not touched.
 * Entries with an invalid id get pos = -1. */
int oracle_positions(const int32_t* topk, int64_t N, int K, int E,
                     const int32_t* offsets, int32_t* pos, int32_t* row_src,
                     int64_t cap) {
    int st = 0;
    int32_t cursor[65536];
    if (E > 65536) return -1;
    for (int64_t r = 0; r < offsets[E] && r < cap; ++r) row_src[r] = -1;
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t t = 0; t < N; ++t)
        for (int k = 0; k < K; ++k) {
            int64_t i = t * K + k;
            int32_t e = topk[i];
            if (e < 0 || e >= E) {
                pos[i] = -1;
                st |= ORC_BAD_EXPERT;
                continue;
            }
            int32_t p = cursor[e]++;
            pos[i] = p;
            if (p >= cap) {
                st |= ORC_CAPACITY;
                continue;
            }
            row_src[p] = (int32_t)i;
        }
    return st;
}

/* All three layout steps in order. */
int oracle_layout(const int32_t* topk, int64_t N, int K, int E, int pad,
                  int32_t* counts, int32_t* offsets, int32_t* pos,
                  int32_t* row_src, int64_t cap) {
    int st = oracle_histogram(topk, N, K, E, counts);
    oracle_expert_offsets(counts, E, pad, offsets);
    st |= oracle_positions(topk, N, K, E, offsets, pos, row_src, cap);
    return st;
}

/* ------------------------------------------------------------------------ */
/* Dispatch                                                                 */
/* ------------------------------------------------------------------------ */

/* bf16 dispatch [EP]/[MEP]: recv[pos[t,k]] = hidden[t] (bit copy),
 * recv_w[pos[t,k]] = w[t,k]. Padding rows (row_src == -1) are all-zero with
 * weight 0. recv_w may be NULL. */
void oracle_dispatch_bf16(const uint16_t* hidden, const float* w,
                          const int32_t* pos, const int32_t* row_src,
                          const int32_t* offsets, int64_t N, int K, int E,
                          int H, int64_t cap, uint16_t* recv, float* recv_w) {
    for (int64_t r = 0; r < offsets[E] && r < cap; ++r)
        if (row_src[r] < 0) {
            for (int h = 0; h < H; ++h) recv[r * H + h] = 0;
            if (recv_w) recv_w[r] = 0.0f;
        }
    for (int64_t t = 0; t < N; ++t)
        for (int k = 0; k < K; ++k) {
            int32_t p = pos[t * K + k];
            if (p < 0 || p >= cap) continue;
            for (int h = 0; h < H; ++h) recv[(int64_t)p * H + h] = hidden[t * H + h];
            if (recv_w) recv_w[p] = w[t * K + k];
        }
}

/* Quantise one token row [DEP "性能": FP8 dispatch]: for each group of 128
 * channels, amax = max |x|, scale = amax / 448 (fp32 division), and each
 * code is the E4M3 encoding of the fp32 quotient x / scale. A zero scale
 * gives all-zero codes. q has H bytes, scales H/128 floats. */
void oracle_quantize_row(const uint16_t* row, int H, uint8_t* q,
                         float* scales) {
    int G = H / 128;
    for (int g = 0; g < G; ++g) {
        float amax = 0.0f;
        for (int c = 0; c < 128; ++c) {
            float v = fabsf(oracle_bf16_to_f32(row[g * 128 + c]));
            if (v > amax) amax = v;
        }
        float scale = amax / 448.0f;
        scales[g] = scale;
        for (int c = 0; c < 128; ++c) {
            if (scale == 0.0f) {
                q[g * 128 + c] = 0;
                continue;
            }
            float x = oracle_bf16_to_f32(row[g * 128 + c]);
            float qf = x / scale;
            q[g * 128 + c] = oracle_e4m3_encode(qf);
        }
    }
}

/* Codes of values quantised by a given scale per group of `group` values:
 * out[i] = e4m3(x[i] / scale[i / group]) with the quotient in fp32 (the
 * inner step of oracle_quantize_row, for arbitrary scales); scale 0 gives
 * code 0. */
void oracle_quantize_by_scale(const float* x, const float* scale, int64_t n,
                              int group, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        float s = scale[i / group];
        if (s == 0.0f) {
            out[i] = 0;
            continue;
        }
        float qf = x[i] / s;
        out[i] = oracle_e4m3_encode(qf);
    }
}

/* FP8 dispatch: each token row is quantised once and its codes and scales
 * copied to the K destination rows. Padding rows: zero codes, zero scales,
 * zero weight. recv_w may be NULL. */
void oracle_dispatch_fp8(const uint16_t* hidden, const float* w,
                         const int32_t* pos, const int32_t* row_src,
                         const int32_t* offsets, int64_t N, int K, int E,
                         int H, int64_t cap, uint8_t* recv, float* scales,
                         float* recv_w) {
    int G = H / 128;
    uint8_t qrow[65536];
    float srow[512];
    if (H > 65536) return;
    for (int64_t r = 0; r < offsets[E] && r < cap; ++r)
        if (row_src[r] < 0) {
            for (int h = 0; h < H; ++h) recv[r * H + h] = 0;
            for (int g = 0; g < G; ++g) scales[r * G + g] = 0.0f;
            if (recv_w) recv_w[r] = 0.0f;
        }
    for (int64_t t = 0; t < N; ++t) {
        oracle_quantize_row(hidden + t * H, H, qrow, srow);
        for (int k = 0; k < K; ++k) {
            int32_t p = pos[t * K + k];
            if (p < 0 || p >= cap) continue;
            for (int h = 0; h < H; ++h) recv[(int64_t)p * H + h] = qrow[h];
            for (int g = 0; g < G; ++g) scales[(int64_t)p * G + g] = srow[g];
            if (recv_w) recv_w[p] = w[t * K + k];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Combine                                                                  */
/* ------------------------------------------------------------------------ */

/* out[t,h] = bf16( sum_k w[t,k] * y[pos[t,k], h] ), accumulated in fp32 with
 * one fused multiply-add per k in order k = 0..K-1 starting from +0, then
 * rounded to bf16 (nearest even) [EP: results are returned and combined;
 * DEP: BF16 combine]. Entries with pos < 0 contribute nothing. */
void oracle_combine(const uint16_t* y, const int32_t* pos, const float* w,
                    int64_t N, int K, int H, int64_t cap, uint16_t* out) {
    for (int64_t t = 0; t < N; ++t)
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                int32_t p = pos[t * K + k];
                if (p < 0 || p >= cap) continue;
                acc = fmaf(w[t * K + k], oracle_bf16_to_f32(y[(int64_t)p * H + h]), acc);
            }
            out[t * H + h] = oracle_f32_to_bf16(acc);
        }
}

/* The same weighted sum in double precision, unrounded: the yardstick for
 * the 1-bf16-ulp bound of the fp32 accumulation. */
void oracle_combine_f64(const uint16_t* y, const int32_t* pos, const float* w,
                        int64_t N, int K, int H, int64_t cap, double* out) {
    for (int64_t t = 0; t < N; ++t)
        for (int h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) {
                int32_t p = pos[t * K + k];
                if (p < 0 || p >= cap) continue;
                acc += (double)w[t * K + k] *
                       (double)oracle_bf16_to_f32(y[(int64_t)p * H + h]);
            }
            out[t * H + h] = acc;
        }
}

/* ------------------------------------------------------------------------ */
/* Balanced plan [MEP "1. 完美负载平衡", "3. 智能内存管理"]                       */
/* ------------------------------------------------------------------------ */

/* The unpadded expert-grouped rows, experts in order, are cut into R chunks
 * of exactly T = S*K rows; chunk d is logical rank d's receive region.
 * Segment = the rows of one expert inside one chunk. An expert whose rows
 * cross a cut is split: the chunk holding its first row reads the expert's
 * own weight row e, and every later chunk it reaches is given the next free
 * prefetch slot b of that rank, weight row E + d*B + b, with
 * slot_expert[d*B + b] = e (slots handed out in increasing e).
 *
 * Outputs per rank d (row-major):
 *   plan_nseg[d]                 number of segments
 *   plan_cu[d*(E+1) + j]         start of segment j inside the chunk;
 *                                entry nseg is T, later entries T as well
 *   plan_expert[d*E + j]         expert of segment j, -1 past nseg
 *   plan_wrow[d*E + j]           weight row of segment j, -1 past nseg
 *   slot_expert[d*B + b]         expert prefetched into slot b, -1 if unused
 * Requires sum(counts) == R*T (ORC_PLAN_TOTAL otherwise, outputs unfilled);
 * running out of slots raises ORC_SLOTS and stores weight row -1. */
int oracle_plan_balanced(const int32_t* counts, int R, int S, int K, int E,
                         int B, int32_t* plan_cu, int32_t* plan_expert,
                         int32_t* plan_wrow, int32_t* plan_nseg,
                         int32_t* slot_expert) {
    int64_t T = (int64_t)S * K;
    int64_t total = 0;
    int st = 0;
    for (int e = 0; e < E; ++e) total += counts[e];
    if (total != (int64_t)R * T) return ORC_PLAN_TOTAL;
    for (int d = 0; d < R; ++d) {
        int64_t lo = (int64_t)d * T, hi = lo + T;
        int nseg = 0, nslot = 0;
        int64_t C = 0; /* first row of expert e */
        for (int b = 0; b < B; ++b) slot_expert[d * B + b] = -1;
        for (int e = 0; e < E; ++e) {
            int64_t a = C, z = C + counts[e];
            C = z;
            int64_t s = a > lo ? a : lo;
            int64_t f = z < hi ? z : hi;
            if (f <= s) continue; /* no rows of e in chunk d */
            plan_cu[d * (E + 1) + nseg] = (int32_t)(s - lo);
            plan_expert[d * E + nseg] = e;
            if (a >= lo) {
                plan_wrow[d * E + nseg] = e; /* first chunk of expert e */
            } else if (nslot < B) {
                slot_expert[d * B + nslot] = e;
                plan_wrow[d * E + nseg] = E + d * B + nslot;
                nslot++;
            } else {
                plan_wrow[d * E + nseg] = -1;
                st |= ORC_SLOTS;
            }
            nseg++;
        }
        plan_nseg[d] = nseg;
        for (int j = nseg; j <= E; ++j) plan_cu[d * (E + 1) + j] = (int32_t)T;
        for (int j = nseg; j < E; ++j) {
            plan_expert[d * E + j] = -1;
            plan_wrow[d * E + j] = -1;
        }
    }
    return st;
}

/* Weight prefetch [MEP "3. 智能内存管理", prefetch_weight]: slot row
 * E + d*B + b receives a copy of expert row slot_expert[d*B+b]; unused slots
 * and every other row are left as they are. W is [E + R*B, elems] of 16-bit
 * elements (one projection; call once per projection). */
void oracle_prefetch(const int32_t* slot_expert, int R, int E, int B,
                     int64_t elems, uint16_t* W) {
    for (int d = 0; d < R; ++d)
        for (int b = 0; b < B; ++b) {
            int32_t e = slot_expert[d * B + b];
            if (e < 0) continue;
            int64_t dst = (int64_t)E + (int64_t)d * B + b;
            for (int64_t i = 0; i < elems; ++i)
                W[dst * elems + i] = W[(int64_t)e * elems + i];
        }
}

/* ------------------------------------------------------------------------ */
/* Backward pair [DEP "DeepEP介绍": kernels for training; MEP "快速上手":    */
/* combine returns gathered_route_weights_sk for the backward pass]          */
/* ------------------------------------------------------------------------ */

/* Dispatch backward (bf16 dispatch): each token's gradient is the sum of the
 * gradients of its K receive rows, in fp32, k = 0..K-1 from +0, rounded to
 * bf16. This is combine with every weight equal to one. */
void oracle_dispatch_backward(const uint16_t* grad_recv, const int32_t* pos,
                              int64_t N, int K, int H, int64_t cap,
                              uint16_t* grad_hidden) {
    for (int64_t t = 0; t < N; ++t)
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                int32_t p = pos[t * K + k];
                if (p < 0 || p >= cap) continue;
                acc = acc + oracle_bf16_to_f32(grad_recv[(int64_t)p * H + h]);
            }
            grad_hidden[t * H + h] = oracle_f32_to_bf16(acc);
        }
}

/* Combine backward, expert-output side: the gradient of receive row
 * pos[t,k] is w[t,k] * grad_out[t], the product in fp32 rounded to bf16.
 * Padding rows (row_src == -1 below offsets[E]) get zeros; rows at and above
 * offsets[E] are not touched. */
void oracle_combine_backward_rows(const uint16_t* grad_out, const float* w,
                                  const int32_t* pos, const int32_t* row_src,
                                  const int32_t* offsets, int64_t N, int K,
                                  int E, int H, int64_t cap,
                                  uint16_t* grad_rows) {
    for (int64_t r = 0; r < offsets[E] && r < cap; ++r)
        if (row_src[r] < 0)
            for (int h = 0; h < H; ++h) grad_rows[r * H + h] = 0;
    for (int64_t t = 0; t < N; ++t)
        for (int k = 0; k < K; ++k) {
            int32_t p = pos[t * K + k];
            if (p < 0 || p >= cap) continue;
            float wk = w[t * K + k];
            for (int h = 0; h < H; ++h) {
                float g = oracle_bf16_to_f32(grad_out[t * H + h]);
                grad_rows[(int64_t)p * H + h] = oracle_f32_to_bf16(wk * g);
            }
        }
}

/* Combine backward, route-weight side: d out[t] / d w[t,k] = y[pos[t,k]], so
 * the weight gradient is the dot product of that row with grad_out[t],
 * computed here in double precision (the yardstick for the fp32 sum of the
 * CUDA path). Entries with pos < 0 get 0. */
void oracle_combine_backward_weights(const uint16_t* grad_out,
                                     const uint16_t* y, const int32_t* pos,
                                     int64_t N, int K, int H, int64_t cap,
                                     double* grad_w) {
    for (int64_t t = 0; t < N; ++t)
        for (int k = 0; k < K; ++k) {
            int32_t p = pos[t * K + k];
            double acc = 0.0;
            if (p >= 0 && p < cap)
                for (int h = 0; h < H; ++h)
                    acc += (double)oracle_bf16_to_f32(y[(int64_t)p * H + h]) *
                           (double)oracle_bf16_to_f32(grad_out[t * H + h]);
            grad_w[t * K + k] = acc;
        }
}

/* gathered_route_weights: the per-row values of the receive side gathered
 * back into token order, out[t,k] = row_vals[pos[t,k]] (0 where pos < 0). */
void oracle_gather_row_values(const float* row_vals, const int32_t* pos,
                              int64_t N, int K, int64_t cap, float* out) {
    for (int64_t i = 0; i < N * K; ++i) {
        int32_t p = pos[i];
        out[i] = (p >= 0 && p < cap) ? row_vals[p] : 0.0f;
    }
}

/* Redundant-slot gradient reduce [MEP "3. 智能内存管理", 图4: the gradient
 * buffer mirrors the weight buffer; gradients of the prefetched copies are
 * reduced into the owners' rows]. G is one projection's gradient buffer
 * [E + R*B, elems] in fp32: rows [0, E) hold each expert's gradient, row
 * E + d*B + b the gradient that rank d computed for its copy of expert
 * slot_expert[d*B+b]. Every used slot is added into its expert's row, slots
 * in (d, b) order, one fp32 addition each; slot rows are left as they are. */
void oracle_reduce_slot_grads(const int32_t* slot_expert, int R, int E, int B,
                              int64_t elems, float* G) {
    for (int d = 0; d < R; ++d)
        for (int b = 0; b < B; ++b) {
            int32_t e = slot_expert[d * B + b];
            if (e < 0 || e >= E) continue;
            int64_t src = (int64_t)E + (int64_t)d * B + b;
            for (int64_t i = 0; i < elems; ++i)
                G[(int64_t)e * elems + i] = G[(int64_t)e * elems + i] + G[src * elems + i];
        }
}
