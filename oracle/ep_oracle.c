/*
 * ep_oracle.c -- plain, slow, single-threaded CPU oracle for MoE expert-parallel
 * token dispatch and combine with logical EP ranks.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  The CUDA library never links
 * or calls it, and this file shares no code, header or table with it.
 *
 * Sources followed (page title, section):
 *  - Ascend CANN "low_latency_dispatch", Function / Formula: the quant_mode 0 and
 *    quant_mode 2 (dynamic int8) formulas, the alltoallv of the quantized rows
 *    and the alltoall of the per-token scale; the zero / copy / constant special
 *    experts.
 *  - same page, Constraints: the receive-row bound
 *    A >= max_tokens_per_rank * ep_world_size * min(local_expert_num, K),
 *    local_expert_num = num_experts / ep_world_size, 0 < K <= 16,
 *    num_experts + zero + copy + const < MAX_INT32, and
 *    "Deterministic Computation: defaults to a deterministic computation".
 *  - same page, Example: special-expert ids follow the routed ones
 *    (num_experts = 32 with one zero and one copy expert uses ids 32 and 33).
 *  - same page, Formula, non-dynamic case: quant_mode 1 (any mode other than 0
 *    and 2) is the static cast CastToInt8(CastToFp32(x) * scales), no scale sent.
 *  - same page, Prototype: the optional per-token x_active_mask.
 *  - DeepEP issue #84 "Profiling dispatch_t for low-latency kernel dispatch
 *    bandwidth", masking experiment: expert g lives on rank g / (E / P) and a
 *    pick set to -1 sends nothing.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - the absmax of the dynamic quantization runs over one token row (d values);
 *  - CastToInt8 rounds half to even and saturates to [-128, 127];
 *  - the scale sent along is inv = 1.0f / s computed in fp32, s = 127.0f / amax;
 *  - amax == 0 or s not finite: the row quantizes to all zeros, inv = 0;
 *  - within one (expert, source rank) run the received rows are in ascending
 *    source-token order (the deterministic stable order);
 *  - a routed id repeated inside one token is routed once (first occurrence);
 *    later copies are dropped and flagged;
 *  - special experts replace the expert output and are weighted like routed picks;
 *    the constant expert is alpha1 * x + alpha2 * v in fp32 (two rounded products,
 *    one rounded sum), no bf16 rounding before weighting;
 *  - combine accumulates acc = fma(w_j, e_j, acc) in fp32 in pick order j and
 *    rounds once to bf16 (nearest even);
 *  - static quantization (mode 1) with no scale given multiplies by nothing;
 *  - x_active_mask: a token whose entry is 0 takes no part at all, as if every
 *    pick of it were -1: no receive row, not counted (special experts included),
 *    no error bits for its ids, and combine returns +0 for it.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Status codes returned by every entry point. */
#define ORC_OK 0
#define ORC_BAD_ARG (-1)

/* Error bits reported for bad routing data (same meaning as the GPU library's,
 * but defined here independently). */
#define ORC_ERR_BAD_ID 0x1u /* id < -1 or id >= E + Z + C + K */
#define ORC_ERR_DUP_ID 0x2u /* a routed id repeated inside one token */

typedef struct {
    int32_t B;          /* tokens over all logical ranks */
    int32_t d;          /* hidden size */
    int32_t k;          /* picks per token */
    int32_t P;          /* logical EP ranks */
    int32_t M;          /* max tokens per rank (receive rows per (expert, rank)) */
    int32_t E;          /* routed experts */
    int32_t n_zero;     /* zero experts */
    int32_t n_copy;     /* copy experts */
    int32_t n_const;    /* constant experts */
    int32_t quant_mode; /* 0: bf16 pass-through, 1: static int8, 2: dynamic int8 */
    int32_t layout;     /* 0: low-latency rows, 1: packed rows */
} orc_cfg;

/* ---- bf16 <-> fp32, written from the format definition ------------------- */

/* A bf16 is the upper half of an IEEE binary32. */
static float bf16_to_f32(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary32 to bf16, nearest with ties to even; NaN stays a quiet NaN. */
static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) {
        return (uint16_t)((u >> 16) | 0x0040u);
    }
    uint32_t keep_lsb = (u >> 16) & 1u;
    u = u + 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

static int cfg_ok(const orc_cfg* c) {
    if (!c) return 0;
    if (c->B < 0 || c->d <= 0 || c->k <= 0 || c->k > 16) return 0;
    if (c->P <= 0 || c->M < 0 || c->E <= 0) return 0;
    if (c->n_zero < 0 || c->n_copy < 0 || c->n_const < 0) return 0;
    if (c->B % c->P != 0 || c->E % c->P != 0) return 0;
    if (c->layout != 0 && c->layout != 1) return 0;
    if (c->layout == 0 && c->B / c->P > c->M) return 0;
    if (c->quant_mode < 0 || c->quant_mode > 2) return 0;
    return 1;
}

/* Receive rows the layout addresses: E*P*M (low-latency) or B*k (packed). */
static int64_t orc_rows(const orc_cfg* c) {
    return c->layout == 1 ? (int64_t)c->B * c->k : (int64_t)c->E * c->P * c->M;
}
int64_t orc_receive_rows(const orc_cfg* c) { return cfg_ok(c) ? orc_rows(c) : -1; }

/* Exported for the tests that pin the format helpers. */
uint16_t orc_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }
float orc_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }
void orc_f32_to_bf16_n(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

/*
 * Layout: counts, exclusive prefix, destination row of every routed pick and
 * the source token of every received row.  slot = the pick's rank among rank
 * r's tokens that routed to g, in token order.  Receive row:
 *   low-latency (layout 0): g*P*M + r*M + slot   (a [E][P*M] buffer; the
 *                           Ascend/DeepEP low-latency form [L][P*M] per rank)
 *   packed      (layout 1): expert_offset[g] + sum_{r' < r} recv_count[g][r'] + slot
 *                           (rows contiguous per expert, then per source rank:
 *                           the dense [A][H] expand_x of the Ascend page)
 *
 * expert_count  [E + Z + C + K]      picks per expert id (routed and special)
 * expert_offset [E + Z + C + K + 1]  exclusive prefix of expert_count
 * recv_count    [E][P]               rows of expert g sent by source rank r
 * dst_pos       [B][k]               global receive row, or -1 if not routed
 * recv_src      [rows]               source token of each received row; -1 in
 *                                    rows nobody wrote (rows = E*P*M or B*k)
 * active        [B] or NULL          x_active_mask: tokens with 0 are skipped
 */
int orc_layout_active(const orc_cfg* c, const int32_t* topk_idx, const uint8_t* active,
                      int32_t* expert_count, int32_t* expert_offset, int32_t* recv_count,
                      int32_t* dst_pos, int32_t* recv_src, uint32_t* err_bits) {
    if (!cfg_ok(c) || !topk_idx || !expert_count || !expert_offset || !recv_count ||
        !dst_pos || !recv_src || !err_bits)
        return ORC_BAD_ARG;
    const int64_t E = c->E, P = c->P, M = c->M, k = c->k;
    const int64_t E_tot = E + c->n_zero + c->n_copy + c->n_const;
    const int64_t T = c->B / c->P;
    uint32_t err = 0;

    const int64_t rows = orc_rows(c);
    for (int64_t g = 0; g < E_tot; ++g) expert_count[g] = 0;
    for (int64_t i = 0; i < E * P; ++i) recv_count[i] = 0;
    for (int64_t i = 0; i < rows; ++i) recv_src[i] = -1;

    for (int64_t r = 0; r < P; ++r) {
        for (int64_t t = r * T; t < (r + 1) * T; ++t) {
            if (active && !active[t]) {              /* inactive token: nothing at all */
                for (int64_t j = 0; j < k; ++j) dst_pos[t * k + j] = -1;
                continue;
            }
            for (int64_t j = 0; j < k; ++j) {
                int64_t g = topk_idx[t * k + j];
                dst_pos[t * k + j] = -1;
                if (g == -1) continue;               /* masked pick: nothing sent */
                if (g < -1 || g >= E_tot) {          /* not an expert id */
                    err |= ORC_ERR_BAD_ID;
                    continue;
                }
                if (g >= E) {                        /* special expert: no transfer */
                    expert_count[g] += 1;
                    continue;
                }
                int repeated = 0;
                for (int64_t jj = 0; jj < j; ++jj)
                    if (topk_idx[t * k + jj] == g) repeated = 1;
                if (repeated) {
                    err |= ORC_ERR_DUP_ID;
                    continue;
                }
                int64_t slot = recv_count[g * P + r];
                recv_count[g * P + r] += 1;
                expert_count[g] += 1;
                if (c->layout == 0) {
                    int64_t row = g * P * M + r * M + slot;
                    dst_pos[t * k + j] = (int32_t)row;
                    recv_src[row] = (int32_t)t;
                } else {
                    dst_pos[t * k + j] = (int32_t)slot; /* turned into a row below */
                }
            }
        }
    }

    int64_t run = 0;
    for (int64_t g = 0; g < E_tot; ++g) {
        expert_offset[g] = (int32_t)run;
        run += expert_count[g];
    }
    expert_offset[E_tot] = (int32_t)run;

    if (c->layout == 1) {
        /* second pass: rows need every rank's counts of the lower experts */
        for (int64_t t = 0; t < c->B; ++t) {
            int64_t r = t / T;
            for (int64_t j = 0; j < k; ++j) {
                int64_t g = topk_idx[t * k + j];
                if (g < 0 || g >= E || dst_pos[t * k + j] < 0) {
                    dst_pos[t * k + j] = -1;
                    continue;
                }
                int64_t base = expert_offset[g];
                for (int64_t rr = 0; rr < r; ++rr) base += recv_count[g * P + rr];
                int64_t row = base + dst_pos[t * k + j];
                dst_pos[t * k + j] = (int32_t)row;
                recv_src[row] = (int32_t)t;
            }
        }
    }
    *err_bits = err;
    return ORC_OK;
}

int orc_layout(const orc_cfg* c, const int32_t* topk_idx, int32_t* expert_count,
               int32_t* expert_offset, int32_t* recv_count, int32_t* dst_pos,
               int32_t* recv_src, uint32_t* err_bits) {
    return orc_layout_active(c, topk_idx, NULL, expert_count, expert_offset, recv_count, dst_pos,
                             recv_src, err_bits);
}

/* Static cast of one row (quant_mode 1): q = CastToInt8(fp32(x) (* scales)), round
 * half to even, saturate; no scale is derived. */
static void cast_row_static(const uint16_t* x, const float* scales, int64_t d, int8_t* q) {
    for (int64_t i = 0; i < d; ++i) {
        float v = bf16_to_f32(x[i]);
        if (scales) v = v * scales[i];
        float y = nearbyintf(v);
        if (y > 127.0f) y = 127.0f;
        else if (y < -128.0f) y = -128.0f;
        q[i] = (int8_t)y;
    }
}

/*
 * Per-token quantization.
 *  quant_mode 0: quant_out = x (bf16 bits copied), token_scale untouched.
 *  quant_mode 1: q = CastToInt8(fp32(x) * smooth), token_scale untouched.
 *  quant_mode 2: x_fp32 = fp32(x) * smooth, s = 127 / max|x_fp32|,
 *                q = CastToInt8(x_fp32 * s), token_scale = 1 / s.
 * smooth is a [d] fp32 vector or NULL (NULL means no multiply at all).
 */
/* One row: x_fp32 = fp32(x) (* smooth), s = 127 / max|x_fp32|, q = CastToInt8(x_fp32 * s).
 * Returns 1 / s, or 0 with q = 0 when amax == 0 or s is not finite.  xf: d floats scratch. */
static float quantize_row(const uint16_t* x, const float* smooth, int64_t d, float* xf, int8_t* q) {
    float amax = 0.0f;
    for (int64_t i = 0; i < d; ++i) {
        float v = bf16_to_f32(x[i]);
        if (smooth) v = v * smooth[i];
        xf[i] = v;
        float a = fabsf(v);
        if (a > amax) amax = a;
    }
    float s = 127.0f / amax;
    if (amax == 0.0f || !isfinite(s)) {
        for (int64_t i = 0; i < d; ++i) q[i] = 0;
        return 0.0f;
    }
    for (int64_t i = 0; i < d; ++i) {
        float y = nearbyintf(xf[i] * s);  /* default rounding: nearest, ties to even */
        if (y > 127.0f) y = 127.0f;
        if (y < -128.0f) y = -128.0f;
        q[i] = (int8_t)y;
    }
    return 1.0f / s;
}

int orc_quantize(const orc_cfg* c, const uint16_t* x, const float* smooth, void* quant_out,
                 float* token_scale) {
    if (!cfg_ok(c) || !x || !quant_out) return ORC_BAD_ARG;
    const int64_t B = c->B, d = c->d;
    if (c->quant_mode == 0) {
        uint16_t* out = (uint16_t*)quant_out;
        for (int64_t i = 0; i < B * d; ++i) out[i] = x[i];
        return ORC_OK;
    }
    int8_t* q = (int8_t*)quant_out;
    if (c->quant_mode == 1) {
        for (int64_t t = 0; t < B; ++t) cast_row_static(x + t * d, smooth, d, q + t * d);
        return ORC_OK;
    }
    if (!token_scale) return ORC_BAD_ARG;
    float* xf = (float*)malloc(sizeof(float) * (size_t)d);
    if (!xf) return ORC_BAD_ARG;
    for (int64_t t = 0; t < B; ++t) token_scale[t] = quantize_row(x + t * d, smooth, d, xf, q + t * d);
    free(xf);
    return ORC_OK;
}

/*
 * Scatter (the alltoallv): every routed pick copies its token's quantized row
 * to its receive row; in quant_mode 2 the row's scale goes along.
 * recv_x has `rows` rows of d elements (int8 or bf16); recv_scale has `rows`
 * entries (quant_mode 2 only).  Rows nobody writes are left untouched.
 */
int orc_dispatch(const orc_cfg* c, const void* quant_out, const float* token_scale,
                 const int32_t* dst_pos, void* recv_x, float* recv_scale, int64_t rows) {
    if (!cfg_ok(c) || !quant_out || !dst_pos || !recv_x) return ORC_BAD_ARG;
    if (c->quant_mode == 2 && (!token_scale || !recv_scale)) return ORC_BAD_ARG;
    const int64_t B = c->B, d = c->d, k = c->k;
    const int64_t esz = (c->quant_mode != 0) ? 1 : 2;
    for (int64_t t = 0; t < B; ++t) {
        for (int64_t j = 0; j < k; ++j) {
            int64_t row = dst_pos[t * k + j];
            if (row < 0) continue;
            if (row >= rows) return ORC_BAD_ARG;
            memcpy((char*)recv_x + row * d * esz, (const char*)quant_out + t * d * esz,
                   (size_t)(d * esz));
            if (c->quant_mode == 2) recv_scale[row] = token_scale[t];
        }
    }
    return ORC_OK;
}

/*
 * Dispatch with a per-expert smooth scale (scales of shape [E][d], as in the
 * Ascend example's quant_mode 2 call): each routed copy (t, g) is quantized on
 * its own,  x_fp32 = fp32(x[t]) * smooth[g], s = 127 / max|x_fp32|,
 * q = CastToInt8(x_fp32 * s), and written with recv_scale = 1 / s to its row.
 * Same readings as orc_quantize (row absmax, round half to even, saturation,
 * amax == 0 or non-finite s -> zeros and scale 0).  In quant_mode 1 each copy is
 * the static cast with its expert's row, q = CastToInt8(fp32(x[t]) * smooth[g]),
 * and recv_scale is not used.
 */
int orc_dispatch_expert_smooth(const orc_cfg* c, const uint16_t* x, const float* smooth,
                               const int32_t* topk_idx, const int32_t* dst_pos, int8_t* recv_x,
                               float* recv_scale, int64_t rows) {
    if (!cfg_ok(c) || c->quant_mode == 0 || !x || !smooth || !topk_idx || !dst_pos || !recv_x)
        return ORC_BAD_ARG;
    if (c->quant_mode == 2 && !recv_scale) return ORC_BAD_ARG;
    const int64_t B = c->B, d = c->d, k = c->k, E = c->E;
    float* xf = (float*)malloc(sizeof(float) * (size_t)d);
    if (!xf) return ORC_BAD_ARG;
    for (int64_t t = 0; t < B; ++t) {
        for (int64_t j = 0; j < k; ++j) {
            const int64_t row = dst_pos[t * k + j];
            const int64_t g = topk_idx[t * k + j];
            if (row < 0) continue;
            if (g < 0 || g >= E || row >= rows) {
                free(xf);
                return ORC_BAD_ARG;
            }
            if (c->quant_mode == 1)
                cast_row_static(x + t * d, smooth + g * d, d, recv_x + row * d);
            else
                recv_scale[row] = quantize_row(x + t * d, smooth + g * d, d, xf, recv_x + row * d);
        }
    }
    free(xf);
    return ORC_OK;
}

/*
 * Combine: y[t] = bf16( sum over j in order of w[t,j] * e(t,j) ), accumulated as
 * acc = fma(w, e, acc) in fp32 from acc = 0.
 *   routed id with dst_pos >= 0 : e = fp32(expert_out[dst_pos])
 *   -1, zero expert, bad id, or routed id with dst_pos < 0 : the term is skipped
 *   copy expert c              : e = fp32(ori_x[t])
 *   const expert c             : e = fp32(a1[c]) * fp32(ori_x[t]) + fp32(a2[c]) * fp32(v[c])
 * expert_out has `rows` rows of d bf16 values.  active ([B] or NULL): a token
 * whose entry is 0 has every term skipped, so y[t] = +0.
 */
int orc_combine_active(const orc_cfg* c, const uint16_t* expert_out, int64_t rows,
                       const int32_t* topk_idx, const float* topk_weights, const int32_t* dst_pos,
                       const uint16_t* ori_x, const uint16_t* a1, const uint16_t* a2,
                       const uint16_t* v, const uint8_t* active, uint16_t* y) {
    if (!cfg_ok(c) || !topk_idx || !topk_weights || !dst_pos || !y) return ORC_BAD_ARG;
    const int64_t B = c->B, d = c->d, k = c->k, E = c->E;
    const int64_t Z = c->n_zero, C = c->n_copy, K = c->n_const;
    if ((C + K) > 0 && !ori_x) return ORC_BAD_ARG;
    if (K > 0 && (!a1 || !a2 || !v)) return ORC_BAD_ARG;
    for (int64_t t = 0; t < B; ++t) {
        const int64_t k_t = (active && !active[t]) ? 0 : k;
        for (int64_t i = 0; i < d; ++i) {
            float acc = 0.0f;
            for (int64_t j = 0; j < k_t; ++j) {
                int64_t g = topk_idx[t * k + j];
                float w = topk_weights[t * k + j];
                float e;
                if (g >= 0 && g < E) {
                    int64_t row = dst_pos[t * k + j];
                    if (row < 0) continue;
                    if (!expert_out || row >= rows) return ORC_BAD_ARG;
                    e = bf16_to_f32(expert_out[row * d + i]);
                } else if (g >= E + Z && g < E + Z + C) {
                    e = bf16_to_f32(ori_x[t * d + i]);
                } else if (g >= E + Z + C && g < E + Z + C + K) {
                    int64_t ci = g - E - Z - C;
                    float p1 = bf16_to_f32(a1[ci * d + i]) * bf16_to_f32(ori_x[t * d + i]);
                    float p2 = bf16_to_f32(a2[ci * d + i]) * bf16_to_f32(v[ci * d + i]);
                    e = p1 + p2;
                } else {
                    continue; /* -1, zero expert, or not an expert id */
                }
                acc = fmaf(w, e, acc);
            }
            y[t * d + i] = f32_to_bf16_rne(acc);
        }
    }
    return ORC_OK;
}

int orc_combine(const orc_cfg* c, const uint16_t* expert_out, int64_t rows,
                const int32_t* topk_idx, const float* topk_weights, const int32_t* dst_pos,
                const uint16_t* ori_x, const uint16_t* a1, const uint16_t* a2,
                const uint16_t* v, uint16_t* y) {
    return orc_combine_active(c, expert_out, rows, topk_idx, topk_weights, dst_pos, ori_x, a1, a2,
                              v, NULL, y);
}
