// Device-side pieces of dispatch shared by the dispatch kernels (ep_dispatch.cu)
// and the fused layout+dispatch kernel (ep_fused.cu).  Internal header.
#pragma once

#include <cuda_bf16.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kSelfRowsMaxT = 256;

struct DispatchArgs {
    const uint16_t* x;       // [B][d] bf16
    const float* smooth;     // [d] or null
    int expert_smooth;       // smooth holds one [d] row per routed expert (expert-major kernel)
    const int32_t* dst_pos;  // [B][k]
    const int32_t* topk_idx; // [B][k]; read instead of dst_pos when self_rows
    const uint8_t* active;   // x_active_mask [B] or null (self_rows only: dst_pos has it)
    int self_rows;           // compute the receive rows here (small T) instead of reading dst_pos
    const int32_t* expert_offset;  // packed rows with self_rows: the layout's counts
    const int32_t* recv_count;
    int T, P, M, E;
    int gstride, rbase;      // self_rows: row of (g, rank r, slot) = g * gstride + r * M + rbase + slot
    void* recv_x;            // [rows][d] int8 or bf16
    float* recv_scale;       // [rows]
    float* token_scale;      // [B]
    unsigned* err;
    long long rows;
    int d, k;
};

// Where a receive row lives.
//  LocalRows: this buffer's recv_x / recv_scale (the layout kernel writes recv_src).
//  ShardRows: the slab of the rank that owns the row's expert (expert g lives on rank
//  g / L, and its rows are slab row = row - q * slab_rows of slab q), through a table of
//  device addresses: a peer GPU's slab mapped through CUDA IPC, or separate
//  allocations on one GPU.  The table is a __grid_constant__ kernel parameter, so a
//  lookup with a computed rank index reads the parameter bank, not a local copy.
//  recv_src is written here too (the sender is the only one that knows the token).
struct LocalRows {
    __device__ __forceinline__ char* x(const DispatchArgs& a, int row, size_t row_bytes) const {
        return reinterpret_cast<char*>(a.recv_x) + (size_t)row * row_bytes;
    }
    __device__ __forceinline__ float* scale(const DispatchArgs& a, int row) const { return a.recv_scale + row; }
    __device__ __forceinline__ void write_src(int, int) const {}
};

struct ShardRows {
    const ShardTable& tab;
    __device__ __forceinline__ char* x(const DispatchArgs&, int row, size_t row_bytes) const {
        const int q = (int)(row / tab.slab_rows);
        return reinterpret_cast<char*>(tab.x[q]) + (size_t)(row - q * tab.slab_rows) * row_bytes;
    }
    __device__ __forceinline__ float* scale(const DispatchArgs&, int row) const {
        const int q = (int)(row / tab.slab_rows);
        return tab.scale[q] + (row - q * tab.slab_rows);
    }
    __device__ __forceinline__ void write_src(int row, int t) const {
        const int q = (int)(row / tab.slab_rows);
        if (tab.src[q]) tab.src[q][row - q * tab.slab_rows] = tab.token_base + t;
    }
};

// Destination row base of pick `threadIdx.x` (threads j < k, after its row is in
// s_rows[j]); null when the pick is not routed.  Not yet published to other threads.
template <class Rows>
__device__ __forceinline__ void resolve_rows(const DispatchArgs& a, int t, const int* s_rows,
                                             char** s_dst, size_t row_bytes, const Rows& rows) {
    if (threadIdx.x < a.k) {
        const int row = s_rows[threadIdx.x];
        char* dst = nullptr;
        if (row >= 0 && ep_in_range(row, a.rows, a.err)) {
            dst = rows.x(a, row, row_bytes);
            rows.write_src(row, t);
        }
        s_dst[threadIdx.x] = dst;
    }
}

// Receive rows of token t computed from the routing alone (used when T is small),
// while the x row load is in flight.
__device__ __forceinline__ void compute_rows(const DispatchArgs& a, int t, int* s_rows, int* s_g,
                                             int* s_cnt) {
    __shared__ uint16_t s_tab[kMaxE];
    routing_rows(a.topk_idx, a.active, t, a.k, a.E, a.T, a.P, a.M, s_rows, s_g, s_cnt, s_tab,
                 a.expert_offset, a.recv_count, a.gstride, a.rbase);
}

// Receive rows of token t into shared memory; out-of-range rows are skipped and flagged.
__device__ __forceinline__ void load_rows(const DispatchArgs& a, int t, int* s_rows) {
    unsigned bad = 0;
    if (threadIdx.x < a.k) {
        int row = a.dst_pos[(size_t)t * a.k + threadIdx.x];
        if (row < -1 || (long long)row >= a.rows) {
            bad = EP_ERRBIT_ROW_RANGE;
            row = -1;
        }
        s_rows[threadIdx.x] = row;
    }
    if (threadIdx.x < 32) report_err(a.err, bad);
}

// x_fp32 of one 16-element unit (two 16-byte bf16 vectors), times the smooth scale
// when given (four 16-byte loads of it, kept in L1 for the second pass).
__device__ __forceinline__ void xf_unit(const uint4 (&r)[2], const float* ss, float (&f)[16]) {
    const uint32_t w[8] = {r[0].x, r[0].y, r[0].z, r[0].w, r[1].x, r[1].y, r[1].z, r[1].w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        f[2 * e] = bf16lo(w[e]);
        f[2 * e + 1] = bf16hi(w[e]);
    }
    if (ss) {
        const float4* s4 = reinterpret_cast<const float4*>(ss);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const float4 m = __ldg(s4 + h);
            f[4 * h] = __fmul_rn(f[4 * h], m.x);
            f[4 * h + 1] = __fmul_rn(f[4 * h + 1], m.y);
            f[4 * h + 2] = __fmul_rn(f[4 * h + 2], m.z);
            f[4 * h + 3] = __fmul_rn(f[4 * h + 3], m.w);
        }
    }
}

// CastToInt8 of v, four at a time: round half to even, saturate, pack the bytes.
// The clamp bounds are integers, so clamping before rounding equals saturating
// after it.  The rounding itself is the classic magic-number conversion: adding
// 1.5 * 2^23 in fp32 (round to nearest even) leaves rne(v) in the low mantissa
// bits, exact for |v| < 2^22; the low byte of the sum is then q mod 256.  This is
// one add and a byte permute per value instead of a float-to-int conversion.
__device__ __forceinline__ uint32_t s8_byte_word(float v) {
    return __float_as_uint(__fadd_rn(fminf(fmaxf(v, -128.0f), 127.0f), 12582912.0f));
}
__device__ __forceinline__ uint32_t cvt_s8x4(float a, float b, float c, float d) {
    const uint32_t lo = __byte_perm(s8_byte_word(a), s8_byte_word(b), 0x0040);
    const uint32_t hi = __byte_perm(s8_byte_word(c), s8_byte_word(d), 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}

// The same for values already known to lie within [-127.5, 127.5): in dynamic
// quantization |x_fp32 * s| <= amax * fl(127 / amax), which is at most
// 127 * (1 + 2^-24)^2 after the two roundings, so the saturation never acts and
// the clamp is left out.
__device__ __forceinline__ uint32_t s8_byte_word_unclamped(float v) {
    return __float_as_uint(__fadd_rn(v, 12582912.0f));
}
__device__ __forceinline__ uint32_t cvt_s8x4_unclamped(float a, float b, float c, float d) {
    const uint32_t lo = __byte_perm(s8_byte_word_unclamped(a), s8_byte_word_unclamped(b), 0x0040);
    const uint32_t hi = __byte_perm(s8_byte_word_unclamped(c), s8_byte_word_unclamped(d), 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}

// quant_mode 2 (dynamic) or 1 (STATIC: q = CastToInt8(x_fp32), no absmax and no
// scale): a unit is 16 elements (two 16-byte bf16 loads -> one 16-byte int8 store).
template <int U, bool STATIC, class Rows = LocalRows>
__device__ __forceinline__ void dispatch_int8_body(const DispatchArgs& a, int t, const Rows& rows = Rows()) {
    __shared__ int s_rows[kMaxK];
    __shared__ char* s_dst[kMaxK];
    __shared__ float s_red[32];
    const int nunits = a.d >> 4;
    const int NT = blockDim.x;

    __shared__ int s_g[kMaxK], s_cnt[kMaxK];

    const uint4* xrow = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d);
    uint4 raw[U][2];
#pragma unroll
    for (int i = 0; i < U; ++i) {
        const int u = threadIdx.x + i * NT;
        if (u < nunits) {
            raw[i][0] = ld_stream_v4(xrow + 2 * u);
            raw[i][1] = ld_stream_v4(xrow + 2 * u + 1);
        } else {
            raw[i][0] = make_uint4(0, 0, 0, 0);
            raw[i][1] = make_uint4(0, 0, 0, 0);
        }
    }
    if (a.self_rows)
        compute_rows(a, t, s_rows, s_g, s_cnt);
    else
        load_rows(a, t, s_rows);
    resolve_rows(a, t, s_rows, s_dst, (size_t)a.d, rows);

    float s = 1.0f, inv = 0.0f;
    bool degenerate = false;
    if (STATIC) {
        __syncthreads();  // publishes s_rows and s_dst
    } else {
        // x_fp32 = fp32(x) * smooth; absmax over the row
        float amax = 0.0f;
        if (a.smooth == nullptr) {
            // max |x| straight on the bf16 bits (fp32(x) is exact): clear the sign bits
            // and take the bf16x2 maximum, which like fmaxf ignores a NaN operand;
            // units past the row are +0
            __nv_bfloat162 m2 = __floats2bfloat162_rn(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < U; ++i) {
                const uint32_t w[8] = {raw[i][0].x, raw[i][0].y, raw[i][0].z, raw[i][0].w,
                                       raw[i][1].x, raw[i][1].y, raw[i][1].z, raw[i][1].w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t m = w[e] & 0x7fff7fffu;
                    m2 = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162*>(&m));
                }
            }
            amax = fmaxf(__low2float(m2), __high2float(m2));
        } else {
#pragma unroll
            for (int i = 0; i < U; ++i) {
                const int u = threadIdx.x + i * NT;
                if (u >= nunits) continue;
                float f[16];
                xf_unit(raw[i], a.smooth + 16 * u, f);
#pragma unroll
                for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[e]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = amax;
        __syncthreads();  // also publishes s_rows and s_dst
        if (threadIdx.x < 32) {
            float m = threadIdx.x < (NT >> 5) ? s_red[threadIdx.x] : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (threadIdx.x == 0) s_red[0] = m;
        }
        __syncthreads();
        amax = s_red[0];
        s = __fdiv_rn(127.0f, amax);
        degenerate = (amax == 0.0f) || isinf(s);
        inv = degenerate ? 0.0f : __fdiv_rn(1.0f, s);
    }
#pragma unroll
    for (int i = 0; i < U; ++i) {
        const int u = threadIdx.x + i * NT;
        if (u >= nunits) continue;
        float f[16];
        xf_unit(raw[i], a.smooth ? a.smooth + 16 * u : nullptr, f);
        if (!STATIC) {
#pragma unroll
            for (int e = 0; e < 16; ++e) f[e] = __fmul_rn(f[e], s);
        }
        uint4 v;
        if (STATIC)
            v = make_uint4(cvt_s8x4(f[0], f[1], f[2], f[3]), cvt_s8x4(f[4], f[5], f[6], f[7]),
                           cvt_s8x4(f[8], f[9], f[10], f[11]), cvt_s8x4(f[12], f[13], f[14], f[15]));
        else
            v = make_uint4(cvt_s8x4_unclamped(f[0], f[1], f[2], f[3]),
                           cvt_s8x4_unclamped(f[4], f[5], f[6], f[7]),
                           cvt_s8x4_unclamped(f[8], f[9], f[10], f[11]),
                           cvt_s8x4_unclamped(f[12], f[13], f[14], f[15]));
        if (degenerate) v = make_uint4(0, 0, 0, 0);
        for (int j = 0; j < a.k; ++j) {
            char* dst = s_dst[j];
            if (dst) st_v4(dst + 16 * u, v);
        }
    }
    if (STATIC) return;
    if (threadIdx.x < a.k && s_dst[threadIdx.x]) *rows.scale(a, s_rows[threadIdx.x]) = inv;
    if (threadIdx.x == 0) a.token_scale[t] = inv;
}

// quant_mode 0: bf16 rows copied as they are; a unit is one 16-byte vector.
template <int U, class Rows = LocalRows>
__device__ __forceinline__ void dispatch_bf16_body(const DispatchArgs& a, int t, const Rows& rows = Rows()) {
    __shared__ int s_rows[kMaxK];
    __shared__ char* s_dst[kMaxK];
    const int nvec = a.d >> 3;
    const int NT = blockDim.x;

    __shared__ int s_g[kMaxK], s_cnt[kMaxK];

    const uint4* xrow = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d);
    uint4 raw[U];
#pragma unroll
    for (int i = 0; i < U; ++i) {
        const int u = threadIdx.x + i * NT;
        raw[i] = (u < nvec) ? ld_stream_v4(xrow + u) : make_uint4(0, 0, 0, 0);
    }
    if (a.self_rows)
        compute_rows(a, t, s_rows, s_g, s_cnt);
    else
        load_rows(a, t, s_rows);
    resolve_rows(a, t, s_rows, s_dst, (size_t)a.d * 2, rows);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < U; ++i) {
        const int u = threadIdx.x + i * NT;
        if (u >= nvec) continue;
        for (int j = 0; j < a.k; ++j) {
            char* dst = s_dst[j];
            if (dst) st_v4(dst + 16 * (size_t)u, raw[i]);
        }
    }
}

// Host-side helpers shared by the dispatch launchers.
inline DispatchArgs make_dispatch_args(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* x,
                                       const float* smooth, const int32_t* topk_idx,
                                       const uint8_t* active) {
    DispatchArgs a;
    a.active = active;
    a.x = x;
    a.smooth = smooth;
    a.expert_smooth = (smooth != nullptr && s.expert_smooth) ? 1 : 0;
    a.dst_pos = p.dst_pos;
    a.recv_x = p.recv_x;
    a.recv_scale = p.recv_scale;
    a.token_scale = p.token_scale;
    a.err = &reinterpret_cast<WsHeader*>(p.workspace)->err;
    a.rows = s.rows;
    a.d = s.d;
    a.k = s.k;
    a.topk_idx = topk_idx;
    a.self_rows = 0;
    a.expert_offset = nullptr;
    a.recv_count = nullptr;
    a.T = s.T;
    a.P = s.P;
    a.M = s.M;
    a.E = s.E;
    a.gstride = s.P * s.M;
    a.rbase = 0;
    return a;
}

inline int pick_units(int n, int max_u, int* U, int* NT) {
    // Smallest power-of-two U <= max_u with ceil(n / U) <= 128 threads: small CTAs
    // (and few registers) so that a decode batch of ~1000 tokens is resident in one
    // wave.  Wider rows fall back to up to 256 threads.
    int u = 1;
    while (u < max_u && (n + u - 1) / u > 128) u *= 2;
    int nt = (n + u - 1) / u;
    nt = ((nt + 31) / 32) * 32;
    if (nt > 256) return EP_ERR_UNSUPPORTED;
    *U = u;
    *NT = nt;
    return EP_OK;
}


}  // namespace
}  // namespace ep
