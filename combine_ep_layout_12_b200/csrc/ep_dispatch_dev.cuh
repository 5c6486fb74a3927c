// Device-side pieces of dispatch shared by the dispatch kernels (ep_dispatch.cu)
// and the fused layout+dispatch kernel (ep_fused.cu).  Internal header.
#pragma once

#include <cuda_bf16.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kSelfRowsMaxT = 256;

// Warp-per-token kernels: tokens (one per warp) per CTA.
constexpr int kWarpTokens = 4;
#ifndef EP_DISPATCH_BULK
#define EP_DISPATCH_BULK 0
#endif
// int8 receive rows written by bulk copies from a staged shared-memory row (1) or
// by the warp's own 32-byte stores (0).
constexpr bool kDispatchBulk = EP_DISPATCH_BULK != 0;

// Units per lane of the warp-per-token kernels for a row of d elements (a unit is
// 32 elements in the int8 modes, 16 in quant_mode 0), rounded up to an
// instantiated count; 0 when the row is too long for one warp (d > 8192).
inline int warp_units(int quant_mode, int d) {
    if (quant_mode != 0) {
        const int nu = ((d + 31) / 32 + 31) / 32;
        if (nu <= 1) return 1;
        if (nu <= 2) return 2;
        if (nu <= 4) return 4;
        if (nu == 7) return 7;
        return nu <= 8 ? 8 : 0;
    }
    const int nu = (d / 16 + 31) / 32;
    if (nu <= 2) return 2;
    if (nu <= 4) return 4;
    if (nu <= 8) return 8;
    if (nu <= 14) return 14;
    return nu <= 16 ? 16 : 0;
}

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
    void* recv_x;            // [rows][d] int8 or bf16
    float* recv_scale;       // [rows]
    float* token_scale;      // [B]
    unsigned* err;
    long long rows;
    int d, k;
    int B;                   // tokens
    int wide_x;              // x is 32-byte aligned: 256-bit loads of it
    int wide_out;            // every receive row starts 32-byte aligned: 256-bit stores
};

// Receive rows of token t computed from the routing alone (used when T is small),
// while the x row load is in flight.
__device__ __forceinline__ void compute_rows(const DispatchArgs& a, int t, int* s_rows, int* s_g,
                                             int* s_cnt) {
    routing_rows(a.topk_idx, a.active, t, a.k, a.E, a.T, a.P, a.M, s_rows, s_g, s_cnt,
                 a.expert_offset, a.recv_count);
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
template <int U, bool STATIC>
__device__ __forceinline__ void dispatch_int8_body(const DispatchArgs& a, int t) {
    __shared__ int s_rows[kMaxK];
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

    float s = 1.0f, inv = 0.0f;
    bool degenerate = false;
    if (STATIC) {
        __syncthreads();  // publishes s_rows
    } else {
        // x_fp32 = fp32(x) * smooth; absmax over the row
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int u = threadIdx.x + i * NT;
            if (u >= nunits) continue;
            float f[16];
            xf_unit(raw[i], a.smooth ? a.smooth + 16 * u : nullptr, f);
#pragma unroll
            for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[e]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = amax;
        __syncthreads();  // also publishes s_rows
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
    int8_t* out = reinterpret_cast<int8_t*>(a.recv_x);

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
            const int row = s_rows[j];
            if (row >= 0 && ep_in_range(row, a.rows, a.err)) st_v4(out + (size_t)row * a.d + 16 * u, v);
        }
    }
    if (STATIC) return;
    if (threadIdx.x < a.k) {
        const int row = s_rows[threadIdx.x];
        if (row >= 0 && ep_in_range(row, a.rows, a.err)) a.recv_scale[row] = inv;
    }
    if (threadIdx.x == 0) a.token_scale[t] = inv;
}

// quant_mode 0: bf16 rows copied as they are; a unit is one 16-byte vector.
template <int U>
__device__ __forceinline__ void dispatch_bf16_body(const DispatchArgs& a, int t) {
    __shared__ int s_rows[kMaxK];
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
    __syncthreads();
    uint4* out = reinterpret_cast<uint4*>(a.recv_x);
#pragma unroll
    for (int i = 0; i < U; ++i) {
        const int u = threadIdx.x + i * NT;
        if (u >= nvec) continue;
        for (int j = 0; j < a.k; ++j) {
            const int row = s_rows[j];
            if (row >= 0 && ep_in_range(row, a.rows, a.err)) st_v4(out + (size_t)row * nvec + u, raw[i]);
        }
    }
}

// ---------------------------------------------------------------------------
// Warp-per-token dispatch, for rows of up to 8192 elements.
//
// Each warp owns one token: it reads the row once with 32-byte loads into
// registers, finds the row's absmax with warp shuffles only (no CTA barrier, so
// no warp waits for another warp's loads), quantizes in registers and writes each
// of the token's receive rows.  A unit is 32 elements in the int8 modes (two
// 32-byte bf16 loads, one 32-byte int8 store per receive row) and 16 elements in
// quant_mode 0 (one 32-byte load and one 32-byte store per receive row).  Lane l
// owns units l, l + 32, ..., so each load and store instruction of the warp covers
// one contiguous span of the row.
//
// BULK (int8 modes): instead of every lane storing its units to each of the k
// receive rows, the warp writes the quantized row once into shared memory and one
// lane issues k bulk copies (cp.async.bulk, shared -> global, no multicast) of the
// whole row, so the copy engine rather than the warp's store instructions carries
// the k-fold write.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void unpack16(const V8& r, float (&f)[16]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        f[2 * e] = bf16lo(r.w[e]);
        f[2 * e + 1] = bf16hi(r.w[e]);
    }
}

// fp32(x) of 16 elements, times the smooth scale ss[0..16) when given.
__device__ __forceinline__ void xf16(const V8& r, const float* ss, float (&f)[16]) {
    unpack16(r, f);
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

// CastToInt8 of 16 values (times s in the dynamic mode) into four words.
template <bool STATIC>
__device__ __forceinline__ void cast16(const float (&f)[16], float s, uint32_t* q) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        if (STATIC)
            q[c] = cvt_s8x4(f[4 * c], f[4 * c + 1], f[4 * c + 2], f[4 * c + 3]);
        else
            q[c] = cvt_s8x4_unclamped(__fmul_rn(f[4 * c], s), __fmul_rn(f[4 * c + 1], s),
                                      __fmul_rn(f[4 * c + 2], s), __fmul_rn(f[4 * c + 3], s));
    }
}

__device__ __forceinline__ void bulk_store_row(void* gdst, const void* ssrc, uint32_t bytes) {
    const uint32_t saddr = (uint32_t)__cvta_generic_to_shared(ssrc);
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(saddr), "r"(bytes)
                 : "memory");
}

template <int NU, int MODE, int KM, bool BULK>
__device__ __forceinline__ void dispatch_warp_body(const DispatchArgs& a, int t, uint16_t* tab,
                                                   unsigned char* stage) {
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int VPU = MODE == 0 ? 1 : 2;  // 32-byte bf16 vectors per unit
    const int lane = threadIdx.x & 31;
    const int n16 = a.d >> 4;  // 16-element vectors in the row
    const char* xrow = reinterpret_cast<const char*>(a.x + (size_t)t * a.d);
    V8 raw[NU][VPU];
#pragma unroll
    for (int i = 0; i < NU; ++i) {
#pragma unroll
        for (int h = 0; h < VPU; ++h) {
            const int v = (lane + 32 * i) * VPU + h;
            if (v < n16) {
                raw[i][h] = ld32(xrow + 32 * (size_t)v, a.wide_x);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) raw[i][h].w[e] = 0u;
            }
        }
    }

    // receive rows of the k picks, in every lane; myrow = the row of pick `lane`
    int row[KM];
    int myrow = -1;
    if (a.self_rows) {
        routing_rows_warp<KM>(a.topk_idx, a.active, t, a.k, a.E, a.T, a.P, a.M, tab, row,
                              a.expert_offset, a.recv_count);
#pragma unroll
        for (int j = 0; j < KM; ++j)
            if (lane == j) myrow = row[j];
    } else {
        unsigned bad = 0;
        if (lane < a.k) {
            int rr = a.dst_pos[(size_t)t * a.k + lane];
            if (rr < -1 || (long long)rr >= a.rows) {
                bad = EP_ERRBIT_ROW_RANGE;
                rr = -1;
            }
            myrow = rr;
        }
        report_err(a.err, bad);
#pragma unroll
        for (int j = 0; j < KM; ++j) row[j] = __shfl_sync(FULL, myrow, j);
    }

    if (MODE == 0) {
        char* out = reinterpret_cast<char*>(a.recv_x);
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (j >= a.k || row[j] < 0 || !ep_in_range(row[j], a.rows, a.err)) continue;
            char* dst = out + (size_t)row[j] * a.d * 2;
#pragma unroll
            for (int i = 0; i < NU; ++i) {
                const int v = lane + 32 * i;
                if (v < n16) st32(dst + 32 * (size_t)v, raw[i][0], a.wide_out);
            }
        }
        return;
    }

    // int8: x_fp32 = fp32(x) * smooth; dynamic mode: s = 127 / max|x_fp32| over the row
    float s = 1.0f, inv = 0.0f;
    bool degenerate = false;
    if (MODE == 2) {
        float amax = 0.0f;
        if (a.smooth == nullptr) {
            // max |x| straight on the bf16 bits (fp32(x) is exact): clear the sign
            // bits and take the bf16x2 maximum; padding vectors are +0
            __nv_bfloat162 m2 = __floats2bfloat162_rn(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < NU; ++i)
#pragma unroll
                for (int h = 0; h < VPU; ++h)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const uint32_t w = raw[i][h].w[e] & 0x7fff7fffu;
                        m2 = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162*>(&w));
                    }
            amax = fmaxf(__low2float(m2), __high2float(m2));
        } else {
#pragma unroll
            for (int i = 0; i < NU; ++i)
#pragma unroll
                for (int h = 0; h < VPU; ++h) {
                    const int v = (lane + 32 * i) * VPU + h;
                    if (v >= n16) continue;
                    float f[16];
                    xf16(raw[i][h], a.smooth + 16 * v, f);
#pragma unroll
                    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[e]));
                }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
        s = __fdiv_rn(127.0f, amax);
        degenerate = (amax == 0.0f) || isinf(s);
        inv = degenerate ? 0.0f : __fdiv_rn(1.0f, s);
    }

    int8_t* out = reinterpret_cast<int8_t*>(a.recv_x);
    V8 q[NU];
#pragma unroll
    for (int i = 0; i < NU; ++i) {
        const int u = lane + 32 * i;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int v = 2 * u + h;
            if (v < n16 && !degenerate) {
                float f[16];
                xf16(raw[i][h], a.smooth ? a.smooth + 16 * v : nullptr, f);
                cast16<MODE == 1>(f, s, q[i].w + 4 * h);
            } else {
                q[i].w[4 * h] = q[i].w[4 * h + 1] = q[i].w[4 * h + 2] = q[i].w[4 * h + 3] = 0u;
            }
        }
    }
    if (BULK) {
#pragma unroll
        for (int i = 0; i < NU; ++i) {
            const int u = lane + 32 * i;
            if (2 * u >= n16) continue;
            uint4* sp = reinterpret_cast<uint4*>(stage + 32 * (size_t)u);
            sp[0] = make_uint4(q[i].w[0], q[i].w[1], q[i].w[2], q[i].w[3]);
            if (2 * u + 1 < n16) sp[1] = make_uint4(q[i].w[4], q[i].w[5], q[i].w[6], q[i].w[7]);
        }
        __syncwarp();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
            int issued = 0;
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                if (j >= a.k || row[j] < 0 || !ep_in_range(row[j], a.rows, a.err)) continue;
                bulk_store_row(out + (size_t)row[j] * a.d, stage, (uint32_t)a.d);
                ++issued;
            }
            if (issued) {
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                // the staging row must stay intact until the copies have read it
                asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            }
        }
        __syncwarp();
    } else {
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (j >= a.k || row[j] < 0 || !ep_in_range(row[j], a.rows, a.err)) continue;
            int8_t* dst = out + (size_t)row[j] * a.d;
#pragma unroll
            for (int i = 0; i < NU; ++i) {
                const int u = lane + 32 * i;
                if (2 * u + 1 < n16)
                    st32(dst + 32 * (size_t)u, q[i], a.wide_out);
                else if (2 * u < n16)
                    st_v4(dst + 32 * (size_t)u, make_uint4(q[i].w[0], q[i].w[1], q[i].w[2], q[i].w[3]));
            }
        }
    }
    if (MODE == 2) {
        if (lane < a.k && myrow >= 0 && ep_in_range(myrow, a.rows, a.err)) a.recv_scale[myrow] = inv;
        if (lane == 0) a.token_scale[t] = inv;
    }
}

// Per-warp shared bytes of dispatch_warp_body: routing table (+ staging row).
inline size_t dispatch_warp_smem(int E, int d, bool bulk, int warps) {
    return (size_t)warps * ((size_t)warp_tab_bytes(E) + (bulk ? (size_t)((d + 15) / 16) * 16 : 0));
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
    a.B = s.B;
    // 256-bit accesses need 32-byte aligned addresses: x rows are 2d bytes apart
    // (a multiple of 32), int8 receive rows d bytes, bf16 ones 2d
    a.wide_x = (reinterpret_cast<uintptr_t>(x) & 31u) == 0;
    a.wide_out = (reinterpret_cast<uintptr_t>(p.recv_x) & 31u) == 0 && (s.quant_mode == 0 || s.d % 32 == 0);
    a.topk_idx = topk_idx;
    a.self_rows = 0;
    a.expert_offset = nullptr;
    a.recv_count = nullptr;
    a.T = s.T;
    a.P = s.P;
    a.M = s.M;
    a.E = s.E;
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
