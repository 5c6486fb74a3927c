// Combine kernel: the weighted gather-reduce of expert outputs back to tokens,
// with the zero, copy and constant special experts (Ascend CANN
// "low_latency_dispatch", Formula, special expert scenario: Moe(ori_x) = 0,
// Moe(ori_x) = ori_x, Moe(ori_x) = alpha1 * ori_x + alpha2 * v; low_latency_combine
// takes the dispatch outputs, topk_weights and ori_x).
//
//   y[t] = bf16_rn( acc ),  acc = 0;  for j = 0..k-1 in order:
//          acc = fma(w[t][j], e(t,j), acc)   (fp32, one rounding per pick)
//   e = fp32(expert_out[dst_pos[t][j]])          routed pick
//       fp32(ori_x[t])                            copy expert
//       a1[c]*ori_x[t] + a2[c]*v[c]  (fp32 ops)   constant expert c
//   -1, zero experts, dropped picks, every pick of an inactive token
//   (x_active_mask): no term, so an inactive token gets y = +0.
//
// Design.  A CTA covers NT consecutive 16-byte column vectors (8 bf16) of one
// token.  The token's k picks are classified once into shared memory, then each
// thread issues all k 16-byte loads of its column before accumulating, so a
// thread keeps k loads in flight; the k-order fused multiply-adds match the
// definition exactly.
#include "ep_internal.cuh"

namespace ep {
namespace {

enum : int { kSkip = 0, kRouted = 1, kCopy = 2, kConst = 3 };

// Per-rank batches up to this size derive their rows from the routing (the scan of
// the earlier tokens' ids stays within one load per thread).  At 256 tokens per
// rank reading dst_pos was measured faster (90 against 102 us per combine at
// P = 16, d = 7168, k = 8): the scan's L2 reads grow with T while dst_pos does not.
constexpr int kCombineSelfRowsMaxT = 128;

struct CombineArgs {
    const uint16_t* expert_out;  // [rows][d]
    const int32_t* topk_idx;     // [B][k]
    const uint8_t* active;       // x_active_mask [B] or null: inactive tokens give +0
    const float* topk_weights;   // [B][k]
    const int32_t* dst_pos;      // [B][k]
    const uint16_t* ori_x;       // [B][d]
    const uint16_t* a1;          // [K][d]
    const uint16_t* a2;
    const uint16_t* v;
    uint16_t* y;                 // [B][d]
    unsigned* err;
    long long rows;
    int d, k, E, Z, C, K;
    int chunks;                  // CTAs per token
    int self_rows;               // derive receive rows from topk_idx instead of reading dst_pos
    const int32_t* expert_offset;  // packed rows with self_rows: the layout's counts
    const int32_t* recv_count;
    int T, P, M;
    int B;                       // tokens
};

__device__ __forceinline__ void unpack8(const uint4& r, float* f) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16lo(w[i]);
        f[2 * i + 1] = bf16hi(w[i]);
    }
}

template <int KMAX>
__global__ void __launch_bounds__(128, (KMAX > 8 ? 4 : 8)) combine_kernel(CombineArgs a) {
    __shared__ int s_kind[KMAX];
    __shared__ long long s_src[KMAX];  // receive row (routed) or const index
    __shared__ float s_w[KMAX];

    // CTA = (token t, column slice c); the slice is swept by the CTA's threads
    const int t = blockIdx.x / a.chunks;
    const int c = blockIdx.x - t * a.chunks;
    const int nvec = a.d >> 3;
    const int span = (nvec + a.chunks - 1) / a.chunks;
    const int v_begin = c * span;
    const int v_end = min(nvec, v_begin + span);

    // With self_rows the prologue only reads the routing (topk_idx, topk_weights),
    // which was complete before the preceding kernels started, so it runs before
    // griddepcontrol.wait and overlaps their tail; the expert outputs are read and
    // y is written only after the wait.
    __shared__ int s_rows[KMAX], s_g[KMAX], s_cnt[KMAX];
    if (a.self_rows) {
        routing_rows(a.topk_idx, a.active, t, a.k, a.E, a.T, a.P, a.M, s_rows, s_g, s_cnt,
                     a.expert_offset, a.recv_count);
    } else {
        pdl_wait();
    }
    pdl_launch_dependents();

    unsigned bad = 0;
    const bool on = !(a.active && !a.active[t]);  // an inactive token has no terms
    if (threadIdx.x < a.k) {
        const size_t i = (size_t)t * a.k + threadIdx.x;
        const int g = on ? a.topk_idx[i] : -1;
        const int dp = a.self_rows ? s_rows[threadIdx.x] : a.dst_pos[i];
        int kind = kSkip;
        long long src = 0;
        if (g >= 0 && g < a.E) {
            if (dp >= 0 && (long long)dp < a.rows) {
                kind = kRouted;
                src = dp;
            } else if (dp != -1) {
                bad = EP_ERRBIT_ROW_RANGE;
            }
        } else if (g >= a.E + a.Z && g < a.E + a.Z + a.C) {
            kind = kCopy;
        } else if (g >= a.E + a.Z + a.C && g < a.E + a.Z + a.C + a.K) {
            kind = kConst;
            src = g - (a.E + a.Z + a.C);
        }
        s_kind[threadIdx.x] = kind;
        s_src[threadIdx.x] = src;
        s_w[threadIdx.x] = a.topk_weights[i];
    }
    if (a.self_rows) pdl_wait();
    if (threadIdx.x < 32) report_err(a.err, bad);
    __syncthreads();

    for (int vcol = v_begin + threadIdx.x; vcol < v_end; vcol += blockDim.x) {
        const size_t col = (size_t)vcol * 8;
        uint4 raw[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            raw[j] = make_uint4(0, 0, 0, 0);
            if (j < a.k) {
                const int kind = s_kind[j];
                if (kind == kRouted)
                    raw[j] = ld_stream_v4(a.expert_out + (size_t)s_src[j] * a.d + col);
                else if (kind != kSkip)
                    raw[j] = ld_stream_v4(a.ori_x + (size_t)t * a.d + col);
            }
        }
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j >= a.k) continue;
            const int kind = s_kind[j];
            if (kind == kSkip) continue;
            float e[8];
            unpack8(raw[j], e);
            if (kind == kConst) {
                const size_t off = (size_t)s_src[j] * a.d + col;
                float f1[8], f2[8], fv[8];
                unpack8(ld_stream_v4(a.a1 + off), f1);
                unpack8(ld_stream_v4(a.a2 + off), f2);
                unpack8(ld_stream_v4(a.v + off), fv);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    e[i] = __fadd_rn(__fmul_rn(f1[i], e[i]), __fmul_rn(f2[i], fv[i]));
            }
            const float w = s_w[j];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(w, e[i], acc[i]);
        }
        uint4 out;
        out.x = pack_bf16x2(acc[0], acc[1]);
        out.y = pack_bf16x2(acc[2], acc[3]);
        out.z = pack_bf16x2(acc[4], acc[5]);
        out.w = pack_bf16x2(acc[6], acc[7]);
        st_v4(a.y + (size_t)t * a.d + col, out);
    }
}

// ---------------------------------------------------------------------------
// Warp-independent combine.  A warp owns one (token, column slice): it classifies
// the token's picks itself (lanes < k read the routing, then broadcast it with
// shuffles), so no warp waits at a CTA barrier for another warp's loads.  Lane l
// takes the row's units l, l + 32, ... of its slice (a unit is VW 32-bit words,
// 2 * VW bf16 values); PIPE keeps the next unit's k loads in flight while the
// current unit is reduced.
// ---------------------------------------------------------------------------
#ifndef EP_COMBINE_VW
#define EP_COMBINE_VW 8
#endif
#ifndef EP_COMBINE_PIPE
#define EP_COMBINE_PIPE 1
#endif
constexpr int kCombineVW = EP_COMBINE_VW;         // words per unit (4: 16 bytes, 8: 32 bytes)
constexpr bool kCombinePipe = EP_COMBINE_PIPE != 0;
constexpr int kCombineWarps = 4;                   // warps per CTA

template <int VW>
struct VecW {
    uint32_t w[VW];
};
template <int VW>
__device__ __forceinline__ VecW<VW> ld_vec(const void* p) {
    VecW<VW> r;
    if constexpr (VW == 8) {
        const V8 v = ld_stream_v8(p);
#pragma unroll
        for (int e = 0; e < 8; ++e) r.w[e] = v.w[e];
    } else {
        const uint4 v = ld_stream_v4(p);
        r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
    }
    return r;
}
template <int VW>
__device__ __forceinline__ void st_vec(void* p, const VecW<VW>& v) {
    if constexpr (VW == 8) {
        V8 o;
#pragma unroll
        for (int e = 0; e < 8; ++e) o.w[e] = v.w[e];
        st_v8(p, o);
    } else {
        st_v4(p, make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]));
    }
}

template <int KM, int VW, bool PIPE>
__global__ void __launch_bounds__(32 * kCombineWarps) combine_warp_kernel(CombineArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int UB = 4 * VW;  // bytes of a unit
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long item = (long long)blockIdx.x * kCombineWarps + warp;
    const int t = (int)(item / a.chunks);
    const int c = (int)(item - (long long)t * a.chunks);
    const bool live = t < a.B;
    const bool on = live && !(a.active && !a.active[t]);

    // routing of token t: every lane ends with kind / src / w of each pick
    const int mine = (live && lane < a.k) ? __ldg(a.topk_idx + (size_t)t * a.k + lane) : -1;
    int rows[KM];
    if (a.self_rows) {
        uint16_t* tab = reinterpret_cast<uint16_t*>(smem + warp * warp_tab_bytes(a.E));
        zero_warp_tab(tab, a.E);
        if (live)
            routing_rows_warp<KM>(a.topk_idx, a.active, t, a.k, a.E, a.T, a.P, a.M, tab, rows,
                                  a.expert_offset, a.recv_count);
        pdl_wait();
    } else {
        pdl_wait();
        const int dp = (live && lane < a.k) ? a.dst_pos[(size_t)t * a.k + lane] : -1;
#pragma unroll
        for (int j = 0; j < KM; ++j) rows[j] = __shfl_sync(FULL, dp, j);
    }
    pdl_launch_dependents();
    const float wmine = (live && lane < a.k) ? a.topk_weights[(size_t)t * a.k + lane] : 0.0f;
    int kind[KM];
    long long src[KM];
    float w[KM];
    unsigned bad = 0;
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        const int g = on ? __shfl_sync(FULL, mine, j) : -1;
        w[j] = __shfl_sync(FULL, wmine, j);
        kind[j] = kSkip;
        src[j] = 0;
        if (j >= a.k || !live) continue;
        if (g >= 0 && g < a.E) {
            const int dp = live ? rows[j] : -1;
            if (dp >= 0 && (long long)dp < a.rows) {
                kind[j] = kRouted;
                src[j] = dp;
            } else if (dp != -1) {
                bad = EP_ERRBIT_ROW_RANGE;
            }
        } else if (g >= a.E + a.Z && g < a.E + a.Z + a.C) {
            kind[j] = kCopy;
        } else if (g >= a.E + a.Z + a.C && g < a.E + a.Z + a.C + a.K) {
            kind[j] = kConst;
            src[j] = g - (a.E + a.Z + a.C);
        }
    }
    if (lane == 0 && bad) atomicOr(a.err, bad);
    if (!live) return;

    const int nunits = (a.d * 2) / UB;
    const char* eo = reinterpret_cast<const char*>(a.expert_out);
    const char* ox = reinterpret_cast<const char*>(a.ori_x) + (size_t)t * a.d * 2;
    char* yrow = reinterpret_cast<char*>(a.y) + (size_t)t * a.d * 2;
    // units of this slice: lane + 32 * (c + chunks * i)
    auto unit_of = [&](int i) { return lane + 32 * (c + a.chunks * i); };
    auto issue = [&](VecW<VW> (&buf)[KM], int u) {
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (j < a.k && kind[j] == kRouted)
                buf[j] = ld_vec<VW>(eo + (size_t)src[j] * a.d * 2 + (size_t)u * UB);
            else if (j < a.k && kind[j] != kSkip)
                buf[j] = ld_vec<VW>(ox + (size_t)u * UB);
        }
    };
    auto reduce = [&](const VecW<VW> (&buf)[KM], int u) {
        float acc[2 * VW];
#pragma unroll
        for (int e = 0; e < 2 * VW; ++e) acc[e] = 0.0f;
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (j >= a.k || kind[j] == kSkip) continue;
            float e[2 * VW];
#pragma unroll
            for (int q = 0; q < VW; ++q) {
                e[2 * q] = bf16lo(buf[j].w[q]);
                e[2 * q + 1] = bf16hi(buf[j].w[q]);
            }
            if (kind[j] == kConst) {
                const size_t off = (size_t)src[j] * a.d * 2 + (size_t)u * UB;
                const VecW<VW> v1 = ld_vec<VW>(reinterpret_cast<const char*>(a.a1) + off);
                const VecW<VW> v2 = ld_vec<VW>(reinterpret_cast<const char*>(a.a2) + off);
                const VecW<VW> vv = ld_vec<VW>(reinterpret_cast<const char*>(a.v) + off);
#pragma unroll
                for (int q = 0; q < VW; ++q) {
                    e[2 * q] = __fadd_rn(__fmul_rn(bf16lo(v1.w[q]), e[2 * q]), __fmul_rn(bf16lo(v2.w[q]), bf16lo(vv.w[q])));
                    e[2 * q + 1] = __fadd_rn(__fmul_rn(bf16hi(v1.w[q]), e[2 * q + 1]), __fmul_rn(bf16hi(v2.w[q]), bf16hi(vv.w[q])));
                }
            }
#pragma unroll
            for (int e2 = 0; e2 < 2 * VW; ++e2) acc[e2] = __fmaf_rn(w[j], e[e2], acc[e2]);
        }
        VecW<VW> out;
#pragma unroll
        for (int q = 0; q < VW; ++q) out.w[q] = pack_bf16x2(acc[2 * q], acc[2 * q + 1]);
        st_vec<VW>(yrow + (size_t)u * UB, out);
    };

    if (PIPE) {
        VecW<VW> cur[KM], nxt[KM];
        int u = unit_of(0);
        if (u < nunits) issue(cur, u);
        for (int i = 0; u < nunits; ++i) {
            const int un = unit_of(i + 1);
            if (un < nunits) issue(nxt, un);
            reduce(cur, u);
#pragma unroll
            for (int j = 0; j < KM; ++j) cur[j] = nxt[j];
            u = un;
        }
    } else {
        for (int i = 0;; ++i) {
            const int u = unit_of(i);
            if (u >= nunits) break;
            VecW<VW> cur[KM];
            issue(cur, u);
            reduce(cur, u);
        }
    }
}

}  // namespace

int launch_combine(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* expert_out,
                   const int32_t* topk_idx, const float* topk_weights, const uint8_t* active,
                   const uint16_t* ori_x,
                   const uint16_t* a1, const uint16_t* a2, const uint16_t* v, uint16_t* y,
                   cudaStream_t stream) {
    if (s.B == 0) return EP_OK;
    CombineArgs a;
    a.expert_out = expert_out;
    a.topk_idx = topk_idx;
    a.active = active;
    a.topk_weights = topk_weights;
    a.dst_pos = p.dst_pos;
    a.ori_x = ori_x;
    a.a1 = a1;
    a.a2 = a2;
    a.v = v;
    a.y = y;
    a.err = &reinterpret_cast<WsHeader*>(p.workspace)->err;
    a.rows = s.rows;
    a.d = s.d;
    a.k = s.k;
    a.E = s.E;
    a.Z = s.Z;
    a.C = s.C;
    a.K = s.K;
    a.T = s.T;
    a.P = s.P;
    a.M = s.M;
    a.B = s.B;
    // packed rows also read the layout's counts, complete before the dispatch that
    // precedes this kernel started
    a.self_rows = s.T <= kCombineSelfRowsMaxT ? 1 : 0;
    a.expert_offset = (a.self_rows && s.layout == 1) ? p.expert_offset : nullptr;
    a.recv_count = (a.self_rows && s.layout == 1) ? p.recv_count : nullptr;
#ifndef EP_COMBINE_OLD
    {
        // 32-byte units need every row base it reads or writes 32-byte aligned (rows
        // are 2d bytes apart, a multiple of 32); otherwise and for k > 8, 16-byte units
        auto al32 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 31u) == 0; };
        const bool wide = kCombineVW == 8 && s.k <= 8 && al32(expert_out) && al32(y) &&
                          (s.C + s.K == 0 || al32(ori_x)) && (s.K == 0 || (al32(a1) && al32(a2) && al32(v)));
        const int UB = wide ? 32 : 16;
        // one warp per (token, column slice): slices only when the batch is too
        // small to give every SM about eight warps
        const int nunits = (s.d * 2) / UB;
        const int max_chunks = (nunits + 31) / 32;
        long long chunks = (long long)num_sms() * 8 / (s.B > 0 ? s.B : 1);
        if (chunks < 1) chunks = 1;
        if (chunks > max_chunks) chunks = max_chunks;
        a.chunks = (int)chunks;
        const long long items = (long long)s.B * a.chunks;
        const long long nblk = (items + kCombineWarps - 1) / kCombineWarps;
        if (nblk > 0x7fffffffLL) return EP_ERR_UNSUPPORTED;
        const size_t smem = a.self_rows ? (size_t)kCombineWarps * warp_tab_bytes(s.E) : 0;
        void (*kern)(CombineArgs);
        if (s.k <= 4)
            kern = wide ? combine_warp_kernel<4, 8, kCombinePipe> : combine_warp_kernel<4, 4, kCombinePipe>;
        else if (s.k <= 8)
            kern = wide ? combine_warp_kernel<8, 8, kCombinePipe> : combine_warp_kernel<8, 4, kCombinePipe>;
        else  // 16 picks: 16-byte units without the prefetch, to stay within the registers
            kern = combine_warp_kernel<16, 4, false>;
        const cudaError_t e = launch_pdl(kern, dim3((unsigned)nblk), dim3(32 * kCombineWarps), smem, stream, a);
        return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
    }
#endif
    // One CTA per token when that fills the GPU in about one wave; otherwise split
    // each token's columns over up to nvec / NT CTAs.
    const int nvec = s.d / 8;
    const int NT = nvec < 128 ? ((nvec + 31) / 32) * 32 : 128;
    const int max_chunks = (nvec + NT - 1) / NT;
    const long long target = (long long)num_sms() * 7;
    long long chunks = target / (s.B > 0 ? s.B : 1);
    if (chunks < 1) chunks = 1;
    if (chunks > max_chunks) chunks = max_chunks;
    a.chunks = (int)chunks;
    const long long nblocks = (long long)s.B * a.chunks;
    if (nblocks > 0x7fffffffLL) return EP_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)nblocks);
    cudaError_t e;
    if (s.k <= 2)
        e = launch_pdl(combine_kernel<2>, grid, dim3(NT), 0, stream, a);
    else if (s.k <= 4)
        e = launch_pdl(combine_kernel<4>, grid, dim3(NT), 0, stream, a);
    else if (s.k <= 8)
        e = launch_pdl(combine_kernel<8>, grid, dim3(NT), 0, stream, a);
    else
        e = launch_pdl(combine_kernel<16>, grid, dim3(NT), 0, stream, a);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

}  // namespace ep
