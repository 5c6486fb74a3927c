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

// Where the receive rows come from.  The routing scan runs before
// griddepcontrol.wait, so it is hidden only while a preceding kernel of the
// library still runs; otherwise its cost is exposed (about 1 us at decode, more
// than the one round trip of reading dst_pos after the wait).  In a model the
// combine follows the expert kernels, so dst_pos is the default.  The scan is kept
// where it measured faster in back-to-back steps: per-rank batches of at most
// kCombineScanMaxT tokens (few earlier tokens to scan), and, up to
// kCombineSelfRowsMaxT tokens, buffers with a per-expert smooth table, whose
// persistent dispatch kernel drains while the scan runs (56.5 against 63.0 us per
// step at decode).  Above kCombineSelfRowsMaxT the scan's L2 reads grow with T.
constexpr int kCombineScanMaxT = 16;
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
};

__device__ __forceinline__ void unpack8(const uint4& r, float* f) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16lo(w[i]);
        f[2 * i + 1] = bf16hi(w[i]);
    }
}

// Where the expert output of a routed row lives: this buffer's expert_out, or the
// slab of the rank that owns the row's expert (see ShardTable).
struct LocalOut {
    __device__ __forceinline__ const uint16_t* row(const CombineArgs& a, int r) const {
        return a.expert_out + (size_t)r * a.d;
    }
};
struct ShardOut {
    const ShardTable& tab;
    __device__ __forceinline__ const uint16_t* row(const CombineArgs& a, int r) const {
        const int q = (int)(r / tab.slab_rows);
        return reinterpret_cast<const uint16_t*>(tab.x[q]) + (size_t)(r - q * tab.slab_rows) * a.d;
    }
};

template <int KMAX, class Out>
__device__ __forceinline__ void combine_body(const CombineArgs& a, const Out& out_rows) {
    __shared__ const uint16_t* s_ptr[KMAX];  // row the pick reads (expert output or ori_x[t]); null: no term
    __shared__ float s_w[KMAX];
    __shared__ int s_const[KMAX];            // constant expert index, -1 for other picks
    __shared__ uint16_t s_tab[kMaxE];

    // CTA = (token t, column slice c); the slice is swept by the CTA's threads
    const int t = blockIdx.x / a.chunks;
    const int c = blockIdx.x - t * a.chunks;
    const int nvec = a.d >> 3;
    const int span = (nvec + a.chunks - 1) / a.chunks;
    const int v_begin = c * span;
    const int v_end = min(nvec, v_begin + span);

    // With self_rows the prologue reads the routing (topk_idx, topk_weights and the
    // optional x_active_mask), which was complete before the preceding kernels
    // started, and in the packed layout also expert_offset and recv_count, which
    // ep_layout's counting kernel finished before the library's later kernels could
    // start.  So it runs before griddepcontrol.wait and overlaps their tail; the
    // expert outputs are read and y is written only after the wait.  (The public
    // header states what a caller may therefore not launch in between.)
    __shared__ int s_rows[KMAX], s_g[KMAX], s_cnt[KMAX];
    // the weights were final before the preceding kernels started (as topk_idx):
    // their load is issued first so its latency overlaps the row lookup
    const float wt = threadIdx.x < a.k ? a.topk_weights[(size_t)t * a.k + threadIdx.x] : 0.0f;
    if (a.self_rows) {
        routing_rows(a.topk_idx, a.active, t, a.k, a.E, a.T, a.P, a.M, s_rows, s_g, s_cnt, s_tab,
                     a.expert_offset, a.recv_count);
    } else {
        pdl_wait();
    }
    pdl_launch_dependents();

    unsigned bad = 0;
    int is_const = 0;
    const bool on = !(a.active && !a.active[t]);  // an inactive token has no terms
    if (threadIdx.x < a.k) {
        const size_t i = (size_t)t * a.k + threadIdx.x;
        const int g = on ? a.topk_idx[i] : -1;
        const int dp = a.self_rows ? s_rows[threadIdx.x] : a.dst_pos[i];
        const uint16_t* ptr = nullptr;
        int cidx = -1;
        if (g >= 0 && g < a.E) {
            if (dp >= 0 && (long long)dp < a.rows)
                ptr = out_rows.row(a, dp);
            else if (dp != -1)
                bad = EP_ERRBIT_ROW_RANGE;
        } else if (g >= a.E + a.Z && g < a.E + a.Z + a.C) {
            ptr = a.ori_x + (size_t)t * a.d;  // copy expert
        } else if (g >= a.E + a.Z + a.C && g < a.E + a.Z + a.C + a.K) {
            ptr = a.ori_x + (size_t)t * a.d;  // constant expert: a1[c] * ori_x + a2[c] * v[c]
            cidx = g - (a.E + a.Z + a.C);
            is_const = 1;
        }
        s_ptr[threadIdx.x] = ptr;
        s_w[threadIdx.x] = wt;
        s_const[threadIdx.x] = cidx;
    }
    if (a.self_rows) pdl_wait();
    if (threadIdx.x < 32) report_err(a.err, bad);
    const int any_const = __syncthreads_or(is_const);

    // picks with a term (CTA-uniform): skipped picks add nothing, exactly as if absent
    unsigned live = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
        if (j < a.k && s_ptr[j] != nullptr) live |= 1u << j;

    for (int vcol = v_begin + threadIdx.x; vcol < v_end; vcol += blockDim.x) {
        const size_t col = (size_t)vcol * 8;
        uint4 raw[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            raw[j] = ((live >> j) & 1u) ? ld_stream_v4(s_ptr[j] + col) : make_uint4(0, 0, 0, 0);
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (!((live >> j) & 1u)) continue;
            float e[8];
            unpack8(raw[j], e);
            if (any_const && s_const[j] >= 0) {
                const size_t off = (size_t)s_const[j] * a.d + col;
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

template <int KMAX>
__global__ void __launch_bounds__(128, (KMAX > 8 ? 4 : 8)) combine_kernel(CombineArgs a) {
    combine_body<KMAX>(a, LocalOut());
}

// Multi-GPU form: expert outputs read from every rank's slab (peer loads).
template <int KMAX>
__global__ void __launch_bounds__(128, (KMAX > 8 ? 4 : 8))
    combine_shard_kernel(CombineArgs a, const __grid_constant__ ShardTable tab) {
    combine_body<KMAX>(a, ShardOut{tab});
}

}  // namespace

namespace {
int launch_combine_impl(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* expert_out,
                        const int32_t* topk_idx, const float* topk_weights, const uint8_t* active,
                        const uint16_t* ori_x, const uint16_t* a1, const uint16_t* a2,
                        const uint16_t* v, uint16_t* y, cudaStream_t stream, const ShardTable* tab) {
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
    // packed rows also read the layout's counts, complete before the dispatch that
    // precedes this kernel started
    a.self_rows = (tab == nullptr && (s.T <= kCombineScanMaxT ||
                                      (s.expert_smooth && s.T <= kCombineSelfRowsMaxT))) ? 1 : 0;
    a.expert_offset = (a.self_rows && s.layout == 1) ? p.expert_offset : nullptr;
    a.recv_count = (a.self_rows && s.layout == 1) ? p.recv_count : nullptr;
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
    if (tab) {
        if (s.k <= 2)
            e = launch_pdl(combine_shard_kernel<2>, grid, dim3(NT), 0, stream, a, *tab);
        else if (s.k <= 4)
            e = launch_pdl(combine_shard_kernel<4>, grid, dim3(NT), 0, stream, a, *tab);
        else if (s.k <= 8)
            e = launch_pdl(combine_shard_kernel<8>, grid, dim3(NT), 0, stream, a, *tab);
        else
            e = launch_pdl(combine_shard_kernel<16>, grid, dim3(NT), 0, stream, a, *tab);
    } else if (s.k <= 2)
        e = launch_pdl(combine_kernel<2>, grid, dim3(NT), 0, stream, a);
    else if (s.k <= 4)
        e = launch_pdl(combine_kernel<4>, grid, dim3(NT), 0, stream, a);
    else if (s.k <= 8)
        e = launch_pdl(combine_kernel<8>, grid, dim3(NT), 0, stream, a);
    else
        e = launch_pdl(combine_kernel<16>, grid, dim3(NT), 0, stream, a);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}
}  // namespace

int launch_combine(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* expert_out,
                   const int32_t* topk_idx, const float* topk_weights, const uint8_t* active,
                   const uint16_t* ori_x,
                   const uint16_t* a1, const uint16_t* a2, const uint16_t* v, uint16_t* y,
                   cudaStream_t stream) {
    return launch_combine_impl(s, p, expert_out, topk_idx, topk_weights, active, ori_x, a1, a2, v, y,
                               stream, nullptr);
}

int launch_shard_combine(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                         const float* topk_weights, const uint8_t* active, const uint16_t* ori_x,
                         const uint16_t* a1, const uint16_t* a2, const uint16_t* v, uint16_t* y,
                         const ShardTable& tab, cudaStream_t stream) {
    return launch_combine_impl(s, p, nullptr, topk_idx, topk_weights, active, ori_x, a1, a2, v, y,
                               stream, &tab);
}

}  // namespace ep
