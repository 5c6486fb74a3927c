// Device-side pieces of the layout shared by the layout kernels (ep_layout.cu)
// and the fused layout+dispatch kernel (ep_fused.cu).  Internal header.
#pragma once

#include "ep_internal.cuh"

namespace ep {
namespace {

struct LayoutArgs {
    const int32_t* topk_idx;
    const uint8_t* active;  // x_active_mask [B] or null
    int32_t* expert_count;
    int32_t* expert_offset;
    int32_t* recv_count;
    int32_t* dst_pos;
    int32_t* recv_src;
    WsHeader* ws;
    int32_t* chunk_cnt;   // larger batches: [P][chunks][E] routed picks per expert and chunk
    int32_t* sp_chunk;    // larger batches: [P][chunks][n_special] special-expert picks
    int B, k, P, M, E, T, n_special, E_tot;
    long long rows;       // receive rows the computed row ids index (E * P * M)
    int warps;            // warps per CTA
    // row of (expert g, rank r, slot) = g * gstride + r * M + rbase + slot: P * M and 0
    // on one GPU; a process that lays out only its own rank's tokens (P = 1 here)
    // uses the global stride and its rank's offset
    int gstride, rbase;
};

// Exclusive prefix of cnt[0..n) into out[0..n], out[n] = total; all threads of the
// CTA call it.  Thread i owns a contiguous chunk; chunk sums go through a warp
// shuffle scan and one pass over the warp totals.  wsum: 32 ints of shared memory.
__device__ void block_exclusive_scan(const int* cnt, int n, int32_t* out, int* wsum) {
    const int per = (n + (int)blockDim.x - 1) / (int)blockDim.x;
    const int lo = min(n, (int)threadIdx.x * per);
    const int hi = min(n, lo + per);
    int local = 0;
    for (int g = lo; g < hi; ++g) local += cnt[g];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int nw = (blockDim.x + 31) >> 5;
        int v = lane < nw ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        wsum[lane] = v;
    }
    __syncthreads();
    int acc = x - local + (warp > 0 ? wsum[warp - 1] : 0);
    for (int g = lo; g < hi; ++g) {
        out[g] = acc;
        acc += cnt[g];
    }
    if (threadIdx.x == blockDim.x - 1) out[n] = acc;
}

// Pick ids of token t into ids[0..k), -1 beyond k.  16-byte loads when each row
// starts on a 16-byte boundary (k % 4 == 0 and an aligned base).
template <int KM>
__device__ __forceinline__ void load_token_ids(const int32_t* topk_idx, int t, int k, bool vec4,
                                               int* ids) {
    if (vec4) {
        const int4* src = reinterpret_cast<const int4*>(topk_idx + (size_t)t * k);
#pragma unroll
        for (int j4 = 0; j4 < KM / 4; ++j4) {
            int4 v = make_int4(-1, -1, -1, -1);
            if (4 * j4 < k) v = __ldg(src + j4);
            ids[4 * j4] = v.x;
            ids[4 * j4 + 1] = v.y;
            ids[4 * j4 + 2] = v.z;
            ids[4 * j4 + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < KM; ++j) ids[j] = (j < k) ? __ldg(topk_idx + (size_t)t * k + j) : -1;
    }
}

// An inactive token (x_active_mask entry 0) is seen as k picks of -1.
template <int KM>
__device__ __forceinline__ void apply_active(const uint8_t* active, int t, int* ids) {
    if (active && !active[t]) {
#pragma unroll
        for (int j = 0; j < KM; ++j) ids[j] = -1;
    }
}

// Classify the picks of one token: returns a mask with bit j set when pick j is
// routed (the first occurrence of an id in [0, E)); repeated routed ids and ids
// outside [-1, E_tot) set error bits; specials are handed to on_special.
template <int KM, typename OnSpecial>
__device__ __forceinline__ unsigned classify_ids(const int* ids, int k, int E, int E_tot,
                                                 unsigned& err, OnSpecial on_special) {
    unsigned routed = 0;
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        if (j >= k) continue;
        const int g = ids[j];
        if (g == -1) continue;
        if (g < -1 || g >= E_tot) {
            err |= EP_ERRBIT_BAD_ID;
            continue;
        }
        if (g >= E) {
            on_special(g - E);
            continue;
        }
        bool dup = false;
#pragma unroll
        for (int jj = 0; jj < KM; ++jj)
            if (jj < j && ids[jj] == g) dup = true;
        if (dup) {
            err |= EP_ERRBIT_DUP_ID;
            continue;
        }
        routed |= 1u << j;
    }
    return routed;
}

// Layout for small per-rank batches (T <= 256), with no dependency between CTAs.
//  - CTA 0 (the count CTA) histograms every token's ids per expert id (routed and
//    special) and writes expert_count and its exclusive prefix expert_offset.
//  - Every other CTA holds whole ranks (warps / ceil(T/32) of them) with one warp per
//    32-token chunk.  A warp sets, in shared memory, one lane bit per routed id of
//    its tokens; after one barrier a token's slot is the popcount of the earlier
//    chunks' masks of its rank plus popc(mask & lanemask_lt) of its own chunk,
//    i.e. its rank among the rank's tokens that routed to g, in token order; the
//    sum of its ranks' chunk popcounts per expert is recv_count.
// Each warp reads only its own tokens' ids, and both halves use order-independent
// shared-memory atomics, so the result is deterministic.
// shard (multi-GPU form, one rank laid out as P = 1): when given, the slot CTA also
// stores each expert's count into column shard->rank of the owning rank's recv_count,
// which is the count exchange of ep_shard_layout_dispatch.
template <int KM>
__device__ __forceinline__ void layout_small_body(const LayoutArgs& a, int cpr, int cta,
                                                  unsigned* smem, const ShardTable* shard = nullptr) {
    const int E = a.E, k = a.k, P = a.P;
    const bool vec4 = (k % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.topk_idx) & 15) == 0);
    unsigned err = 0;

    if (cta == 0) {
        // count CTA: picks per expert id over all tokens, then the exclusive prefix
        int* ec = reinterpret_cast<int*>(smem);  // [E_tot]
        int* wsum = ec + a.E_tot;                // [32]
        for (int i = threadIdx.x; i < a.E_tot; i += blockDim.x) ec[i] = 0;
        __syncthreads();
        // four tokens per thread per pass, their id loads issued together
        const int stride = blockDim.x;
        for (int t0 = threadIdx.x; t0 < a.B; t0 += 4 * stride) {
            int ids[4][KM];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int t = t0 + b * stride;
                if (t < a.B) {
                    load_token_ids<KM>(a.topk_idx, t, k, vec4, ids[b]);
                    apply_active<KM>(a.active, t, ids[b]);
                } else {
#pragma unroll
                    for (int j = 0; j < KM; ++j) ids[b][j] = -1;
                }
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                if (t0 + b * stride >= a.B) continue;
                const unsigned rb = classify_ids<KM>(ids[b], k, E, a.E_tot, err,
                                                     [&](int sidx) { atomicAdd(&ec[E + sidx], 1); });
#pragma unroll
                for (int j = 0; j < KM; ++j)
                    if (rb & (1u << j)) atomicAdd(&ec[ids[b][j]], 1);
            }
        }
        __syncthreads();
        for (int g = threadIdx.x; g < a.E_tot; g += blockDim.x) a.expert_count[g] = ec[g];
        report_err(&a.ws->err, err);
        block_exclusive_scan(ec, a.E_tot, a.expert_offset, wsum);
        return;
    }

    // slot CTAs: whole ranks per CTA (warps / cpr of them), one warp per 32-token chunk
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ranks_per_cta = (int)(blockDim.x >> 5) / cpr;
    const int lr = warp / cpr, c = warp - lr * cpr;
    const int r = (cta - 1) * ranks_per_cta + lr;
    const bool holds_rank = lr < ranks_per_cta && r < P;
    unsigned* mask = reinterpret_cast<unsigned*>(smem);  // [warps][E]
    unsigned* my_mask = mask + (size_t)warp * E;
    for (int g = lane; g < E; g += 32) my_mask[g] = 0u;
    __syncthreads();
    const int t = a.T * r + c * 32 + lane;
    const bool valid = holds_rank && c * 32 + lane < a.T;
    int ids[KM];
    unsigned rb = 0;
    if (valid) {
        load_token_ids<KM>(a.topk_idx, t, k, vec4, ids);
        apply_active<KM>(a.active, t, ids);
        rb = classify_ids<KM>(ids, k, E, a.E_tot, err, [](int) {});
    }
#pragma unroll
    for (int j = 0; j < KM; ++j)
        if (rb & (1u << j)) atomicOr(&my_mask[ids[j]], 1u << lane);
    __syncthreads();
    if (valid) {
        const unsigned lt = lanemask_lt();
        const unsigned* rank_masks = mask + (size_t)(lr * cpr) * E;
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (j >= k) continue;
            int row = -1;
            if (rb & (1u << j)) {
                const int g = ids[j];
                int before = 0;  // the rank's tokens in its earlier chunks that routed to g
                for (int cc = 0; cc < c; ++cc) before += __popc(rank_masks[(size_t)cc * E + g]);
                row = g * a.gstride + r * a.M + a.rbase + before + __popc(my_mask[g] & lt);
                if (!ep_in_range(row, a.rows, &a.ws->err)) row = -1;
                else if (a.recv_src) a.recv_src[row] = t;
            }
            a.dst_pos[(size_t)t * k + j] = row;
        }
    }
    // recv_count of this CTA's ranks: every chunk's popcount, per expert
    for (int i = threadIdx.x; i < ranks_per_cta * E; i += blockDim.x) {
        const int lrr = i / E, g = i - lrr * E;
        const int rr = (cta - 1) * ranks_per_cta + lrr;
        if (rr >= P) continue;
        int n = 0;
        for (int cc = 0; cc < cpr; ++cc) n += __popc(mask[(size_t)(lrr * cpr + cc) * E + g]);
        a.recv_count[(size_t)g * P + rr] = n;
        if (shard) {
            const int q = g / shard->L;
            if (shard->count[q]) shard->count[q][(size_t)(g - q * shard->L) * shard->P + shard->rank] = n;
        }
    }
    // errors of the chunk's own tokens only (the count CTA reports the same bits)
    report_err(&a.ws->err, err);
}

}  // namespace
}  // namespace ep
