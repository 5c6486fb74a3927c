// Routing layout kernel.
//
// Computes, from topk_idx[B][k], the per-expert counts, the per-(expert, source
// rank) counts, their exclusive prefix and the low-latency receive row of every
// routed pick (Ascend CANN "low_latency_dispatch": Formula, the alltoallv of the
// quantized rows; Constraints, the row bound A >= M * P * min(L, K) and the
// deterministic computation).  Expert g lives on rank g / (E / P) (DeepEP issue
// #84, masking experiment); id -1 sends nothing.
//
// Design.  One CTA per source rank r.  The rank's tokens are processed in rounds
// of (warps x 32) tokens, one token per lane.  In a round every warp builds, in
// shared memory, a 32-bit lane mask per routed expert (atomicOr of bit `lane`
// for each of its token's routed ids).  Because OR is order-independent the
// masks, and everything derived from them, are deterministic.  An exclusive scan
// over the warps of popc(mask) per expert, plus the counts of earlier rounds,
// gives each warp's base; a token's slot inside its (expert, rank) run is then
//     base[w][g] + popc(mask[w][g] & lanemask_lt)
// i.e. its rank among rank r's tokens that routed to g, in ascending token order.
// The last CTA to finish (a ticket counter in the workspace; no CTA ever waits on
// another) adds the per-rank counts into expert_count and scans expert_offset.
#include <mutex>

#include "ep_internal.cuh"
#include "ep_layout_dev.cuh"

namespace ep {
namespace {

template <int KM>
__global__ void __launch_bounds__(256) layout_small_kernel(LayoutArgs a, int cpr) {
    extern __shared__ unsigned smem[];
    pdl_wait();
    pdl_launch_dependents();
    layout_small_body<KM>(a, cpr, blockIdx.x, smem);
}

template <int KM>
__global__ void __launch_bounds__(1024) layout_kernel(LayoutArgs a) {
    extern __shared__ unsigned smem[];
    const int W = a.warps;
    unsigned* mask = smem;                                         // [W][E]
    int* pre = reinterpret_cast<int*>(smem + (size_t)W * a.E);     // [W][E]
    int* run = pre + (size_t)W * a.E;                              // [E] count so far
    int* spc = run + a.E;                                          // [n_special]
    __shared__ int s_last;

    const int r = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int E = a.E, k = a.k;

    pdl_wait();
    pdl_launch_dependents();

    for (int g = threadIdx.x; g < E; g += blockDim.x) run[g] = 0;
    for (int s = threadIdx.x; s < a.n_special; s += blockDim.x) spc[s] = 0;

    unsigned err = 0;
    const int tok_begin = r * a.T;
    const int tok_end = tok_begin + a.T;
    const int per_round = W * 32;
    unsigned* my_mask = mask + (size_t)warp * E;
    int* my_pre = pre + (size_t)warp * E;

    for (int round0 = tok_begin; round0 < tok_end; round0 += per_round) {
        // (1) clear this warp's masks (the previous round's readers of my_mask
        //     are this warp's own lanes, so a warp barrier suffices)
        __syncwarp();
        for (int g = lane; g < E; g += 32) my_mask[g] = 0u;
        __syncthreads();  // also orders run[] / spc[] init before first use

        const int t = round0 + warp * 32 + lane;
        const bool valid = t < tok_end;
        int ids[KM];
        bool routed[KM];
        const bool on = valid && !(a.active && !a.active[t]);  // x_active_mask
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            ids[j] = -1;
            routed[j] = false;
            if (j < k && on) ids[j] = a.topk_idx[(size_t)t * k + j];
        }
        // (2) classify; routed ids set their lane bit
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (j >= k || !valid) continue;
            const int g = ids[j];
            if (g == -1) continue;
            if (g < -1 || g >= a.E_tot) {
                err |= EP_ERRBIT_BAD_ID;
                continue;
            }
            if (g >= E) {
                atomicAdd(&spc[g - E], 1);
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
            routed[j] = true;
            atomicOr(&my_mask[g], 1u << lane);
        }
        __syncthreads();
        // (3) per expert: exclusive scan of the warps' popcounts, on top of the
        //     counts of earlier rounds
        for (int g = threadIdx.x; g < E; g += blockDim.x) {
            int c = run[g];
            for (int w = 0; w < W; ++w) {
                pre[(size_t)w * E + g] = c;
                c += __popc(mask[(size_t)w * E + g]);
            }
            run[g] = c;
        }
        __syncthreads();
        // (4) slots, receive rows, source map
        if (valid) {
            const unsigned lt = lanemask_lt();
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                if (j >= k) continue;
                int row = -1;
                if (routed[j]) {
                    const int g = ids[j];
                    const int slot = my_pre[g] + __popc(my_mask[g] & lt);
                    row = g * a.P * a.M + r * a.M + slot;
                    if (!ep_in_range(row, a.rows, &a.ws->err)) row = -1;
                    else if (a.recv_src) a.recv_src[row] = t;
                }
                a.dst_pos[(size_t)t * k + j] = row;
            }
        }
    }
    __syncthreads();

    // per-rank outputs
    for (int g = threadIdx.x; g < E; g += blockDim.x) a.recv_count[(size_t)g * a.P + r] = run[g];
    for (int s = threadIdx.x; s < a.n_special; s += blockDim.x)
        a.sp_partial[(size_t)r * a.n_special + s] = spc[s];
    report_err(&a.ws->err, err);

    // ticket: the last CTA of this launch reduces over ranks
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned ticket = atomicAdd(&a.ws->done, 1u);
        s_last = (ticket == (unsigned)a.P - 1u);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // expert_count over all ids, then its exclusive prefix into expert_offset.
    // The rank loop is unrolled so a thread's loads are in flight together.
    int* ec = reinterpret_cast<int*>(smem);            // reuse: [E_tot]
    int* wsum = ec + a.E_tot;                          // [32]
    for (int g = threadIdx.x; g < a.E_tot; g += blockDim.x) {
        int v = 0;
        if (g < E) {
            const int32_t* src = a.recv_count + (size_t)g * a.P;
#pragma unroll 8
            for (int q = 0; q < a.P; ++q) v += __ldcg(src + q);
        } else {
#pragma unroll 8
            for (int q = 0; q < a.P; ++q) v += __ldcg(&a.sp_partial[(size_t)q * a.n_special + (g - E)]);
        }
        ec[g] = v;
        a.expert_count[g] = v;
    }
    __syncthreads();
    block_exclusive_scan(ec, a.E_tot, a.expert_offset, wsum);
    if (threadIdx.x == 0) a.ws->done = 0u;  // re-arm the ticket for the next launch
}

// Packed layout, second step: the layout kernels left each routed pick's row in
// low-latency form with stride T (g*P*T + r*T + slot); with every rank's counts
// known, the row becomes expert_offset[g] + sum_{r' < r} recv_count[g][r'] + slot,
// and recv_src is written at it.  Each CTA builds the (expert, rank) base table in
// shared memory, then converts a grid-strided share of the picks.
__global__ void __launch_bounds__(256) layout_pack_kernel(const int32_t* expert_offset,
                                                          const int32_t* recv_count, int32_t* dst_pos,
                                                          int32_t* recv_src, int B, int k, int P,
                                                          int T, int E, unsigned* err) {
    extern __shared__ int base[];  // [E][P]
    pdl_wait();
    pdl_launch_dependents();
    for (int g = threadIdx.x; g < E; g += blockDim.x) {
        int run = expert_offset[g];
        for (int r = 0; r < P; ++r) {
            base[g * P + r] = run;
            run += recv_count[g * P + r];
        }
    }
    __syncthreads();
    const long long n = (long long)B * k;
    const int PT = P * T;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const int v = dst_pos[i];
        if (v < 0) continue;
        const int g = v / PT;
        const int rem = v - g * PT;
        const int r = rem / T;
        if (!ep_in_range((long long)g * P + r, (long long)E * P, err)) {
            dst_pos[i] = -1;
            continue;
        }
        const int row = base[g * P + r] + (rem - r * T);
        if (!ep_in_range(row, n, err)) {
            dst_pos[i] = -1;
            continue;
        }
        dst_pos[i] = row;
        recv_src[row] = (int)(i / k);
    }
}

}  // namespace

int launch_layout(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                  const uint8_t* active, cudaStream_t stream) {
    if (s.layout == 1 && s.B > 0) {
        // counts and low-latency-form rows (stride T, no recv_src), then pack
        Shape ll = s;
        ll.layout = 0;
        ll.M = s.T;
        ll.rows = (long long)s.E * s.P * s.T;
        ep_buffer_ptrs q = p;
        q.recv_src = nullptr;
        const int st = launch_layout(ll, q, topk_idx, active, stream);
        if (st != EP_OK) return st;
        const size_t smem = sizeof(int) * (size_t)s.E * s.P;
        static bool attr_pack[kDeviceSlots] = {false};
        int dev = 0;
        cudaGetDevice(&dev);
        if (first_on_device(attr_pack, dev)) {
            if (cudaFuncSetAttribute(layout_pack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(sizeof(int) * kMaxPackedEP)) != cudaSuccess)
                return EP_ERR_CUDA;
            mark_device(attr_pack, dev);
        }
        long long grid = ((long long)s.B * s.k + 1023) / 1024;
        if (grid > (long long)num_sms() * 4) grid = (long long)num_sms() * 4;
        if (grid < 1) grid = 1;
        cudaError_t e = launch_pdl(layout_pack_kernel, dim3((unsigned)grid), dim3(256), smem, stream,
                                   (const int32_t*)p.expert_offset, (const int32_t*)p.recv_count,
                                   p.dst_pos, p.recv_src, s.B, s.k, s.P, s.T, s.E,
                                   &reinterpret_cast<WsHeader*>(p.workspace)->err);
        return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
    }
    if (s.B == 0) {
        // no tokens: counts are all zero
        cudaError_t e1 = cudaMemsetAsync(p.expert_count, 0, sizeof(int32_t) * s.E_tot, stream);
        cudaError_t e2 = cudaMemsetAsync(p.expert_offset, 0, sizeof(int32_t) * (s.E_tot + 1), stream);
        cudaError_t e3 = cudaMemsetAsync(p.recv_count, 0, sizeof(int32_t) * s.E * s.P, stream);
        return (e1 || e2 || e3) ? EP_ERR_CUDA : EP_OK;
    }
    const size_t budget = 160 * 1024;
    static bool attr_small[kDeviceSlots] = {false};
    int dev0 = 0;
    cudaGetDevice(&dev0);
    // small per-rank batches: count CTA + slot CTAs, no inter-CTA dependency
    const int cpr = (s.T + 31) / 32;
    const size_t smem_count = sizeof(int) * ((size_t)s.E_tot + 32);
    const size_t smem_slot = sizeof(int) * (size_t)8 * s.E;
    const size_t smem_small = smem_count > smem_slot ? smem_count : smem_slot;
    if (s.T <= 256 && smem_small <= budget) {
        if (first_on_device(attr_small, dev0)) {
            if (cudaFuncSetAttribute(layout_small_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget) ||
                cudaFuncSetAttribute(layout_small_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget) ||
                cudaFuncSetAttribute(layout_small_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget) ||
                cudaFuncSetAttribute(layout_small_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget))
                return EP_ERR_CUDA;
            mark_device(attr_small, dev0);
        }
        LayoutArgs a1;
        a1.topk_idx = topk_idx;
        a1.active = active;
        a1.expert_count = p.expert_count;
        a1.expert_offset = p.expert_offset;
        a1.recv_count = p.recv_count;
        a1.dst_pos = p.dst_pos;
        a1.recv_src = p.recv_src;
        a1.ws = reinterpret_cast<WsHeader*>(p.workspace);
        a1.sp_partial = nullptr;
        a1.B = s.B; a1.k = s.k; a1.P = s.P; a1.M = s.M; a1.E = s.E; a1.T = s.T;
        a1.n_special = s.n_special; a1.E_tot = s.E_tot;
        a1.rows = s.rows;
        a1.warps = 8;
        const int ranks_per_cta = 8 / cpr;
        const int grid = 1 + (s.P + ranks_per_cta - 1) / ranks_per_cta;
        cudaError_t e;
        if (s.k <= 2)
            e = launch_pdl(layout_small_kernel<2>, dim3(grid), dim3(256), smem_small, stream, a1, cpr);
        else if (s.k <= 4)
            e = launch_pdl(layout_small_kernel<4>, dim3(grid), dim3(256), smem_small, stream, a1, cpr);
        else if (s.k <= 8)
            e = launch_pdl(layout_small_kernel<8>, dim3(grid), dim3(256), smem_small, stream, a1, cpr);
        else
            e = launch_pdl(layout_small_kernel<16>, dim3(grid), dim3(256), smem_small, stream, a1, cpr);
        return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
    }
    // multi-CTA path: one CTA per rank; warps per CTA enough for one round of the
    // rank's tokens, at most 32, within the shared-memory budget (two [warps][E]
    // arrays plus [E] + specials)
    const size_t fixed = sizeof(int) * ((size_t)s.E + s.n_special);
    int warps = (s.T + 31) / 32;
    if (warps > 32) warps = 32;
    if (warps < 1) warps = 1;
    while (warps > 1 && fixed + (size_t)warps * s.E * 8 > budget) --warps;
    size_t smem = fixed + (size_t)warps * s.E * 8;
    const size_t need_tail = sizeof(int) * ((size_t)s.E_tot + 32);  // counts + scan of the last CTA
    if (smem < need_tail) smem = need_tail;
    if (smem > budget) return EP_ERR_UNSUPPORTED;

    static bool attr_set[kDeviceSlots] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (first_on_device(attr_set, dev)) {
        if (cudaFuncSetAttribute(layout_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget) ||
            cudaFuncSetAttribute(layout_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget) ||
            cudaFuncSetAttribute(layout_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget) ||
            cudaFuncSetAttribute(layout_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget))
            return EP_ERR_CUDA;
        mark_device(attr_set, dev);
    }

    LayoutArgs a;
    a.topk_idx = topk_idx;
    a.active = active;
    a.expert_count = p.expert_count;
    a.expert_offset = p.expert_offset;
    a.recv_count = p.recv_count;
    a.dst_pos = p.dst_pos;
    a.recv_src = p.recv_src;
    a.ws = reinterpret_cast<WsHeader*>(p.workspace);
    a.sp_partial = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.workspace) + sizeof(WsHeader));
    a.B = s.B; a.k = s.k; a.P = s.P; a.M = s.M; a.E = s.E; a.T = s.T;
    a.n_special = s.n_special; a.E_tot = s.E_tot;
    a.rows = s.rows;
    a.warps = warps;
    cudaError_t e;
    if (s.k <= 2)
        e = launch_pdl(layout_kernel<2>, dim3(s.P), dim3(warps * 32), smem, stream, a);
    else if (s.k <= 4)
        e = launch_pdl(layout_kernel<4>, dim3(s.P), dim3(warps * 32), smem, stream, a);
    else if (s.k <= 8)
        e = launch_pdl(layout_kernel<8>, dim3(s.P), dim3(warps * 32), smem, stream, a);
    else
        e = launch_pdl(layout_kernel<16>, dim3(s.P), dim3(warps * 32), smem, stream, a);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// ep_layout_static_scratch: the layout for callers that cannot allocate.
//
// The regular entry point keeps its scratch (ticket counter, error word, per-rank
// special-expert counts) in a workspace the caller allocates.  Some callers have
// no way to do that: a serving engine that has already handed every byte of the
// GPU to its own pool, code that must not call cudaMalloc because it can
// synchronize the whole device and stall other streams, or a plain C host without
// a tensor library.  This variant keeps that scratch in a fixed array in the
// library's own device memory instead.  It launches the same layout kernel.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = 64 * 1024;  // 256-byte header + P*(Z+C+K) int32 counts

// Lives on every GPU that loads this library, until the process exits.
static __device__ __align__(256) unsigned char g_layout_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_layout_scratch on the current device.  Looked up once per
// device with that device current; in host code the symbol itself is only a
// host-side stand-in and must never be handed to a kernel.
cudaError_t static_scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0) return cudaErrorInvalidDevice;
    if (dev >= kMaxDevices) return cudaGetSymbolAddress(out, g_layout_scratch);  // not cached
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_layout_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace ep

extern "C" int ep_layout_static_scratch(const ep_config* cfg, const int32_t* topk_idx,
                                        int32_t* expert_count, int32_t* expert_offset,
                                        int32_t* recv_count, int32_t* dst_pos, int32_t* recv_src,
                                        uint32_t* err_word, ep_stream_t stream) {
    ep_buffer_sizes sz;
    const int st = ep_buffer_size(cfg, &sz);  // validates cfg
    if (st != EP_OK) return st;
    const size_t need = ep::workspace_layout_bytes(ep::make_shape(*cfg));
    if (need > ep::kStaticScratchBytes) return EP_ERR_CAPACITY;
    auto bad = [](const void* p, size_t size) {
        return size != 0 && (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 3u) != 0);
    };
    if (bad(expert_count, sz.expert_count) || bad(expert_offset, sz.expert_offset) ||
        bad(recv_count, sz.recv_count) || bad(dst_pos, sz.dst_pos) || bad(recv_src, sz.recv_src) ||
        bad(topk_idx, sz.dst_pos) || bad(err_word, err_word ? 4 : 0))
        return EP_ERR_INVALID_ARG;
    void* scratch = nullptr;
    if (ep::static_scratch_address(&scratch) != cudaSuccess) return EP_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: start from zero every call.
    if (cudaMemsetAsync(scratch, 0, need, s) != cudaSuccess) return EP_ERR_CUDA;
    ep_buffer_ptrs p = {};
    p.expert_count = expert_count;
    p.expert_offset = expert_offset;
    p.recv_count = recv_count;
    p.dst_pos = dst_pos;
    p.recv_src = recv_src;
    p.workspace = scratch;
    const int lst = ep::launch_layout(ep::make_shape(*cfg), p, topk_idx, nullptr, s);
    if (lst != EP_OK) return lst;
    if (err_word) {
        const auto* hdr = reinterpret_cast<const ep::WsHeader*>(scratch);
        if (cudaMemcpyAsync(err_word, &hdr->err, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
            return EP_ERR_CUDA;
    }
    return EP_OK;
}
