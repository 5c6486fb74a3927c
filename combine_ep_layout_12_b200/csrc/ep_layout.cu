// Routing layout kernel.
//
// Computes, from topk_idx[B][k], the per-expert counts, the per-(expert, source
// rank) counts, their exclusive prefix and the low-latency receive row of every
// routed pick (Ascend CANN "low_latency_dispatch": Formula, the alltoallv of the
// quantized rows; Constraints, the row bound A >= M * P * min(L, K) and the
// deterministic computation).  Expert g lives on rank g / (E / P) (DeepEP issue
// #84, masking experiment); id -1 sends nothing.
//
// Design.  Every variant builds, in shared memory, one 32-bit lane mask per
// routed expert for each warp's 32 tokens (atomicOr of bit `lane` for each of the
// token's routed ids).  OR is order-independent, so the masks and everything
// derived from them are deterministic.  A token's slot inside its (expert, rank)
// run is the count of the rank's earlier tokens that picked g plus
// popc(mask[w][g] & lanemask_lt), i.e. its rank among rank r's tokens that routed
// to g, in ascending token order.  Batches of up to 256 tokens per rank use one
// kernel (ep_layout_dev.cuh); larger ones two kernels over 256-token chunks, below.
// No CTA ever waits on another.
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

// Layout for larger per-rank batches (T > 256), in two kernels over (chunk, rank)
// CTAs, a chunk being 256 consecutive tokens of one rank; no CTA ever waits on
// another.
//  - Count kernel: each CTA builds the lane masks of its chunk (one warp per 32
//    tokens, as in the small-batch layout), writes the chunk's routed picks per
//    expert and its special-expert counts to the workspace, and leaves each routed
//    pick's slot within the chunk in dst_pos.
//  - Rows kernel: each CTA sums the counts of its rank's earlier chunks per expert
//    (all the loads spread over the CTA at once) and turns the in-chunk slots into
//    receive rows; the rank's last chunk also writes recv_count.  The last CTA to
//    finish (a ticket counter) adds the counts over ranks into expert_count and
//    scans expert_offset.
// Slots stay in ascending token order: the earlier chunks' counts come first, then
// the lane-mask rank inside the chunk.
constexpr int kChunkTokens = 256;

template <int KM>
__global__ void __launch_bounds__(kChunkTokens) layout_chunk_count_kernel(LayoutArgs a, int n_chunks) {
    extern __shared__ unsigned smem[];
    const int E = a.E, k = a.k;
    constexpr int W = kChunkTokens / 32;
    unsigned* mask = smem;                                     // [W][E]
    int* spc = reinterpret_cast<int*>(smem + (size_t)W * E);  // [n_special]
    pdl_wait();
    pdl_launch_dependents();
    const int c = blockIdx.x, r = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) mask[i] = 0u;
    for (int i = threadIdx.x; i < a.n_special; i += blockDim.x) spc[i] = 0;
    __syncthreads();
    const int tr = c * kChunkTokens + (int)threadIdx.x;  // token index inside the rank
    const bool valid = tr < a.T;
    const int t = r * a.T + tr;
    const bool vec4 = (k % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.topk_idx) & 15) == 0);
    int ids[KM];
    unsigned rb = 0, err = 0;
    if (valid) {
        load_token_ids<KM>(a.topk_idx, t, k, vec4, ids);
        apply_active<KM>(a.active, t, ids);
        rb = classify_ids<KM>(ids, k, E, a.E_tot, err, [&](int sidx) { atomicAdd(&spc[sidx], 1); });
    }
#pragma unroll
    for (int j = 0; j < KM; ++j)
        if (rb & (1u << j)) atomicOr(&mask[(size_t)warp * E + ids[j]], 1u << lane);
    __syncthreads();
    if (valid) {
        const unsigned lt = lanemask_lt();
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (j >= k) continue;
            int slot = -1;
            if (rb & (1u << j)) {
                const int g = ids[j];
                slot = __popc(mask[(size_t)warp * E + g] & lt);
                for (int w = 0; w < warp; ++w) slot += __popc(mask[(size_t)w * E + g]);
            }
            a.dst_pos[(size_t)t * k + j] = slot;  // in-chunk slot; the rows kernel adds the rest
        }
    }
    int32_t* cnt = a.chunk_cnt + ((size_t)r * n_chunks + c) * E;
    for (int g = threadIdx.x; g < E; g += blockDim.x) {
        int n = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) n += __popc(mask[(size_t)w * E + g]);
        cnt[g] = n;
    }
    int32_t* sp = a.sp_chunk + ((size_t)r * n_chunks + c) * a.n_special;
    for (int i = threadIdx.x; i < a.n_special; i += blockDim.x) sp[i] = spc[i];
    report_err(&a.ws->err, err);
}

template <int KM>
__global__ void __launch_bounds__(kChunkTokens) layout_chunk_rows_kernel(LayoutArgs a, int n_chunks) {
    extern __shared__ int pre[];  // [max(E, E_tot) + 32]: earlier chunks' counts, later the totals
    __shared__ int s_last;
    const int E = a.E, k = a.k;
    pdl_wait();
    pdl_launch_dependents();
    const int c = blockIdx.x, r = blockIdx.y;
    for (int g = threadIdx.x; g < E; g += blockDim.x) pre[g] = 0;
    __syncthreads();
    // the rank's picks per expert in chunks 0..c-1 (the rank's last chunk adds its own
    // to get recv_count); the loads of all (chunk, expert) pairs are spread at once
    const int32_t* cnt_r = a.chunk_cnt + (size_t)r * n_chunks * E;
    const int upto = (c == n_chunks - 1) ? c + 1 : c;
    for (int i = threadIdx.x; i < upto * E; i += blockDim.x) {
        const int cc = i / E, g = i - cc * E;
        if (cc < c) atomicAdd(&pre[g], __ldcg(cnt_r + i));
    }
    __syncthreads();
    if (c == n_chunks - 1) {
        const int32_t* own = cnt_r + (size_t)c * E;
        for (int g = threadIdx.x; g < E; g += blockDim.x)
            a.recv_count[(size_t)g * a.P + r] = pre[g] + __ldcg(own + g);
    }
    const int tr = c * kChunkTokens + (int)threadIdx.x;
    if (tr < a.T) {
        const int t = r * a.T + tr;
        const bool vec4 = (k % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.topk_idx) & 15) == 0);
        int ids[KM];
        load_token_ids<KM>(a.topk_idx, t, k, vec4, ids);
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (j >= k) continue;
            const int slot = __ldcg(a.dst_pos + (size_t)t * k + j);
            if (slot < 0) continue;  // not routed (the count kernel left -1)
            const int g = ids[j];
            int row = -1;
            if (ep_in_range(g, E, &a.ws->err)) {
                row = g * a.gstride + r * a.M + a.rbase + pre[g] + slot;
                if (!ep_in_range(row, a.rows, &a.ws->err)) row = -1;
                else if (a.recv_src) a.recv_src[row] = t;
            }
            a.dst_pos[(size_t)t * k + j] = row;
        }
    }

    // ticket: the last CTA of this launch reduces over ranks and scans
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned ticket = atomicAdd(&a.ws->done, 1u);
        s_last = (ticket == gridDim.x * gridDim.y - 1u);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    int* ec = pre;                 // [E_tot]
    int* wsum = pre + a.E_tot;     // [32]
    for (int g = threadIdx.x; g < a.E_tot; g += blockDim.x) ec[g] = 0;
    __syncthreads();
    // totals per expert id: recv_count [E][P] and the chunks' special counts
    // [P][chunks][n_special], both read contiguously with every load in flight at once
    for (int i = threadIdx.x; i < E * a.P; i += blockDim.x) atomicAdd(&ec[i / a.P], __ldcg(a.recv_count + i));
    const int n_sp = a.P * n_chunks * a.n_special;
    for (int i = threadIdx.x; i < n_sp; i += blockDim.x) atomicAdd(&ec[E + i % a.n_special], __ldcg(a.sp_chunk + i));
    __syncthreads();
    for (int g = threadIdx.x; g < a.E_tot; g += blockDim.x) a.expert_count[g] = ec[g];
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
                  const uint8_t* active, cudaStream_t stream, int gstride, int rbase) {
    if (gstride < 0) gstride = s.P * s.M;
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
        a1.chunk_cnt = nullptr;
        a1.sp_chunk = nullptr;
        a1.B = s.B; a1.k = s.k; a1.P = s.P; a1.M = s.M; a1.E = s.E; a1.T = s.T;
        a1.n_special = s.n_special; a1.E_tot = s.E_tot;
        a1.rows = s.rows;
        a1.warps = 8;
        a1.gstride = gstride;
        a1.rbase = rbase;
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
    // larger batches: the chunked count and rows kernels
    const int n_chunks = (s.T + kChunkTokens - 1) / kChunkTokens;
    const size_t smem_count_k = sizeof(unsigned) * (size_t)(kChunkTokens / 32) * s.E + sizeof(int) * s.n_special;
    const size_t smem_rows_k = sizeof(int) * (((size_t)s.E > (size_t)s.E_tot ? s.E : s.E_tot) + 32);
    if (smem_count_k > budget || smem_rows_k > budget) return EP_ERR_UNSUPPORTED;
    static bool attr_chunk[kDeviceSlots] = {false};
    if (first_on_device(attr_chunk, dev0)) {
        if (cudaFuncSetAttribute(layout_chunk_count_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget) ||
            cudaFuncSetAttribute(layout_chunk_count_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget) ||
            cudaFuncSetAttribute(layout_chunk_count_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget) ||
            cudaFuncSetAttribute(layout_chunk_count_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget))
            return EP_ERR_CUDA;
        mark_device(attr_chunk, dev0);
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
    int32_t* words = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.workspace) + sizeof(WsHeader));
    a.chunk_cnt = words;                                                   // [P][n_chunks][E]
    a.sp_chunk = words + (size_t)s.P * n_chunks * s.E;                     // [P][n_chunks][n_special]
    a.B = s.B; a.k = s.k; a.P = s.P; a.M = s.M; a.E = s.E; a.T = s.T;
    a.n_special = s.n_special; a.E_tot = s.E_tot;
    a.rows = s.rows;
    a.warps = kChunkTokens / 32;
    a.gstride = gstride;
    a.rbase = rbase;
    const dim3 grid((unsigned)n_chunks, (unsigned)s.P), block(kChunkTokens);
    cudaError_t e;
    if (s.k <= 2)
        e = launch_pdl(layout_chunk_count_kernel<2>, grid, block, smem_count_k, stream, a, n_chunks);
    else if (s.k <= 4)
        e = launch_pdl(layout_chunk_count_kernel<4>, grid, block, smem_count_k, stream, a, n_chunks);
    else if (s.k <= 8)
        e = launch_pdl(layout_chunk_count_kernel<8>, grid, block, smem_count_k, stream, a, n_chunks);
    else
        e = launch_pdl(layout_chunk_count_kernel<16>, grid, block, smem_count_k, stream, a, n_chunks);
    if (e != cudaSuccess) return EP_ERR_CUDA;
    if (s.k <= 2)
        e = launch_pdl(layout_chunk_rows_kernel<2>, grid, block, smem_rows_k, stream, a, n_chunks);
    else if (s.k <= 4)
        e = launch_pdl(layout_chunk_rows_kernel<4>, grid, block, smem_rows_k, stream, a, n_chunks);
    else if (s.k <= 8)
        e = launch_pdl(layout_chunk_rows_kernel<8>, grid, block, smem_rows_k, stream, a, n_chunks);
    else
        e = launch_pdl(layout_chunk_rows_kernel<16>, grid, block, smem_rows_k, stream, a, n_chunks);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// ep_layout_static_scratch: the layout for callers that cannot allocate.
//
// The regular entry point keeps its scratch (ticket counter, error word, and the
// chunked layout's per-chunk counts) in a workspace the caller allocates.  Some callers have
// no way to do that: a serving engine that has already handed every byte of the
// GPU to its own pool, code that must not call cudaMalloc because it can
// synchronize the whole device and stall other streams, or a plain C host without
// a tensor library.  This variant keeps that scratch in a fixed array in the
// library's own device memory instead.  It launches the same layout kernel.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = 64 * 1024;  // 256-byte header + P*ceil(T/256)*(E+Z+C+K) int32 chunk counts when T > 256

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
