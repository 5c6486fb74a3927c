// Layout and dispatch in one grid, for small per-rank batches (T <= 128).
//
// The first CTAs of the grid run the layout (a count CTA and rank-holding slot
// CTAs, see ep_layout_dev.cuh); every other CTA is the dispatch of one token,
// which derives its receive rows from the routing itself (the count of earlier
// tokens of its rank that picked the same expert), so no CTA of the grid waits
// on another.  Compared with two launches this removes one kernel launch from
// the critical path, and the grid completes only when both parts have, so the
// combine that follows on the stream sees a finished layout and payload.
#include "ep_internal.cuh"
#include "ep_layout_dev.cuh"
#include "ep_dispatch_dev.cuh"

namespace ep {
namespace {

// MODE: quant_mode (0 bf16 pass-through, 1 static int8, 2 dynamic int8).
template <int KM, int U, int MODE>
__global__ void __launch_bounds__(128, (U <= 4 ? 8 : 4))
    layout_dispatch_kernel(LayoutArgs la, DispatchArgs da, int cpr, int n_layout) {
    extern __shared__ unsigned smem[];
    pdl_wait();
    pdl_launch_dependents();
    if ((int)blockIdx.x < n_layout) {
        layout_small_body<KM>(la, cpr, blockIdx.x, smem);
    } else if (MODE == 0) {
        dispatch_bf16_body<U>(da, blockIdx.x - n_layout);
    } else {
        dispatch_int8_body<U, MODE == 1>(da, blockIdx.x - n_layout);
    }
}

// Multi-GPU form of the same grid for one rank (laid out as P = 1 with global rows):
// the slot CTAs also store the rank's counts into the owners' recv_count (the count
// exchange), and the dispatch CTAs store every copy into the owning rank's slab.
template <int KM, int U, int MODE>
__global__ void __launch_bounds__(128, (U <= 4 ? 8 : 4))
    layout_dispatch_shard_kernel(LayoutArgs la, DispatchArgs da, const __grid_constant__ ShardTable tab, int cpr,
                                 int n_layout) {
    extern __shared__ unsigned smem[];
    pdl_wait();
    pdl_launch_dependents();
    if ((int)blockIdx.x < n_layout) {
        layout_small_body<KM>(la, cpr, blockIdx.x, smem, &tab);
    } else if (MODE == 0) {
        dispatch_bf16_body<U>(da, blockIdx.x - n_layout, ShardRows{tab});
    } else {
        dispatch_int8_body<U, MODE == 1>(da, blockIdx.x - n_layout, ShardRows{tab});
    }
}

template <int KM, int MODE>
cudaError_t launch_fused_shard_u(int U, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 const LayoutArgs& la, const DispatchArgs& da, const ShardTable& tab, int cpr,
                                 int n_layout) {
    switch (U) {
        case 1: return launch_pdl(layout_dispatch_shard_kernel<KM, 1, MODE>, grid, block, smem, stream, la, da, tab, cpr, n_layout);
        case 2: return launch_pdl(layout_dispatch_shard_kernel<KM, 2, MODE>, grid, block, smem, stream, la, da, tab, cpr, n_layout);
        case 4: return launch_pdl(layout_dispatch_shard_kernel<KM, 4, MODE>, grid, block, smem, stream, la, da, tab, cpr, n_layout);
        default: return launch_pdl(layout_dispatch_shard_kernel<KM, 8, MODE>, grid, block, smem, stream, la, da, tab, cpr, n_layout);
    }
}

template <int KM>
cudaError_t launch_fused_shard_mode(int mode, int U, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                    const LayoutArgs& la, const DispatchArgs& da, const ShardTable& tab, int cpr,
                                    int n_layout) {
    if (mode == 0) return launch_fused_shard_u<KM, 0>(U, grid, block, smem, stream, la, da, tab, cpr, n_layout);
    if (mode == 1) return launch_fused_shard_u<KM, 1>(U, grid, block, smem, stream, la, da, tab, cpr, n_layout);
    return launch_fused_shard_u<KM, 2>(U, grid, block, smem, stream, la, da, tab, cpr, n_layout);
}

template <int KM, int MODE>
cudaError_t launch_fused_u(int U, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                           const LayoutArgs& la, const DispatchArgs& da, int cpr, int n_layout) {
    switch (U) {
        case 1: return launch_pdl(layout_dispatch_kernel<KM, 1, MODE>, grid, block, smem, stream, la, da, cpr, n_layout);
        case 2: return launch_pdl(layout_dispatch_kernel<KM, 2, MODE>, grid, block, smem, stream, la, da, cpr, n_layout);
        case 4: return launch_pdl(layout_dispatch_kernel<KM, 4, MODE>, grid, block, smem, stream, la, da, cpr, n_layout);
        default: return launch_pdl(layout_dispatch_kernel<KM, 8, MODE>, grid, block, smem, stream, la, da, cpr, n_layout);
    }
}

template <int KM>
cudaError_t launch_fused_mode(int mode, int U, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              const LayoutArgs& la, const DispatchArgs& da, int cpr, int n_layout) {
    if (mode == 0) return launch_fused_u<KM, 0>(U, grid, block, smem, stream, la, da, cpr, n_layout);
    if (mode == 1) return launch_fused_u<KM, 1>(U, grid, block, smem, stream, la, da, cpr, n_layout);
    return launch_fused_u<KM, 2>(U, grid, block, smem, stream, la, da, cpr, n_layout);
}

// Whether layout and dispatch of shape s run as one grid, and its geometry.
struct FusedPlan {
    int cpr, U, NT, threads, n_layout;
    size_t smem;
};

bool plan_fused(const Shape& s, const float* smooth, FusedPlan* f) {
    f->cpr = (s.T + 31) / 32;
    const int units = s.quant_mode != 0 ? s.d / 16 : s.d / 8;
    const bool fits = s.B > 0 && s.layout == 0 && f->cpr <= 4 && s.k <= 8 && !(smooth && s.expert_smooth) &&
                      pick_units(units, 8, &f->U, &f->NT) == EP_OK && f->NT <= 128 && f->U <= 8;
    if (!fits) return false;
    f->threads = f->NT > 32 * f->cpr ? f->NT : 32 * f->cpr;  // the layout part needs one warp per chunk
    const int warps = f->threads / 32;
    const int ranks_per_cta = warps / f->cpr;
    f->n_layout = 1 + (s.P + ranks_per_cta - 1) / ranks_per_cta;
    const size_t smem_count = sizeof(int) * ((size_t)s.E_tot + 32);
    const size_t smem_slot = sizeof(int) * (size_t)warps * s.E;
    f->smem = smem_count > smem_slot ? smem_count : smem_slot;  // <= 32 KB here
    return true;
}

LayoutArgs fused_layout_args(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                             const uint8_t* active, int warps, int gstride, int rbase) {
    LayoutArgs la;
    la.topk_idx = topk_idx;
    la.active = active;
    la.expert_count = p.expert_count;
    la.expert_offset = p.expert_offset;
    la.recv_count = p.recv_count;
    la.dst_pos = p.dst_pos;
    la.recv_src = p.recv_src;
    la.ws = reinterpret_cast<WsHeader*>(p.workspace);
    la.chunk_cnt = nullptr;
    la.sp_chunk = nullptr;
    la.B = s.B; la.k = s.k; la.P = s.P; la.M = s.M; la.E = s.E; la.T = s.T;
    la.n_special = s.n_special; la.E_tot = s.E_tot;
    la.rows = s.rows;
    la.warps = warps;
    la.gstride = gstride;
    la.rbase = rbase;
    return la;
}

}  // namespace

int launch_layout_dispatch(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                           const uint8_t* active, const uint16_t* x, const float* smooth,
                           cudaStream_t stream) {
    FusedPlan f;
    if (!plan_fused(s, smooth, &f)) {
        const int st = launch_layout(s, p, topk_idx, active, stream);
        return st != EP_OK ? st : launch_dispatch(s, p, x, smooth, topk_idx, active, stream);
    }
    const LayoutArgs la = fused_layout_args(s, p, topk_idx, active, f.threads / 32, s.P * s.M, 0);
    DispatchArgs da = make_dispatch_args(s, p, x, smooth, topk_idx, active);
    da.self_rows = 1;

    const dim3 grid((unsigned)(f.n_layout + s.B)), block((unsigned)f.threads);
    cudaError_t e;
    if (s.k <= 2)
        e = launch_fused_mode<2>(s.quant_mode, f.U, grid, block, f.smem, stream, la, da, f.cpr, f.n_layout);
    else if (s.k <= 4)
        e = launch_fused_mode<4>(s.quant_mode, f.U, grid, block, f.smem, stream, la, da, f.cpr, f.n_layout);
    else
        e = launch_fused_mode<8>(s.quant_mode, f.U, grid, block, f.smem, stream, la, da, f.cpr, f.n_layout);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

int launch_shard_layout_dispatch(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                                 const uint8_t* active, const uint16_t* x, const float* smooth,
                                 const ShardTable& tab, int gstride, int rbase, cudaStream_t stream) {
    FusedPlan f;
    if (!plan_fused(s, smooth, &f)) {
        // separate launches: the layout writes send_count, the dispatch exchanges it
        const int st = launch_layout(s, p, topk_idx, active, stream, gstride, rbase);
        if (st != EP_OK) return st;
        ShardTable t = tab;
        t.send_count = p.recv_count;
        return launch_shard_dispatch(s, p, x, smooth, t, stream);
    }
    const LayoutArgs la = fused_layout_args(s, p, topk_idx, active, f.threads / 32, gstride, rbase);
    DispatchArgs da = make_dispatch_args(s, p, x, smooth, topk_idx, active);
    da.self_rows = 1;
    da.gstride = gstride;
    da.rbase = rbase;

    const dim3 grid((unsigned)(f.n_layout + s.B)), block((unsigned)f.threads);
    cudaError_t e;
    if (s.k <= 2)
        e = launch_fused_shard_mode<2>(s.quant_mode, f.U, grid, block, f.smem, stream, la, da, tab, f.cpr, f.n_layout);
    else if (s.k <= 4)
        e = launch_fused_shard_mode<4>(s.quant_mode, f.U, grid, block, f.smem, stream, la, da, tab, f.cpr, f.n_layout);
    else
        e = launch_fused_shard_mode<8>(s.quant_mode, f.U, grid, block, f.smem, stream, la, da, tab, f.cpr, f.n_layout);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

}  // namespace ep
