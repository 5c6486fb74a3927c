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

}  // namespace

int launch_layout_dispatch(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                           const uint8_t* active, const uint16_t* x, const float* smooth,
                           cudaStream_t stream) {
    const int cpr = (s.T + 31) / 32;
    int U = 0, NT = 0;
    const int units = s.quant_mode != 0 ? s.d / 16 : s.d / 8;
    const bool fits = s.B > 0 && s.layout == 0 && cpr <= 4 && s.k <= 8 &&
                      !(smooth && s.expert_smooth) &&
                      pick_units(units, 8, &U, &NT) == EP_OK &&
                      NT <= 128 && U <= 8;
    if (!fits) {
        const int st = launch_layout(s, p, topk_idx, active, stream);
        return st != EP_OK ? st : launch_dispatch(s, p, x, smooth, topk_idx, active, stream);
    }
    const int threads = NT > 32 * cpr ? NT : 32 * cpr;  // the layout part needs one warp per chunk
    const int warps = threads / 32;
    const int ranks_per_cta = warps / cpr;
    const int n_layout = 1 + (s.P + ranks_per_cta - 1) / ranks_per_cta;
    const size_t smem_count = sizeof(int) * ((size_t)s.E_tot + 32);
    const size_t smem_slot = sizeof(int) * (size_t)warps * s.E;
    const size_t smem = smem_count > smem_slot ? smem_count : smem_slot;  // <= 32 KB here

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
    la.gstride = s.P * s.M;
    la.rbase = 0;
    DispatchArgs da = make_dispatch_args(s, p, x, smooth, topk_idx, active);
    da.self_rows = 1;

    const dim3 grid((unsigned)(n_layout + s.B)), block((unsigned)threads);
    cudaError_t e;
    if (s.k <= 2)
        e = launch_fused_mode<2>(s.quant_mode, U, grid, block, smem, stream, la, da, cpr, n_layout);
    else if (s.k <= 4)
        e = launch_fused_mode<4>(s.quant_mode, U, grid, block, smem, stream, la, da, cpr, n_layout);
    else
        e = launch_fused_mode<8>(s.quant_mode, U, grid, block, smem, stream, la, da, cpr, n_layout);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

}  // namespace ep
