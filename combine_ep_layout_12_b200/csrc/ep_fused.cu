// Layout and dispatch in one grid, for small per-rank batches (T <= 128).
//
// The first CTAs of the grid run the layout (a count CTA and rank-holding slot
// CTAs, see ep_layout_dev.cuh); every other CTA dispatches kWarpTokens tokens, one
// per warp, each warp deriving its token's receive rows from the routing itself
// (the count of earlier tokens of its rank that picked the same expert), so no
// CTA of the grid waits on another.  Compared with two launches this removes one
// kernel launch from the critical path, and the grid completes only when both
// parts have, so the combine that follows on the stream sees a finished layout
// and payload.
#include "ep_internal.cuh"
#include "ep_layout_dev.cuh"
#include "ep_dispatch_dev.cuh"

namespace ep {
namespace {

// MODE: quant_mode (0 bf16 pass-through, 1 static int8, 2 dynamic int8).  The
// layout CTAs and the dispatch CTAs (kWarpTokens tokens each, one per warp) share
// the block shape; k <= 8.
template <int NU, int MODE, bool BULK>
__global__ void __launch_bounds__(32 * kWarpTokens)
    layout_dispatch_kernel(LayoutArgs la, DispatchArgs da, int cpr, int n_layout) {
    extern __shared__ __align__(16) unsigned smem[];
    pdl_wait();
    pdl_launch_dependents();
    if ((int)blockIdx.x < n_layout) {
        layout_small_body<8>(la, cpr, blockIdx.x, smem);
        return;
    }
    const int warp = threadIdx.x >> 5;
    const int t = ((int)blockIdx.x - n_layout) * kWarpTokens + warp;
    const size_t per = (size_t)warp_tab_bytes(da.E) + (BULK ? (size_t)da.d : 0);
    unsigned char* mine = reinterpret_cast<unsigned char*>(smem) + warp * per;
    uint16_t* tab = reinterpret_cast<uint16_t*>(mine);
    if (t < da.B) {
        zero_warp_tab(tab, da.E);
        dispatch_warp_body<NU, MODE, 8, BULK>(da, t, tab, mine + warp_tab_bytes(da.E));
    }
}

using FusedKernel = void (*)(LayoutArgs, DispatchArgs, int, int);

template <int MODE>
FusedKernel fused_kernel_nu(int NU) {
    constexpr bool BULK = MODE != 0 && kDispatchBulk;
    if constexpr (MODE == 0) {
        switch (NU) {
            case 2: return layout_dispatch_kernel<2, MODE, BULK>;
            case 4: return layout_dispatch_kernel<4, MODE, BULK>;
            case 8: return layout_dispatch_kernel<8, MODE, BULK>;
            case 14: return layout_dispatch_kernel<14, MODE, BULK>;
            default: return layout_dispatch_kernel<16, MODE, BULK>;
        }
    } else {
        switch (NU) {
            case 1: return layout_dispatch_kernel<1, MODE, BULK>;
            case 2: return layout_dispatch_kernel<2, MODE, BULK>;
            case 4: return layout_dispatch_kernel<4, MODE, BULK>;
            case 7: return layout_dispatch_kernel<7, MODE, BULK>;
            default: return layout_dispatch_kernel<8, MODE, BULK>;
        }
    }
}

}  // namespace

int launch_layout_dispatch(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                           const uint8_t* active, const uint16_t* x, const float* smooth,
                           cudaStream_t stream) {
    const int cpr = (s.T + 31) / 32;
    const int NU = warp_units(s.quant_mode, s.d);
    const bool fits = s.B > 0 && s.layout == 0 && cpr <= kWarpTokens && s.k <= 8 &&
                      !(smooth && s.expert_smooth) && NU > 0;
    if (!fits) {
        const int st = launch_layout(s, p, topk_idx, active, stream);
        return st != EP_OK ? st : launch_dispatch(s, p, x, smooth, topk_idx, active, stream);
    }
    const int warps = kWarpTokens;  // the layout part needs one warp per 32-token chunk
    const int ranks_per_cta = warps / cpr;
    const int n_layout = 1 + (s.P + ranks_per_cta - 1) / ranks_per_cta;
    const size_t smem_count = sizeof(int) * ((size_t)s.E_tot + 32);
    const size_t smem_slot = sizeof(int) * (size_t)warps * s.E;
    const size_t smem_disp = dispatch_warp_smem(s.E, s.d, s.quant_mode != 0 && kDispatchBulk, warps);
    size_t smem = smem_count > smem_slot ? smem_count : smem_slot;
    if (smem_disp > smem) smem = smem_disp;

    FusedKernel kern = s.quant_mode == 0 ? fused_kernel_nu<0>(NU)
                       : s.quant_mode == 1 ? fused_kernel_nu<1>(NU) : fused_kernel_nu<2>(NU);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return EP_ERR_CUDA;

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
    DispatchArgs da = make_dispatch_args(s, p, x, smooth, topk_idx, active);
    da.self_rows = 1;

    const int n_disp = (s.B + kWarpTokens - 1) / kWarpTokens;
    const dim3 grid((unsigned)(n_layout + n_disp)), block((unsigned)(32 * warps));
    const cudaError_t e = launch_pdl(kern, grid, block, smem, stream, la, da, cpr, n_layout);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

}  // namespace ep
