// Dispatch kernels: per-token quantization and the scatter of every routed pick
// into the low-latency receive buffer (Ascend CANN "low_latency_dispatch",
// Formula: quant_out = x for quant_mode 0; for quant_mode 2
//   x_fp32 = fp32(x) * scales, s = 127 / max|x_fp32|, quant_out = CastToInt8(x_fp32 * s),
// expand_x = alltoallv(quant_out), dynamic_scales = alltoall(1 / s)).
//
// Readings (shared with the CPU oracle, written independently): the absmax runs
// over one token row; CastToInt8 rounds half to even and saturates; the scale
// returned is 1.0f / s in fp32; a row with amax == 0 or a non-finite s quantizes
// to zeros with scale 0.
//
// Design.  One CTA per token row.  The row is read once with 16-byte loads into
// registers (each thread owns U units, strided by the CTA width so every load
// instruction of a warp covers a contiguous span), reduced to the row absmax with
// warp shuffles and one shared-memory pass, quantized in registers, and written
// to each of the token's k receive rows with 16-byte stores.  The read happens
// once per token; the k writes are the bulk of the traffic.
#include "ep_internal.cuh"
#include "ep_dispatch_dev.cuh"

namespace ep {
namespace {

// Dispatch kernels.  With self_rows the kernel needs nothing the layout kernel
// writes, so it runs alongside it and waits for it only before exiting (so that
// whatever follows on the stream sees a finished layout); otherwise it waits first.
template <int U>
__global__ void __launch_bounds__(256) dispatch_int8_kernel(DispatchArgs a) {
    if (!a.self_rows) pdl_wait();
    pdl_launch_dependents();
    dispatch_int8_body<U>(a, blockIdx.x);
    if (a.self_rows) pdl_wait();
}

template <int U>
__global__ void __launch_bounds__(256) dispatch_bf16_kernel(DispatchArgs a) {
    if (!a.self_rows) pdl_wait();
    pdl_launch_dependents();
    dispatch_bf16_body<U>(a, blockIdx.x);
    if (a.self_rows) pdl_wait();
}

}  // namespace

int launch_dispatch(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* x,
                    const float* smooth, const int32_t* topk_idx, cudaStream_t stream) {
    if (s.B == 0) return EP_OK;
    DispatchArgs a = make_dispatch_args(s, p, x, smooth, topk_idx);
    // Small batches per rank: each CTA derives its rows from the routing itself
    // (at most kSelfRowsMaxT earlier tokens to scan), so dispatch overlaps layout.
    a.self_rows = (topk_idx != nullptr && s.layout == 0 && s.T <= kSelfRowsMaxT) ? 1 : 0;
    int U = 0, NT = 0;
    cudaError_t e = cudaSuccess;
    const dim3 grid(s.B);
    if (s.quant_mode == 2) {
        if (pick_units(s.d / 16, 8, &U, &NT) != EP_OK) return EP_ERR_UNSUPPORTED;
        switch (U) {
            case 1: e = launch_pdl(dispatch_int8_kernel<1>, grid, dim3(NT), 0, stream, a); break;
            case 2: e = launch_pdl(dispatch_int8_kernel<2>, grid, dim3(NT), 0, stream, a); break;
            case 4: e = launch_pdl(dispatch_int8_kernel<4>, grid, dim3(NT), 0, stream, a); break;
            default: e = launch_pdl(dispatch_int8_kernel<8>, grid, dim3(NT), 0, stream, a); break;
        }
    } else {
        if (pick_units(s.d / 8, 16, &U, &NT) != EP_OK) return EP_ERR_UNSUPPORTED;
        switch (U) {
            case 1: e = launch_pdl(dispatch_bf16_kernel<1>, grid, dim3(NT), 0, stream, a); break;
            case 2: e = launch_pdl(dispatch_bf16_kernel<2>, grid, dim3(NT), 0, stream, a); break;
            case 4: e = launch_pdl(dispatch_bf16_kernel<4>, grid, dim3(NT), 0, stream, a); break;
            case 8: e = launch_pdl(dispatch_bf16_kernel<8>, grid, dim3(NT), 0, stream, a); break;
            default: e = launch_pdl(dispatch_bf16_kernel<16>, grid, dim3(NT), 0, stream, a); break;
        }
    }
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

}  // namespace ep
