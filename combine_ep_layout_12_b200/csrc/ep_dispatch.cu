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

namespace ep {
namespace {

struct DispatchArgs {
    const uint16_t* x;       // [B][d] bf16
    const float* smooth;     // [d] or null
    const int32_t* dst_pos;  // [B][k]
    void* recv_x;            // [rows][d] int8 or bf16
    float* recv_scale;       // [rows]
    float* token_scale;      // [B]
    unsigned* err;
    long long rows;
    int d, k;
};

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

// quant_mode 2: a unit is 16 elements (two 16-byte bf16 loads -> one 16-byte int8 store).
template <int U>
__global__ void __launch_bounds__(256) dispatch_int8_kernel(DispatchArgs a) {
    __shared__ int s_rows[kMaxK];
    __shared__ float s_red[32];
    const int t = blockIdx.x;
    const int nunits = a.d >> 4;
    const int NT = blockDim.x;

    pdl_wait();
    pdl_launch_dependents();
    load_rows(a, t, s_rows);

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

    // x_fp32 = fp32(x) * smooth; absmax over the row
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < U; ++i) {
        const int u = threadIdx.x + i * NT;
        if (u >= nunits) continue;
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&raw[i][0]);
        float4 ss[4];
        if (a.smooth) {
            const float4* sp = reinterpret_cast<const float4*>(a.smooth + 16 * u);
#pragma unroll
            for (int q = 0; q < 4; ++q) ss[q] = __ldg(sp + q);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float lo = bf16lo(w[e]), hi = bf16hi(w[e]);
            if (a.smooth) {
                const float* sf = reinterpret_cast<const float*>(ss);
                lo = __fmul_rn(lo, sf[2 * e]);
                hi = __fmul_rn(hi, sf[2 * e + 1]);
            }
            amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
        }
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

    const float s = __fdiv_rn(127.0f, amax);
    const bool degenerate = (amax == 0.0f) || isinf(s);
    const float inv = degenerate ? 0.0f : __fdiv_rn(1.0f, s);

    int rows[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) rows[j] = (j < a.k) ? s_rows[j] : -1;
    int8_t* out = reinterpret_cast<int8_t*>(a.recv_x);

#pragma unroll
    for (int i = 0; i < U; ++i) {
        const int u = threadIdx.x + i * NT;
        if (u >= nunits) continue;
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&raw[i][0]);
        float4 ss[4];
        if (a.smooth) {
            const float4* sp = reinterpret_cast<const float4*>(a.smooth + 16 * u);
#pragma unroll
            for (int q = 0; q < 4; ++q) ss[q] = __ldg(sp + q);
        }
        uint32_t packed[4];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float lo = bf16lo(w[e]), hi = bf16hi(w[e]);
            if (a.smooth) {
                const float* sf = reinterpret_cast<const float*>(ss);
                lo = __fmul_rn(lo, sf[2 * e]);
                hi = __fmul_rn(hi, sf[2 * e + 1]);
            }
            int qlo = 0, qhi = 0;
            if (!degenerate) {
                qlo = min(127, max(-128, __float2int_rn(__fmul_rn(lo, s))));
                qhi = min(127, max(-128, __float2int_rn(__fmul_rn(hi, s))));
            }
            const uint32_t pair = (uint32_t)(qlo & 0xff) | ((uint32_t)(qhi & 0xff) << 8);
            if (e & 1)
                packed[e >> 1] |= pair << 16;
            else
                packed[e >> 1] = pair;
        }
        const uint4 v = make_uint4(packed[0], packed[1], packed[2], packed[3]);
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            if (rows[j] >= 0) st_v4(out + (size_t)rows[j] * a.d + 16 * u, v);
        }
    }
    if (threadIdx.x < a.k) {
        const int row = s_rows[threadIdx.x];
        if (row >= 0) a.recv_scale[row] = inv;
    }
    if (threadIdx.x == 0) a.token_scale[t] = inv;
}

// quant_mode 0: bf16 rows copied as they are; a unit is one 16-byte vector.
template <int U>
__global__ void __launch_bounds__(256) dispatch_bf16_kernel(DispatchArgs a) {
    __shared__ int s_rows[kMaxK];
    const int t = blockIdx.x;
    const int nvec = a.d >> 3;
    const int NT = blockDim.x;

    pdl_wait();
    pdl_launch_dependents();
    load_rows(a, t, s_rows);

    const uint4* xrow = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d);
    uint4 raw[U];
#pragma unroll
    for (int i = 0; i < U; ++i) {
        const int u = threadIdx.x + i * NT;
        raw[i] = (u < nvec) ? ld_stream_v4(xrow + u) : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    int rows[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) rows[j] = (j < a.k) ? s_rows[j] : -1;
    uint4* out = reinterpret_cast<uint4*>(a.recv_x);
#pragma unroll
    for (int i = 0; i < U; ++i) {
        const int u = threadIdx.x + i * NT;
        if (u >= nvec) continue;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            if (rows[j] >= 0) st_v4(out + (size_t)rows[j] * nvec + u, raw[i]);
        }
    }
}

int pick_units(int n, int max_u, int* U, int* NT) {
    // smallest power-of-two U <= max_u with ceil(n / U) <= 256 threads
    int u = 1;
    while (u < max_u && (n + u - 1) / u > 256) u *= 2;
    int nt = (n + u - 1) / u;
    nt = ((nt + 31) / 32) * 32;
    if (nt > 256) return EP_ERR_UNSUPPORTED;
    *U = u;
    *NT = nt;
    return EP_OK;
}

}  // namespace

int launch_dispatch(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* x,
                    const float* smooth, cudaStream_t stream) {
    if (s.B == 0) return EP_OK;
    DispatchArgs a;
    a.x = x;
    a.smooth = smooth;
    a.dst_pos = p.dst_pos;
    a.recv_x = p.recv_x;
    a.recv_scale = p.recv_scale;
    a.token_scale = p.token_scale;
    a.err = &reinterpret_cast<WsHeader*>(p.workspace)->err;
    a.rows = s.rows;
    a.d = s.d;
    a.k = s.k;
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
