// Dispatch kernels: per-token quantization and the scatter of every routed pick
// into the low-latency receive buffer (Ascend CANN "low_latency_dispatch",
// Formula: quant_out = x for quant_mode 0; CastToInt8(CastToFp32(x) * scales) for
// the static mode 1; for quant_mode 2
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
template <int U, bool STATIC>
__global__ void __launch_bounds__(256) dispatch_int8_kernel(DispatchArgs a) {
    if (!a.self_rows) pdl_wait();
    pdl_launch_dependents();
    dispatch_int8_body<U, STATIC>(a, blockIdx.x);
    if (a.self_rows) pdl_wait();
}

template <int U>
__global__ void __launch_bounds__(256) dispatch_bf16_kernel(DispatchArgs a) {
    if (!a.self_rows) pdl_wait();
    pdl_launch_dependents();
    dispatch_bf16_body<U>(a, blockIdx.x);
    if (a.self_rows) pdl_wait();
}

template <bool STATIC>
cudaError_t launch_int8(int U, dim3 grid, dim3 block, cudaStream_t stream, const DispatchArgs& a) {
    switch (U) {
        case 1: return launch_pdl(dispatch_int8_kernel<1, STATIC>, grid, block, 0, stream, a);
        case 2: return launch_pdl(dispatch_int8_kernel<2, STATIC>, grid, block, 0, stream, a);
        case 4: return launch_pdl(dispatch_int8_kernel<4, STATIC>, grid, block, 0, stream, a);
        default: return launch_pdl(dispatch_int8_kernel<8, STATIC>, grid, block, 0, stream, a);
    }
}

// ---------------------------------------------------------------------------
// Per-expert smooth scale ([E][d], the scales of shape [E, h] in the Ascend
// example): every routed copy (t, g) is quantized on its own,
//   x_fp32 = fp32(x[t]) * smooth[g];  dynamic: s = 127 / max|x_fp32|,
//   q = CastToInt8(x_fp32 * s), recv_scale[row] = 1 / s;  static: q = CastToInt8(x_fp32).
//
// Design (expert-major).  Each copy needs a whole fp32 smooth row, four times the
// bytes of the int8 row it produces, so reading it per token (k rows per token)
// makes the kernel bound by L2 reads of the table.  Instead a CTA takes one
// expert g and a share of its receive rows: it stages smooth[g] in shared memory
// once, finds the source token of each of its rows through recv_src, and
// quantizes the rows one at a time with all its threads.  A thread holds GP
// groups of 4 elements of the row in registers (the x row is read once, from L2),
// the absmax is one CTA reduction behind one barrier (two alternating sets of
// reduction slots), and the next row's x is loaded before that barrier so its
// latency overlaps the reduction.  Loads, stores and the float4 shared-memory
// reads are all lane-contiguous.  The receive rows come from the layout
// (recv_count, recv_src, expert_offset), so the kernel waits for it first.
// ---------------------------------------------------------------------------
struct ExpertArgs {
    const uint16_t* x;             // [B][d]
    const float* smooth;           // [E][d]
    const int32_t* expert_offset;  // packed layout: first row of each expert
    const int32_t* recv_count;     // [E][P]
    const int32_t* recv_src;       // [rows]
    int8_t* recv_x;                // [rows][d]
    float* recv_scale;             // [rows] (dynamic only)
    unsigned* err;
    long long rows;
    int B, d, P, M, E, parts, layout;
};

template <int GP>
__device__ __forceinline__ void load_x_groups(const ExpertArgs& a, int t, int nq, uint2 (&v)[GP]) {
    const uint2* xr = reinterpret_cast<const uint2*>(a.x + (size_t)(t < 0 ? 0 : t) * a.d);
#pragma unroll
    for (int m = 0; m < GP; ++m) {
        const int q = threadIdx.x + m * blockDim.x;
        v[m] = (t >= 0 && q < nq) ? __ldg(xr + q) : make_uint2(0, 0);
    }
}

template <int GP, int MAXT, bool STATIC>
__global__ void __launch_bounds__(MAXT) dispatch_expert_major_kernel(ExpertArgs a) {
    extern __shared__ float4 s_sm4[];                                          // [d / 4]
    const int NT = blockDim.x;
    long long* s_row = reinterpret_cast<long long*>(s_sm4 + (a.d >> 2));    // [NT]
    int* s_t = reinterpret_cast<int*>(s_row + NT);                           // [NT]
    int* s_pre = s_t + NT;                                                   // [P + 1]
    __shared__ float s_red[2][32];
    pdl_wait();
    pdl_launch_dependents();
    const int g = blockIdx.x / a.parts, part = blockIdx.x - g * a.parts;
    const int nq = a.d >> 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = NT >> 5;

    const float4* srow = reinterpret_cast<const float4*>(a.smooth + (size_t)g * a.d);
    for (int q = threadIdx.x; q < nq; q += NT) s_sm4[q] = __ldg(srow + q);
    if (a.layout == 0 && warp == 0) {
        // exclusive prefix over source ranks of this expert's row counts
        int run = 0;
        for (int r0 = 0; r0 < a.P; r0 += 32) {
            const int r = r0 + lane;
            const int c = r < a.P ? a.recv_count[(size_t)g * a.P + r] : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (r < a.P) s_pre[r] = run + incl - c;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_pre[a.P] = run;
    }
    __syncthreads();
    int n = a.layout == 0 ? s_pre[a.P] : a.expert_offset[g + 1] - a.expert_offset[g];
    // an expert holds at most one copy per token (P * M rows in the low-latency form)
    n = max(0, min(n, a.layout == 0 ? a.P * a.M : a.B));
    const int chunk = (n + a.parts - 1) / a.parts;
    const int i0 = part * chunk, i1 = min(n, i0 + chunk);

    int par = 0;  // reduction slot set of the current row
    for (int b0 = i0; b0 < i1; b0 += NT) {
        const int nb = min(NT, i1 - b0);
        // receive row and source token of each copy of this batch
        if (threadIdx.x < nb) {
            const int i = b0 + threadIdx.x;
            long long row;
            if (a.layout == 0) {
                int lo = 0, hi = a.P - 1;  // the last rank whose run starts at or before i
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (s_pre[mid] <= i) lo = mid; else hi = mid - 1;
                }
                row = (long long)g * a.P * a.M + (long long)lo * a.M + (i - s_pre[lo]);
            } else {
                row = (long long)a.expert_offset[g] + i;
            }
            const int t = (row >= 0 && row < a.rows) ? a.recv_src[row] : -1;
            const bool ok = t >= 0 && t < a.B;
            report_err(a.err, ok ? 0u : EP_ERRBIT_ROW_RANGE);
            s_row[threadIdx.x] = row;
            s_t[threadIdx.x] = ok ? t : -1;
        }
        __syncthreads();
        uint2 cur[GP], nxt[GP];
        load_x_groups<GP>(a, s_t[0], nq, cur);
        for (int j = 0; j < nb; ++j) {
            const int t = s_t[j];
            const long long row = s_row[j];
            if (j + 1 < nb) load_x_groups<GP>(a, s_t[j + 1], nq, nxt);
            float s = 1.0f;
            bool degenerate = false;
            if (!STATIC) {
                float amax = 0.0f;
#pragma unroll
                for (int m = 0; m < GP; ++m) {
                    const int q = threadIdx.x + m * NT;
                    if (q >= nq) continue;
                    const float4 sm = s_sm4[q];
                    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(__fmul_rn(bf16lo(cur[m].x), sm.x)),
                                                   fabsf(__fmul_rn(bf16hi(cur[m].x), sm.y))),
                                             fmaxf(fabsf(__fmul_rn(bf16lo(cur[m].y), sm.z)),
                                                   fabsf(__fmul_rn(bf16hi(cur[m].y), sm.w)))));
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                if (lane == 0) s_red[par][warp] = amax;
                __syncthreads();
                amax = s_red[par][0];
                for (int w2 = 1; w2 < nw; ++w2) amax = fmaxf(amax, s_red[par][w2]);
                par ^= 1;
                s = __fdiv_rn(127.0f, amax);
                degenerate = (amax == 0.0f) || isinf(s);
            }
            if (t >= 0) {
                uint32_t* out = reinterpret_cast<uint32_t*>(a.recv_x + row * a.d);
#pragma unroll
                for (int m = 0; m < GP; ++m) {
                    const int q = threadIdx.x + m * NT;
                    if (q >= nq) continue;
                    const float4 sm = s_sm4[q];
                    float f0 = __fmul_rn(bf16lo(cur[m].x), sm.x), f1 = __fmul_rn(bf16hi(cur[m].x), sm.y);
                    float f2 = __fmul_rn(bf16lo(cur[m].y), sm.z), f3 = __fmul_rn(bf16hi(cur[m].y), sm.w);
                    if (!STATIC) {
                        f0 = __fmul_rn(f0, s); f1 = __fmul_rn(f1, s);
                        f2 = __fmul_rn(f2, s); f3 = __fmul_rn(f3, s);
                    }
                    out[q] = degenerate ? 0u : cvt_s8x4(f0, f1, f2, f3);
                }
                if (!STATIC && threadIdx.x == 0)
                    a.recv_scale[row] = degenerate ? 0.0f : __fdiv_rn(1.0f, s);
            }
#pragma unroll
            for (int m = 0; m < GP; ++m) cur[m] = nxt[m];
        }
        __syncthreads();  // s_row / s_t are rewritten by the next batch
    }
}

// GP groups per thread; up to 256 threads, or 1024 for rows above 8192 elements.
template <bool STATIC>
cudaError_t launch_expert_gp(int GP, int NT, dim3 grid, size_t smem, cudaStream_t stream,
                             const ExpertArgs& a) {
    const dim3 block((unsigned)NT);
    switch (GP) {
        case 1: return launch_pdl(dispatch_expert_major_kernel<1, 256, STATIC>, grid, block, smem, stream, a);
        case 2: return launch_pdl(dispatch_expert_major_kernel<2, 256, STATIC>, grid, block, smem, stream, a);
        case 4: return launch_pdl(dispatch_expert_major_kernel<4, 256, STATIC>, grid, block, smem, stream, a);
        default:
            return NT <= 256
                ? launch_pdl(dispatch_expert_major_kernel<8, 256, STATIC>, grid, block, smem, stream, a)
                : launch_pdl(dispatch_expert_major_kernel<8, 1024, STATIC>, grid, block, smem, stream, a);
    }
}

template <int GP, int MAXT>
cudaError_t set_expert_smem(int cap) {
    cudaError_t e = cudaFuncSetAttribute(dispatch_expert_major_kernel<GP, MAXT, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(dispatch_expert_major_kernel<GP, MAXT, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
}

int launch_dispatch_expert(const Shape& sh, const ep_buffer_ptrs& p, const uint16_t* x,
                           const float* smooth, cudaStream_t stream) {
    ExpertArgs a;
    a.x = x;
    a.smooth = smooth;
    a.expert_offset = p.expert_offset;
    a.recv_count = p.recv_count;
    a.recv_src = p.recv_src;
    a.recv_x = reinterpret_cast<int8_t*>(p.recv_x);
    a.recv_scale = p.recv_scale;
    a.err = &reinterpret_cast<WsHeader*>(p.workspace)->err;
    a.rows = sh.rows;
    a.B = sh.B; a.d = sh.d; a.P = sh.P; a.M = sh.M; a.E = sh.E; a.layout = sh.layout;
    // groups of 4 elements per thread: the smallest GP in {1, 2, 4, 8} with at most
    // 256 threads, else GP = 8 with up to 1024 threads (d <= 32768)
    const int nq = sh.d / 4;
    int GP = 1;
    while (GP < 8 && (nq + GP - 1) / GP > 256) GP *= 2;
    int NT = (nq + GP - 1) / GP;
    NT = ((NT + 31) / 32) * 32;
    if (NT > 1024) return EP_ERR_UNSUPPORTED;
    // about four CTAs per SM in total, split evenly over the experts
    const long long target = (long long)num_sms() * 4;
    long long parts = (target + sh.E - 1) / sh.E;
    if (parts < 1) parts = 1;
    a.parts = (int)parts;
    const size_t smem = sizeof(float) * (size_t)sh.d + (sizeof(long long) + sizeof(int)) * (size_t)NT +
                        sizeof(int) * ((size_t)sh.P + 1);
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        const int cap = (int)(sizeof(float) * kMaxD + (sizeof(long long) + sizeof(int)) * 1024 +
                              sizeof(int) * (kMaxE + 1));
        if (set_expert_smem<1, 256>(cap) || set_expert_smem<2, 256>(cap) ||
            set_expert_smem<4, 256>(cap) || set_expert_smem<8, 256>(cap) ||
            set_expert_smem<8, 1024>(cap))
            return EP_ERR_CUDA;
        attr_set[dev] = true;
    }
    const dim3 grid((unsigned)((long long)sh.E * a.parts));
    const cudaError_t e = sh.quant_mode == 1 ? launch_expert_gp<true>(GP, NT, grid, smem, stream, a)
                                             : launch_expert_gp<false>(GP, NT, grid, smem, stream, a);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

}  // namespace

int launch_dispatch(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* x,
                    const float* smooth, const int32_t* topk_idx, const uint8_t* active,
                    cudaStream_t stream) {
    if (s.B == 0) return EP_OK;
    DispatchArgs a = make_dispatch_args(s, p, x, smooth, topk_idx, active);
    // Small batches per rank: each CTA derives its rows from the routing itself
    // (at most kSelfRowsMaxT earlier tokens to scan), so dispatch overlaps layout.
    a.self_rows = (topk_idx != nullptr && s.layout == 0 && s.T <= kSelfRowsMaxT) ? 1 : 0;
    int U = 0, NT = 0;
    cudaError_t e = cudaSuccess;
    const dim3 grid(s.B);
    if (a.expert_smooth) return launch_dispatch_expert(s, p, x, smooth, stream);
    if (s.quant_mode != 0) {
        if (pick_units(s.d / 16, 8, &U, &NT) != EP_OK) return EP_ERR_UNSUPPORTED;
        e = s.quant_mode == 1 ? launch_int8<true>(U, grid, dim3(NT), stream, a)
                              : launch_int8<false>(U, grid, dim3(NT), stream, a);
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
