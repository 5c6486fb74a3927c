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
#include <mutex>

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

// Multi-GPU form: rows read from dst_pos, stored into the owning rank's slab.  The
// count exchange rides along: the threads of one CTA store this rank's send_count of
// each expert g into column `rank` of the owner's recv_count (owner q = g / L, entry
// [g - q L][rank]), plain stores to the owner's memory like the rows themselves.
__device__ __forceinline__ void store_counts(const ShardTable& tab, int E) {
    if (!tab.send_count) return;
    for (int g = threadIdx.x; g < E; g += blockDim.x) {
        const int q = g / tab.L;
        int32_t* dst = tab.count[q];
        if (dst) dst[(size_t)(g - q * tab.L) * tab.P + tab.rank] = tab.send_count[g];
    }
}

template <int U, bool STATIC>
__global__ void __launch_bounds__(256)
    dispatch_int8_shard_kernel(DispatchArgs a, const __grid_constant__ ShardTable tab) {
    pdl_wait();
    pdl_launch_dependents();
    if (blockIdx.x == 0) store_counts(tab, a.E);
    dispatch_int8_body<U, STATIC>(a, blockIdx.x, ShardRows{tab});
}

template <int U>
__global__ void __launch_bounds__(256)
    dispatch_bf16_shard_kernel(DispatchArgs a, const __grid_constant__ ShardTable tab) {
    pdl_wait();
    pdl_launch_dependents();
    if (blockIdx.x == 0) store_counts(tab, a.E);
    dispatch_bf16_body<U>(a, blockIdx.x, ShardRows{tab});
}

// A rank without tokens still sends its (zero) counts.
__global__ void __launch_bounds__(256) shard_counts_kernel(const __grid_constant__ ShardTable tab, int E) {
    pdl_wait();
    pdl_launch_dependents();
    store_counts(tab, E);
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
// makes the kernel bound by L2 reads of the table.  Instead the work is split by
// expert.  Rows of up to 8192 elements take the column-owning kernel further
// down; the row-wide kernel here takes any row length.  A CTA takes one
// expert g and a share of its receive rows: it stages smooth[g] in shared memory
// once, finds the source token of each of its rows through recv_src, and
// quantizes the rows one at a time with all its threads.  Per-copy quantization
// does k times the arithmetic of the per-token form, so the loop is written for
// few instructions per element: a thread owns GP units of 8 elements (one 16-byte
// x load and one 8-byte store per unit), x_fp32 is formed once per element and
// kept in registers for the cast, the smooth row sits in two float4 planes so
// the shared-memory reads are conflict-free, and the absmax is one CTA reduction
// behind one barrier (two alternating slot sets).  The next row's x is loaded
// before that barrier so its latency overlaps the reduction.  The receive rows
// come from the layout (recv_count, recv_src, expert_offset), so the kernel
// waits for it first.
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

// EXACT: the CTA's threads times GP cover the d / 8 units exactly (no bounds checks).
template <int GP, bool EXACT>
__device__ __forceinline__ void load_x_units(const ExpertArgs& a, int t, int nu, uint4 (&v)[GP]) {
    const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)(t < 0 ? 0 : t) * a.d);
#pragma unroll
    for (int m = 0; m < GP; ++m) {
        const int u = threadIdx.x + m * blockDim.x;
        v[m] = (t >= 0 && (EXACT || u < nu)) ? __ldg(xr + u) : make_uint4(0, 0, 0, 0);
    }
}

template <int GP, int MAXT, bool STATIC, bool EXACT>
__global__ void __launch_bounds__(MAXT) dispatch_expert_major_kernel(ExpertArgs a) {
    extern __shared__ float4 s_sm4[];                                        // 2 planes of [d / 8]
    const int NT = blockDim.x;
    const int nu = a.d >> 3;
    float4* s_lo = s_sm4;                                                    // elements 8u .. 8u+3
    float4* s_hi = s_sm4 + nu;                                               // elements 8u+4 .. 8u+7
    long long* s_row = reinterpret_cast<long long*>(s_sm4 + 2 * nu);        // [NT]
    int* s_t = reinterpret_cast<int*>(s_row + NT);                           // [NT]
    int* s_pre = s_t + NT;                                                   // [P + 1]
    __shared__ float s_red[2][32];
    pdl_wait();
    pdl_launch_dependents();
    const int g = blockIdx.x / a.parts, part = blockIdx.x - g * a.parts;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = NT >> 5;

    const float4* srow = reinterpret_cast<const float4*>(a.smooth + (size_t)g * a.d);
    for (int u = threadIdx.x; u < nu; u += NT) {
        s_lo[u] = __ldg(srow + 2 * u);
        s_hi[u] = __ldg(srow + 2 * u + 1);
    }
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
        uint4 cur[GP], nxt[GP];
        load_x_units<GP, EXACT>(a, s_t[0], nu, cur);
        for (int j = 0; j < nb; ++j) {
            const int t = s_t[j];
            const long long row = s_row[j];
            // x_fp32 = fp32(x) * smooth[g], formed once per element and kept for the cast
            float f[GP][8];
            float amax = 0.0f;
#pragma unroll
            for (int m = 0; m < GP; ++m) {
                const int u = threadIdx.x + m * NT;
                const bool in = EXACT || u < nu;
                const float4 lo4 = in ? s_lo[u] : make_float4(0.f, 0.f, 0.f, 0.f);
                const float4 hi4 = in ? s_hi[u] : make_float4(0.f, 0.f, 0.f, 0.f);
                f[m][0] = __fmul_rn(bf16lo(cur[m].x), lo4.x);
                f[m][1] = __fmul_rn(bf16hi(cur[m].x), lo4.y);
                f[m][2] = __fmul_rn(bf16lo(cur[m].y), lo4.z);
                f[m][3] = __fmul_rn(bf16hi(cur[m].y), lo4.w);
                f[m][4] = __fmul_rn(bf16lo(cur[m].z), hi4.x);
                f[m][5] = __fmul_rn(bf16hi(cur[m].z), hi4.y);
                f[m][6] = __fmul_rn(bf16lo(cur[m].w), hi4.z);
                f[m][7] = __fmul_rn(bf16hi(cur[m].w), hi4.w);
                if (!STATIC) {
#pragma unroll
                    for (int e = 0; e < 8; e += 2)
                        amax = fmaxf(amax, fmaxf(fabsf(f[m][e]), fabsf(f[m][e + 1])));
                }
            }
            if (j + 1 < nb) load_x_units<GP, EXACT>(a, s_t[j + 1], nu, nxt);
            float s = 1.0f;
            bool degenerate = false;
            if (!STATIC) {
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
                uint2* out = reinterpret_cast<uint2*>(a.recv_x + row * a.d);
#pragma unroll
                for (int m = 0; m < GP; ++m) {
                    const int u = threadIdx.x + m * NT;
                    if (!EXACT && u >= nu) continue;
                    uint2 word;
                    if (STATIC) {
                        word.x = cvt_s8x4(f[m][0], f[m][1], f[m][2], f[m][3]);
                        word.y = cvt_s8x4(f[m][4], f[m][5], f[m][6], f[m][7]);
                    } else {
                        word.x = cvt_s8x4_unclamped(__fmul_rn(f[m][0], s), __fmul_rn(f[m][1], s),
                                                    __fmul_rn(f[m][2], s), __fmul_rn(f[m][3], s));
                        word.y = cvt_s8x4_unclamped(__fmul_rn(f[m][4], s), __fmul_rn(f[m][5], s),
                                                    __fmul_rn(f[m][6], s), __fmul_rn(f[m][7], s));
                        if (degenerate) word = make_uint2(0, 0);
                    }
                    out[u] = word;
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

// Column-owning form, for rows of up to 128 * 8 units of 8 elements (d <= 8192;
// the row-wide kernel above takes longer rows).  A CTA of 128 threads (4 warps)
// quantizes one receive row at a time, and thread i owns the same GP units
// u = i + 128 m of every row, so the smooth values of its columns are loaded into
// registers once per expert, and the per-row costs (the absmax reduction over four
// warps, the scale division, the row bookkeeping) are spread over 8 GP elements per
// thread.  x_fp32 is kept in registers between the absmax and the cast; the next
// row's x is loaded while the current one is reduced.  The grid is one resident
// wave: CTA b takes rows [N b / G, N (b + 1) / G) of the N routed rows in expert
// order (row q of that order is copy q - expert_offset[g] of the expert g with
// expert_offset[g] <= q < expert_offset[g + 1]), so every CTA has the same number
// of rows and reloads the smooth row where its share crosses into the next expert.
// Instruction savings that keep the bits: the absmax takes two elements per
// three-operand maximum, and x_fp32 * s is formed two products per packed
// multiply (each product rounded on its own; the add that follows is scalar, so no
// multiply-add contraction can reach it).  A degenerate row takes s = 0, which
// turns every finite x_fp32 into +-0 and so into the int8 code 0.
constexpr int kColsThreads = 128;

// (a.x * b.x, a.y * b.y), each product rounded to nearest even (one packed instruction)
__device__ __forceinline__ float2 fmul2_rn(float2 a, float2 b) {
    unsigned long long ra, rb, rd;
    asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
    float2 d;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
    return d;
}

// max(a, |b|, |c|) in one three-operand maximum (NaN operands ignored, as fmaxf)
__device__ __forceinline__ float fmax_abs2(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
    return r;
}

template <int GP, bool STATIC, bool EXACT>
struct ColsRow {
    const ExpertArgs& a;
    const float4 (&sl)[GP];  // smooth[g][8u .. 8u + 3] of this thread's units
    const float4 (&sh)[GP];  // smooth[g][8u + 4 .. 8u + 7]
    int nu;
    float (&red)[2][4];

    // Quantizes the row (t, row) whose x is in cur; loads x of token t_next into nxt.
    __device__ __forceinline__ void run(int t, long long row, int t_next, int& par, uint4 (&cur)[GP],
                                        uint4 (&nxt)[GP]) const {
        float f[GP][8];
        float amax = 0.0f;
#pragma unroll
        for (int m = 0; m < GP; ++m) {
            f[m][0] = __fmul_rn(bf16lo(cur[m].x), sl[m].x);
            f[m][1] = __fmul_rn(bf16hi(cur[m].x), sl[m].y);
            f[m][2] = __fmul_rn(bf16lo(cur[m].y), sl[m].z);
            f[m][3] = __fmul_rn(bf16hi(cur[m].y), sl[m].w);
            f[m][4] = __fmul_rn(bf16lo(cur[m].z), sh[m].x);
            f[m][5] = __fmul_rn(bf16hi(cur[m].z), sh[m].y);
            f[m][6] = __fmul_rn(bf16lo(cur[m].w), sh[m].z);
            f[m][7] = __fmul_rn(bf16hi(cur[m].w), sh[m].w);
            if (!STATIC) {
#pragma unroll
                for (int e = 0; e < 8; e += 2) amax = fmax_abs2(amax, f[m][e], f[m][e + 1]);
            }
        }
        const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)(t_next < 0 ? 0 : t_next) * a.d);
#pragma unroll
        for (int m = 0; m < GP; ++m) {
            const int u = threadIdx.x + m * kColsThreads;
            nxt[m] = (t_next >= 0 && (EXACT || u < nu)) ? __ldg(xr + u) : make_uint4(0, 0, 0, 0);
        }
        float s = 1.0f;
        bool degenerate = false;
        if (!STATIC) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            if ((threadIdx.x & 31) == 0) red[par][threadIdx.x >> 5] = amax;
            __syncthreads();
            const float4 r4 = *reinterpret_cast<const float4*>(red[par]);
            par ^= 1;
            amax = fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w));
            s = __fdiv_rn(127.0f, amax);
            degenerate = (amax == 0.0f) || isinf(s);
            if (degenerate) s = 0.0f;
        }
        if (t < 0) return;
        uint2* out = reinterpret_cast<uint2*>(a.recv_x + row * a.d);
#pragma unroll
        for (int m = 0; m < GP; ++m) {
            const int u = threadIdx.x + m * kColsThreads;
            if (!EXACT && u >= nu) continue;
            uint2 word;
            if (STATIC) {
                word.x = cvt_s8x4(f[m][0], f[m][1], f[m][2], f[m][3]);
                word.y = cvt_s8x4(f[m][4], f[m][5], f[m][6], f[m][7]);
            } else {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const float2 p = fmul2_rn(make_float2(f[m][e], f[m][e + 1]), make_float2(s, s));
                    v[e] = p.x;
                    v[e + 1] = p.y;
                }
                word.x = cvt_s8x4_unclamped(v[0], v[1], v[2], v[3]);
                word.y = cvt_s8x4_unclamped(v[4], v[5], v[6], v[7]);
            }
            out[u] = word;
        }
        if (!STATIC && threadIdx.x == 0) a.recv_scale[row] = degenerate ? 0.0f : __fdiv_rn(1.0f, s);
    }
};

template <int GP, bool STATIC, bool EXACT>
__global__ void __launch_bounds__(kColsThreads, 3) dispatch_expert_cols_kernel(ExpertArgs a) {
    extern __shared__ int s_pre[];  // [P + 1]
    __shared__ long long s_row[kColsThreads];
    __shared__ int s_t[kColsThreads];
    __shared__ __align__(16) float s_red[2][4];
    constexpr int NT = kColsThreads;
    const int nu = a.d >> 3;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_launch_dependents();
    const long long N = min((long long)max(a.expert_offset[a.E], 0), a.rows);
    long long q = N * blockIdx.x / gridDim.x;
    const long long q1 = N * (blockIdx.x + 1) / gridDim.x;
    int g = 0;
    {
        int lo = 0, hi = a.E - 1;  // the last expert whose rows start at or before q
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (a.expert_offset[mid] <= q) lo = mid; else hi = mid - 1;
        }
        g = lo;
    }
    float4 sl[GP], sh[GP];
    const ColsRow<GP, STATIC, EXACT> body{a, sl, sh, nu, s_red};
    int par = 0;
    while (q < q1) {
        while (g < a.E - 1 && a.expert_offset[g + 1] <= q) ++g;  // skip experts without rows
        const long long off = a.expert_offset[g];
        const long long end = min(q1, max(q + 1, (long long)a.expert_offset[g + 1]));
        const float4* srow = reinterpret_cast<const float4*>(a.smooth + (size_t)g * a.d);
#pragma unroll
        for (int m = 0; m < GP; ++m) {
            const int u = threadIdx.x + m * NT;
            const bool in = EXACT || u < nu;
            sl[m] = in ? __ldg(srow + 2 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
            sh[m] = in ? __ldg(srow + 2 * u + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
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
        // copies of expert g that exist (an expert holds at most one copy per token)
        const long long n = a.layout == 0 ? min((long long)s_pre[a.P], (long long)a.P * a.M) : end - off;
        for (long long b0 = q; b0 < end; b0 += NT) {
            const int nb = (int)min((long long)NT, end - b0);
            if (threadIdx.x < nb) {
                const long long i = b0 + threadIdx.x - off;
                long long row = -1;
                if (i >= 0 && i < n) {
                    if (a.layout == 0) {
                        int lo = 0, hi = a.P - 1;  // the last rank whose run starts at or before i
                        while (lo < hi) {
                            const int mid = (lo + hi + 1) >> 1;
                            if (s_pre[mid] <= i) lo = mid; else hi = mid - 1;
                        }
                        row = (long long)g * a.P * a.M + (long long)lo * a.M + (i - s_pre[lo]);
                    } else {
                        row = b0 + threadIdx.x;
                    }
                }
                const int t = (row >= 0 && row < a.rows) ? a.recv_src[row] : -1;
                const bool ok = t >= 0 && t < a.B;
                report_err(a.err, ok ? 0u : EP_ERRBIT_ROW_RANGE);
                s_row[threadIdx.x] = row;
                s_t[threadIdx.x] = ok ? t : -1;
            }
            __syncthreads();
            uint4 xa[GP], xb[GP];
            {
                const int t0 = s_t[0];
                const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)(t0 < 0 ? 0 : t0) * a.d);
#pragma unroll
                for (int m = 0; m < GP; ++m) {
                    const int u = threadIdx.x + m * NT;
                    xa[m] = (t0 >= 0 && (EXACT || u < nu)) ? __ldg(xr + u) : make_uint4(0, 0, 0, 0);
                }
            }
            // two rows per iteration, so the current and the prefetched x swap roles
            // without register copies
            for (int j = 0; j < nb; j += 2) {
                body.run(s_t[j], s_row[j], j + 1 < nb ? s_t[j + 1] : -1, par, xa, xb);
                if (j + 1 < nb) body.run(s_t[j + 1], s_row[j + 1], j + 2 < nb ? s_t[j + 2] : -1, par, xb, xa);
            }
            __syncthreads();  // s_row / s_t (and s_pre) are rewritten next
        }
        q = end;
        g = min(g + 1, a.E - 1);
    }
}

using ExpertKernel = void (*)(ExpertArgs);

ExpertKernel pick_cols_kernel(bool st, int GP, bool exact) {
#define EP_COLS_K(G) \
    (st ? (exact ? dispatch_expert_cols_kernel<G, true, true> : dispatch_expert_cols_kernel<G, true, false>) \
        : (exact ? dispatch_expert_cols_kernel<G, false, true> : dispatch_expert_cols_kernel<G, false, false>))
    switch (GP) {
        case 1: return EP_COLS_K(1);
        case 2: return EP_COLS_K(2);
        case 3: return EP_COLS_K(3);
        case 4: return EP_COLS_K(4);
        case 5: return EP_COLS_K(5);
        case 6: return EP_COLS_K(6);
        case 7: return EP_COLS_K(7);
        default: return EP_COLS_K(8);
    }
#undef EP_COLS_K
}

// GP units of 8 elements per thread, up to 256 threads (1024 for rows above 8192
// elements), and whether NT * GP covers the row exactly.
ExpertKernel pick_expert_kernel(bool st, int GP, int NT, bool exact) {
#define EP_EXPERT_K(G, T)                                                                          \
    (st ? (exact ? dispatch_expert_major_kernel<G, T, true, true> : dispatch_expert_major_kernel<G, T, true, false>) \
        : (exact ? dispatch_expert_major_kernel<G, T, false, true> : dispatch_expert_major_kernel<G, T, false, false>))
    switch (GP) {
        case 1: return EP_EXPERT_K(1, 256);
        case 2: return EP_EXPERT_K(2, 256);
        default: return NT <= 256 ? EP_EXPERT_K(4, 256) : EP_EXPERT_K(4, 1024);
    }
#undef EP_EXPERT_K
}

// Resident CTAs per SM of one kernel configuration, queried once per device and
// configuration (the result depends only on the kernel's resources).
int expert_occupancy(ExpertKernel kern, int NT, size_t smem) {
    struct Entry { int dev; ExpertKernel k; int nt; size_t smem; int occ; };
    static Entry cache[32];
    static int n_cache = 0;
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n_cache; ++i)
        if (cache[i].dev == dev && cache[i].k == kern && cache[i].nt == NT && cache[i].smem == smem)
            return cache[i].occ;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, NT, smem) != cudaSuccess || occ < 1)
        occ = 1;
    if (n_cache < 32) cache[n_cache++] = {dev, kern, NT, smem, occ};
    return occ;
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
    const int nu = sh.d / 8;
    if (nu <= kColsThreads * 8) {
        const int GP = (nu + kColsThreads - 1) / kColsThreads;
        const ExpertKernel kern = pick_cols_kernel(sh.quant_mode == 1, GP, GP * kColsThreads == nu);
        const size_t smem = sizeof(int) * ((size_t)sh.P + 1);
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return EP_ERR_CUDA;
        // one resident wave of CTAs, each with an equal share of the rows
        const int occ = expert_occupancy(kern, kColsThreads, smem);
        a.parts = 1;
        const dim3 grid((unsigned)(num_sms() * occ));
        const cudaError_t e = launch_pdl(kern, grid, dim3(kColsThreads), smem, stream, a);
        return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
    }
    // units of 8 elements per thread: the smallest GP in {1, 2, 4} with at most 256
    // threads, else GP = 4 with up to 1024 threads (d <= 32768)
    int GP = 1;
    while (GP < 4 && (nu + GP - 1) / GP > 256) GP *= 2;
    int NT = (nu + GP - 1) / GP;
    NT = ((NT + 31) / 32) * 32;
    if (NT > 1024) return EP_ERR_UNSUPPORTED;
    const bool exact = NT * GP == nu;
    const ExpertKernel kern = pick_expert_kernel(sh.quant_mode == 1, GP, NT, exact);
    const size_t smem = sizeof(float) * (size_t)sh.d + (sizeof(long long) + sizeof(int)) * (size_t)NT +
                        sizeof(int) * ((size_t)sh.P + 1);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return EP_ERR_CUDA;
    // about four waves of resident CTAs, split evenly over the experts
    const int occ = expert_occupancy(kern, NT, smem);
    const long long target = 4LL * num_sms() * occ;
    long long parts = (target + sh.E - 1) / sh.E;
    if (parts < 1) parts = 1;
    a.parts = (int)parts;
    const dim3 grid((unsigned)((long long)sh.E * a.parts));
    const cudaError_t e = launch_pdl(kern, grid, dim3((unsigned)NT), smem, stream, a);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

}  // namespace

int launch_dispatch(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* x,
                    const float* smooth, const int32_t* topk_idx, const uint8_t* active,
                    cudaStream_t stream) {
    if (s.B == 0) return EP_OK;
    DispatchArgs a = make_dispatch_args(s, p, x, smooth, topk_idx, active);
    // Where the rows come from.  Low-latency layout: dst_pos, read after the wait
    // (one round trip; a CTA deriving its rows from the routing before the wait
    // gains only while the layout kernel is still running, and a caller that wants
    // that overlap has ep_layout_dispatch, whose one grid does it).  Packed layout,
    // small batches per rank (at most kSelfRowsMaxT earlier tokens to scan): each
    // CTA derives its rows from the routing and the first layout kernel's counts.
    // ep_layout ends with the pack kernel, which starts only after the counting
    // kernel has finished, so a dispatch started by the pack kernel can read them
    // and run alongside it.
    a.self_rows = (topk_idx != nullptr && s.layout == 1 && s.T <= kSelfRowsMaxT) ? 1 : 0;
    if (a.self_rows) {
        a.expert_offset = p.expert_offset;
        a.recv_count = p.recv_count;
    }
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

int launch_shard_dispatch(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* x,
                          const float* smooth, const ShardTable& tab, cudaStream_t stream) {
    if (s.B == 0) {
        if (!tab.send_count) return EP_OK;
        return launch_pdl(shard_counts_kernel, dim3(1), dim3(256), 0, stream, tab, s.E) == cudaSuccess ? EP_OK
                                                                                                  : EP_ERR_CUDA;
    }
    DispatchArgs a = make_dispatch_args(s, p, x, smooth, nullptr, nullptr);
    a.self_rows = 0;
    int U = 0, NT = 0;
    cudaError_t e = cudaSuccess;
    const dim3 grid(s.B);
    if (s.quant_mode != 0) {
        if (pick_units(s.d / 16, 8, &U, &NT) != EP_OK) return EP_ERR_UNSUPPORTED;
        const bool st = s.quant_mode == 1;
        switch (U) {
            case 1: e = launch_pdl(st ? dispatch_int8_shard_kernel<1, true> : dispatch_int8_shard_kernel<1, false>, grid, dim3(NT), 0, stream, a, tab); break;
            case 2: e = launch_pdl(st ? dispatch_int8_shard_kernel<2, true> : dispatch_int8_shard_kernel<2, false>, grid, dim3(NT), 0, stream, a, tab); break;
            case 4: e = launch_pdl(st ? dispatch_int8_shard_kernel<4, true> : dispatch_int8_shard_kernel<4, false>, grid, dim3(NT), 0, stream, a, tab); break;
            default: e = launch_pdl(st ? dispatch_int8_shard_kernel<8, true> : dispatch_int8_shard_kernel<8, false>, grid, dim3(NT), 0, stream, a, tab); break;
        }
    } else {
        if (pick_units(s.d / 8, 16, &U, &NT) != EP_OK) return EP_ERR_UNSUPPORTED;
        switch (U) {
            case 1: e = launch_pdl(dispatch_bf16_shard_kernel<1>, grid, dim3(NT), 0, stream, a, tab); break;
            case 2: e = launch_pdl(dispatch_bf16_shard_kernel<2>, grid, dim3(NT), 0, stream, a, tab); break;
            case 4: e = launch_pdl(dispatch_bf16_shard_kernel<4>, grid, dim3(NT), 0, stream, a, tab); break;
            case 8: e = launch_pdl(dispatch_bf16_shard_kernel<8>, grid, dim3(NT), 0, stream, a, tab); break;
            default: e = launch_pdl(dispatch_bf16_shard_kernel<16>, grid, dim3(NT), 0, stream, a, tab); break;
        }
    }
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

}  // namespace ep
