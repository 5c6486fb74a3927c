// Internal declarations shared by the libep translation units (host launchers,
// the buffer object, device helpers).  Not part of the public ABI (include/ep.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"

namespace ep {

// Workspace header at the start of the caller's workspace array.  The layout
// kernel's per-rank special-expert partial counts follow it.
struct WsHeader {
    unsigned int done;  // CTAs of the current layout launch that have finished
    unsigned int err;   // device error word (EP_ERRBIT_*)
    unsigned int pad[62];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

constexpr int kMaxE = 2048;        // routed experts (Ascend: local_expert_num * ranks <= 2048)
constexpr int kMaxSpecial = 2048;  // zero + copy + const experts
constexpr int kMaxK = 16;          // picks per token (Ascend: 0 < K <= 16)
constexpr int kMaxD = 32768;     // 256 threads x 8 units of 16 elements

constexpr int kMaxPackedEP = 24576;  // E * P of the packed layout (the pack kernel's shared table)

struct Shape {
    int B, d, k, P, M, E, Z, C, K, T, L, E_tot, n_special;
    int quant_mode;     // 0 bf16, 1 static int8, 2 dynamic int8
    int expert_smooth;  // 1: a given smooth scale is [E][d], one row per routed expert
    int layout;      // 0 low-latency, 1 packed
    long long rows;  // receive rows: E * P * M (low-latency) or B * k (packed)
};

inline Shape make_shape(const ep_config& c) {
    Shape s;
    s.B = c.B; s.d = c.d; s.k = c.k; s.P = c.P; s.M = c.M; s.E = c.E;
    s.Z = c.n_zero; s.C = c.n_copy; s.K = c.n_const;
    s.T = c.B / c.P;
    s.L = c.E / c.P;
    s.n_special = c.n_zero + c.n_copy + c.n_const;
    s.E_tot = c.E + s.n_special;
    s.quant_mode = c.quant_mode;
    s.expert_smooth = c.smooth_rows > 1 ? 1 : 0;
    s.layout = c.layout;
    s.rows = c.layout == 1 ? (long long)c.B * c.k : (long long)c.E * c.P * c.M;
    return s;
}

// Workspace layout: WsHeader, then, for batches of more than 256 tokens per rank
// (the chunked layout kernels), the per-chunk counts [P][chunks][E] and special
// counts [P][chunks][n_special], chunks = ceil(T / 256).
inline size_t workspace_layout_bytes(const Shape& s) {
    const size_t chunks = s.T > 256 ? ((size_t)s.T + 255) / 256 : 0;
    return sizeof(WsHeader) + 4 * (size_t)s.P * chunks * ((size_t)s.E + s.n_special);
}
inline size_t workspace_bytes(const Shape& s) {
    return (workspace_layout_bytes(s) + 255) & ~(size_t)255;
}

// Host launchers (one per kernel family); each returns an EP_* status.
// active: x_active_mask [B] (nonzero = active) or null; an inactive token takes no
// part (as if every pick were -1).
int launch_layout(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                  const uint8_t* active, cudaStream_t stream);
// topk_idx: the routing of the latest layout on this buffer (lets dispatch derive
// its receive rows itself for small per-rank batches); may be null, except with a
// per-expert smooth scale, where it names each copy's expert.
int launch_dispatch(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* x,
                    const float* smooth, const int32_t* topk_idx, const uint8_t* active,
                    cudaStream_t stream);
// Layout and dispatch of the same routing in one grid when the batch per rank is
// small (T <= 128, k <= 8); otherwise the two launches above, in order.
int launch_layout_dispatch(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                           const uint8_t* active, const uint16_t* x, const float* smooth,
                           cudaStream_t stream);
int launch_combine(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* expert_out,
                   const int32_t* topk_idx, const float* topk_weights, const uint8_t* active,
                   const uint16_t* ori_x,
                   const uint16_t* a1, const uint16_t* a2, const uint16_t* v, uint16_t* y,
                   cudaStream_t stream);

// Streaming multiprocessors of the current device (queried once per device).
inline int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64 && cached[dev] != 0) return cached[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev < 64) cached[dev] = n;
    return n;
}

// One-time per-device setup (a kernel's shared-memory opt-in is a per-device
// attribute).  first_on_device is true until mark_device records the device; past
// the table it stays true, so the setup simply runs on every call there.  Setting
// the same attribute twice is harmless, so concurrent first calls need no lock.
constexpr int kDeviceSlots = 64;
inline bool first_on_device(const bool* done, int dev) {
    return dev < 0 || dev >= kDeviceSlots || !done[dev];
}
inline void mark_device(bool* done, int dev) {
    if (dev >= 0 && dev < kDeviceSlots) done[dev] = true;
}

// Launch with programmatic dependent launch enabled: the kernel may begin while
// the previous kernel on the stream drains; every kernel here executes
// griddepcontrol.wait before it touches memory a predecessor may still use.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace ep

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
#ifdef __CUDACC__

namespace ep {

__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 16-byte streaming load through the non-coherent path, not kept in L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// 32 bytes per thread (sm_100 256-bit global accesses): one load or store moves 16
// bf16 values, the source of one 16-byte int8 vector.
struct V8 {
    uint32_t w[8];
};
__device__ __forceinline__ V8 ld_stream_v8(const void* p) {
    V8 r;
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]),
                   "=r"(r.w[5]), "=r"(r.w[6]), "=r"(r.w[7])
                 : "l"(p));
    return r;
}
__device__ __forceinline__ void st_v8(void* p, const V8& v) {
    asm volatile("st.global.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v.w[0]),
                 "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]), "r"(v.w[6]),
                 "r"(v.w[7])
                 : "memory");
}

// 32 bytes at p: one 256-bit access when `wide` (the host has checked that every
// such address is 32-byte aligned), else two 16-byte accesses (the ABI promises
// only 16-byte alignment, and an int8 row of d % 32 == 16 bytes leaves every
// other row on a 16-byte boundary).
__device__ __forceinline__ V8 ld32(const void* p, bool wide) {
    if (wide) return ld_stream_v8(p);
    const uint4 a = ld_stream_v4(p);
    const uint4 b = ld_stream_v4(reinterpret_cast<const char*>(p) + 16);
    V8 r;
    r.w[0] = a.x; r.w[1] = a.y; r.w[2] = a.z; r.w[3] = a.w;
    r.w[4] = b.x; r.w[5] = b.y; r.w[6] = b.z; r.w[7] = b.w;
    return r;
}
__device__ __forceinline__ void st32(void* p, const V8& v, bool wide) {
    if (wide) {
        st_v8(p, v);
    } else {
        st_v4(p, make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]));
        st_v4(reinterpret_cast<char*>(p) + 16, make_uint4(v.w[4], v.w[5], v.w[6], v.w[7]));
    }
}

// bf16 bits <-> fp32: a bf16 is the high half of a binary32.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 -> packed bf16x2, round to nearest even (cvt.rn.bf16x2.f32; NaN stays NaN).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Checked build (-DEP_CHECKED): every row or offset a kernel computes is tested
// against the extent of the array it indexes before the access; one outside it
// sets EP_ERRBIT_CHECKED in the error word and the access is skipped.  Without
// EP_CHECKED the test compiles away (the kernels' own range checks stay).
#ifdef EP_CHECKED
__device__ __forceinline__ bool ep_in_range(long long idx, long long n, unsigned* err_word) {
    if (idx >= 0 && idx < n) return true;
    atomicOr(err_word, EP_ERRBIT_CHECKED);
    return false;
}
#else
__device__ __forceinline__ bool ep_in_range(long long, long long, unsigned*) { return true; }
#endif

// OR `bits` into the device error word, one atomic per group of converged lanes.
__device__ __forceinline__ void report_err(unsigned* err_word, unsigned bits) {
    const unsigned active = __activemask();
    const unsigned all = __reduce_or_sync(active, bits);
    if (all && (int)(threadIdx.x & 31) == __ffs(active) - 1) atomicOr(err_word, all);
}

// Shared memory of one warp of the warp-per-token kernels: the routing table
// (E uint16, 16-byte padded); the dispatch kernels may add a staging row after it.
__host__ __device__ __forceinline__ int warp_tab_bytes(int E) { return ((2 * E + 15) / 16) * 16; }

// Zero this warp's routing table (E uint16) before its first use.
__device__ __forceinline__ void zero_warp_tab(uint16_t* tab, int E) {
    uint32_t* w = reinterpret_cast<uint32_t*>(tab);
    const int n = warp_tab_bytes(E) / 4;
    for (int i = threadIdx.x & 31; i < n; i += 32) w[i] = 0u;
    __syncwarp();
}

// Receive rows of token t derived from the routing alone, for small per-rank
// batches: the slot of a routed id g is the number of earlier tokens of the same
// rank that picked g (a token counts once), which is exactly the slot the layout
// kernels assign; a routed id repeated inside the token gets row -1 after its
// first occurrence.  Inactive tokens (active[t] == 0, when a mask is given) route
// nothing and are not counted.  The earlier tokens' ids come from L2.  s_rows,
// s_g, s_cnt: k-entry shared arrays.  All threads of the CTA call it; on return
// s_rows[j] is written by thread j (j < k) and not yet published to the other threads.
// Packed rows (expert_offset and recv_count given): the row is expert_offset[g] +
// sum_{r' < r} recv_count[g][r'] + slot.  Those counts come from the layout kernel,
// which the caller guarantees complete; they are read through L2 (another grid
// wrote them).
__device__ inline void routing_rows(const int32_t* topk_idx, const uint8_t* active, int t, int k,
                                    int E, int T, int P, int M, int* s_rows, int* s_g, int* s_cnt,
                                    const int32_t* expert_offset = nullptr,
                                    const int32_t* recv_count = nullptr) {
    if (threadIdx.x < k) {
        const int j = threadIdx.x;
        const int g = topk_idx[(size_t)t * k + j];
        bool routed = g >= 0 && g < E && !(active && !active[t]);
        for (int jj = 0; jj < j; ++jj)
            if (topk_idx[(size_t)t * k + jj] == g) routed = false;  // repeated id: dropped
        s_g[j] = routed ? g : -1;
        s_cnt[j] = 0;
    }
    __syncthreads();
    const int r = t / T;
    for (int tt = r * T + (int)threadIdx.x; tt < t; tt += blockDim.x) {
        if (active && !active[tt]) continue;
        const int32_t* ids = topk_idx + (size_t)tt * k;
        unsigned hit = 0;
        for (int jj = 0; jj < k; ++jj) {
            const int v = __ldg(ids + jj);
            for (int j = 0; j < k; ++j) {
                const int g = s_g[j];
                if (g >= 0 && v == g) hit |= 1u << j;
            }
        }
        while (hit) {
            const int j = __ffs(hit) - 1;
            hit &= hit - 1;
            atomicAdd(&s_cnt[j], 1);
        }
    }
    if (expert_offset) {
        // packed: add each pick's base (expert_offset[g] and the r lower ranks' counts)
        // to its slot, all the loads spread over the CTA's threads at once
        const int per = r + 1;
        for (int i = threadIdx.x; i < k * per; i += blockDim.x) {
            const int j = i / per, rr = i - j * per;
            const int g = s_g[j];
            if (g >= 0)
                atomicAdd(&s_cnt[j], rr < r ? __ldcg(recv_count + (size_t)g * P + rr) : __ldcg(expert_offset + g));
        }
    }
    __syncthreads();
    if (threadIdx.x < k) {
        const int g = s_g[threadIdx.x];
        int row = -1;
        if (g >= 0) row = expert_offset ? s_cnt[threadIdx.x] : g * P * M + r * M + s_cnt[threadIdx.x];
        s_rows[threadIdx.x] = row;
    }
}

// The same receive rows computed by one warp on its own, for kernels whose warps
// each own a token (no CTA barrier).  tab: this warp's shared table of E uint16
// entries, all zero on entry and zero again on return; entry g holds the bit of
// the pick of this token that routes to g.  An earlier token of the rank looks
// each of its ids up in the table, so it costs k shared loads instead of k * k
// compares, and a token counts once per expert however often it repeats an id.
// On return row[j] is the receive row of pick j (-1: not routed) in every lane.
template <int KM>
__device__ __forceinline__ void routing_rows_warp(const int32_t* __restrict__ topk_idx,
                                                  const uint8_t* active, int t, int k, int E,
                                                  int T, int P, int M, uint16_t* tab,
                                                  int (&row)[KM],
                                                  const int32_t* expert_offset = nullptr,
                                                  const int32_t* recv_count = nullptr) {
    static_assert(KM <= 16, "pick bits are kept in 16-bit table entries");
    const unsigned FULL = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    const bool on = !(active && !active[t]);
    const int mine = lane < k ? __ldg(topk_idx + (size_t)t * k + lane) : -1;
    int g[KM];
    unsigned rb = 0;  // routed picks: an id in [0, E), its first occurrence, token active
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        g[j] = __shfl_sync(FULL, mine, j);
        bool routed = on && j < k && g[j] >= 0 && g[j] < E;
#pragma unroll
        for (int jj = 0; jj < j; ++jj)
            if (g[jj] == g[j]) routed = false;
        if (routed) rb |= 1u << j;
    }
    if ((rb >> lane) & 1u) tab[mine] = (uint16_t)(1u << lane);
    __syncwarp();
    const int r = t / T;
    int cnt[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) cnt[j] = 0;
    const bool vec4 = (k % 4 == 0) && ((reinterpret_cast<uintptr_t>(topk_idx) & 15) == 0);
    for (int tt = r * T + lane; tt < t; tt += 32) {
        if (active && !active[tt]) continue;
        const int32_t* ids = topk_idx + (size_t)tt * k;
        unsigned hit = 0;
        if (vec4) {
#pragma unroll
            for (int j4 = 0; j4 < KM / 4; ++j4) {
                if (4 * j4 >= k) continue;
                const int4 v = __ldg(reinterpret_cast<const int4*>(ids) + j4);
                hit |= (unsigned)v.x < (unsigned)E ? tab[v.x] : 0u;
                hit |= (unsigned)v.y < (unsigned)E ? tab[v.y] : 0u;
                hit |= (unsigned)v.z < (unsigned)E ? tab[v.z] : 0u;
                hit |= (unsigned)v.w < (unsigned)E ? tab[v.w] : 0u;
            }
        } else {
#pragma unroll
            for (int jj = 0; jj < KM; ++jj) {
                if (jj >= k) continue;
                const int v = __ldg(ids + jj);
                hit |= (unsigned)v < (unsigned)E ? tab[v] : 0u;
            }
        }
#pragma unroll
        for (int j = 0; j < KM; ++j) cnt[j] += (hit >> j) & 1u;
    }
#pragma unroll
    for (int j = 0; j < KM; ++j) cnt[j] = (int)__reduce_add_sync(FULL, (unsigned)cnt[j]);
    if (expert_offset) {
        // packed: add expert_offset[g] and the r lower ranks' counts of g
        const int per = r + 1;
        int part[KM];
#pragma unroll
        for (int j = 0; j < KM; ++j) part[j] = 0;
        for (int i = lane; i < k * per; i += 32) {
            const int jsel = i / per, rr = i - jsel * per;
            int gsel = -1;
#pragma unroll
            for (int j = 0; j < KM; ++j)
                if (j == jsel && ((rb >> j) & 1u)) gsel = g[j];
            if (gsel < 0) continue;
            const int val = rr < r ? __ldcg(recv_count + (size_t)gsel * P + rr) : __ldcg(expert_offset + gsel);
#pragma unroll
            for (int j = 0; j < KM; ++j)
                if (j == jsel) part[j] += val;
        }
#pragma unroll
        for (int j = 0; j < KM; ++j) cnt[j] += (int)__reduce_add_sync(FULL, (unsigned)part[j]);
    }
    __syncwarp();
    if ((rb >> lane) & 1u) tab[mine] = 0;
    __syncwarp();
#pragma unroll
    for (int j = 0; j < KM; ++j)
        row[j] = ((rb >> j) & 1u) ? (expert_offset ? cnt[j] : g[j] * P * M + r * M + cnt[j]) : -1;
}

}  // namespace ep

#endif  // __CUDACC__
