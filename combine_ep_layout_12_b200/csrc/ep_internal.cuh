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

// Receive slabs of the ranks of a multi-GPU run (a kernel parameter): slab q holds
// the slab_rows = L * P * M low-latency rows of experts q*L .. q*L+L-1.
struct ShardTable {
    void* x[EP_SHARD_MAX_RANKS];        // recv_x slabs (dispatch) or expert-output slabs (combine)
    float* scale[EP_SHARD_MAX_RANKS];   // recv_scale slabs (dispatch, quant_mode 2)
    int32_t* src[EP_SHARD_MAX_RANKS];   // recv_src slabs (dispatch; may be null)
    int32_t* count[EP_SHARD_MAX_RANKS]; // recv_count [L][P] of each rank (dispatch; may be null)
    const int32_t* send_count;          // this rank's picks per expert [E] (dispatch; may be null)
    long long slab_rows;
    int token_base;                     // global index of this rank's first token
    int rank, P, L;                     // this rank, the ranks, experts per rank
};

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
// gstride / rbase: see LayoutArgs (default: gstride = P * M, rbase = 0).
int launch_layout(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                  const uint8_t* active, cudaStream_t stream, int gstride = -1, int rbase = 0);
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

// Multi-GPU forms (one process per logical rank; see ShardTable).  s is the local
// view: B = T tokens of this rank, rows = the global E * P * M.
int launch_shard_dispatch(const Shape& s, const ep_buffer_ptrs& p, const uint16_t* x,
                          const float* smooth, const ShardTable& tab, cudaStream_t stream);
// Layout and dispatch of one rank (s: P = 1, global rows via gstride and rbase) with
// the count exchange, in one grid when T <= 128 and k <= 8; p.recv_count is the
// rank's send_count [E].
int launch_shard_layout_dispatch(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                                 const uint8_t* active, const uint16_t* x, const float* smooth,
                                 const ShardTable& tab, int gstride, int rbase, cudaStream_t stream);
int launch_shard_combine(const Shape& s, const ep_buffer_ptrs& p, const int32_t* topk_idx,
                         const float* topk_weights, const uint8_t* active, const uint16_t* ori_x,
                         const uint16_t* a1, const uint16_t* a2, const uint16_t* v, uint16_t* y,
                         const ShardTable& tab, cudaStream_t stream);

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

// 16-byte store.  No "memory" clobber: nothing in the library reads back, within
// the same kernel, what these stores write, so the compiler may keep shared-memory
// values (row pointers, weights) in registers across the stores.
__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w));
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

// Receive rows of token t derived from the routing alone, for small per-rank
// batches: the slot of a routed id g is the number of earlier tokens of the same
// rank that picked g (a token counts once), which is exactly the slot the layout
// kernels assign; a routed id repeated inside the token gets row -1 after its
// first occurrence.  Inactive tokens (active[t] == 0, when a mask is given) route
// nothing and are not counted.  The earlier tokens' ids come from L2.
// s_rows, s_g, s_cnt: k-entry shared arrays; tab: E uint16 of shared memory, set
// here to one bit per routed pick of this token at the pick's expert, so that an
// earlier token costs k table lookups rather than k * k compares.  All threads of
// the CTA call it; on return s_rows[j] is written by thread j (j < k) and not yet
// published to the other threads.
// Packed rows (expert_offset and recv_count given): the row is expert_offset[g] +
// sum_{r' < r} recv_count[g][r'] + slot.  Those counts come from the layout kernel,
// which the caller guarantees complete; they are read through L2 (another grid
// wrote them).
__device__ inline void routing_rows(const int32_t* topk_idx, const uint8_t* active, int t, int k,
                                    int E, int T, int P, int M, int* s_rows, int* s_g, int* s_cnt,
                                    uint16_t* tab, const int32_t* expert_offset = nullptr,
                                    const int32_t* recv_count = nullptr, int gstride = -1, int rbase = 0) {
    uint32_t* tw = reinterpret_cast<uint32_t*>(tab);
    for (int i = threadIdx.x; i < (E + 1) / 2; i += blockDim.x) tw[i] = 0u;
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
    if (threadIdx.x < k && s_g[threadIdx.x] >= 0) tab[s_g[threadIdx.x]] = (uint16_t)(1u << threadIdx.x);
    __syncthreads();
    const int r = t / T;
    const bool vec4 = (k % 4 == 0) && ((reinterpret_cast<uintptr_t>(topk_idx) & 15) == 0);
    for (int tt = r * T + (int)threadIdx.x; tt < t; tt += blockDim.x) {
        if (active && !active[tt]) continue;
        const int32_t* ids = topk_idx + (size_t)tt * k;
        unsigned hit = 0;
        if (vec4) {
            for (int j4 = 0; 4 * j4 < k; ++j4) {
                const int4 v = __ldg(reinterpret_cast<const int4*>(ids) + j4);
                hit |= (unsigned)v.x < (unsigned)E ? tab[v.x] : 0u;
                hit |= (unsigned)v.y < (unsigned)E ? tab[v.y] : 0u;
                hit |= (unsigned)v.z < (unsigned)E ? tab[v.z] : 0u;
                hit |= (unsigned)v.w < (unsigned)E ? tab[v.w] : 0u;
            }
        } else {
            for (int jj = 0; jj < k; ++jj) {
                const int v = __ldg(ids + jj);
                hit |= (unsigned)v < (unsigned)E ? tab[v] : 0u;
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
        if (g >= 0)
            row = expert_offset ? s_cnt[threadIdx.x]
                                : g * (gstride < 0 ? P * M : gstride) + r * M + rbase + s_cnt[threadIdx.x];
        s_rows[threadIdx.x] = row;
    }
}

}  // namespace ep

#endif  // __CUDACC__
