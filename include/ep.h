/*
 * ep.h -- C ABI of libep: MoE expert-parallel token dispatch and combine on one
 * B200, with the EP ranks as logical partitions of the GPU's memory.
 *
 * The operation (sources: Ascend CANN page "low_latency_dispatch", sections
 * Function / Formula, Constraints and Example; DeepEP issue #84 "Profiling
 * dispatch_t for low-latency kernel dispatch bandwidth"):
 *
 *   B tokens x[B][d] (bf16) are split over P logical ranks, T = B / P tokens each;
 *   token t belongs to source rank r = t / T.  Each token picks k experts
 *   topk_idx[t][j].  Routed experts are ids [0, E); expert g lives on rank g / L,
 *   L = E / P (DeepEP issue #84, masking experiment).  Ids E .. E+Z-1 are zero
 *   experts, then C copy experts, then K constant experts (Ascend Example:
 *   num_experts = 32 with one zero and one copy expert uses ids 32 and 33).
 *   Id -1 means "not routed" (DeepEP issue #84 masks picks with -1).
 *
 *   ep_layout   counts per expert and per (expert, source rank), their exclusive
 *               prefix, the receive row of every routed pick and the source token
 *               of every receive row.  Low-latency receive layout (layout 0):
 *               row = g * P * M + r * M + slot, i.e. a [E][P*M][d] buffer that
 *               rank q reads as [L][P*M][d] starting at expert q*L.  Packed
 *               layout (layout 1): rows contiguous per expert, then per source
 *               rank, with no padding (the dense expand_x [A][H] of the Ascend
 *               page).  slot is the rank of token t among rank r's tokens that
 *               routed to g, ascending t (the page states the computation is
 *               deterministic).
 *   ep_dispatch quant_mode 0: expand_x row = x[t] (bf16 bits copied).
 *               quant_mode 1 (static; the Formula's non-dynamic case with a mode
 *               other than 0): q = CastToInt8(fp32(x) * smooth_scale) (round half
 *               to even, saturate; no smooth scale = no multiply), no scale sent.
 *               quant_mode 2: xf = fp32(x) * smooth_scale, s = 127 / max|xf| over
 *               the row, q = CastToInt8(xf * s) (round half to even, saturate),
 *               inv = 1 / s; q goes to every receive row of t and inv to
 *               recv_scale of those rows and to token_scale[t]
 *               (Ascend Formula, dynamic quantization scenario).  With a
 *               per-expert smooth scale ([E][d], the scales of shape
 *               [num_experts, h] in the Ascend Example) each routed copy (t, g)
 *               is quantized on its own with xf = fp32(x) * smooth_scale[g]: its
 *               own absmax, q and inv (in recv_scale of its row); token_scale is
 *               then not written.  In quant_mode 1 a per-expert scale gives each
 *               copy CastToInt8(fp32(x) * smooth_scale[g]).
 *   x_active_mask (Ascend Prototype: the optional x_active_mask of
 *               low_latency_dispatch; uint8 [B], nonzero = active, NULL = all
 *               active): an inactive token takes no part, exactly as if each of
 *               its picks were -1: no receive row, not counted in any count
 *               (special experts included), no error bit for its ids, and combine
 *               writes y[t] = +0.  In quant_mode 2 its token_scale is still written.
 *   ep_combine  y[t] = bf16( sum_j w[t][j] * e(t,j) ), fp32 fused multiply-add in
 *               pick order j from 0, rounded once to bf16 (nearest even), where
 *               e(t,j) = expert_out[dst_pos[t][j]] for a routed pick, ori_x[t]
 *               for a copy expert, a1[c] * ori_x[t] + a2[c] * v[c] (fp32) for
 *               constant expert c, and the term is skipped for -1 and zero
 *               experts (Ascend Formula, special expert scenario).
 *
 * Conventions for every entry point:
 *  - All device pointers are owned by the caller (e.g. torch tensors).  The
 *    library never allocates or frees device memory; ep_buffer_create allocates
 *    one small host struct.
 *  - bf16 values travel as their uint16_t bit patterns.  Arrays are dense,
 *    row-major, with the shapes given below.  Pointers to bf16/int8 row data
 *    must be 16-byte aligned (d % 16 == 0 keeps every row aligned).
 *  - Launching calls are asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and return after the launch.  Host-side validation
 *    failures return a negative status and launch nothing.  Bad routing data
 *    found on the device (ids outside [-1, E+Z+C+K), a routed id repeated inside
 *    a token) does not trap: the pick is dropped and a bit is set in the buffer's
 *    device error word, read by ep_buffer_check.
 *  - The device that runs the kernels is the one current on the calling thread
 *    (the CUDA context current when the call is made).
 *  - An ep_buffer is not thread-safe: calls on one buffer must not overlap on the
 *    host, and its kernels must be ordered on one stream (each call reuses the
 *    buffer's arrays and the routing of its latest layout).  Different buffers
 *    are independent.
 *  - Entry points make no device allocation and, apart from ep_buffer_create and
 *    ep_buffer_check, no synchronizing call, so they can be captured into CUDA
 *    graphs (make one eager call of each per device first: the first launch of a
 *    kernel sets its shared-memory opt-in).
 */
#ifndef EP_H
#define EP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols keep default visibility even when the library is built with
 * -fvisibility=hidden. */
#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* ep_stream_t;

/* Status codes. */
#define EP_OK 0
#define EP_ERR_INVALID_ARG (-1) /* null or misaligned pointer, bad config field */
#define EP_ERR_UNSUPPORTED (-2) /* well-formed but outside what this build supports */
#define EP_ERR_CAPACITY (-3)    /* T > M, or int32 row ids would overflow */
#define EP_ERR_CUDA (-4)        /* a CUDA runtime call or a launch failed */

/* Bits of the device error word. */
#define EP_ERRBIT_BAD_ID 0x1u /* an id < -1 or >= E+Z+C+K: that pick was dropped */
#define EP_ERRBIT_DUP_ID 0x2u /* a routed id repeated in one token: later copies dropped */
#define EP_ERRBIT_ROW_RANGE 0x4u /* a dst_pos outside [-1, E*P*M) reached dispatch or
                                    combine (e.g. no ep_layout ran): that pick was skipped */
#define EP_ERRBIT_CHECKED 0x8u /* checked build only (libep_checked.so, -DEP_CHECKED): a
                                   row or offset a kernel computed fell outside the array it
                                   indexes; that access was skipped.  Never set by libep.so. */

/*
 * Problem description.  Constraints checked by ep_buffer_size/ep_buffer_create:
 *   B >= 0, P >= 1, B % P == 0, E >= 1, E % P == 0 (Ascend Example: num_experts must
 *   be a multiple of the MoE rank count), E <= 2048 (Constraints:
 *   local_expert_num * ep_world_size <= 2048), 1 <= k <= 16 (Constraints:
 *   0 < K <= 16), T = B / P <= M, Z, C, K >= 0 with Z + C + K <= 2048,
 *   E*P*M < 2^31 (int32 row ids), 16 <= d <= 32768 with d % 16 == 0,
 *   quant_mode in {0, 1, 2}, smooth_rows in {0, 1, E} (E > 1 needs quant_mode 1 or 2),
 *   layout in {0, 1}.  The T <= M
 *   and E*P*M bounds apply to layout 0; layout 1 needs E*B < 2^31 and
 *   E*P <= 24576.
 */
typedef struct {
    int32_t B;           /* tokens over all logical ranks */
    int32_t d;           /* hidden size */
    int32_t k;           /* picks per token */
    int32_t P;           /* logical EP ranks */
    int32_t M;           /* max tokens per rank (rows per (expert, source rank)) */
    int32_t E;           /* routed experts */
    int32_t n_zero;      /* zero experts  (ids E .. E+Z-1) */
    int32_t n_copy;      /* copy experts  (next C ids) */
    int32_t n_const;     /* constant experts (next K ids) */
    int32_t quant_mode;  /* 0: bf16 pass-through; 1: static int8; 2: dynamic per-token int8 */
    int32_t smooth_rows; /* 0: no smooth scale; 1: one fp32 [d] vector may be given;
                            E: one fp32 [d] row per routed expert ([E][d]) may be given */
    int32_t layout;      /* 0: low-latency [E][P*M][d] receive layout;
                            1: packed [B*k][d]: the rows of expert g start at
                               expert_offset[g], those of source rank r after the
                               lower ranks' (expert_offset[g] + sum_{r'<r}
                               recv_count[g][r'] + slot); rank q reads rows
                               [expert_offset[q*L], expert_offset[(q+1)*L]).
                               M is not used. */
} ep_config;

/* Byte sizes of the caller-allocated device arrays (0 = not needed). */
typedef struct {
    size_t expert_count;  /* int32 [E+Z+C+K]    picks per expert id */
    size_t expert_offset; /* int32 [E+Z+C+K+1]  exclusive prefix of expert_count */
    size_t recv_count;    /* int32 [E][P]       rows of expert g from source rank r
                             (per receiving rank q: [L][P] = ep_recv_counts) */
    size_t dst_pos;       /* int32 [B][k]       receive row of each pick, -1 if none */
    size_t recv_src;      /* int32 [rows]       source token of each receive row
                             (the combine's source map); rows past a run's count
                             are not written.  rows = E*P*M (layout 0) or B*k
                             (layout 1; rows past expert_offset[E] unused) */
    size_t recv_x;        /* [rows][d] int8 (quant_mode 1, 2) or bf16 (quant_mode 0) */
    size_t recv_scale;    /* fp32 [rows]        1/s of the row's copy (quant_mode 2) */
    size_t token_scale;   /* fp32 [B]           1/s per token (quant_mode 2; not
                             written with a per-expert smooth scale) */
    size_t workspace;     /* scratch words; zero-filled by ep_buffer_create */
} ep_buffer_sizes;

/* Device pointers matching ep_buffer_sizes (NULL where the size is 0). */
typedef struct {
    int32_t* expert_count;
    int32_t* expert_offset;
    int32_t* recv_count;
    int32_t* dst_pos;
    int32_t* recv_src;
    void* recv_x;
    float* recv_scale;
    float* token_scale;
    void* workspace;
} ep_buffer_ptrs;

typedef struct ep_buffer ep_buffer;

/* Validate `cfg` and report the byte size of every array.  Host only, no CUDA call.
 * Returns EP_OK, EP_ERR_INVALID_ARG, EP_ERR_UNSUPPORTED or EP_ERR_CAPACITY. */
EP_API int ep_buffer_size(const ep_config* cfg, ep_buffer_sizes* out);

/* Wrap caller memory into a buffer object (a host struct; no device allocation).
 * Every pointer whose size is non-zero must be non-NULL and 16-byte aligned.
 * Zero-fills the workspace with a synchronous cudaMemset on the current device.
 * On success *out owns the host struct until ep_buffer_destroy. */
EP_API int ep_buffer_create(const ep_config* cfg, const ep_buffer_ptrs* ptrs, ep_buffer** out);

/* Free the host struct.  Device memory stays with the caller.  NULL is accepted. */
EP_API int ep_buffer_destroy(ep_buffer* buf);

/* Routing layout from topk_idx (int32 [B][k], device) and the optional
 * x_active_mask (uint8 [B], device, or NULL).  Writes expert_count, expert_offset,
 * recv_count, dst_pos and the written rows of recv_src. */
EP_API int ep_layout(ep_buffer* buf, const int32_t* topk_idx, const uint8_t* x_active_mask,
                     ep_stream_t stream);

/* Quantize (quant_mode 2) or pass through (0) x (bf16 [B][d], device) and scatter
 * every routed pick into recv_x (plus recv_scale, token_scale in mode 2), to the
 * receive rows of the latest ep_layout on this buffer.  smooth_scale is an fp32
 * device array of cfg.smooth_rows rows of d ([d], or [E][d] per routed expert) or
 * NULL; it must be NULL when cfg.smooth_rows == 0.  With a per-expert scale the
 * kernel works expert by expert over the receive rows of that ep_layout
 * (recv_count, expert_offset and recv_src), so one must have run on this buffer
 * (else EP_ERR_INVALID_ARG); it starts after the layout kernel has finished.  A
 * receive row whose recv_src is not a token sets EP_ERRBIT_ROW_RANGE and is skipped.
 * In the packed layout with T = B/P <= 256 the kernel derives those rows from the
 * topk_idx (and mask) passed to that ep_layout (which must still hold the same
 * values) and the per-expert counts its first kernel wrote, instead of reading
 * dst_pos, so it can run alongside the layout's second kernel; it finishes only
 * after the layout kernels have.  Call it on the stream of that ep_layout, after it.
 * Ordering: in that packed small-batch form the kernel reads x, the routing and
 * those counts and writes recv_x, recv_scale and token_scale before it waits for the
 * kernel ahead of it on the stream.  That is safe because ep_layout's kernels wait
 * for everything before them first.  So no kernel that is launched with
 * programmatic dependent launch and triggers its dependents early may sit between
 * ep_layout and ep_dispatch on the stream (ordinary launches, copies and event
 * waits may).  In every other form the kernel waits before reading anything.
 * (ep_layout_dispatch overlaps layout and dispatch in the low-latency layout.) */
EP_API int ep_dispatch(ep_buffer* buf, const uint16_t* x, const float* smooth_scale,
                ep_stream_t stream);

/* ep_layout followed by ep_dispatch on the same stream, as one call: same
 * outputs, bit for bit.  When T = B/P <= 128 and k <= 8 both run in a single
 * grid (the layout in its first CTAs, one token's dispatch in each of the
 * others, which derives its receive rows from the routing itself), saving one
 * kernel launch on the critical path; otherwise the two kernels are launched in
 * order.  Arguments as for ep_layout and ep_dispatch. */
EP_API int ep_layout_dispatch(ep_buffer* buf, const int32_t* topk_idx,
                              const uint8_t* x_active_mask, const uint16_t* x,
                              const float* smooth_scale, ep_stream_t stream);

/* Weighted combine into y (bf16 [B][d], device).  expert_out: bf16 [E*P*M][d]
 * receive-layout expert outputs (may alias recv_x when quant_mode is 0);
 * topk_idx int32 [B][k] and topk_weights fp32 [B][k] as given to ep_layout;
 * x_active_mask uint8 [B] or NULL, the mask given to ep_layout (inactive tokens
 * get y = +0);
 * ori_x bf16 [B][d] (required when C + K > 0, else may be NULL);
 * a1, a2, v bf16 [K][d] (required iff K > 0).  Uses the latest layout's dst_pos,
 * or, for T = B/P <= 16 and for T <= 128 on a buffer with a per-expert smooth table
 * (smooth_rows > 1), derives the same rows from topk_idx (which must hold the ids
 * given to that layout) and the layout's counts.
 * y must not overlap any input.
 * Ordering: in that small-batch form the kernel reads topk_idx, topk_weights,
 * x_active_mask and (packed layout) expert_offset and recv_count before it waits for
 * the kernel ahead of it on the stream, and reads expert outputs and writes y only
 * after.  The library's own kernels before it (ep_layout, ep_dispatch) let it start
 * only once those counts are final.  A kernel launched with programmatic dependent
 * launch that triggers its dependents early and writes those inputs or counts must
 * not be the one right before ep_combine on the stream. */
EP_API int ep_combine(ep_buffer* buf, const uint16_t* expert_out, const int32_t* topk_idx,
               const float* topk_weights, const uint8_t* x_active_mask, const uint16_t* ori_x,
               const uint16_t* a1, const uint16_t* a2, const uint16_t* v, uint16_t* y,
               ep_stream_t stream);

/* Layout for callers that cannot allocate device memory.  The pages have no
 * counterpart to this entry point; it exists for this library's users.
 *
 * Same outputs, bit for bit, as ep_layout on the same topk_idx with no
 * x_active_mask (every token active), but without an
 * ep_buffer or a workspace: the caller passes only the inputs and the outputs
 * (device arrays sized as ep_buffer_size reports; cfg is validated the same
 * way).  Meant for callers that cannot allocate a workspace: an engine whose
 * memory pool already owns all of the GPU's memory, code that must not call
 * cudaMalloc because it can synchronize the device and stall other streams, or
 * a plain C host without a tensor library.  This call itself allocates nothing
 * (no cudaMalloc, no cudaFree, no allocating library routine).
 *
 * Its scratch is a 64 KiB array in the library's static device memory, present
 * on every GPU that loads the library until the process exits.  It holds a
 * 256-byte header and, for batches of more than 256 tokens per rank, one int32
 * per (rank, 256-token chunk, expert id): configurations that need more, i.e.
 * P * ceil(T / 256) * (E + Z + C + K) > 16320 with T > 256, are rejected with
 * EP_ERR_CAPACITY.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every call on a device shares the one array, and each call clears the part
 *    it uses on `stream` first.  Calls whose work can overlap on the GPU (other
 *    streams, other host threads) race on it: order them on one stream.
 *  - err_word: device uint32 that receives this call's error bits (EP_ERRBIT_*,
 *    overwritten, not OR-ed); NULL to not report them.
 * Returns EP_OK, a validation status, EP_ERR_CAPACITY or EP_ERR_CUDA. */
EP_API int ep_layout_static_scratch(const ep_config* cfg, const int32_t* topk_idx,
                                    int32_t* expert_count, int32_t* expert_offset,
                                    int32_t* recv_count, int32_t* dst_pos, int32_t* recv_src,
                                    uint32_t* err_word, ep_stream_t stream);

/* Synchronize `stream`, read the device error word into *err_bits and clear it. */
EP_API int ep_buffer_check(ep_buffer* buf, ep_stream_t stream, uint32_t* err_bits);

/*
 * ---------------------------------------------------------------------------
 * Expert parallelism across GPUs: one process per GPU (the wide expert
 * parallelism of the Wide-EP blog (getimpala.ai), sections on wide EP and DBO; the
 * low-latency layout of DeepEP issue #84, where each rank's receive buffer holds
 * [local_experts][ranks * max_tokens][hidden]).
 *
 * Logical rank r is one process.  It holds its own T = B / P tokens (x, topk_idx,
 * topk_weights and x_active_mask of global tokens r*T .. r*T+T-1, indexed locally
 * 0 .. T-1) and receive slab r: the low-latency rows of its experts r*L .. r*L+L-1,
 * [L][P*M][d], slab row = global row - r*L*P*M, where the global row of (expert g,
 * source rank r, slot) is g*P*M + r*M + slot exactly as on one GPU.  A sender
 * therefore places its tokens with no information from other ranks:
 *   ep_shard_layout    its picks' global rows (dst_pos [T][k]) and send_count [E],
 *                      its routed picks per expert: entries q*L .. q*L+L-1 are
 *                      column r of rank q's recv_count [L][P];
 *   (count exchange)   done by the caller, e.g. one all-to-all of send_count;
 *   ep_shard_dispatch  quantizes its tokens (as ep_dispatch) and stores every routed
 *                      copy straight into the owning rank's slab, with the row's
 *                      recv_scale and recv_src (global token index);
 *   ep_shard_combine   reads each routed pick's expert output from the owning
 *                      rank's slab and reduces as ep_combine into y [T][d].
 * The slabs are reached through an ep_shard_table of device addresses: this
 * process's own slab and the peers' slabs mapped into it (CUDA IPC; every access is
 * a plain load or store over NVLink, no bulk or multicast copy), or, on one GPU,
 * P separate allocations.  Between a rank's dispatch and another rank's reads of
 * its slab the caller orders the GPUs (e.g. a collective or a barrier on the
 * stream); the library itself never waits on another rank.
 * Low-latency layout (layout 0) only; smooth_rows 0 or 1; P <= EP_SHARD_MAX_RANKS.
 */
#define EP_SHARD_MAX_RANKS 64

typedef struct {
    int32_t rank;                           /* this process's logical rank, 0 <= rank < P */
    void* recv_x[EP_SHARD_MAX_RANKS];       /* [P] device address of rank q's slab: recv_x rows
                                               [L*P*M][d] (int8, or bf16 in quant_mode 0) for
                                               ep_shard_dispatch; bf16 expert outputs of the same
                                               rows for ep_shard_combine */
    float* recv_scale[EP_SHARD_MAX_RANKS];  /* [P] recv_scale slabs [L*P*M] (quant_mode 2, dispatch) */
    int32_t* recv_src[EP_SHARD_MAX_RANKS];  /* [P] recv_src slabs [L*P*M] (dispatch); NULL = not written */
    int32_t* recv_count[EP_SHARD_MAX_RANKS]; /* [P] rank q's recv_count [L][P] (dispatch, with a
                                               send_count): the count exchange.  ep_shard_dispatch
                                               stores column `rank` of every owner's array, entry
                                               [l][rank] = this rank's picks of q's local expert l.
                                               NULL = that rank's column is not written. */
} ep_shard_table;

/* Bytes of the device workspace of the ep_shard_* calls (one per process; the caller
 * allocates it and zero-fills it once before the first call). */
EP_API int ep_shard_workspace_size(const ep_config* cfg, size_t* bytes);

/* Layout of rank `rank`'s T tokens (topk_idx int32 [T][k], x_active_mask uint8 [T] or
 * NULL): dst_pos int32 [T][k] (global low-latency rows, -1 if not routed) and
 * send_count int32 [E].  Error bits go to the workspace (ep_shard_check). */
EP_API int ep_shard_layout(const ep_config* cfg, int32_t rank, const int32_t* topk_idx,
                           const uint8_t* x_active_mask, int32_t* dst_pos, int32_t* send_count,
                           void* workspace, ep_stream_t stream);

/* Dispatch of rank tab->rank's tokens x (bf16 [T][d]) to the rows dst_pos of its
 * ep_shard_layout, into the slabs of `tab` (recv_x, recv_scale in quant_mode 2, recv_src
 * = rank*T + local token).  token_scale: fp32 [T] (quant_mode 2), else NULL.
 * send_count: the int32 [E] of the same ep_shard_layout, or NULL.  When given, the
 * kernel also performs the count exchange: it stores send_count[q*L + l] into
 * tab->recv_count[q][l*P + rank] for every rank q whose table entry is set (also when
 * T = 0, so an owner never keeps a stale column).  Like the rows, those stores are
 * ordered before another rank's reads by the caller's barrier after this call. */
EP_API int ep_shard_dispatch(const ep_config* cfg, const ep_shard_table* tab, const uint16_t* x,
                             const float* smooth_scale, const int32_t* dst_pos, const int32_t* send_count,
                             float* token_scale, void* workspace, ep_stream_t stream);

/* ep_shard_layout and ep_shard_dispatch of rank tab->rank as one call, with the count
 * exchange (send_count stored into every owner's tab->recv_count column): same
 * outputs.  When T <= 128 and k <= 8 all of it runs in one grid, as ep_layout_dispatch
 * on one GPU: the first CTAs lay out the rank's tokens and store its counts, every
 * other CTA derives one token's global rows from the routing and stores its copies;
 * otherwise the two kernels run in order.  Arguments as for those two calls. */
EP_API int ep_shard_layout_dispatch(const ep_config* cfg, const ep_shard_table* tab, const int32_t* topk_idx,
                                    const uint8_t* x_active_mask, const uint16_t* x,
                                    const float* smooth_scale, int32_t* dst_pos, int32_t* send_count,
                                    float* token_scale, void* workspace, ep_stream_t stream);

/* Combine of rank tab->rank's tokens into y (bf16 [T][d]); tab->recv_x[q] are the bf16
 * expert-output slabs; other arguments as ep_combine, local to this rank. */
EP_API int ep_shard_combine(const ep_config* cfg, const ep_shard_table* tab,
                            const int32_t* topk_idx, const float* topk_weights,
                            const uint8_t* x_active_mask, const int32_t* dst_pos,
                            const uint16_t* ori_x, const uint16_t* a1, const uint16_t* a2,
                            const uint16_t* v, uint16_t* y, void* workspace, ep_stream_t stream);

/* Synchronize `stream`, read the shard workspace's error word into *err_bits, clear it. */
EP_API int ep_shard_check(void* workspace, ep_stream_t stream, uint32_t* err_bits);

/* Static text for a status code. */
EP_API const char* ep_status_str(int status);

#ifdef __cplusplus
}
#endif

#endif /* EP_H */
