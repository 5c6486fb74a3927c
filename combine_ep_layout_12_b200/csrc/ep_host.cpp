// Host side of libep: configuration checks, buffer sizing, the buffer object and
// the exported C entry points declared in include/ep.h.  Every entry point
// validates its arguments before touching CUDA and launches nothing on failure.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <new>

#include "ep.h"
#include "ep_internal.cuh"

struct ep_buffer {
    ep_config cfg;
    ep_buffer_ptrs ptrs;
    ep_buffer_sizes sizes;
    const int32_t* last_topk_idx;  // routing of the latest ep_layout (dispatch may re-read it)
    const uint8_t* last_active;    // its x_active_mask (or null)
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_config(const ep_config* c) {
    if (!c) return EP_ERR_INVALID_ARG;
    if (c->B < 0 || c->P < 1 || c->E < 1 || c->k < 1 || c->M < 0 || c->d < 1)
        return EP_ERR_INVALID_ARG;
    if (c->n_zero < 0 || c->n_copy < 0 || c->n_const < 0) return EP_ERR_INVALID_ARG;
    if (c->B % c->P != 0 || c->E % c->P != 0) return EP_ERR_INVALID_ARG;
    if (c->quant_mode < 0 || c->quant_mode > 2) return EP_ERR_INVALID_ARG;
    if (c->smooth_rows != 0 && c->smooth_rows != 1 && c->smooth_rows != c->E) return EP_ERR_INVALID_ARG;
    if (c->smooth_rows > 1 && c->quant_mode == 0) return EP_ERR_INVALID_ARG;
    if (c->layout != 0 && c->layout != 1) return EP_ERR_UNSUPPORTED;
    if (c->d % 16 != 0) return EP_ERR_INVALID_ARG;
    if (c->k > ep::kMaxK) return EP_ERR_INVALID_ARG;
    if (c->d > ep::kMaxD) return EP_ERR_UNSUPPORTED;
    if (c->E > ep::kMaxE) return EP_ERR_UNSUPPORTED;
    const long long n_special = (long long)c->n_zero + c->n_copy + c->n_const;
    if (n_special > ep::kMaxSpecial) return EP_ERR_UNSUPPORTED;
    if ((long long)c->B * c->k >= (1LL << 31)) return EP_ERR_CAPACITY;
    if (c->layout == 0) {
        if (c->B / c->P > c->M) return EP_ERR_CAPACITY;
        if ((long long)c->E * c->P * c->M >= (1LL << 31)) return EP_ERR_CAPACITY;
    } else {
        // packed rows are derived from low-latency-form rows with stride T
        if ((long long)c->E * c->B >= (1LL << 31)) return EP_ERR_CAPACITY;
        if ((long long)c->E * c->P > ep::kMaxPackedEP) return EP_ERR_UNSUPPORTED;
    }
    return EP_OK;
}

void fill_sizes(const ep_config* c, ep_buffer_sizes* s) {
    const size_t E_tot = (size_t)c->E + c->n_zero + c->n_copy + c->n_const;
    const size_t n_special = (size_t)c->n_zero + c->n_copy + c->n_const;
    const size_t rows = (size_t)ep::make_shape(*c).rows;
    const size_t esz = c->quant_mode != 0 ? 1 : 2;
    s->expert_count = 4 * E_tot;
    s->expert_offset = 4 * (E_tot + 1);
    s->recv_count = 4 * (size_t)c->E * c->P;
    s->dst_pos = 4 * (size_t)c->B * c->k;
    s->recv_src = 4 * rows;
    s->recv_x = rows * (size_t)c->d * esz;
    s->recv_scale = c->quant_mode == 2 ? 4 * rows : 0;
    s->token_scale = c->quant_mode == 2 ? 4 * (size_t)c->B : 0;
    (void)n_special;
    s->workspace = ep::workspace_bytes(ep::make_shape(*c));
}

bool ptr_ok(const void* p, size_t size) { return size == 0 || (p != nullptr && aligned16(p)); }

}  // namespace

extern "C" {

int ep_buffer_size(const ep_config* cfg, ep_buffer_sizes* out) {
    if (!out) return EP_ERR_INVALID_ARG;
    const int st = check_config(cfg);
    if (st != EP_OK) return st;
    fill_sizes(cfg, out);
    return EP_OK;
}

int ep_buffer_create(const ep_config* cfg, const ep_buffer_ptrs* ptrs, ep_buffer** out) {
    if (!out || !ptrs) return EP_ERR_INVALID_ARG;
    *out = nullptr;
    const int st = check_config(cfg);
    if (st != EP_OK) return st;
    ep_buffer_sizes s;
    fill_sizes(cfg, &s);
    if (!ptr_ok(ptrs->expert_count, s.expert_count) || !ptr_ok(ptrs->expert_offset, s.expert_offset) ||
        !ptr_ok(ptrs->recv_count, s.recv_count) || !ptr_ok(ptrs->dst_pos, s.dst_pos) ||
        !ptr_ok(ptrs->recv_src, s.recv_src) || !ptr_ok(ptrs->recv_x, s.recv_x) ||
        !ptr_ok(ptrs->recv_scale, s.recv_scale) || !ptr_ok(ptrs->token_scale, s.token_scale) ||
        !ptr_ok(ptrs->workspace, s.workspace))
        return EP_ERR_INVALID_ARG;
    if (cudaMemset(ptrs->workspace, 0, s.workspace) != cudaSuccess) return EP_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return EP_ERR_CUDA;
    ep_buffer* b = new (std::nothrow) ep_buffer;
    if (!b) return EP_ERR_INVALID_ARG;
    b->cfg = *cfg;
    b->ptrs = *ptrs;
    b->sizes = s;
    b->last_topk_idx = nullptr;
    b->last_active = nullptr;
    *out = b;
    return EP_OK;
}

int ep_buffer_destroy(ep_buffer* buf) {
    delete buf;
    return EP_OK;
}

int ep_layout(ep_buffer* buf, const int32_t* topk_idx, const uint8_t* x_active_mask,
              ep_stream_t stream) {
    if (!buf) return EP_ERR_INVALID_ARG;
    if (buf->cfg.B > 0 && (!topk_idx || !aligned4(topk_idx))) return EP_ERR_INVALID_ARG;
    const int st = ep::launch_layout(ep::make_shape(buf->cfg), buf->ptrs, topk_idx, x_active_mask,
                                     reinterpret_cast<cudaStream_t>(stream));
    buf->last_topk_idx = st == EP_OK ? topk_idx : nullptr;
    buf->last_active = st == EP_OK ? x_active_mask : nullptr;
    return st;
}

int ep_dispatch(ep_buffer* buf, const uint16_t* x, const float* smooth_scale, ep_stream_t stream) {
    if (!buf) return EP_ERR_INVALID_ARG;
    const ep_config& c = buf->cfg;
    if (c.B > 0 && (!x || !aligned16(x))) return EP_ERR_INVALID_ARG;
    if (smooth_scale && (c.smooth_rows == 0 || !aligned16(smooth_scale))) return EP_ERR_INVALID_ARG;
    if (smooth_scale && c.quant_mode == 0) return EP_ERR_INVALID_ARG;
    if (smooth_scale && c.smooth_rows > 1 && c.B > 0 && !buf->last_topk_idx) return EP_ERR_INVALID_ARG;
    return ep::launch_dispatch(ep::make_shape(c), buf->ptrs, x, smooth_scale, buf->last_topk_idx,
                               buf->last_active, reinterpret_cast<cudaStream_t>(stream));
}

int ep_layout_dispatch(ep_buffer* buf, const int32_t* topk_idx, const uint8_t* x_active_mask,
                       const uint16_t* x, const float* smooth_scale, ep_stream_t stream) {
    if (!buf) return EP_ERR_INVALID_ARG;
    const ep_config& c = buf->cfg;
    if (c.B > 0 && (!topk_idx || !aligned4(topk_idx))) return EP_ERR_INVALID_ARG;
    if (c.B > 0 && (!x || !aligned16(x))) return EP_ERR_INVALID_ARG;
    if (smooth_scale && (c.smooth_rows == 0 || !aligned16(smooth_scale))) return EP_ERR_INVALID_ARG;
    if (smooth_scale && c.quant_mode == 0) return EP_ERR_INVALID_ARG;
    const int st = ep::launch_layout_dispatch(ep::make_shape(c), buf->ptrs, topk_idx, x_active_mask,
                                              x, smooth_scale, reinterpret_cast<cudaStream_t>(stream));
    buf->last_topk_idx = st == EP_OK ? topk_idx : nullptr;
    buf->last_active = st == EP_OK ? x_active_mask : nullptr;
    return st;
}

int ep_combine(ep_buffer* buf, const uint16_t* expert_out, const int32_t* topk_idx,
               const float* topk_weights, const uint8_t* x_active_mask, const uint16_t* ori_x,
               const uint16_t* a1, const uint16_t* a2, const uint16_t* v, uint16_t* y,
               ep_stream_t stream) {
    if (!buf) return EP_ERR_INVALID_ARG;
    const ep_config& c = buf->cfg;
    if (c.B > 0) {
        if (!expert_out || !aligned16(expert_out)) return EP_ERR_INVALID_ARG;
        if (!topk_idx || !aligned4(topk_idx) || !topk_weights || !aligned4(topk_weights))
            return EP_ERR_INVALID_ARG;
        if (!y || !aligned16(y)) return EP_ERR_INVALID_ARG;
        if (c.n_copy + c.n_const > 0 && (!ori_x || !aligned16(ori_x))) return EP_ERR_INVALID_ARG;
        if (c.n_const > 0 && (!a1 || !a2 || !v || !aligned16(a1) || !aligned16(a2) || !aligned16(v)))
            return EP_ERR_INVALID_ARG;
        if (y == ori_x || y == expert_out) return EP_ERR_INVALID_ARG;
    }
    return ep::launch_combine(ep::make_shape(c), buf->ptrs, expert_out, topk_idx, topk_weights,
                              x_active_mask, ori_x, a1, a2, v, y,
                              reinterpret_cast<cudaStream_t>(stream));
}

int ep_buffer_check(ep_buffer* buf, ep_stream_t stream, uint32_t* err_bits) {
    if (!buf || !err_bits) return EP_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    auto* hdr = reinterpret_cast<ep::WsHeader*>(buf->ptrs.workspace);
    unsigned host = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return EP_ERR_CUDA;
    if (cudaMemcpy(&host, &hdr->err, sizeof host, cudaMemcpyDeviceToHost) != cudaSuccess)
        return EP_ERR_CUDA;
    if (cudaMemset(&hdr->err, 0, sizeof host) != cudaSuccess) return EP_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return EP_ERR_CUDA;
    *err_bits = host;
    return EP_OK;
}

// ---------------------------------------------------------------------------
// Multi-GPU forms (one process per logical rank).
// ---------------------------------------------------------------------------
namespace {

// Shard workspace: the layout workspace of this rank's tokens laid out as a one-rank
// problem (header and, above 256 tokens, the chunk counts), then the layout's
// expert_count [E_tot] and expert_offset [E_tot + 1] scratch.
struct ShardWs {
    size_t layout_bytes, count_off, offset_off, total;
};

int shard_local(const ep_config* cfg, ep::Shape* ls, ShardWs* ws) {
    const int st = check_config(cfg);
    if (st != EP_OK) return st;
    if (cfg->layout != 0 || cfg->smooth_rows > 1 || cfg->P > EP_SHARD_MAX_RANKS) return EP_ERR_UNSUPPORTED;
    ep::Shape s = ep::make_shape(*cfg);  // global rows E * P * M
    s.B = s.T;                           // this rank's tokens
    s.P = 1;                             // laid out as a one-rank problem (global rows via gstride)
    *ls = s;
    ws->layout_bytes = ep::workspace_bytes(s);
    ws->count_off = ws->layout_bytes;
    ws->offset_off = ws->count_off + 4 * (size_t)s.E_tot;
    ws->total = (ws->offset_off + 4 * ((size_t)s.E_tot + 1) + 255) & ~(size_t)255;
    return EP_OK;
}

int shard_table(const ep_config* cfg, const ep_shard_table* tab, bool combine, ep::ShardTable* out) {
    if (!tab || tab->rank < 0 || tab->rank >= cfg->P) return EP_ERR_INVALID_ARG;
    for (int q = 0; q < cfg->P; ++q) {
        if (!tab->recv_x[q] || !aligned16(tab->recv_x[q])) return EP_ERR_INVALID_ARG;
        if (!combine && cfg->quant_mode == 2 && (!tab->recv_scale[q] || !aligned4(tab->recv_scale[q])))
            return EP_ERR_INVALID_ARG;
        if (!combine && tab->recv_src[q] && !aligned4(tab->recv_src[q])) return EP_ERR_INVALID_ARG;
        if (!combine && tab->recv_count[q] && !aligned4(tab->recv_count[q])) return EP_ERR_INVALID_ARG;
        out->x[q] = tab->recv_x[q];
        out->scale[q] = combine ? nullptr : tab->recv_scale[q];
        out->src[q] = combine ? nullptr : tab->recv_src[q];
        out->count[q] = combine ? nullptr : tab->recv_count[q];
    }
    for (int q = cfg->P; q < EP_SHARD_MAX_RANKS; ++q) {
        out->x[q] = nullptr;
        out->scale[q] = nullptr;
        out->src[q] = nullptr;
        out->count[q] = nullptr;
    }
    out->send_count = nullptr;
    out->slab_rows = (long long)(cfg->E / cfg->P) * cfg->P * cfg->M;
    out->token_base = tab->rank * (cfg->B / cfg->P);
    out->rank = tab->rank;
    out->P = cfg->P;
    out->L = cfg->E / cfg->P;
    return EP_OK;
}

}  // namespace

int ep_shard_workspace_size(const ep_config* cfg, size_t* bytes) {
    if (!bytes) return EP_ERR_INVALID_ARG;
    ep::Shape ls;
    ShardWs ws;
    const int st = shard_local(cfg, &ls, &ws);
    if (st != EP_OK) return st;
    *bytes = ws.total;
    return EP_OK;
}

int ep_shard_layout(const ep_config* cfg, int32_t rank, const int32_t* topk_idx,
                    const uint8_t* x_active_mask, int32_t* dst_pos, int32_t* send_count,
                    void* workspace, ep_stream_t stream) {
    ep::Shape ls;
    ShardWs ws;
    const int st = shard_local(cfg, &ls, &ws);
    if (st != EP_OK) return st;
    if (rank < 0 || rank >= cfg->P) return EP_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace) || !send_count || !aligned4(send_count)) return EP_ERR_INVALID_ARG;
    if (ls.B > 0 && (!topk_idx || !aligned4(topk_idx) || !dst_pos || !aligned4(dst_pos)))
        return EP_ERR_INVALID_ARG;
    ep_buffer_ptrs p = {};
    char* w = static_cast<char*>(workspace);
    p.expert_count = reinterpret_cast<int32_t*>(w + ws.count_off);
    p.expert_offset = reinterpret_cast<int32_t*>(w + ws.offset_off);
    p.recv_count = send_count;  // [E][1]: this rank's column
    p.dst_pos = dst_pos;
    p.recv_src = nullptr;       // written by the dispatch, into the owners' slabs
    p.workspace = workspace;
    return ep::launch_layout(ls, p, topk_idx, x_active_mask, reinterpret_cast<cudaStream_t>(stream),
                             cfg->P * cfg->M, rank * cfg->M);
}

int ep_shard_dispatch(const ep_config* cfg, const ep_shard_table* tab, const uint16_t* x,
                      const float* smooth_scale, const int32_t* dst_pos, const int32_t* send_count,
                      float* token_scale, void* workspace, ep_stream_t stream) {
    ep::Shape ls;
    ShardWs ws;
    int st = shard_local(cfg, &ls, &ws);
    if (st != EP_OK) return st;
    ep::ShardTable t;
    st = shard_table(cfg, tab, false, &t);
    if (st != EP_OK) return st;
    if (!workspace || !aligned16(workspace)) return EP_ERR_INVALID_ARG;
    if (ls.B > 0 && (!x || !aligned16(x) || !dst_pos || !aligned4(dst_pos))) return EP_ERR_INVALID_ARG;
    if (ls.B > 0 && cfg->quant_mode == 2 && (!token_scale || !aligned4(token_scale))) return EP_ERR_INVALID_ARG;
    if (smooth_scale && (cfg->smooth_rows == 0 || cfg->quant_mode == 0 || !aligned16(smooth_scale)))
        return EP_ERR_INVALID_ARG;
    if (send_count && !aligned4(send_count)) return EP_ERR_INVALID_ARG;
    t.send_count = send_count;
    ep_buffer_ptrs p = {};
    p.dst_pos = const_cast<int32_t*>(dst_pos);
    p.token_scale = token_scale;
    p.workspace = workspace;
    return ep::launch_shard_dispatch(ls, p, x, smooth_scale, t, reinterpret_cast<cudaStream_t>(stream));
}

int ep_shard_layout_dispatch(const ep_config* cfg, const ep_shard_table* tab, const int32_t* topk_idx,
                             const uint8_t* x_active_mask, const uint16_t* x, const float* smooth_scale,
                             int32_t* dst_pos, int32_t* send_count, float* token_scale, void* workspace,
                             ep_stream_t stream) {
    ep::Shape ls;
    ShardWs ws;
    int st = shard_local(cfg, &ls, &ws);
    if (st != EP_OK) return st;
    ep::ShardTable t;
    st = shard_table(cfg, tab, false, &t);
    if (st != EP_OK) return st;
    if (!workspace || !aligned16(workspace) || !send_count || !aligned4(send_count)) return EP_ERR_INVALID_ARG;
    if (ls.B > 0 && (!topk_idx || !aligned4(topk_idx) || !dst_pos || !aligned4(dst_pos) || !x || !aligned16(x)))
        return EP_ERR_INVALID_ARG;
    if (ls.B > 0 && cfg->quant_mode == 2 && (!token_scale || !aligned4(token_scale))) return EP_ERR_INVALID_ARG;
    if (smooth_scale && (cfg->smooth_rows == 0 || cfg->quant_mode == 0 || !aligned16(smooth_scale)))
        return EP_ERR_INVALID_ARG;
    ep_buffer_ptrs p = {};
    char* w = static_cast<char*>(workspace);
    p.expert_count = reinterpret_cast<int32_t*>(w + ws.count_off);
    p.expert_offset = reinterpret_cast<int32_t*>(w + ws.offset_off);
    p.recv_count = send_count;  // [E][1]: this rank's column
    p.dst_pos = dst_pos;
    p.recv_src = nullptr;       // written by the dispatch, into the owners' slabs
    p.token_scale = token_scale;
    p.workspace = workspace;
    return ep::launch_shard_layout_dispatch(ls, p, topk_idx, x_active_mask, x, smooth_scale, t, cfg->P * cfg->M,
                                            tab->rank * cfg->M, reinterpret_cast<cudaStream_t>(stream));
}

int ep_shard_combine(const ep_config* cfg, const ep_shard_table* tab, const int32_t* topk_idx,
                     const float* topk_weights, const uint8_t* x_active_mask, const int32_t* dst_pos,
                     const uint16_t* ori_x, const uint16_t* a1, const uint16_t* a2, const uint16_t* v,
                     uint16_t* y, void* workspace, ep_stream_t stream) {
    ep::Shape ls;
    ShardWs ws;
    int st = shard_local(cfg, &ls, &ws);
    if (st != EP_OK) return st;
    ep::ShardTable t;
    st = shard_table(cfg, tab, true, &t);
    if (st != EP_OK) return st;
    if (!workspace || !aligned16(workspace)) return EP_ERR_INVALID_ARG;
    if (ls.B > 0) {
        if (!topk_idx || !aligned4(topk_idx) || !topk_weights || !aligned4(topk_weights) || !dst_pos ||
            !aligned4(dst_pos))
            return EP_ERR_INVALID_ARG;
        if (!y || !aligned16(y)) return EP_ERR_INVALID_ARG;
        if (cfg->n_copy + cfg->n_const > 0 && (!ori_x || !aligned16(ori_x))) return EP_ERR_INVALID_ARG;
        if (cfg->n_const > 0 && (!a1 || !a2 || !v || !aligned16(a1) || !aligned16(a2) || !aligned16(v)))
            return EP_ERR_INVALID_ARG;
        if (y == ori_x) return EP_ERR_INVALID_ARG;
    }
    ep_buffer_ptrs p = {};
    p.dst_pos = const_cast<int32_t*>(dst_pos);
    p.workspace = workspace;
    return ep::launch_shard_combine(ls, p, topk_idx, topk_weights, x_active_mask, ori_x, a1, a2, v, y, t,
                                    reinterpret_cast<cudaStream_t>(stream));
}

int ep_shard_check(void* workspace, ep_stream_t stream, uint32_t* err_bits) {
    if (!workspace || !err_bits) return EP_ERR_INVALID_ARG;
    auto* hdr = reinterpret_cast<ep::WsHeader*>(workspace);
    unsigned host = 0;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return EP_ERR_CUDA;
    if (cudaMemcpy(&host, &hdr->err, sizeof host, cudaMemcpyDeviceToHost) != cudaSuccess) return EP_ERR_CUDA;
    if (cudaMemset(&hdr->err, 0, sizeof host) != cudaSuccess) return EP_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return EP_ERR_CUDA;
    *err_bits = host;
    return EP_OK;
}

const char* ep_status_str(int status) {
    switch (status) {
        case EP_OK: return "ok";
        case EP_ERR_INVALID_ARG: return "invalid argument";
        case EP_ERR_UNSUPPORTED: return "unsupported configuration";
        case EP_ERR_CAPACITY: return "capacity exceeded (T > M or row ids overflow int32)";
        case EP_ERR_CUDA: return "CUDA error";
        default: return "unknown status";
    }
}

}  // extern "C"
