"""ctypes binding of libep.so: the C ABI of include/ep.h, one Python function per
entry point with the same name.  Argument marshalling only; every step of the
path runs in the library's CUDA kernels.  Pointers are passed as Python ints
(device addresses); streams as cudaStream_t handles (ints, 0 = default stream).
"""
import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libep.so")

EP_OK = 0
EP_ERR_INVALID_ARG = -1
EP_ERR_UNSUPPORTED = -2
EP_ERR_CAPACITY = -3
EP_ERR_CUDA = -4

ERRBIT_BAD_ID = 0x1
ERRBIT_DUP_ID = 0x2
ERRBIT_ROW_RANGE = 0x4

_CONFIG_FIELDS = ("B", "d", "k", "P", "M", "E", "n_zero", "n_copy", "n_const", "quant_mode",
                  "smooth_rows", "layout")
BUFFER_FIELDS = ("expert_count", "expert_offset", "recv_count", "dst_pos", "recv_src", "recv_x",
                 "recv_scale", "token_scale", "workspace")


class ep_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in _CONFIG_FIELDS]


class ep_buffer_sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in BUFFER_FIELDS]


class ep_buffer_ptrs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in BUFFER_FIELDS]


SHARD_MAX_RANKS = 64


class ep_shard_table(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_int32),
                ("recv_x", ctypes.c_void_p * SHARD_MAX_RANKS),
                ("recv_scale", ctypes.c_void_p * SHARD_MAX_RANKS),
                ("recv_src", ctypes.c_void_p * SHARD_MAX_RANKS),
                ("recv_count", ctypes.c_void_p * SHARD_MAX_RANKS)]


def make_shard_table(rank, recv_x, recv_scale=None, recv_src=None, recv_count=None):
    """ep_shard_table from per-rank device addresses (lists of ints; None entries or
    lists mean NULL)."""
    t = ep_shard_table()
    t.rank = int(rank)
    for name, vals in (("recv_x", recv_x), ("recv_scale", recv_scale), ("recv_src", recv_src),
                       ("recv_count", recv_count)):
        if vals is None:
            continue
        if len(vals) > SHARD_MAX_RANKS:
            raise ValueError("at most %d ranks" % SHARD_MAX_RANKS)
        arr = getattr(t, name)
        for q, v in enumerate(vals):
            arr[q] = v
    return t


class EPError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (where, ep_status_str(status), status))


LIB_CHECKED_PATH = os.path.join(_PKG, "libep_checked.so")
ERRBIT_CHECKED = 0x8

_libs = {}
_use_checked = False


def use_checked(flag=True):
    """Route every following call to libep_checked.so (flag True) or libep.so.
    A buffer must be used with the library that created it."""
    global _use_checked
    _use_checked = bool(flag)


def lib():
    """The loaded libep.so (or libep_checked.so after use_checked()).  Raises if the
    library has not been built: there is no fallback implementation."""
    path = LIB_CHECKED_PATH if _use_checked else LIB_PATH
    L = _libs.get(path)
    if L is not None:
        return L
    if not os.path.exists(path):
        raise RuntimeError("%s is missing; build it with "
                           "`python -m combine_ep_layout_12_b200.build`" % path)
    L = _load(path)
    _libs[path] = L
    return L


def _load(path):
    L = ctypes.CDLL(path)
    vp, i = ctypes.c_void_p, ctypes.c_int
    L.ep_buffer_size.argtypes = [ctypes.POINTER(ep_config), ctypes.POINTER(ep_buffer_sizes)]
    L.ep_buffer_create.argtypes = [ctypes.POINTER(ep_config), ctypes.POINTER(ep_buffer_ptrs),
                                   ctypes.POINTER(vp)]
    L.ep_buffer_destroy.argtypes = [vp]
    L.ep_layout.argtypes = [vp, vp, vp, vp]
    L.ep_dispatch.argtypes = [vp, vp, vp, vp]
    L.ep_layout_dispatch.argtypes = [vp] * 6
    L.ep_combine.argtypes = [vp] * 11
    L.ep_buffer_check.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    L.ep_layout_static_scratch.argtypes = [ctypes.POINTER(ep_config)] + [vp] * 8
    L.ep_shard_workspace_size.argtypes = [ctypes.POINTER(ep_config), ctypes.POINTER(ctypes.c_size_t)]
    L.ep_shard_layout.argtypes = [ctypes.POINTER(ep_config), ctypes.c_int32] + [vp] * 6
    L.ep_shard_dispatch.argtypes = [ctypes.POINTER(ep_config), ctypes.POINTER(ep_shard_table)] + [vp] * 7
    L.ep_shard_layout_dispatch.argtypes = [ctypes.POINTER(ep_config), ctypes.POINTER(ep_shard_table)] + [vp] * 9
    L.ep_shard_combine.argtypes = [ctypes.POINTER(ep_config), ctypes.POINTER(ep_shard_table)] + [vp] * 11
    L.ep_shard_check.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    for f in (L.ep_buffer_size, L.ep_buffer_create, L.ep_buffer_destroy, L.ep_layout,
              L.ep_dispatch, L.ep_layout_dispatch, L.ep_combine, L.ep_buffer_check,
              L.ep_layout_static_scratch, L.ep_shard_workspace_size, L.ep_shard_layout,
              L.ep_shard_dispatch, L.ep_shard_layout_dispatch, L.ep_shard_combine, L.ep_shard_check):
        f.restype = i
    L.ep_status_str.argtypes = [i]
    L.ep_status_str.restype = ctypes.c_char_p
    return L


def make_config(B, d, k, P, M, E, n_zero=0, n_copy=0, n_const=0, quant_mode=0, smooth_rows=0,
                layout=0):
    return ep_config(B, d, k, P, M, E, n_zero, n_copy, n_const, quant_mode, smooth_rows, layout)


def _check(status, where):
    if status != EP_OK:
        raise EPError(status, where)


def ep_status_str(status):
    return lib().ep_status_str(int(status)).decode()


def ep_buffer_size(cfg):
    out = ep_buffer_sizes()
    _check(lib().ep_buffer_size(ctypes.byref(cfg), ctypes.byref(out)), "ep_buffer_size")
    return out


def ep_buffer_create(cfg, ptrs):
    h = ctypes.c_void_p()
    _check(lib().ep_buffer_create(ctypes.byref(cfg), ctypes.byref(ptrs), ctypes.byref(h)),
           "ep_buffer_create")
    return h


def ep_buffer_destroy(handle):
    _check(lib().ep_buffer_destroy(handle), "ep_buffer_destroy")


def ep_layout(handle, topk_idx, x_active_mask=None, stream=0):
    _check(lib().ep_layout(handle, topk_idx, x_active_mask, stream), "ep_layout")


def ep_dispatch(handle, x, smooth_scale=None, stream=0):
    _check(lib().ep_dispatch(handle, x, smooth_scale, stream), "ep_dispatch")


def ep_layout_dispatch(handle, topk_idx, x_active_mask, x, smooth_scale=None, stream=0):
    _check(lib().ep_layout_dispatch(handle, topk_idx, x_active_mask, x, smooth_scale, stream),
           "ep_layout_dispatch")


def ep_combine(handle, expert_out, topk_idx, topk_weights, x_active_mask, ori_x, a1, a2, v, y,
               stream=0):
    _check(lib().ep_combine(handle, expert_out, topk_idx, topk_weights, x_active_mask, ori_x, a1,
                            a2, v, y, stream), "ep_combine")


def ep_buffer_check(handle, stream=0):
    bits = ctypes.c_uint32()
    _check(lib().ep_buffer_check(handle, stream, ctypes.byref(bits)), "ep_buffer_check")
    return int(bits.value)


def ep_layout_static_scratch(cfg, topk_idx, expert_count, expert_offset, recv_count, dst_pos,
                             recv_src, err_word=None, stream=0):
    """Layout without a caller workspace (scratch in the library's static device
    memory); for callers that cannot allocate.  All arguments after cfg are device
    addresses (ints); err_word may be None."""
    _check(lib().ep_layout_static_scratch(ctypes.byref(cfg), topk_idx, expert_count,
                                          expert_offset, recv_count, dst_pos, recv_src,
                                          err_word, stream), "ep_layout_static_scratch")


def ep_shard_workspace_size(cfg):
    n = ctypes.c_size_t()
    _check(lib().ep_shard_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "ep_shard_workspace_size")
    return int(n.value)


def ep_shard_layout(cfg, rank, topk_idx, x_active_mask, dst_pos, send_count, workspace, stream=0):
    _check(lib().ep_shard_layout(ctypes.byref(cfg), int(rank), topk_idx, x_active_mask, dst_pos,
                                 send_count, workspace, stream), "ep_shard_layout")


def ep_shard_dispatch(cfg, table, x, smooth_scale, dst_pos, send_count, token_scale, workspace, stream=0):
    _check(lib().ep_shard_dispatch(ctypes.byref(cfg), ctypes.byref(table), x, smooth_scale, dst_pos,
                                   send_count, token_scale, workspace, stream), "ep_shard_dispatch")


def ep_shard_layout_dispatch(cfg, table, topk_idx, x_active_mask, x, smooth_scale, dst_pos, send_count,
                             token_scale, workspace, stream=0):
    _check(lib().ep_shard_layout_dispatch(ctypes.byref(cfg), ctypes.byref(table), topk_idx, x_active_mask, x,
                                          smooth_scale, dst_pos, send_count, token_scale, workspace, stream),
           "ep_shard_layout_dispatch")


def ep_shard_combine(cfg, table, topk_idx, topk_weights, x_active_mask, dst_pos, ori_x, a1, a2, v, y,
                     workspace, stream=0):
    _check(lib().ep_shard_combine(ctypes.byref(cfg), ctypes.byref(table), topk_idx, topk_weights,
                                  x_active_mask, dst_pos, ori_x, a1, a2, v, y, workspace, stream),
           "ep_shard_combine")


def ep_shard_check(workspace, stream=0):
    bits = ctypes.c_uint32()
    _check(lib().ep_shard_check(workspace, stream, ctypes.byref(bits)), "ep_shard_check")
    return int(bits.value)
