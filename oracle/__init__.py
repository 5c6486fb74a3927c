"""ctypes front end of the CPU oracle (ep_oracle.c).

TEST INFRASTRUCTURE ONLY.  Imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg; the product library (combine_ep_layout_12_b200)
never imports it, and it imports nothing from the product.

bf16 arrays are numpy uint16 bit patterns; int8 payloads are numpy int8.
Every function allocates its outputs with numpy and returns them.
"""
import ctypes
import os

import numpy as np

from . import build as _build

ERR_BAD_ID = 0x1
ERR_DUP_ID = 0x2


class OrcCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "B", "d", "k", "P", "M", "E", "n_zero", "n_copy", "n_const", "quant_mode", "layout")]


_lib = None
_lib_path = None


def load(path=None):
    """Load (building first if needed) the oracle library; `path` selects another build."""
    global _lib, _lib_path
    if path is None:
        if _lib is not None and _lib_path == _build.LIB:
            return _lib
        path = _build.build()
    lib = ctypes.CDLL(os.path.abspath(path))
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    lib.orc_layout.argtypes = [P] * 8
    lib.orc_quantize.argtypes = [P] * 5
    lib.orc_dispatch.argtypes = [P, P, P, P, P, P, i64]
    lib.orc_combine.argtypes = [P, P, i64, P, P, P, P, P, P, P, P]
    for f in (lib.orc_layout, lib.orc_quantize, lib.orc_dispatch, lib.orc_combine):
        f.restype = ctypes.c_int
    lib.orc_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.orc_f32_to_bf16.restype = ctypes.c_uint16
    lib.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.orc_bf16_to_f32.restype = ctypes.c_float
    lib.orc_f32_to_bf16_n.argtypes = [P, P, i64]
    lib.orc_f32_to_bf16_n.restype = None
    lib.orc_receive_rows.argtypes = [P]
    lib.orc_receive_rows.restype = i64
    lib.orc_dispatch_expert_smooth.argtypes = [P, P, P, P, P, P, P, i64]
    lib.orc_dispatch_expert_smooth.restype = ctypes.c_int
    lib.orc_layout_active.argtypes = [P] * 9
    lib.orc_layout_active.restype = ctypes.c_int
    lib.orc_combine_active.argtypes = [P, P, i64, P, P, P, P, P, P, P, P, P]
    lib.orc_combine_active.restype = ctypes.c_int
    if path == _build.LIB or os.path.abspath(path) == os.path.abspath(_build.LIB):
        _lib, _lib_path = lib, _build.LIB
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def make_cfg(B, d, k, P, M, E, n_zero=0, n_copy=0, n_const=0, quant_mode=0, layout=0):
    """layout 0: low-latency receive rows (E*P*M); 1: packed rows (B*k)."""
    return OrcCfg(B, d, k, P, M, E, n_zero, n_copy, n_const, quant_mode, layout)


def receive_rows(cfg, lib=None):
    lib = lib or load()
    n = int(lib.orc_receive_rows(ctypes.byref(cfg)))
    if n < 0:
        raise ValueError("oracle rejected the configuration")
    return n


def _check(rc, name):
    if rc != 0:
        raise ValueError("oracle %s rejected its arguments (status %d)" % (name, rc))


def layout(cfg, topk_idx, lib=None, active=None):
    """Returns dict(expert_count, expert_offset, recv_count [E,P], dst_pos [B,k],
    recv_src [rows], err); rows = E*P*M (low-latency) or B*k (packed).
    active: optional [B] x_active_mask (nonzero = active)."""
    lib = lib or load()
    E_tot = cfg.E + cfg.n_zero + cfg.n_copy + cfg.n_const
    idx = _c(topk_idx, np.int32)
    out = dict(
        expert_count=np.zeros(E_tot, np.int32),
        expert_offset=np.zeros(E_tot + 1, np.int32),
        recv_count=np.zeros((cfg.E, cfg.P), np.int32),
        dst_pos=np.zeros((cfg.B, cfg.k), np.int32),
        recv_src=np.zeros(receive_rows(cfg, lib), np.int32),
    )
    err = np.zeros(1, np.uint32)
    act = None if active is None else (np.asarray(active) != 0).astype(np.uint8)
    rc = lib.orc_layout_active(ctypes.byref(cfg), _ptr(idx), _ptr(act), _ptr(out["expert_count"]),
                               _ptr(out["expert_offset"]), _ptr(out["recv_count"]),
                               _ptr(out["dst_pos"]), _ptr(out["recv_src"]), _ptr(err))
    _check(rc, "layout")
    out["err"] = int(err[0])
    return out


def quantize(cfg, x_bits, smooth=None, lib=None):
    """Returns (quant_out [B,d] int8 or uint16, token_scale [B] float32 or None);
    quant_mode 1 (static cast) returns no scale."""
    lib = lib or load()
    x = _c(x_bits, np.uint16)
    ss = _c(smooth, np.float32)
    if cfg.quant_mode == 1:
        q = np.zeros((cfg.B, cfg.d), np.int8)
        sc = None
    elif cfg.quant_mode == 2:
        q = np.zeros((cfg.B, cfg.d), np.int8)
        sc = np.zeros(cfg.B, np.float32)
    else:
        q = np.zeros((cfg.B, cfg.d), np.uint16)
        sc = None
    rc = lib.orc_quantize(ctypes.byref(cfg), _ptr(x), _ptr(ss), _ptr(q), _ptr(sc))
    _check(rc, "quantize")
    return q, sc


def dispatch(cfg, quant_out, token_scale, dst_pos, rows, lib=None):
    """Scatter into a fresh receive buffer of `rows` rows (zero-filled; only the
    rows named by dst_pos are written).  Returns (recv_x, recv_scale or None)."""
    lib = lib or load()
    q = np.ascontiguousarray(quant_out)
    dp = _c(dst_pos, np.int32)
    recv_x = np.zeros((rows, cfg.d), q.dtype)
    recv_scale = np.zeros(rows, np.float32) if cfg.quant_mode == 2 else None
    ts = _c(token_scale, np.float32)
    rc = lib.orc_dispatch(ctypes.byref(cfg), _ptr(q), _ptr(ts), _ptr(dp), _ptr(recv_x),
                          _ptr(recv_scale), rows)
    _check(rc, "dispatch")
    return recv_x, recv_scale


def dispatch_expert_smooth(cfg, x_bits, smooth_E, topk_idx, dst_pos, rows, lib=None):
    """Per-copy quantization with a [E, d] smooth scale, scattered to `rows` receive
    rows.  Returns (recv_x int8 [rows, d], recv_scale float32 [rows], or None in
    quant_mode 1); rows no pick maps to stay zero."""
    lib = lib or load()
    recv_x = np.zeros((rows, cfg.d), np.int8)
    recv_scale = np.zeros(rows, np.float32) if cfg.quant_mode == 2 else None
    rc = lib.orc_dispatch_expert_smooth(ctypes.byref(cfg), _ptr(_c(x_bits, np.uint16)),
                                        _ptr(_c(smooth_E, np.float32)), _ptr(_c(topk_idx, np.int32)),
                                        _ptr(_c(dst_pos, np.int32)), _ptr(recv_x), _ptr(recv_scale),
                                        rows)
    _check(rc, "dispatch_expert_smooth")
    return recv_x, recv_scale


def combine(cfg, expert_out, topk_idx, topk_weights, dst_pos, ori_x=None, a1=None, a2=None,
            v=None, lib=None, active=None):
    """Returns y [B,d] as bf16 bits (uint16).  expert_out is [rows, d] bf16 bits;
    active: optional [B] x_active_mask (inactive tokens give +0)."""
    lib = lib or load()
    eo = _c(expert_out, np.uint16)
    rows = 0 if eo is None else eo.shape[0]
    y = np.zeros((cfg.B, cfg.d), np.uint16)
    act = None if active is None else (np.asarray(active) != 0).astype(np.uint8)
    rc = lib.orc_combine_active(ctypes.byref(cfg), _ptr(eo), rows, _ptr(_c(topk_idx, np.int32)),
                                _ptr(_c(topk_weights, np.float32)), _ptr(_c(dst_pos, np.int32)),
                                _ptr(_c(ori_x, np.uint16)), _ptr(_c(a1, np.uint16)),
                                _ptr(_c(a2, np.uint16)), _ptr(_c(v, np.uint16)), _ptr(act), _ptr(y))
    _check(rc, "combine")
    return y


def f32_to_bf16(f, lib=None):
    lib = lib or load()
    return int(lib.orc_f32_to_bf16(float(f)))


def f32_to_bf16_array(a, lib=None):
    lib = lib or load()
    src = np.ascontiguousarray(a, dtype=np.float32).ravel()
    out = np.zeros(src.shape, np.uint16)
    lib.orc_f32_to_bf16_n(_ptr(src), _ptr(out), src.size)
    return out.reshape(np.shape(a))


def bf16_to_f32(h, lib=None):
    lib = lib or load()
    return float(lib.orc_bf16_to_f32(int(h)))
