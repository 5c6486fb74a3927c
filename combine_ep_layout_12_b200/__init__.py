"""B200-native MoE expert-parallel token dispatch and combine, with the EP ranks
as logical partitions of one GPU's memory.

The compute path is libep.so (CUDA kernels for sm_100a behind the C ABI of
include/ep.h).  `_binding` holds the one-to-one ctypes functions; `EPBuffer`
below is a convenience wrapper that allocates the caller-owned arrays as torch
tensors and passes their addresses through.  torch supplies device memory and
streams only.  There is no CPU or torch fallback: every call fails loudly if
libep.so is missing.

Usage (one decode step of 8 logical ranks x 128 tokens, DeepSeek-V3 shape):

    cfg = make_config(B=1024, d=7168, k=8, P=8, M=128, E=256, quant_mode=2, smooth_rows=1)
    buf = EPBuffer(cfg, device="cuda")
    buf.layout_dispatch(topk_idx, x)          # int32 [B, k], bf16 [B, d]
    # buf.recv_x [E*P*M, d] int8 and buf.recv_scale [E*P*M]: rank q's experts
    # q*L .. q*L+L-1 own rows [q*L*P*M, (q+1)*L*P*M); buf.recv_count [E, P] counts
    # them per source rank.  Run the experts, write bf16 outputs to expert_out
    # at the same rows, then:
    y = buf.combine(expert_out, topk_idx, topk_weights, ori_x=x)

Across GPUs (one process per GPU, each holding one logical rank's tokens and its
receive slab): see shard.py (ep_shard_layout / ep_shard_dispatch / ep_shard_layout_dispatch /
ep_shard_combine).

Options: quant_mode 0 (bf16) / 1 (static int8) / 2 (dynamic int8); smooth_rows
= E for a per-expert [E, d] smooth scale; layout=1 for rows packed per expert
(rank q reads [expert_offset[q*L], expert_offset[(q+1)*L])); n_zero / n_copy /
n_const special experts (combine then needs ori_x, and a1, a2, v for constant
experts); x_active_mask= on layout / layout_dispatch / combine.
"""
import torch

from . import _binding as abi
from ._binding import (EPError, ep_buffer_check, ep_buffer_create, ep_buffer_destroy,
                       ep_buffer_size, ep_combine, ep_dispatch, ep_layout, ep_layout_dispatch,
                       ep_layout_static_scratch, ep_shard_check, ep_shard_combine, ep_shard_dispatch,
                       ep_shard_layout, ep_shard_layout_dispatch, ep_shard_workspace_size, ep_status_str, make_config,
                       make_shard_table)

__all__ = ["EPBuffer", "EPError", "abi", "ep_buffer_check", "ep_buffer_create",
           "ep_buffer_destroy", "ep_buffer_size", "ep_combine", "ep_dispatch", "ep_layout",
           "ep_layout_dispatch", "ep_layout_static_scratch", "ep_shard_check", "ep_shard_combine",
           "ep_shard_dispatch", "ep_shard_layout", "ep_shard_layout_dispatch", "ep_shard_workspace_size", "ep_status_str",
           "make_config", "make_shard_table"]


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need(t, name, dtype, shape, device):
    if t is None:
        raise ValueError("%s is required" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.device != device:
        raise ValueError("%s must be on %s, got %s" % (name, device, t.device))
    return t


class EPBuffer:
    """Caller-owned arrays of one dispatch/combine problem plus the libep handle.

    cfg: an ep_config (see make_config) or any object with the config fields
    (B, d, k, P, M, E, n_zero, n_copy, n_const, quant_mode[, smooth_rows]).
    Views: expert_count [E_tot], expert_offset [E_tot+1], recv_count [E, P],
    dst_pos [B, k], recv_src [rows], recv_x [rows, d] (int8 or bf16),
    recv_scale [rows], token_scale [B]; rows = E*P*M (low-latency layout) or
    B*k (packed layout).  alloc(shape, dtype) -> tensor, if given, provides the
    arrays (e.g. carved out of larger allocations); default torch.empty.
    """

    def __init__(self, cfg, device=None, alloc=None):
        if not isinstance(cfg, abi.ep_config):
            cfg = make_config(cfg.B, cfg.d, cfg.k, cfg.P, cfg.M, cfg.E, cfg.n_zero, cfg.n_copy,
                              cfg.n_const, cfg.quant_mode, getattr(cfg, "smooth_rows", 1),
                              getattr(cfg, "layout", 0))
        self.cfg = cfg
        dev = torch.device("cuda" if device is None else device)
        if dev.type != "cuda":
            raise ValueError("EPBuffer lives on a CUDA device, got %s" % dev)
        self.device = dev if dev.index is not None else torch.device("cuda", torch.cuda.current_device())
        sizes = ep_buffer_size(cfg)
        self.sizes = {n: int(getattr(sizes, n)) for n in abi.BUFFER_FIELDS}
        c = cfg
        self.E_tot = c.E + c.n_zero + c.n_copy + c.n_const
        self.rows = c.B * c.k if c.layout == 1 else c.E * c.P * c.M
        dev = self.device
        if alloc is None:
            def alloc(shape, dtype):
                return torch.empty(shape, dtype=dtype, device=dev)
        self.expert_count = alloc((self.E_tot,), torch.int32)
        self.expert_offset = alloc((self.E_tot + 1,), torch.int32)
        self.recv_count = alloc((c.E, c.P), torch.int32)
        self.dst_pos = alloc((c.B, c.k), torch.int32)
        self.recv_src = alloc((self.rows,), torch.int32)
        xdt = torch.int8 if c.quant_mode != 0 else torch.bfloat16
        self.recv_x = alloc((self.rows, c.d), xdt)
        q = c.quant_mode == 2
        self.recv_scale = alloc((self.rows,), torch.float32) if q else None
        self.token_scale = alloc((c.B,), torch.float32) if q else None
        self.workspace = alloc((self.sizes["workspace"],), torch.uint8)
        ptrs = abi.ep_buffer_ptrs(*[_ptr(getattr(self, n)) for n in abi.BUFFER_FIELDS])
        with torch.cuda.device(dev):
            self.handle = ep_buffer_create(cfg, ptrs)

    def close(self):
        if getattr(self, "handle", None) is not None:
            ep_buffer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _mask(self, x_active_mask):
        """x_active_mask: None or a [B] bool/uint8 device tensor (nonzero = active)."""
        if x_active_mask is None:
            return None
        t = x_active_mask
        if t.dtype not in (torch.bool, torch.uint8):
            raise ValueError("x_active_mask must be bool or uint8, got %s" % t.dtype)
        if tuple(t.shape) != (self.cfg.B,) or not t.is_contiguous() or t.device != self.device:
            raise ValueError("x_active_mask must be a contiguous [B] tensor on %s" % self.device)
        return _ptr(t)

    def _smooth(self, smooth_scale):
        """Checked pointer of a smooth scale: [d] (or [1, d]) for smooth_rows 1,
        [smooth_rows, d] per routed expert otherwise; None passes through."""
        if smooth_scale is None:
            return None
        c = self.cfg
        if c.smooth_rows <= 1 and smooth_scale.dim() == 2 and smooth_scale.shape[0] == 1:
            smooth_scale = smooth_scale[0]
        shape = (c.d,) if c.smooth_rows <= 1 else (c.smooth_rows, c.d)
        return _ptr(_need(smooth_scale, "smooth_scale", torch.float32, shape, self.device))

    # -- hot path ---------------------------------------------------------------
    def layout(self, topk_idx, x_active_mask=None, stream=None):
        c = self.cfg
        _need(topk_idx, "topk_idx", torch.int32, (c.B, c.k), self.device)
        ep_layout(self.handle, _ptr(topk_idx), self._mask(x_active_mask), _stream(stream))

    def dispatch(self, x, smooth_scale=None, stream=None):
        c = self.cfg
        _need(x, "x", torch.bfloat16, (c.B, c.d), self.device)
        ep_dispatch(self.handle, _ptr(x), self._smooth(smooth_scale), _stream(stream))

    def layout_dispatch(self, topk_idx, x, smooth_scale=None, x_active_mask=None, stream=None):
        """layout(topk_idx) then dispatch(x), as one call (one grid when T <= 128)."""
        c = self.cfg
        _need(topk_idx, "topk_idx", torch.int32, (c.B, c.k), self.device)
        _need(x, "x", torch.bfloat16, (c.B, c.d), self.device)
        ep_layout_dispatch(self.handle, _ptr(topk_idx), self._mask(x_active_mask), _ptr(x),
                           self._smooth(smooth_scale), _stream(stream))

    def combine(self, expert_out, topk_idx, topk_weights, ori_x=None, a1=None, a2=None, v=None,
                y=None, x_active_mask=None, stream=None):
        c = self.cfg
        _need(expert_out, "expert_out", torch.bfloat16, (self.rows, c.d), self.device)
        _need(topk_idx, "topk_idx", torch.int32, (c.B, c.k), self.device)
        _need(topk_weights, "topk_weights", torch.float32, (c.B, c.k), self.device)
        if c.n_copy + c.n_const > 0:
            _need(ori_x, "ori_x", torch.bfloat16, (c.B, c.d), self.device)
        if c.n_const > 0:
            for n, t in (("a1", a1), ("a2", a2), ("v", v)):
                _need(t, n, torch.bfloat16, (c.n_const, c.d), self.device)
        if y is None:
            y = torch.empty((c.B, c.d), dtype=torch.bfloat16, device=self.device)
        else:
            _need(y, "y", torch.bfloat16, (c.B, c.d), self.device)
        ep_combine(self.handle, _ptr(expert_out), _ptr(topk_idx), _ptr(topk_weights),
                   self._mask(x_active_mask), _ptr(ori_x), _ptr(a1), _ptr(a2), _ptr(v), _ptr(y),
                   _stream(stream))
        return y

    def check(self, stream=None):
        """Synchronize and return (and clear) the device error bits."""
        return ep_buffer_check(self.handle, _stream(stream))
