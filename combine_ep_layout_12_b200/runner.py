"""Device plumbing around EPBuffer: move a workload's numpy inputs into torch
tensors and run the hot path (layout -> dispatch -> combine) on a stream.
No dispatch/combine arithmetic lives here; every step is a libep call."""
import numpy as np
import torch

from . import EPBuffer


def bf16_tensor(bits, device):
    """numpy uint16 bf16 bit patterns -> torch.bfloat16 tensor on `device`."""
    a = np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)
    return torch.from_numpy(a).to(device).view(torch.bfloat16)


def bf16_bits(t):
    """torch.bfloat16 tensor -> numpy uint16 bit patterns (on the host)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_device(inp, device, pin=False):
    """Inputs of workloads.generate() as device tensors (or pinned host tensors if pin)."""
    out = {}
    for name in ("x", "a1", "a2", "v"):
        a = inp.get(name)
        if a is None:
            out[name] = None
        elif pin:
            out[name] = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
                torch.bfloat16).pin_memory()
        else:
            out[name] = bf16_tensor(a, device)
    for name, dt in (("topk_idx", torch.int32), ("topk_weights", torch.float32),
                     ("smooth", torch.float32), ("active", torch.uint8)):
        a = inp.get(name)
        if a is None:
            out[name] = None
        else:
            t = torch.from_numpy(np.ascontiguousarray(a))
            out[name] = t.pin_memory() if pin else t.to(device)
    return out


class Pipeline:
    """One workload's buffers plus the expert-output buffer combine reads.

    expert_out: for quant_mode 0 it may alias recv_x (identity expert); otherwise a
    separate bf16 [E*P*M, d] buffer the caller fills (the expert computation is
    not part of dispatch/combine).
    """

    def __init__(self, w, device, alias_expert_out=None, alloc=None):
        self.w = w
        self.device = torch.device(device)
        self.buf = EPBuffer(w, device=self.device, alloc=alloc)
        if alloc is None:
            def alloc(shape, dtype):
                return torch.empty(shape, dtype=dtype, device=self.device)
        if alias_expert_out is None:
            alias_expert_out = w.quant_mode == 0
        if alias_expert_out:
            assert w.quant_mode == 0
            self.expert_out = self.buf.recv_x
        else:
            self.expert_out = alloc((w.rows, w.d), torch.bfloat16)
        self.y = alloc((w.B, w.d), torch.bfloat16)

    def layout(self, dev_inp, stream=None):
        self.buf.layout(dev_inp["topk_idx"], x_active_mask=dev_inp.get("active"), stream=stream)

    def dispatch(self, dev_inp, stream=None):
        self.buf.dispatch(dev_inp["x"], dev_inp.get("smooth"), stream=stream)

    def combine(self, dev_inp, stream=None):
        return self.buf.combine(self.expert_out, dev_inp["topk_idx"], dev_inp["topk_weights"],
                                ori_x=dev_inp["x"], a1=dev_inp.get("a1"), a2=dev_inp.get("a2"),
                                v=dev_inp.get("v"), y=self.y, x_active_mask=dev_inp.get("active"),
                                stream=stream)

    def layout_dispatch(self, dev_inp, stream=None):
        self.buf.layout_dispatch(dev_inp["topk_idx"], dev_inp["x"], dev_inp.get("smooth"),
                                 x_active_mask=dev_inp.get("active"), stream=stream)

    def step(self, dev_inp, stream=None, fused=True):
        """layout -> dispatch -> combine; fused=True issues the first two as one call."""
        if fused:
            self.layout_dispatch(dev_inp, stream)
        else:
            self.layout(dev_inp, stream)
            self.dispatch(dev_inp, stream)
        return self.combine(dev_inp, stream)
