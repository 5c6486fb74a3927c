"""Out-of-bounds detection on the GPU, in place of a sanitizer.

Two independent checks over the parity cases:
  * guard bands: every device array the library writes (the buffer's arrays,
    expert outputs and y) is carved out of a larger allocation with GUARD bytes
    of a fill pattern on both sides; after the case the bands must be intact;
  * the checked build (libep_checked.so, -DEP_CHECKED): every row or offset a
    kernel computes is tested against its array's extent before the access and
    reported as EP_ERRBIT_CHECKED, which the parity checks would see as an
    unexpected error bit.
Both run against the same oracle comparisons as tests/test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_12_b200 import _binding as abi
from combine_ep_layout_12_b200 import build as ep_build
from combine_ep_layout_12_b200 import runner
from combine_ep_layout_12_b200 import workloads as wl
from tests import gpu_parity as gp

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side (keeps the 16-byte alignment of the arrays)
FILL = 0xA5


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ep_build.build()
    ep_build.build_checked()
    torch.cuda.set_device(0)
    yield torch.device("cuda", 0)
    abi.use_checked(False)


@pytest.fixture(params=["checked", "regular"])
def library(request):
    abi.use_checked(request.param == "checked")
    yield request.param
    abi.use_checked(False)


class Guarded:
    """Allocator of device tensors with FILL guard bands around each one."""

    def __init__(self, device):
        self.device = device
        self.blocks = []

    def __call__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((n + 2 * GUARD,), FILL, dtype=torch.uint8, device=self.device)
        self.blocks.append((raw, n))
        return raw[GUARD:GUARD + n].view(dtype).view(shape)

    def damaged(self):
        torch.cuda.synchronize(self.device)
        bad = 0
        for raw, n in self.blocks:
            bad += int((raw[:GUARD] != FILL).sum()) + int((raw[GUARD + n:] != FILL).sum())
        return bad


def small(name, **kw):
    base = dict(B=96, d=128, k=4, P=4, M=24, E=16, quant_mode=2)
    base.update(kw)
    return wl.Workload(name, **base)


CASES = [
    wl.get("tiny_q0"),
    wl.get("tiny_q2"),
    wl.get("decode"),
    wl.get("skewed"),
    wl.get("decode_packed"),
    wl.get("skewed_packed"),
    wl.get("decode_expert_smooth"),
    wl.get("decode_static"),
    wl.get("decode_active"),
    wl.get("sweep_T256_q0"),
    wl.get("decode").with_(name="decode_expert_static_active_packed", quant_mode=1, smooth="expert",
                           active_frac=0.7, layout=1),
    wl.Workload("ragged", B=111, d=272, k=3, P=3, M=40, E=9, n_zero=1, n_copy=1, n_const=1,
                quant_mode=2, smooth="rand", seed=5),
    wl.Workload("k16", B=8 * 40, d=64, k=16, P=8, M=48, E=64, quant_mode=2, seed=16),
    wl.Workload("e2048", B=8 * 600, d=64, k=8, P=8, M=600, E=2048, quant_mode=0, seed=11),
    wl.Workload("d32768", B=32, d=32768, k=2, P=2, M=16, E=8, quant_mode=2, smooth="expert", seed=7),
    small("M_equals_T", M=24),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
@pytest.mark.parametrize("fused", [False, True])
def test_no_out_of_bounds(dev, library, w, fused):
    guard = Guarded(dev)
    gp.full_check(w, dev, fused=fused, alloc=guard)
    assert guard.damaged() == 0, "%s: writes outside the arrays (%s build)" % (w.name, library)


def test_dirty_routing_no_out_of_bounds(dev, library):
    """Bad, repeated and masked ids, with specials, a mask and the packed layout."""
    for layout in (0, 1):
        w = wl.Workload("dirty_l%d" % layout, B=111, d=272, k=3, P=3, M=40, E=9, n_zero=1, n_copy=1,
                        n_const=1, quant_mode=2, smooth="rand", seed=21, layout=layout,
                        active_frac=0.8)
        inp = wl.generate(w)
        rng = np.random.default_rng(21)
        idx = np.stack([rng.permutation(w.E_tot)[:w.k] for _ in range(w.B)]).astype(np.int32)
        idx[3, 1] = -1
        idx[7, 0] = w.E_tot + 2
        idx[8, 2] = -9
        idx[10] = [4, 5, 4]
        inp["topk_idx"] = idx
        inp["active"][[7, 8, 10]] = 1
        guard = Guarded(dev)
        dev_inp = runner.to_device(inp, dev)
        pipe = runner.Pipeline(w, dev, alias_expert_out=False, alloc=guard)
        pipe.layout(dev_inp)
        pipe.dispatch(dev_inp)
        err = pipe.buf.check()
        ref = oracle.layout(gp.ocfg(w), idx, active=inp["active"])
        assert err == ref["err"] == (oracle.ERR_BAD_ID | oracle.ERR_DUP_ID)
        rep = gp.Report()
        gp.check_layout(rep, w, pipe, ref)
        gp.check_dispatch(rep, w, pipe, inp, ref)
        gp.check_combine(rep, w, pipe, inp, dev_inp, ref)
        rep.assert_ok()
        assert guard.damaged() == 0
