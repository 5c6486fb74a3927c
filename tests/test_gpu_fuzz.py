"""Seeded random configurations on the GPU against the oracle.

Each case draws a small problem (B, d, k, P, M, E, special experts, quant mode,
receive layout, smooth-scale form, active mask, dirty ids) from a fixed seed and
runs layout, dispatch and combine through the C ABI (split calls and the one-call
layout+dispatch), compares everything with the oracle, and checks guard bands
around every device array.  Half of the cases use the bounds-checked library.
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
from tests.test_gpu_checked import Guarded

pytestmark = pytest.mark.gpu

N_CASES = 300


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ep_build.build()
    ep_build.build_checked()
    torch.cuda.set_device(0)
    yield torch.device("cuda", 0)
    abi.use_checked(False)


def draw_case(i):
    rng = np.random.default_rng(np.random.SeedSequence([20261202, i]))
    P = int(rng.choice([1, 2, 3, 4, 8, 16]))
    T = int(rng.choice([1, 2, 7, 31, 32, 33, 64, 100, 128, 129, 256, 300]))
    B = P * T
    L = int(rng.choice([1, 2, 3, 4, 8]))
    E = P * L
    Z, C, K = (int(v) for v in rng.integers(0, 3, 3))
    E_tot = E + Z + C + K
    k = int(rng.integers(1, min(16, E_tot) + 1))
    d = int(16 * rng.choice([1, 2, 3, 8, 17, 64, 130]))
    layout = int(rng.integers(0, 2))
    M = T + int(rng.choice([0, 0, 1, 9]))
    qm = int(rng.choice([0, 1, 2]))
    smooth = "none"
    if qm:
        smooth = str(rng.choice(["none", "ones", "rand", "expert"]))
    active_frac = None if rng.random() < 0.6 else float(rng.choice([0.0, 0.3, 0.9]))
    w = wl.Workload("fuzz%d" % i, B=B, d=d, k=k, P=P, M=M, E=E, n_zero=Z, n_copy=C, n_const=K,
                    quant_mode=qm, smooth=smooth, seed=i, layout=layout, active_frac=active_frac,
                    routing="zipf")
    inp = wl.generate(w)
    # routing: k distinct ids per token over all E_tot ids, then some dirt
    idx = np.stack([rng.permutation(E_tot)[:k] for _ in range(B)]).astype(np.int32)
    dirty = rng.random() < 0.4
    if dirty and B:
        n = max(1, B // 10)
        rows = rng.integers(0, B, n)
        cols = rng.integers(0, k, n)
        kinds = rng.integers(0, 3, n)
        for r, c, kd in zip(rows, cols, kinds):
            if kd == 0:
                idx[r, c] = -1
            elif kd == 1:
                idx[r, c] = E_tot + int(rng.integers(0, 5))      # not an id
            elif k > 1:
                idx[r, c] = idx[r, (c + 1) % k]                 # repeated id
    inp["topk_idx"] = idx
    return w, inp, bool(rng.random() < 0.5)


@pytest.mark.parametrize("i", range(N_CASES))
def test_fuzz(dev, i):
    w, inp, checked = draw_case(i)
    abi.use_checked(checked)
    try:
        for fused in (False, True):
            guard = Guarded(dev)
            dev_inp = runner.to_device(inp, dev)
            pipe = runner.Pipeline(w, dev, alias_expert_out=False, alloc=guard)
            if fused:
                pipe.layout_dispatch(dev_inp)
            else:
                pipe.layout(dev_inp)
                pipe.dispatch(dev_inp)
            err = pipe.buf.check()
            ref = oracle.layout(gp.ocfg(w), inp["topk_idx"], active=inp.get("active"))
            rep = gp.Report()
            rep.check(err == ref["err"], "%s: device error bits %#x, oracle %#x" % (w.name, err, ref["err"]))
            gp.check_layout(rep, w, pipe, ref)
            gp.check_dispatch(rep, w, pipe, inp, ref)
            gp.check_combine(rep, w, pipe, inp, dev_inp, ref)
            rep.check(pipe.buf.check() == 0, "%s: error bits after combine" % w.name)
            rep.check(guard.damaged() == 0, "%s: writes outside the arrays" % w.name)
            rep.assert_ok()
    finally:
        abi.use_checked(False)
