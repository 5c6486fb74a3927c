"""ep_layout_static_scratch: the layout entry point for callers that cannot
allocate device memory (for example an engine whose memory pool already owns the
whole GPU, or code that must not call cudaMalloc because it can synchronize the
device).  Its scratch lives in the library's own static device memory.

Checked here through the C ABI: two calls in a row give exactly the outputs of
the regular ep_layout and of the CPU oracle (integer results, so the tolerance
is bit equality), the error word is delivered, a configuration that fills the
static array exactly works, and one whose scratch would not fit is refused.  This file is collected last on purpose and must pass
on its own in a fresh process as well as after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_12_b200 import EPBuffer
from combine_ep_layout_12_b200 import _binding as abi
from combine_ep_layout_12_b200 import build as ep_build
from combine_ep_layout_12_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ep_build.build()
    torch.cuda.set_device(0)
    return torch.device("cuda", 0)


def _outputs(w, dev):
    rows = w.rows
    return {
        "expert_count": torch.full((w.E_tot,), -7, dtype=torch.int32, device=dev),
        "expert_offset": torch.full((w.E_tot + 1,), -7, dtype=torch.int32, device=dev),
        "recv_count": torch.full((w.E, w.P), -7, dtype=torch.int32, device=dev),
        "dst_pos": torch.full((w.B, w.k), -7, dtype=torch.int32, device=dev),
        "recv_src": torch.full((rows,), -1, dtype=torch.int32, device=dev),
        "err": torch.full((1,), 0xDEAD, dtype=torch.int32, device=dev),
    }


def _cfg(w):
    return abi.make_config(w.B, w.d, w.k, w.P, w.M, w.E, w.n_zero, w.n_copy, w.n_const,
                           w.quant_mode, 1, w.layout)


def _static_layout(w, topk_idx, out, stream):
    abi.ep_layout_static_scratch(_cfg(w), topk_idx.data_ptr(), out["expert_count"].data_ptr(),
                                 out["expert_offset"].data_ptr(), out["recv_count"].data_ptr(),
                                 out["dst_pos"].data_ptr(), out["recv_src"].data_ptr(),
                                 out["err"].data_ptr(), stream.cuda_stream)


def _dirty(w):
    inp = wl.generate(w, with_x=False)
    idx = inp["topk_idx"].copy()
    idx[3, 0] = w.E_tot + 5          # not an expert id
    idx[9, :2] = 5                   # routed id 5 twice in one token
    return idx


def _case(name):
    if name == "dirty":
        w = wl.get("skewed").with_(name="dirty", n_zero=2, n_copy=1, n_const=3, k=5)
        return w, _dirty(w)
    if name == "ragged257":
        # 257 tokens per rank: a second 256-token chunk holding one token, with specials
        w = wl.Workload("ragged257", B=2 * 257, d=16, k=4, P=2, M=257, E=16, n_zero=1, n_copy=1,
                        n_const=1, routing="zipf", seed=11)
        return w, wl.generate(w, with_x=False)["topk_idx"]
    if name == "full_array":
        # P * ceil(T / 256) * (E + Z + C + K) = 8 * 2 * 1020 = 16320 counts: with the
        # 256-byte header the scratch fills the 64 KiB array exactly
        w = wl.Workload("full_array", B=8 * 300, d=16, k=2, P=8, M=300, E=1016, n_zero=2, n_copy=1,
                        n_const=1, routing="zipf", seed=12)
        return w, wl.generate(w, with_x=False)["topk_idx"]
    w = wl.get(name)
    return w, wl.generate(w, with_x=False)["topk_idx"]


def _check_oracle(w, idx_np, out, err):
    ref = oracle.layout(oracle.make_cfg(w.B, w.d, w.k, w.P, w.M, w.E, w.n_zero, w.n_copy, w.n_const,
                                        w.quant_mode, layout=w.layout), idx_np)
    for n in ("expert_count", "expert_offset", "recv_count", "dst_pos"):
        assert np.array_equal(out[n].cpu().numpy(), ref[n]), "%s differs from the oracle" % n
    rows = np.nonzero(ref["recv_src"] >= 0)[0]
    got = out["recv_src"].cpu().numpy()[rows]
    assert np.array_equal(got, ref["recv_src"][rows]), "recv_src differs from the oracle"
    assert err == ref["err"], "error bits %#x, oracle %#x" % (err, ref["err"])


@pytest.mark.parametrize("name", ["decode", "skewed", "dirty", "decode_packed", "ragged257", "full_array"])
def test_static_scratch_layout_matches_ep_layout(dev, name):
    w, idx_np = _case(name)
    idx = torch.from_numpy(idx_np).to(dev)
    stream = torch.cuda.current_stream(dev)

    # regular entry point, with its caller-allocated workspace
    buf = EPBuffer(w, device=dev)
    buf.recv_src.fill_(-1)
    buf.layout(idx)
    ref_err = buf.check()
    ref = {n: getattr(buf, n).clone() for n in
           ("expert_count", "expert_offset", "recv_count", "dst_pos", "recv_src")}
    if name == "dirty":
        assert ref_err == abi.ERRBIT_BAD_ID | abi.ERRBIT_DUP_ID

    # the static-scratch entry point, twice in a row on the same stream, against the
    # regular entry point and against the CPU oracle
    for call in range(2):
        out = _outputs(w, dev)
        _static_layout(w, idx, out, stream)
        torch.cuda.synchronize(dev)
        for n, t in ref.items():
            assert torch.equal(out[n], t), "call %d: %s differs from ep_layout" % (call, n)
        assert int(out["err"].item()) == ref_err, "call %d: error word" % call
        _check_oracle(w, idx_np, out, int(out["err"].item()))


def test_static_scratch_refuses_configs_beyond_its_array(dev):
    # above 256 tokens per rank the chunked layout keeps P * ceil(T / 256) * (E + Z + C + K)
    # int32 counts next to the 256-byte header; 8 * 16 * 256 of them exceed 64 KiB
    w = wl.Workload("too_many_chunks", B=8 * 4096, d=16, k=2, P=8, M=4096, E=256, quant_mode=0)
    out = _outputs(w, dev)
    idx = torch.zeros((w.B, w.k), dtype=torch.int32, device=dev)
    with pytest.raises(abi.EPError) as ei:
        _static_layout(w, idx, out, torch.cuda.current_stream(dev))
    assert ei.value.status == abi.EP_ERR_CAPACITY
    # one count beyond the array: P * ceil(T / 256) * (E + Z + C + K) = 1 * 19 * 859 = 16321
    w1 = wl.Workload("one_count_over", B=19 * 256, d=16, k=2, P=1, M=19 * 256, E=800, n_zero=59,
                     quant_mode=0)
    out1 = _outputs(w1, dev)
    idx1 = torch.zeros((w1.B, w1.k), dtype=torch.int32, device=dev)
    with pytest.raises(abi.EPError) as ei:
        _static_layout(w1, idx1, out1, torch.cuda.current_stream(dev))
    assert ei.value.status == abi.EP_ERR_CAPACITY
    # small batches need only the header, whatever the number of special experts
    w2 = wl.Workload("many_specials", B=16, d=16, k=2, P=16, M=1, E=16, n_zero=1100, quant_mode=0)
    out2 = _outputs(w2, dev)
    idx2 = torch.zeros((w2.B, w2.k), dtype=torch.int32, device=dev)
    _static_layout(w2, idx2, out2, torch.cuda.current_stream(dev))
    torch.cuda.synchronize(dev)
    assert int(out2["expert_count"][0].item()) == w2.B  # every pick is expert 0, once per token
