"""GPU parity: libep (through the C ABI) against the CPU oracle on the named
workloads and on edge cases.  Layout, source maps, int8/bf16 payloads and scales
must be bit-exact; combine must be within 8e-3 relative (one bf16 ulp of the
accumulated magnitude near zero) and, with the same fused multiply-add order on
both sides, is also required to be bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_12_b200 import EPBuffer, runner
from combine_ep_layout_12_b200 import workloads as wl
from combine_ep_layout_12_b200 import build as ep_build
from tests import gpu_parity as gp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="session")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ep_build.build()
    torch.cuda.set_device(0)
    return torch.device("cuda", 0)


same_as_x = gp.same_as_x
free_bytes = gp.free_bytes
need_bytes = gp.need_bytes
full_check = gp.full_check


# ----------------------------------------------------------------------------- named workloads


@pytest.mark.parametrize("name", ["tiny_q0", "tiny_q2"])
def test_tiny(dev, name):
    full_check(wl.get(name), dev)


def test_tiny_q2_random_smooth(dev):
    full_check(wl.get("tiny_q2").with_(name="tiny_q2_rand_smooth", smooth="rand", seed=3), dev)


def test_decode(dev):
    """DeepSeek-V3-shaped decode in the launch configuration the benchmark times."""
    full_check(wl.get("decode"), dev)


def test_skewed_specials(dev):
    full_check(wl.get("skewed"), dev)


@pytest.mark.parametrize("T", [1, 4, 16, 64, 256])
@pytest.mark.parametrize("qm", [0, 2])
def test_sweep_small(dev, T, qm):
    full_check(wl.get("sweep_T%d_q%d" % (T, qm)), dev)


@pytest.mark.parametrize("qm", [0, 2])
def test_sweep_T1024_sampled(dev, qm):
    w = wl.get("sweep_T1024_q%d" % qm)
    rng = np.random.default_rng(1024)
    tokens = np.sort(rng.choice(w.B, 512, replace=False))
    full_check(w, dev, tokens=tokens, sample_picks=8192, separate=(qm == 2))


def test_sweep_T4096_q2_sampled(dev):
    """120 GB int8 receive buffer; combine is checked through the mode-0 aliasing
    path of the bf16 workloads (a bf16 expert_out of this shape is 240 GB)."""
    w = wl.get("sweep_T4096_q2")
    if need_bytes(w, False) > free_bytes() - (4 << 30):
        pytest.skip("needs %.1f GB" % (need_bytes(w, False) / 1e9))
    inp = wl.generate(w)
    dev_inp = runner.to_device(inp, dev)
    buf = EPBuffer(w, device=dev)
    buf.layout(dev_inp["topk_idx"])
    buf.dispatch(dev_inp["x"])
    rep = gp.Report()
    ref = oracle.layout(gp.ocfg(w), inp["topk_idx"])
    err = buf.check()
    rep.check(err == ref["err"], "error bits")

    class P:
        pass
    pipe = P()
    pipe.buf = buf
    gp.check_layout(rep, w, pipe, ref)
    gp.check_dispatch(rep, w, pipe, inp, ref, sample_picks=8192)
    rep.assert_ok()


def test_prefill(dev):
    """High-throughput prefill, bf16 payload, 120 GB low-latency buffer.  Layout
    bit-exact in full, payload on sampled picks, combine(dispatch(x)) == x with
    one-hot weights in full, and combine against the oracle on sampled tokens."""
    w = wl.get("prefill")
    if need_bytes(w, False) > free_bytes() - (4 << 30):
        pytest.skip("needs %.1f GB" % (need_bytes(w, False) / 1e9))
    inp = wl.generate(w)
    dev_inp = runner.to_device(inp, dev)
    pipe = runner.Pipeline(w, dev, alias_expert_out=True)
    rep = gp.Report()
    pipe.layout(dev_inp)
    pipe.dispatch(dev_inp)
    ref = oracle.layout(gp.ocfg(w), inp["topk_idx"])
    rep.check(pipe.buf.check() == ref["err"], "error bits")
    gp.check_layout(rep, w, pipe, ref)
    gp.check_dispatch(rep, w, pipe, inp, ref, sample_picks=16384)
    # identity expert + one-hot weights: y == x bitwise, every token
    rng = np.random.default_rng(77)
    onehot = np.zeros((w.B, w.k), np.float32)
    onehot[np.arange(w.B), rng.integers(0, w.k, w.B)] = 1.0
    dev1 = dict(dev_inp)
    dev1["topk_weights"] = torch.from_numpy(onehot).to(dev)
    y = pipe.combine(dev1)
    rep.check(same_as_x(y, dev_inp["x"]), "prefill: combine(dispatch(x)) != x with one-hot weights")
    # sampled tokens against the oracle with softmax weights
    tokens = np.sort(rng.choice(w.B, 512, replace=False))
    gp.check_combine(rep, w, pipe, inp, dev_inp, ref, tokens=tokens)
    rep.assert_ok()


# ----------------------------------------------------------------------------- packed layout


@pytest.mark.parametrize("name", ["tiny_q0_packed", "tiny_q2_packed", "decode_packed", "skewed_packed",
                                  "sweep_T1_q2_packed", "sweep_T16_q2_packed", "sweep_T256_q0_packed"])
def test_packed(dev, name):
    """Packed receive rows (contiguous per expert, then per source rank)."""
    full_check(wl.get(name), dev)


@pytest.mark.parametrize("name", ["prefill_packed", "sweep_T4096_q0_packed", "sweep_T4096_q2_packed"])
def test_packed_large_sampled(dev, name):
    """The largest configurations in the packed layout (3.8-11 GB instead of
    120-360 GB low-latency buffers): layout in full, payload on sampled picks,
    combine on sampled tokens."""
    w = wl.get(name)
    rng = np.random.default_rng(4096)
    tokens = np.sort(rng.choice(w.B, 512, replace=False))
    full_check(w, dev, tokens=tokens, sample_picks=16384, separate=(w.quant_mode == 2))


def test_packed_dirty(dev):
    w = wl.Workload("ragged_packed", B=111, d=272, k=3, P=3, M=0, E=9, n_zero=1, n_copy=1, n_const=1,
                    quant_mode=2, smooth="rand", seed=8, layout=1)
    inp = wl.generate(w)
    rng = np.random.default_rng(8)
    idx = np.stack([rng.permutation(w.E_tot)[:w.k] for _ in range(w.B)]).astype(np.int32)
    idx[1, 2] = -1
    idx[4, 0] = w.E_tot + 1
    idx[9] = [2, 2, 5]
    inp["topk_idx"] = idx
    dev_inp = runner.to_device(inp, dev)
    pipe = runner.Pipeline(w, dev, alias_expert_out=False)
    pipe.layout_dispatch(dev_inp)
    err = pipe.buf.check()
    ref = oracle.layout(gp.ocfg(w), idx)
    assert err == ref["err"] == (oracle.ERR_BAD_ID | oracle.ERR_DUP_ID)
    rep = gp.Report()
    gp.check_layout(rep, w, pipe, ref)
    gp.check_dispatch(rep, w, pipe, inp, ref)
    gp.check_combine(rep, w, pipe, inp, dev_inp, ref)
    rep.assert_ok()


# ----------------------------------------------------------------------------- per-expert smooth scale


@pytest.mark.parametrize("name,kw", [
    ("tiny_expert", dict(base="tiny_q2")),                       # T = 128: rows from the routing
    ("decode_expert_smooth", dict()),                            # decode shape, T = 128
    ("skewed_expert", dict(base="skewed")),                      # T = 1024: rows from dst_pos, specials
    ("decode_expert_packed", dict(base="decode", layout=1)),     # packed rows
])
def test_expert_smooth(dev, name, kw):
    """Per-expert smooth scale [E, d]: every routed copy quantized on its own."""
    kw = dict(kw)
    base = kw.pop("base", None)
    w = wl.get(name) if base is None else wl.get(base).with_(name=name, smooth="expert", **kw)
    full_check(w, dev)
    full_check(w.with_(name=name + "_fused"), dev, fused=True)


@pytest.mark.parametrize("qm", [1, 2])
@pytest.mark.parametrize("d", [16, 272, 4112, 8192, 8208, 32768])
def test_expert_smooth_widths(dev, d, qm):
    """Rows that do not tile the CTA (d = 16, 272, 4112), the widest rows with
    columns owned per thread (8192), the first width past them (8208) and the
    widest rows (1024 threads)."""
    w = wl.Workload("expert_d%d_q%d" % (d, qm), B=3 * 37, d=d, k=3, P=3, M=40, E=9, quant_mode=qm,
                    smooth="expert", seed=d)
    full_check(w, dev)


@pytest.mark.parametrize("qm", [1, 2])
def test_expert_smooth_degenerate_rows(dev, qm):
    """Per-copy quantization of all-zero rows, rows whose 127/amax overflows and a
    lone subnormal: q = 0 and scale 0 where the copy is degenerate."""
    w = small("degenerate_expert", d=7168, smooth="expert", quant_mode=qm)
    inp = wl.generate(w)
    inp["x"][0] = 0
    inp["x"][5] = 0x0080          # 2^-126 in every element: 127/amax overflows fp32
    inp["x"][6, :] = 0
    inp["x"][6, 3] = 0x8001       # a single negative subnormal
    full_check(w, dev, inp=inp)


def test_expert_smooth_dirty(dev):
    """Bad and repeated ids with a per-expert scale: those picks get no row, the
    others are quantized per copy."""
    w = wl.Workload("ragged_expert", B=111, d=272, k=3, P=3, M=40, E=9, n_zero=1, n_copy=1,
                    n_const=1, quant_mode=2, smooth="expert", seed=9)
    inp = wl.generate(w)
    rng = np.random.default_rng(9)
    idx = np.stack([rng.permutation(w.E_tot)[:w.k] for _ in range(w.B)]).astype(np.int32)
    idx[2, 0] = -1
    idx[5, 1] = w.E_tot
    idx[11] = [3, 7, 3]
    inp["topk_idx"] = idx
    inp["x"][20] = 0                   # degenerate copies: q = 0, scale 0
    for name, fused in (("dirty", False), ("dirty_fused", True)):
        dev_inp = runner.to_device(inp, dev)
        pipe = runner.Pipeline(w, dev, alias_expert_out=False)
        if fused:
            pipe.layout_dispatch(dev_inp)
        else:
            pipe.layout(dev_inp)
            pipe.dispatch(dev_inp)
        err = pipe.buf.check()
        ref = oracle.layout(gp.ocfg(w), idx)
        assert err == ref["err"] == (oracle.ERR_BAD_ID | oracle.ERR_DUP_ID), name
        rep = gp.Report()
        gp.check_layout(rep, w, pipe, ref)
        gp.check_dispatch(rep, w, pipe, inp, ref)
        gp.check_combine(rep, w, pipe, inp, dev_inp, ref)
        rep.assert_ok()


def test_expert_smooth_identical_rows_match_token_scale(dev):
    """Closed form on the GPU: an [E, d] scale whose rows are all one [d] vector
    gives the same receive rows and scales as that vector given per token."""
    w = wl.get("decode").with_(name="decode_same_rows", smooth="rand")
    inp = wl.generate(w)
    dev_inp = runner.to_device(inp, dev)
    pipe = runner.Pipeline(w, dev)
    we = w.with_(smooth="expert")
    pipe_e = runner.Pipeline(we, dev)
    dev_e = dict(dev_inp)
    dev_e["smooth"] = dev_inp["smooth"].expand(w.E, w.d).contiguous()
    pipe.layout(dev_inp)
    pipe.dispatch(dev_inp)
    pipe_e.layout(dev_e)
    pipe_e.dispatch(dev_e)
    torch.cuda.synchronize()
    dp = pipe.buf.dst_pos.flatten()
    rows = dp[dp >= 0].long()
    assert torch.equal(pipe.buf.recv_x[rows], pipe_e.buf.recv_x[rows])
    assert torch.equal(pipe.buf.recv_scale[rows], pipe_e.buf.recv_scale[rows])
    assert pipe.buf.check() == 0 and pipe_e.buf.check() == 0


def test_expert_smooth_needs_layout(dev):
    """A per-expert scale names the copies' experts through the latest layout's
    routing: ep_dispatch before any ep_layout is refused on the host."""
    from combine_ep_layout_12_b200 import _binding as abi
    w = small("expert_no_layout", smooth="expert")
    inp = wl.generate(w)
    dev_inp = runner.to_device(inp, dev)
    buf = EPBuffer(w, device=dev)
    with pytest.raises(abi.EPError) as ei:
        buf.dispatch(dev_inp["x"], dev_inp["smooth"])
    assert ei.value.status == abi.EP_ERR_INVALID_ARG


# ----------------------------------------------------------------------------- static int8 and x_active_mask


@pytest.mark.parametrize("name,kw", [
    ("tiny_static", dict(base="tiny_q2", quant_mode=1, smooth="rand")),
    ("tiny_static_noscale", dict(base="tiny_q2", quant_mode=1, smooth="none")),
    ("decode_static", dict()),
    ("skewed_static", dict(base="skewed", quant_mode=1, smooth="rand")),
    ("decode_static_packed", dict(base="decode", quant_mode=1, smooth="rand", layout=1)),
    ("decode_static_expert", dict(base="decode", quant_mode=1, smooth="expert")),
])
def test_static_quant(dev, name, kw):
    """quant_mode 1: CastToInt8(CastToFp32(x) * scales), no scale sent."""
    kw = dict(kw)
    base = kw.pop("base", None)
    w = wl.get(name) if base is None else wl.get(base).with_(name=name, **kw)
    full_check(w, dev)
    full_check(w.with_(name=name + "_fused"), dev, fused=True)


def test_static_quant_closed_forms(dev):
    """Integers pass through, x.5 ties go to even, beyond [-128, 127] saturates."""
    w = wl.Workload("static_cf", B=4, d=32, k=2, P=2, M=2, E=4, quant_mode=1, seed=3)
    inp = wl.generate(w)
    vals = np.array([0, 1, -1, 2.5, 3.5, -2.5, -0.5, 0.5, 126, 127, 127.5, 128, 300,
                     -128, -128.5, -129, -300, 1.5, -1.5, 64.25], np.float32)
    want = np.array([0, 1, -1, 2, 4, -2, 0, 0, 126, 127, 127, 127, 127, -128, -128, -128, -128,
                     2, -2, 64], np.int8)
    xv = np.zeros((w.B, w.d), np.float32)
    xv[:, :vals.size] = vals
    inp["x"] = wl.f32_to_bf16_bits(xv)
    pipe, *_ = full_check(w, dev, inp=inp)
    dp = pipe.buf.dst_pos.flatten()
    rows = dp[dp >= 0].long()
    got = pipe.buf.recv_x[rows][:, :vals.size].cpu().numpy()
    assert (got == want[None, :]).all()


@pytest.mark.parametrize("name,kw", [
    ("tiny_active", dict(base="tiny_q2", active_frac=0.5)),
    ("decode_active", dict()),                                          # T = 128, one grid
    ("decode_active_bf16", dict(base="decode", quant_mode=0, active_frac=0.75)),
    ("skewed_active", dict(base="skewed", active_frac=0.6)),            # chunked layout, specials
    ("decode_active_packed", dict(base="decode", active_frac=0.75, layout=1)),
    ("sweep_T256_active", dict(base="sweep_T256_q2", active_frac=0.8)),
    ("decode_active_expert", dict(base="decode", active_frac=0.75, smooth="expert")),
    ("decode_active_none", dict(base="decode", active_frac=0.0)),
])
def test_active_mask(dev, name, kw):
    """x_active_mask: inactive tokens route nothing, count nowhere and get y = +0."""
    kw = dict(kw)
    base = kw.pop("base", None)
    w = wl.get(name) if base is None else wl.get(base).with_(name=name, **kw)
    pipe, dev_inp, inp, ref = full_check(w, dev)
    off = np.nonzero(inp["active"] == 0)[0]
    if off.size:
        y = pipe.y[torch.from_numpy(off).to(dev)]
        assert int(y.view(torch.int16).abs().max()) == 0
    full_check(w.with_(name=name + "_fused"), dev, fused=True)


def test_active_mask_ignores_bad_ids_of_inactive_tokens(dev):
    """An inactive token's ids are not looked at: bad or repeated ids there raise
    no error bit, while the same ids in an active token do."""
    w = wl.Workload("active_dirty", B=111, d=272, k=3, P=3, M=40, E=9, n_zero=1, n_copy=1,
                    n_const=1, quant_mode=2, smooth="rand", seed=13, active_frac=1.0)
    inp = wl.generate(w)
    rng = np.random.default_rng(13)
    idx = np.stack([rng.permutation(w.E_tot)[:w.k] for _ in range(w.B)]).astype(np.int32)
    idx[5, 1] = w.E_tot + 4
    idx[11] = [3, 7, 3]
    inp["topk_idx"] = idx
    for act5, want in ((0, oracle.ERR_DUP_ID), (1, oracle.ERR_DUP_ID | oracle.ERR_BAD_ID)):
        inp["active"] = np.ones(w.B, np.uint8)
        inp["active"][5] = act5
        inp["active"][40:50] = 0
        for fused in (False, True):
            dev_inp = runner.to_device(inp, dev)
            pipe = runner.Pipeline(w, dev, alias_expert_out=False)
            if fused:
                pipe.layout_dispatch(dev_inp)
            else:
                pipe.layout(dev_inp)
                pipe.dispatch(dev_inp)
            err = pipe.buf.check()
            ref = oracle.layout(gp.ocfg(w), idx, active=inp["active"])
            assert err == ref["err"] == want
            rep = gp.Report()
            gp.check_layout(rep, w, pipe, ref)
            gp.check_dispatch(rep, w, pipe, inp, ref)
            gp.check_combine(rep, w, pipe, inp, dev_inp, ref)
            rep.assert_ok()


# ----------------------------------------------------------------------------- fused call


@pytest.mark.parametrize("name", ["tiny_q0", "tiny_q2", "decode", "sweep_T1_q2", "sweep_T16_q0",
                                  "sweep_T64_q2", "sweep_T256_q0", "skewed"])
def test_layout_dispatch_one_call(dev, name):
    """ep_layout_dispatch (one grid when T <= 128 and k <= 8, else two launches)
    against the oracle: identical to ep_layout followed by ep_dispatch."""
    full_check(wl.get(name), dev, fused=True)


def test_layout_dispatch_one_call_dirty(dev):
    w = wl.Workload("ragged_fused", B=111, d=272, k=3, P=3, M=40, E=9, n_zero=1, n_copy=1,
                    n_const=1, quant_mode=2, smooth="rand", seed=5)
    inp = wl.generate(w)
    rng = np.random.default_rng(6)
    idx = np.stack([rng.permutation(w.E_tot)[:w.k] for _ in range(w.B)]).astype(np.int32)
    idx[2, 0] = -1
    idx[5, 1] = w.E_tot
    idx[11] = [3, 7, 3]
    inp["topk_idx"] = idx
    dev_inp = runner.to_device(inp, dev)
    pipe = runner.Pipeline(w, dev, alias_expert_out=False)
    pipe.layout_dispatch(dev_inp)
    err = pipe.buf.check()
    ref = oracle.layout(gp.ocfg(w), idx)
    assert err == ref["err"] == (oracle.ERR_BAD_ID | oracle.ERR_DUP_ID)
    rep = gp.Report()
    gp.check_layout(rep, w, pipe, ref)
    gp.check_dispatch(rep, w, pipe, inp, ref)
    gp.check_combine(rep, w, pipe, inp, dev_inp, ref)
    rep.assert_ok()


# ----------------------------------------------------------------------------- edge cases


def small(name, **kw):
    base = dict(B=96, d=128, k=4, P=4, M=24, E=16, quant_mode=2)
    base.update(kw)
    return wl.Workload(name, **base)


def test_empty_batch(dev):
    w = small("empty", B=0)
    buf = EPBuffer(w, device=dev)
    idx = torch.empty((0, w.k), dtype=torch.int32, device=dev)
    x = torch.empty((0, w.d), dtype=torch.bfloat16, device=dev)
    wts = torch.empty((0, w.k), dtype=torch.float32, device=dev)
    eo = torch.zeros((w.rows, w.d), dtype=torch.bfloat16, device=dev)
    buf.layout(idx)
    buf.dispatch(x)
    y = buf.combine(eo, idx, wts, ori_x=x)
    assert buf.check() == 0
    assert y.shape == (0, w.d)
    assert int(buf.expert_count.sum()) == 0 and int(buf.expert_offset[-1]) == 0
    assert int(buf.recv_count.abs().sum()) == 0


def test_ragged_dirty_specials(dev):
    """T = 37 (not a warp multiple), d = 272 (17 int8 units), 3 ranks, special
    experts, smooth scale, -1 picks, out-of-range ids and a duplicate id."""
    w = wl.Workload("ragged", B=111, d=272, k=3, P=3, M=40, E=9, n_zero=1, n_copy=1, n_const=1,
                    quant_mode=2, smooth="rand", seed=5)
    inp = wl.generate(w)
    rng = np.random.default_rng(5)
    idx = np.stack([rng.permutation(w.E_tot)[:w.k] for _ in range(w.B)]).astype(np.int32)
    idx[3, 1] = -1
    idx[7, 0] = w.E_tot + 2      # not an expert id
    idx[8, 2] = -9               # not an expert id
    idx[10] = [4, 5, 4]          # routed id 4 twice: the second copy is dropped
    inp["topk_idx"] = idx
    # errors are expected here, so run the steps by hand
    dev_inp = runner.to_device(inp, dev)
    pipe = runner.Pipeline(w, dev, alias_expert_out=False)
    pipe.layout(dev_inp)
    pipe.dispatch(dev_inp)
    err = pipe.buf.check()
    ref = oracle.layout(gp.ocfg(w), idx)
    assert ref["err"] == (oracle.ERR_BAD_ID | oracle.ERR_DUP_ID)
    assert err == ref["err"]
    rep = gp.Report()
    gp.check_layout(rep, w, pipe, ref)
    gp.check_dispatch(rep, w, pipe, inp, ref)
    gp.check_combine(rep, w, pipe, inp, dev_inp, ref)
    rep.assert_ok()


@pytest.mark.parametrize("k,E,P", [(1, 8, 2), (16, 32, 2), (16, 64, 8)])
def test_k_extremes(dev, k, E, P):
    w = wl.Workload("k%d" % k, B=P * 40, d=64, k=k, P=P, M=48, E=E, quant_mode=2, seed=k)
    full_check(w, dev)


def test_max_experts(dev):
    """E = 2048 (the pages' cap on local_expert_num * ranks): the layout kernel
    runs with fewer warps per CTA (shared-memory budget) and several rounds."""
    w = wl.Workload("e2048", B=8 * 600, d=64, k=8, P=8, M=600, E=2048, quant_mode=0, seed=11)
    full_check(w, dev)


def test_many_rounds(dev):
    """2500 tokens per rank: ten 256-token chunks per rank, the last one ragged."""
    w = wl.Workload("rounds", B=2 * 2500, d=32, k=6, P=2, M=2600, E=64, quant_mode=2, seed=12)
    full_check(w, dev)


@pytest.mark.parametrize("d", [16, 32768])
def test_d_extremes(dev, d):
    w = wl.Workload("d%d" % d, B=32, d=d, k=2, P=2, M=16, E=8, quant_mode=2, seed=d)
    full_check(w, dev)
    full_check(w.with_(quant_mode=0, name="d%d_q0" % d), dev)


def test_degenerate_rows(dev):
    """All-zero rows and rows whose 127/amax overflows give q = 0 and scale 0."""
    w = small("degenerate")
    inp = wl.generate(w)
    inp["x"][0] = 0
    inp["x"][5] = 0x0080          # 2^-126 in every element: 127/amax overflows fp32
    inp["x"][6, :] = 0
    inp["x"][6, 3] = 0x8001       # a single negative subnormal
    full_check(w, dev, inp=inp)


def test_all_specials(dev):
    """Copy experts with dyadic weights give x; zero experts and -1 give +0."""
    w = small("specials", n_zero=1, n_copy=1, n_const=1, quant_mode=0)
    inp = wl.generate(w)
    dev_inp = runner.to_device(inp, dev)
    pipe = runner.Pipeline(w, dev)
    idx = np.full((w.B, w.k), w.E + 1, np.int32)              # copy expert everywhere
    wts = np.tile(np.array([0.5, 0.25, 0.125, 0.125], np.float32), (w.B, 1))
    dev_inp["topk_idx"] = torch.from_numpy(idx).to(dev)
    dev_inp["topk_weights"] = torch.from_numpy(wts).to(dev)
    y = pipe.step(dev_inp)
    assert same_as_x(y, dev_inp["x"])
    idx[:] = w.E                                               # zero expert
    idx[:, 1] = -1
    dev_inp["topk_idx"] = torch.from_numpy(idx).to(dev)
    y = pipe.step(dev_inp)
    assert int(y.view(torch.int16).abs().max()) == 0
    assert pipe.buf.check() == 0


def test_mask_rank0_decode(dev):
    """DeepEP issue #84 masking: every pick of rank 0's experts set to -1; rank 0
    then receives nothing and combine ignores the masked picks."""
    w = wl.get("decode")
    inp = wl.generate(w)
    idx = inp["topk_idx"].copy()
    idx[idx // w.L == 0] = -1
    inp["topk_idx"] = idx
    pipe, *_ = full_check(w.with_(name="decode_masked"), dev, inp=inp)
    rc = pipe.buf.recv_count.cpu().numpy().reshape(w.P, w.L, w.P)
    assert rc[0].sum() == 0


@pytest.mark.parametrize("T", [74, 75, 127])
@pytest.mark.parametrize("qm", [1, 2])
def test_dispatch_ragged_batches(dev, T, qm):
    """Decode shape with per-rank batches that are not a power of two (592, 600 and
    1016 tokens over 8 ranks), static and dynamic int8."""
    w = wl.get("decode").with_(name="decode_T%d_q%d" % (T, qm), B=8 * T, M=T, quant_mode=qm,
                               smooth="rand" if qm == 1 else "none")
    full_check(w, dev)


def test_dispatch_rewrites_every_row_on_every_call(dev):
    """With the receive rows and scales overwritten by sentinels before every call,
    each call of ep_dispatch writes every routed row and scale again, bit for bit as
    the first, and the last one matches the oracle."""
    w = wl.get("decode")
    inp = wl.generate(w)
    dev_inp = runner.to_device(inp, dev)
    pipe = runner.Pipeline(w, dev)
    pipe.layout(dev_inp)
    torch.cuda.synchronize()
    dp = pipe.buf.dst_pos.cpu().numpy()
    rows = torch.from_numpy(dp[dp >= 0].astype(np.int64)).to(dev)
    outs = []
    for _ in range(4):
        pipe.buf.recv_x.view(torch.uint8).fill_(0x5A)
        pipe.buf.recv_scale.fill_(float("nan"))
        pipe.buf.token_scale.fill_(float("nan"))
        pipe.dispatch(dev_inp)
        torch.cuda.synchronize()
        outs.append((pipe.buf.recv_x[rows].clone(), pipe.buf.recv_scale[rows].clone(),
                     pipe.buf.token_scale.clone()))
    assert not torch.isnan(outs[0][1]).any() and not torch.isnan(outs[0][2]).any()
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    assert pipe.buf.check() == 0
    # the last call against the oracle
    rep = gp.Report()
    ref = oracle.layout(gp.ocfg(w), inp["topk_idx"], active=inp.get("active"))
    gp.check_dispatch(rep, w, pipe, inp, ref)
    rep.assert_ok()


def test_repeated_calls_are_identical(dev):
    """The layout's ticket counter re-arms itself; a second pass over the same
    inputs reproduces every output bit for bit and raises no error bits."""
    w = wl.get("skewed")
    inp = wl.generate(w)
    dev_inp = runner.to_device(inp, dev)
    pipe = runner.Pipeline(w, dev)
    outs = []
    for _ in range(3):
        pipe.layout(dev_inp)
        pipe.dispatch(dev_inp)
        torch.cuda.synchronize()
        outs.append([t.clone() for t in (pipe.buf.expert_count, pipe.buf.expert_offset,
                                         pipe.buf.recv_count, pipe.buf.dst_pos,
                                         pipe.buf.token_scale)])
    for a, b in zip(outs[0], outs[-1]):
        assert torch.equal(a, b)
    assert pipe.buf.check() == 0


def test_roundtrip_identity_decode_shape_bf16(dev):
    """combine(dispatch(x)) == x with one-hot weights at the decode shape in bf16."""
    w = wl.get("decode").with_(name="decode_q0", quant_mode=0)
    inp = wl.generate(w)
    dev_inp = runner.to_device(inp, dev)
    pipe = runner.Pipeline(w, dev, alias_expert_out=True)
    rng = np.random.default_rng(2)
    onehot = np.zeros((w.B, w.k), np.float32)
    onehot[np.arange(w.B), rng.integers(0, w.k, w.B)] = 1.0
    dev_inp["topk_weights"] = torch.from_numpy(onehot).to(dev)
    y = pipe.step(dev_inp)
    assert same_as_x(y, dev_inp["x"])


# ----------------------------------------------------------------------------- boundaries of the paths


@pytest.mark.parametrize("kw", [dict(layout=1), dict(quant_mode=1, smooth="rand"),
                                dict(smooth="expert"), dict(layout=1, smooth="expert")],
                         ids=["packed", "static", "expert", "packed_expert"])
def test_empty_batch_variants(dev, kw):
    w = small("empty_v", B=0, **kw)
    buf = EPBuffer(w, device=dev)
    idx = torch.empty((0, w.k), dtype=torch.int32, device=dev)
    x = torch.empty((0, w.d), dtype=torch.bfloat16, device=dev)
    wts = torch.empty((0, w.k), dtype=torch.float32, device=dev)
    eo = torch.zeros((w.rows, w.d), dtype=torch.bfloat16, device=dev)
    sm = None
    if w.smooth == "rand":
        sm = torch.ones(w.d, dtype=torch.float32, device=dev)
    elif w.smooth == "expert":
        sm = torch.ones((w.E, w.d), dtype=torch.float32, device=dev)
    buf.layout(idx)
    buf.dispatch(x, sm)
    y = buf.combine(eo, idx, wts, ori_x=x)
    assert buf.check() == 0
    assert y.shape == (0, w.d)
    assert int(buf.expert_count.sum()) == 0 and int(buf.expert_offset[-1]) == 0


@pytest.mark.parametrize("T", [257, 512])
@pytest.mark.parametrize("layout", [0, 1])
def test_chunk_boundaries(dev, T, layout):
    """Tokens per rank just past one 256-token chunk (a one-token last chunk) and
    exactly two chunks, with special experts, a mask and both layouts."""
    w = wl.Workload("chunks_T%d_l%d" % (T, layout), B=3 * T, d=64, k=5, P=3, M=T + 3, E=12,
                    n_zero=1, n_copy=1, n_const=1, quant_mode=2, routing="zipf", zipf_s=0.8,
                    seed=T + layout, layout=layout, active_frac=0.9)
    full_check(w, dev)
    full_check(w.with_(name=w.name + "_fused"), dev, fused=True)
