"""Parity harness: run libep on the GPU and compare with the CPU oracle.

Expected values come only from the oracle (or from the seeded input generators);
nothing the GPU computes is fed back into the oracle.  Expert outputs for the
combine check are drawn by the seeded generator and placed at the receive rows
the oracle's layout names, so the GPU combine reads them through its own
dst_pos.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_12_b200 import runner
from combine_ep_layout_12_b200 import workloads as wl

COMBINE_REL_TOL = 8e-3


def ocfg(w, B=None, P=None, M=None, layout=None):
    return oracle.make_cfg(w.B if B is None else B, w.d, w.k, w.P if P is None else P,
                           w.M if M is None else M, w.E, w.n_zero, w.n_copy, w.n_const,
                           w.quant_mode, layout=w.layout if layout is None else layout)


def bf16_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


class Report:
    def __init__(self):
        self.fails = []
        self.notes = {}

    def check(self, cond, msg):
        if not cond:
            self.fails.append(msg)

    def assert_ok(self):
        assert not self.fails, "\n".join(self.fails)


def check_layout(rep, w, pipe, ref):
    buf = pipe.buf
    rep.check(np.array_equal(buf.expert_count.cpu().numpy(), ref["expert_count"]),
              "%s: expert_count differs" % w.name)
    rep.check(np.array_equal(buf.expert_offset.cpu().numpy(), ref["expert_offset"]),
              "%s: expert_offset differs" % w.name)
    rep.check(np.array_equal(buf.recv_count.cpu().numpy(), ref["recv_count"]),
              "%s: recv_count differs" % w.name)
    dp = buf.dst_pos.cpu().numpy()
    rep.check(np.array_equal(dp, ref["dst_pos"]), "%s: dst_pos differs (%d picks)"
              % (w.name, int((dp != ref["dst_pos"]).sum())))
    rows = np.nonzero(ref["recv_src"] >= 0)[0]
    got = buf.recv_src[torch.from_numpy(rows).to(buf.device)].cpu().numpy()
    rep.check(np.array_equal(got, ref["recv_src"][rows]), "%s: recv_src differs" % w.name)


def check_dispatch(rep, w, pipe, inp, ref_lay, sample_picks=None, rng=None):
    """quant_out / scales of the oracle vs the GPU receive rows of routed picks."""
    if w.smooth == "expert" and inp["smooth"] is not None:
        return check_dispatch_expert_smooth(rep, w, pipe, inp, ref_lay, sample_picks, rng)
    cfg = ocfg(w)
    q, ts = oracle.quantize(cfg, inp["x"], inp["smooth"])
    dp = ref_lay["dst_pos"]
    tt, jj = np.nonzero(dp >= 0)
    if sample_picks is not None and tt.size > sample_picks:
        sel = (rng or np.random.default_rng(0)).choice(tt.size, sample_picks, replace=False)
        sel.sort()
        tt, jj = tt[sel], jj[sel]
    rows = dp[tt, jj]
    buf = pipe.buf
    rows_d = torch.from_numpy(rows.astype(np.int64)).to(buf.device)
    got = buf.recv_x[rows_d]
    if w.quant_mode == 1:
        got = got.cpu().numpy()
        bad = np.nonzero(np.any(got != q[tt], axis=1))[0]
        rep.check(bad.size == 0, "%s: static int8 payload differs in %d of %d rows"
                  % (w.name, bad.size, rows.size))
    elif w.quant_mode == 2:
        got = got.cpu().numpy()
        bad = np.nonzero(np.any(got != q[tt], axis=1))[0]
        rep.check(bad.size == 0, "%s: int8 payload differs in %d of %d rows" % (w.name, bad.size, rows.size))
        gs = buf.recv_scale[rows_d].cpu().numpy()
        rep.check(np.array_equal(gs.view(np.uint32), ts[tt].view(np.uint32)),
                  "%s: recv_scale differs" % w.name)
        gts = buf.token_scale.cpu().numpy()
        rep.check(np.array_equal(gts.view(np.uint32), ts.view(np.uint32)),
                  "%s: token_scale differs in %d tokens" % (w.name, int((gts != ts).sum())))
    else:
        got = runner.bf16_bits(got)
        bad = np.nonzero(np.any(got != q[tt], axis=1))[0]
        rep.check(bad.size == 0, "%s: bf16 payload differs in %d of %d rows" % (w.name, bad.size, rows.size))
    rep.notes["dispatch_rows_checked"] = int(rows.size)
    return q, ts


def check_dispatch_expert_smooth(rep, w, pipe, inp, ref_lay, sample_picks=None, rng=None):
    """Per-expert smooth scale: every checked copy against the oracle's per-copy
    quantization, computed on the checked tokens only into compact rows."""
    dp = ref_lay["dst_pos"]
    tt, jj = np.nonzero(dp >= 0)
    if sample_picks is not None and tt.size > sample_picks:
        sel = (rng or np.random.default_rng(0)).choice(tt.size, sample_picks, replace=False)
        sel.sort()
        tt, jj = tt[sel], jj[sel]
    toks, tpos = np.unique(tt, return_inverse=True)
    compact = np.full((toks.size, w.k), -1, np.int32)
    compact[tpos, jj] = np.arange(tt.size, dtype=np.int32)
    sub = ocfg(w, B=toks.size, P=1, M=max(toks.size, 1), layout=0)
    rx, rsc = oracle.dispatch_expert_smooth(sub, inp["x"][toks], inp["smooth"],
                                            inp["topk_idx"][toks], compact, max(tt.size, 1))
    rows_d = torch.from_numpy(dp[tt, jj].astype(np.int64)).to(pipe.buf.device)
    got = pipe.buf.recv_x[rows_d].cpu().numpy()
    bad = np.nonzero(np.any(got != rx[:tt.size], axis=1))[0]
    rep.check(bad.size == 0, "%s: per-expert int8 payload differs in %d of %d rows"
              % (w.name, bad.size, tt.size))
    if w.quant_mode == 2:
        gs = pipe.buf.recv_scale[rows_d].cpu().numpy()
        rep.check(np.array_equal(gs.view(np.uint32), rsc[:tt.size].view(np.uint32)),
                  "%s: per-expert recv_scale differs" % w.name)
    rep.notes["dispatch_rows_checked"] = int(tt.size)
    return rx, rsc


def place_expert_rows(w, pipe, ref_lay, tokens, seed_offset=0):
    """Draw expert outputs for every routed pick of `tokens`, write them to the GPU
    expert_out at the oracle's rows; return the compact rows and compact dst_pos."""
    dp = ref_lay["dst_pos"][tokens]
    routed = dp >= 0
    n = int(routed.sum())
    vals = wl.gen_expert_rows(w, max(n, 1), seed_offset)[:n]
    compact = np.full(dp.shape, -1, np.int32)
    compact[routed] = np.arange(n, dtype=np.int32)
    if n:
        rows_d = torch.from_numpy(dp[routed].astype(np.int64)).to(pipe.device)
        pipe.expert_out[rows_d] = runner.bf16_tensor(vals, pipe.device)
    return vals, compact


def check_combine(rep, w, pipe, inp, dev_inp, ref_lay, tokens=None, seed_offset=0, run=True):
    if tokens is None:
        tokens = np.arange(w.B)
    vals, compact = place_expert_rows(w, pipe, ref_lay, tokens, seed_offset)
    if run:
        torch.cuda.synchronize()
        pipe.combine(dev_inp)
    y_gpu = runner.bf16_bits(pipe.y[torch.from_numpy(tokens).to(pipe.device)])
    sub = ocfg(w, B=len(tokens), P=1, M=max(len(tokens), 1), layout=0)
    idx = inp["topk_idx"][tokens]
    wts = inp["topk_weights"][tokens]
    x = inp["x"][tokens]
    act = None if inp.get("active") is None else inp["active"][tokens]
    y_ref = oracle.combine(sub, vals if vals.shape[0] else None, idx, wts, compact, x,
                           inp["a1"], inp["a2"], inp["v"], active=act)
    compare_combine(rep, w.name, y_gpu, y_ref, idx, wts, compact, vals, x, w)


def compare_combine(rep, name, y_gpu, y_ref, idx, wts, compact, vals, x, w):
    exact = y_gpu == y_ref
    n_diff = int((~exact).sum())
    rep.notes["combine_elements"] = int(exact.size)
    rep.notes["combine_not_bitexact"] = n_diff
    if n_diff == 0:
        return
    # tolerance: |d| <= 8e-3 |y_ref|  or  |d| <= 2^-8 * sum_j |w_j e_j|
    g = bf16_to_f32(y_gpu).astype(np.float64)
    r = bf16_to_f32(y_ref).astype(np.float64)
    mag = np.zeros_like(r)
    E, Z, C = w.E, w.n_zero, w.n_copy
    xf = bf16_to_f32(x).astype(np.float64)
    for j in range(idx.shape[1]):
        gsel = idx[:, j]
        e = np.zeros_like(r)
        routed = compact[:, j] >= 0
        if routed.any():
            e[routed] = bf16_to_f32(vals[compact[routed, j]])
        cp = (gsel >= E + Z) & (gsel < E + Z + C)
        e[cp] = xf[cp]
        mag += np.abs(wts[:, j:j + 1].astype(np.float64) * e)
    ok = (np.abs(g - r) <= COMBINE_REL_TOL * np.abs(r)) | (np.abs(g - r) <= 2.0**-8 * mag)
    rep.check(bool(ok.all()), "%s: combine outside tolerance at %d elements" % (name, int((~ok).sum())))
    rep.check(n_diff == 0, "%s: combine not bit-exact at %d elements (within tolerance: %s)"
              % (name, n_diff, bool(ok.all())))


def same_as_x(y, x):
    """y == x bitwise, except that -0 in x must come back as +0 (an exact sum of
    zeros rounds to +0)."""
    xi = x.view(torch.int16)
    want = torch.where(xi == -32768, torch.zeros_like(xi), xi)
    return torch.equal(y.view(torch.int16), want)


def free_bytes():
    torch.cuda.empty_cache()
    return torch.cuda.mem_get_info()[0]


def need_bytes(w, separate_expert_out):
    rows = w.rows
    esz = 1 if w.quant_mode != 0 else 2
    total = rows * w.d * esz + rows * 4 * (3 if w.quant_mode == 2 else 1)
    if separate_expert_out:
        total += rows * w.d * 2
    total += 2 * w.B * w.d * 2 + 16 * w.B * w.k
    return total


def full_check(w, dev, inp=None, tokens=None, sample_picks=None, separate=True, fused=False,
               alloc=None):
    """Layout + dispatch + combine of one workload against the oracle.  fused: issue
    layout and dispatch as the single ep_layout_dispatch call; alloc: how the
    device arrays are allocated (see EPBuffer)."""
    inp = inp if inp is not None else wl.generate(w)
    if need_bytes(w, separate) > free_bytes() - (4 << 30):
        pytest.skip("%s needs %.1f GB of device memory" % (w.name, need_bytes(w, separate) / 1e9))
    dev_inp = runner.to_device(inp, dev)
    pipe = runner.Pipeline(w, dev, alias_expert_out=not separate, alloc=alloc)
    rep = Report()
    if fused:
        pipe.layout_dispatch(dev_inp)
    else:
        pipe.layout(dev_inp)
        pipe.dispatch(dev_inp)
    err = pipe.buf.check()
    ref = oracle.layout(ocfg(w), inp["topk_idx"], active=inp.get("active"))
    rep.check(err == ref["err"], "%s: device error bits %#x, oracle %#x" % (w.name, err, ref["err"]))
    check_layout(rep, w, pipe, ref)
    check_dispatch(rep, w, pipe, inp, ref, sample_picks=sample_picks)
    check_combine(rep, w, pipe, inp, dev_inp, ref, tokens=tokens)
    err = pipe.buf.check()
    rep.check(err == 0, "%s: error bits after combine %#x" % (w.name, err))
    rep.assert_ok()
    return pipe, dev_inp, inp, ref
