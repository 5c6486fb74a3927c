"""Pins of the CPU oracle: checks of the oracle against things other than itself.

Each pin returns a list of failure messages (empty = the oracle passes).  The
plain test suite asserts every pin passes on the oracle as built; the mutation
test builds deliberately broken copies of the oracle and asserts each one fails
at least one pin, which shows the pins would catch that kind of mistake.

What pins what:
  * bf16 format helpers   -> torch's fp32<->bf16 casts (a library routine)
  * layout                -> pure-Python brute force (tests/brute.py) on the two
                             topk_idx matrices printed in the Ascend CANN
                             "low_latency_dispatch" examples and on random tiny
                             cases; counts read off those printed matrices; the
                             invariants of the layout (sums, injectivity, bound
                             A >= M * P * min(L, K) from the same page's
                             Constraints); the DeepEP issue #84 masking experiment
  * quantization          -> brute force with exact fp32 rounding; closed forms
                             (max |q| = 127, error bound, one-hot rows, ties)
  * scatter               -> brute force
  * combine               -> brute force with an exact fused multiply-add;
                             closed forms (copy expert with dyadic weights gives x,
                             identity expert with one-hot weights gives x, zero
                             experts give 0, a single constant pick gives
                             alpha1 * x + alpha2 * v)
"""
import os
import struct

import numpy as np
import torch

import oracle
from tests import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_topk_fixture(name):
    meta, rows = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line.startswith("# meta:"):
                for kv in line[len("# meta:"):].split():
                    key, val = kv.split("=")
                    meta[key] = int(val)
            elif line and not line.startswith("#"):
                rows.append([int(v) for v in line.split()])
    return np.array(rows, dtype=np.int32), meta


def _bits_f32(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def _torch_bf16(a):
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_to_f32(h):
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------- format


def pin_bf16_format(lib):
    fails = []
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    # ties: low half exactly 0x8000 with both parities of the kept bit, and
    # values just below / above a tie
    hi = rng.integers(0, 2**16, size=4096, dtype=np.uint64).astype(np.uint32)
    ties = np.concatenate([(hi << 16) | 0x8000, (hi << 16) | 0x7FFF, (hi << 16) | 0x8001])
    edge = np.array([0x7F7F8000, 0x7F7F7FFF, 0xFF7F8000, 0x00008000, 0x00018000,
                     0x80008000, 0x7F800000, 0xFF800000, 0, 0x80000000, 0x00000001], np.uint32)
    allb = np.concatenate([bits, ties, edge])
    f = allb.view(np.float32)
    finite_or_inf = ~np.isnan(f)
    got = oracle.f32_to_bf16_array(f[finite_or_inf], lib=lib)
    want = _torch_bf16(f[finite_or_inf])
    bad = np.nonzero(got != want)[0]
    if bad.size:
        i = bad[0]
        fails.append("f32->bf16 differs from torch at %d values, e.g. 0x%08x -> 0x%04x (torch 0x%04x)"
                     % (bad.size, f[finite_or_inf].view(np.uint32)[i], got[i], want[i]))
    nan = np.array([np.nan, -np.nan], np.float32)
    nn = oracle.f32_to_bf16_array(nan, lib=lib)
    if not np.all(np.isnan(_bf16_to_f32(nn))):
        fails.append("f32->bf16 of NaN is not NaN")
    allh = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    tf = torch.from_numpy(allh.view(np.int16)).view(torch.bfloat16).float().numpy()
    for h in (0x0000, 0x3F80, 0xC2FE, 0x0001, 0x7F7F, 0x8000):
        if oracle.bf16_to_f32(h, lib=lib) != tf[h]:
            fails.append("bf16->f32 differs from torch at 0x%04x" % h)
    return fails


# ----------------------------------------------------------------------------- layout


def _compare_layout(name, out, ref, B, k, P, M, E, rows=None):
    fails = []
    ec, rc, dp, rs, err = ref
    if list(out["expert_count"]) != list(ec):
        fails.append("%s: expert_count differs from brute force" % name)
    pre = [0]
    for c in ec:
        pre.append(pre[-1] + c)
    if list(out["expert_offset"]) != pre:
        fails.append("%s: expert_offset is not the exclusive prefix of the counts" % name)
    if out["recv_count"].tolist() != rc:
        fails.append("%s: recv_count differs from brute force" % name)
    if out["dst_pos"].tolist() != dp:
        fails.append("%s: dst_pos differs from brute force" % name)
    want_src = np.full(E * P * M if rows is None else rows, -1, np.int64)
    for row, t in rs.items():
        want_src[row] = t
    if not np.array_equal(out["recv_src"].astype(np.int64), want_src):
        fails.append("%s: recv_src differs from brute force" % name)
    if out["err"] != err:
        fails.append("%s: error bits %#x, brute force %#x" % (name, out["err"], err))
    return fails


def pin_layout_golden(lib):
    fails = []
    for fx in ("ascend_topk_single_operator.txt", "ascend_topk_graph_mode.txt"):
        mat, meta = read_topk_fixture(fx)
        E, Z, C, K, k = meta["E"], meta["n_zero"], meta["n_copy"], meta["n_const"], meta["k"]
        for P in (1, 2, 16):
            for M in (8, 128):
                idx = np.tile(mat, (P, 1))
                B = idx.shape[0]
                cfg = oracle.make_cfg(B, 16, k, P, M, E, Z, C, K, 0)
                out = oracle.layout(cfg, idx, lib=lib)
                ref = brute.layout(idx.tolist(), B, k, P, M, E, Z + C + K)
                fails += _compare_layout("%s P=%d M=%d" % (fx, P, M), out, ref, B, k, P, M, E)
                if int(out["expert_count"].sum()) != B * k:
                    fails.append("%s: counts do not sum to B*k" % fx)
        if fx == "ascend_topk_single_operator.txt":
            # Read off the printed matrix: id 32 (the zero expert) appears once
            # (row 3) and id 33 (the copy expert) three times (rows 3, 5, 7);
            # expert 17 appears in rows 1, 3, 4, 5, 7, 8.
            out = oracle.layout(oracle.make_cfg(8, 16, 8, 1, 8, 32, 1, 1, 0, 0), mat, lib=lib)
            ec = out["expert_count"]
            if (ec[32], ec[33], ec[17]) != (1, 3, 6):
                fails.append("single-operator matrix: counts of ids 32/33/17 are %d/%d/%d, "
                             "the printed matrix has 1/3/6" % (ec[32], ec[33], ec[17]))
            # With P = 16 ranks of 2 local experts, expert 17 lives on rank 8 and
            # token 0 of every rank routes to it at pick 2: rank r's copy lands in
            # row 17*16*M + r*M + 0 of the low-latency buffer.
            M = 8
            idx = np.tile(mat, (16, 1))
            out = oracle.layout(oracle.make_cfg(128, 16, 8, 16, M, 32, 1, 1, 0, 0), idx, lib=lib)
            for r in range(16):
                if out["dst_pos"][r * 8, 2] != 17 * 16 * M + r * M:
                    fails.append("single-operator matrix: rank %d token 0 pick 2 not at the "
                                 "first row of its (expert 17, rank) run" % r)
                    break
    return fails


def pin_layout_random_brute(lib):
    fails = []
    rng = np.random.default_rng(5)
    for trial in range(12):
        P = int(rng.integers(1, 4))
        T = int(rng.integers(1, 7))
        B = P * T
        M = T + int(rng.integers(0, 3))
        L = int(rng.integers(1, 4))
        E = L * P
        Z, C, K = (int(v) for v in rng.integers(0, 2, 3))
        k = int(rng.integers(1, 6))
        E_tot = E + Z + C + K
        dirty = trial % 3 == 0
        if dirty:
            idx = rng.integers(-2, E_tot + 2, size=(B, k)).astype(np.int32)
        else:
            idx = np.stack([rng.permutation(E_tot)[:k] if k <= E_tot else
                            np.concatenate([rng.permutation(E_tot), -np.ones(k - E_tot, int)])
                            for _ in range(B)]).astype(np.int32)
        cfg = oracle.make_cfg(B, 16, k, P, M, E, Z, C, K, 0)
        out = oracle.layout(cfg, idx, lib=lib)
        ref = brute.layout(idx.tolist(), B, k, P, M, E, Z + C + K)
        fails += _compare_layout("random trial %d" % trial, out, ref, B, k, P, M, E)
    # a case built to hit both error kinds at known places
    idx = np.array([[0, 0, 1], [2, -1, 9], [-5, 1, 3]], np.int32)
    cfg = oracle.make_cfg(3, 16, 3, 1, 3, 4, 0, 0, 0, 0)
    out = oracle.layout(cfg, idx, lib=lib)
    if out["err"] != (brute.ERR_BAD_ID | brute.ERR_DUP_ID):
        fails.append("bad/duplicate ids: error bits %#x" % out["err"])
    if out["dst_pos"][0].tolist() != [0 * 3 + 0, -1, 1 * 3 + 0]:
        fails.append("duplicate id: first occurrence must be routed, the second dropped")
    return fails


def pin_layout_packed_brute(lib):
    """Packed rows against the brute force's definition (rows after every pick of a
    lower expert, then after the lower ranks' rows of the same expert)."""
    fails = []
    rng = np.random.default_rng(15)
    for trial in range(10):
        P = int(rng.integers(1, 4))
        T = int(rng.integers(1, 7))
        B = P * T
        L = int(rng.integers(1, 4))
        E = L * P
        Z, C, K = (int(v) for v in rng.integers(0, 2, 3))
        k = int(rng.integers(1, 6))
        E_tot = E + Z + C + K
        if trial % 3 == 0:
            idx = rng.integers(-2, E_tot + 2, size=(B, k)).astype(np.int32)
        else:
            idx = np.stack([np.concatenate([rng.permutation(E_tot), -np.ones(max(0, k - E_tot), int)])[:k]
                            for _ in range(B)]).astype(np.int32)
        cfg = oracle.make_cfg(B, 16, k, P, 0, E, Z, C, K, 0, layout=1)
        out = oracle.layout(cfg, idx, lib=lib)
        ref = brute.layout(idx.tolist(), B, k, P, 0, E, Z + C + K, packed=True)
        fails += _compare_layout("packed trial %d" % trial, out, ref, B, k, P, 0, E, rows=B * k)
    for fx in ("ascend_topk_single_operator.txt", "ascend_topk_graph_mode.txt"):
        mat, meta = read_topk_fixture(fx)
        E, k = meta["E"], meta["k"]
        for P in (1, 16):
            idx = np.tile(mat, (P, 1))
            B = idx.shape[0]
            cfg = oracle.make_cfg(B, 16, k, P, 0, E, meta["n_zero"], meta["n_copy"], 0, 0, layout=1)
            out = oracle.layout(cfg, idx, lib=lib)
            ref = brute.layout(idx.tolist(), B, k, P, 0, E, meta["n_zero"] + meta["n_copy"], packed=True)
            fails += _compare_layout("%s packed P=%d" % (fx, P), out, ref, B, k, P, 0, E, rows=B * k)
    return fails


def packed_invariant_failures(packed, ll, idx, B, k, P, M, E, name=""):
    """Properties of the packed rows, and their relation to the low-latency rows of
    the same routing."""
    fails = []
    T, L = B // P, E // P
    ec, eo, rc = packed["expert_count"], packed["expert_offset"], packed["recv_count"]
    dp, rs = packed["dst_pos"], packed["recv_src"]
    for name_, arr in (("expert_count", "expert_count"), ("expert_offset", "expert_offset"),
                       ("recv_count", "recv_count")):
        if not np.array_equal(packed[arr], ll[arr]):
            fails.append("%s: %s differs between the layouts" % (name, name_))
    ok = dp >= 0
    if not np.array_equal(ok, ll["dst_pos"] >= 0):
        fails.append("%s: routed picks differ between the layouts" % name)
    rows = dp[ok]
    if np.unique(rows).size != rows.size or (rows.size and rows.max() >= eo[E]):
        fails.append("%s: packed rows not a permutation of [0, routed picks)" % name)
    tt = np.repeat(np.arange(B), k).reshape(B, k)
    if not np.array_equal(rs[dp[ok]], tt[ok]):
        fails.append("%s: recv_src[dst_pos[t,j]] != t" % name)
    g = idx[ok]
    r = tt[ok] // T
    base = eo[g] + np.array([rc[gg, :rr].sum() for gg, rr in zip(g, r)], dtype=np.int64)
    ll_slot = ll["dst_pos"][ok] - (g * P * M + r * M)
    if not np.array_equal(rows - base, ll_slot):
        fails.append("%s: packed row - run base differs from the low-latency slot" % name)
    for q in range(P):
        lo, hi = eo[q * L], eo[(q + 1) * L]
        mine = (g // L) == q
        if rows[mine].size and (rows[mine].min() < lo or rows[mine].max() >= hi):
            fails.append("%s: rank %d's rows are not contiguous" % (name, q))
            break
    return fails


def pin_layout_packed_invariants(lib):
    from combine_ep_layout_12_b200 import workloads as wl
    fails = []
    for name in ("decode", "skewed"):
        w = wl.get(name)
        idx = wl.generate(w, with_x=False)["topk_idx"]
        args = (w.B, w.d, w.k, w.P, w.M, w.E, w.n_zero, w.n_copy, w.n_const, w.quant_mode)
        ll = oracle.layout(oracle.make_cfg(*args, layout=0), idx, lib=lib)
        pk = oracle.layout(oracle.make_cfg(*args, layout=1), idx, lib=lib)
        fails += packed_invariant_failures(pk, ll, idx, w.B, w.k, w.P, w.M, w.E, name=name)
    return fails


def layout_invariant_failures(out, idx, B, k, P, M, E, Z=0, C=0, K=0, name=""):
    """Invariants that hold for any valid routing (distinct ids per token)."""
    fails = []
    T = B // P
    L = E // P
    ec, rc, dp, rs = out["expert_count"], out["recv_count"], out["dst_pos"], out["recv_src"]
    n_masked = int((idx == -1).sum())
    if int(ec.sum()) != B * k - n_masked:
        fails.append("%s: sum of expert_count != B*k - #(-1)" % name)
    if not np.array_equal(rc.sum(axis=1), ec[:E]):
        fails.append("%s: sum_r recv_count[g][r] != expert_count[g]" % name)
    if rc.max(initial=0) > T:
        fails.append("%s: recv_count above T" % name)
    routed = dp[dp >= 0]
    if np.unique(routed).size != routed.size:
        fails.append("%s: dst_pos not injective" % name)
    tt = np.repeat(np.arange(B), k).reshape(B, k)
    if not np.array_equal(rs[dp[dp >= 0]], tt[dp >= 0]):
        fails.append("%s: recv_src[dst_pos[t,j]] != t" % name)
    g_of = dp // (P * M)
    r_of = (dp % (P * M)) // M
    slot = dp % M
    ok = dp >= 0
    if not np.array_equal(g_of[ok], idx[ok]):
        fails.append("%s: row of a pick is not in its expert's block" % name)
    if not np.array_equal(r_of[ok], (tt // T)[ok]):
        fails.append("%s: row of a pick is not in its source rank's run" % name)
    if np.any(slot[ok] >= rc[idx[ok], (tt // T)[ok]]):
        fails.append("%s: slot beyond the run's count" % name)
    recv_per_rank = rc.reshape(P, L, P).sum(axis=(1, 2))
    if recv_per_rank.max(initial=0) > M * P * min(L, k):
        fails.append("%s: rows received by a rank exceed M*P*min(L,k)" % name)
    for g in range(E):
        for r in range(P):
            n = rc[g, r]
            run = rs[g * P * M + r * M: g * P * M + r * M + n]
            if n and (np.any(np.diff(run) <= 0) or run.min() < r * T or run.max() >= (r + 1) * T):
                fails.append("%s: run (%d,%d) not ascending source tokens of its rank" % (name, g, r))
                return fails
    return fails


def pin_layout_invariants(lib):
    from combine_ep_layout_12_b200 import workloads as wl
    w = wl.get("decode")
    inp = wl.generate(w, with_x=False)
    cfg = oracle.make_cfg(w.B, w.d, w.k, w.P, w.M, w.E, 0, 0, 0, 2)
    out = oracle.layout(cfg, inp["topk_idx"], lib=lib)
    fails = layout_invariant_failures(out, inp["topk_idx"], w.B, w.k, w.P, w.M, w.E, name="decode")
    if out["err"]:
        fails.append("decode routing flagged as bad")
    return fails


def pin_mask_experiment(lib):
    from combine_ep_layout_12_b200 import workloads as wl
    _, meta = read_topk_fixture("deepep_mask_experiment.txt")
    P, T, E, k = meta["P"], meta["T"], meta["E"], meta["k"]
    B, L = P * T, E // P
    rng = np.random.default_rng(84)
    idx = wl.gen_topk_uniform(rng, B, E, k)
    masked = idx.copy()
    masked[masked // L == meta["masked_rank"]] = -1
    cfg = oracle.make_cfg(B, 16, k, P, T, E, 0, 0, 0, 0)
    out = oracle.layout(cfg, masked, lib=lib)
    fails = layout_invariant_failures(out, masked, B, k, P, T, E, name="masked")
    rc = out["recv_count"].reshape(P, L, P)
    if rc[0].sum() != 0:
        fails.append("masked: rank 0 still receives rows")
    if np.any(rc[1:].sum(axis=(1, 2)) == 0):
        fails.append("masked: another rank receives nothing")
    if np.any(out["dst_pos"][masked == -1] != -1):
        fails.append("masked: a -1 pick got a receive row")
    # combine ignores masked picks: same result as zero weight on them
    d = 16
    x = wl.gen_x(rng, B, d)
    wts = wl.gen_weights(rng, B, k)
    rows = E * P * T
    eo = np.zeros((rows, d), np.uint16)
    ref_full = oracle.layout(cfg, idx, lib=lib)
    vals = wl.gen_x(rng, B * k, d).reshape(B, k, d)
    eo[ref_full["dst_pos"].ravel()] = vals.reshape(B * k, d)
    y_mask = oracle.combine(cfg, eo, masked, wts, out["dst_pos"], lib=lib)
    # reference: every pick routed, masked ones weighted 0; rows via the full layout
    w0 = wts.copy()
    w0[masked == -1] = 0.0
    y_zero = oracle.combine(cfg, eo, idx, w0, ref_full["dst_pos"], lib=lib)
    if not np.array_equal(y_mask, y_zero):
        fails.append("masked: combine differs from zero-weighting the masked picks")
    return fails


# ----------------------------------------------------------------------------- quantization


def pin_quant_brute(lib):
    fails = []
    rng = np.random.default_rng(3)
    B, d = 6, 32
    x = _torch_bf16(rng.standard_normal((B, d)).astype(np.float32))
    x[1] = 0                                      # all-zero row
    x[2] = _torch_bf16(np.full(d, 1e-38, np.float32) * rng.choice([-1, 1], d))  # s overflows
    x[3] = _torch_bf16(rng.standard_normal(d).astype(np.float32) * 1e-30)        # tiny, finite s
    for smooth in (None, np.ones(d, np.float32), rng.uniform(0.5, 2.0, d).astype(np.float32)):
        cfg = oracle.make_cfg(B, d, 1, 1, B, 1, 0, 0, 0, 2)
        q, inv = oracle.quantize(cfg, x, smooth, lib=lib)
        for t in range(B):
            bq, binv = brute.quantize_row(x[t].tolist(), None if smooth is None else smooth.tolist())
            if q[t].tolist() != bq or struct.pack("<f", inv[t]) != struct.pack("<f", binv):
                fails.append("quantize row %d (smooth %s) differs from brute force"
                             % (t, "none" if smooth is None else "set"))
    return fails


def pin_quant_properties(lib):
    fails = []
    rng = np.random.default_rng(4)
    B, d = 256, 512
    x = _torch_bf16(rng.standard_normal((B, d)).astype(np.float32) * rng.uniform(1e-3, 1e3, (B, 1)).astype(np.float32))
    smooth = rng.uniform(0.5, 2.0, d).astype(np.float32)
    cfg = oracle.make_cfg(B, d, 1, 1, B, 1, 0, 0, 0, 2)
    for ss in (None, smooth):
        q, inv = oracle.quantize(cfg, x, ss, lib=lib)
        xf = _bf16_to_f32(x).astype(np.float32)
        if ss is not None:
            xf = (xf * ss[None, :]).astype(np.float32)
        if not np.all(np.abs(q.astype(np.int32)).max(axis=1) == 127):
            fails.append("max |q| != 127 on a non-zero row")
        err = np.abs(xf.astype(np.float64) - q.astype(np.float64) * inv[:, None].astype(np.float64))
        bound = 0.5 * inv[:, None].astype(np.float64) * (1 + 2.0**-22) + np.abs(xf) * 2.0**-22
        if np.any(err > bound):
            fails.append("dequantization error above half a step")
        if np.any((np.sign(q) != np.sign(xf)) & (q != 0)):
            fails.append("sign of q differs from sign of x")
    q1, i1 = oracle.quantize(cfg, x, None, lib=lib)
    q2, i2 = oracle.quantize(cfg, x, np.ones(d, np.float32), lib=lib)
    if not (np.array_equal(q1, q2) and np.array_equal(i1.view(np.uint32), i2.view(np.uint32))):
        fails.append("smooth scale of ones differs from no smooth scale")
    # one-hot rows c * e_i
    xo = np.zeros((4, d), np.uint16)
    cs = [1.0, -3.5, 1e-20, 6.0e4]
    pos = [0, 7, 100, d - 1]
    for r, (c, i) in enumerate(zip(cs, pos)):
        xo[r, i] = _torch_bf16(np.array([c], np.float32))[0]
    cfg4 = oracle.make_cfg(4, d, 1, 1, 4, 1, 0, 0, 0, 2)
    q, inv = oracle.quantize(cfg4, xo, None, lib=lib)
    for r, (c, i) in enumerate(zip(cs, pos)):
        want = np.zeros(d, np.int8)
        want[i] = 127 if c > 0 else -127
        cv = float(_bf16_to_f32(xo[r, i]))
        s = brute.f32(127.0 / abs(cv))
        if not np.array_equal(q[r], want) or inv[r] != brute.f32(1.0 / s):
            fails.append("one-hot row %d wrong" % r)
    zero = oracle.quantize(cfg4, np.zeros((4, d), np.uint16), None, lib=lib)
    if np.any(zero[0] != 0) or np.any(zero[1] != 0):
        fails.append("all-zero row must give q = 0 and scale 0")
    return fails


def pin_quant_ties(lib):
    """amax = 127 makes s = 1 exactly, so q = round(x) and x.5 values are ties."""
    vals = np.array([127.0, 2.5, 3.5, -2.5, 0.5, -0.5, 1.5, -1.5, 126.5, -0.25, 5.0, -127.0],
                    np.float32)
    want = [127, 2, 4, -2, 0, 0, 2, -2, 126, 0, 5, -127]
    cfg = oracle.make_cfg(1, vals.size, 1, 1, 1, 1, 0, 0, 0, 2)
    q, inv = oracle.quantize(cfg, _torch_bf16(vals)[None, :], None, lib=lib)
    fails = []
    if q[0].tolist() != want:
        fails.append("ties: got %s, round-half-to-even gives %s" % (q[0].tolist(), want))
    if inv[0] != 1.0:
        fails.append("ties: scale %r, expected 1" % inv[0])
    return fails


def pin_quant_inv_order(lib):
    """The returned scale is 1/s with s = 127/amax (two roundings), which differs
    from amax/127 for some amax; pick such amax values and check the oracle."""
    cands = []
    for h in range(0x3C00, 0x4400):
        a = brute.bf16_bits_to_float(h)
        s = brute.f32(127.0 / a)
        if brute.f32(1.0 / s) != brute.f32(a / 127.0):
            cands.append(h)
        if len(cands) == 16:
            break
    fails = []
    if not cands:
        return ["no amax found where 1/(127/amax) != amax/127"]
    d = 16
    x = np.zeros((len(cands), d), np.uint16)
    x[:, 3] = cands
    cfg = oracle.make_cfg(len(cands), d, 1, 1, len(cands), 1, 0, 0, 0, 2)
    _, inv = oracle.quantize(cfg, x, None, lib=lib)
    for r, h in enumerate(cands):
        a = brute.bf16_bits_to_float(h)
        if inv[r] != brute.f32(1.0 / brute.f32(127.0 / a)):
            fails.append("scale for amax bits 0x%04x is not 1/(127/amax)" % h)
            break
    return fails


def pin_expert_smooth(lib):
    """Per-expert smooth scale: against the brute force per routed copy, and the
    closed form that identical expert rows reproduce the per-token [d] result."""
    fails = []
    rng = np.random.default_rng(21)
    B, d, k, P, M, E = 10, 32, 3, 2, 5, 6
    idx = np.stack([rng.permutation(E)[:k] for _ in range(B)]).astype(np.int32)
    idx[3, 1] = -1
    x = _torch_bf16(rng.standard_normal((B, d)).astype(np.float32))
    x[4] = 0
    smooth = rng.uniform(0.25, 4.0, (E, d)).astype(np.float32)
    cfg = oracle.make_cfg(B, d, k, P, M, E, 0, 0, 0, 2)
    lay = oracle.layout(cfg, idx, lib=lib)
    rows = E * P * M
    rx, rsc = oracle.dispatch_expert_smooth(cfg, x, smooth, idx, lay["dst_pos"], rows, lib=lib)
    for t in range(B):
        for j in range(k):
            row = lay["dst_pos"][t, j]
            if row < 0:
                continue
            bq, binv = brute.quantize_row(x[t].tolist(), smooth[idx[t, j]].tolist())
            if rx[row].tolist() != bq or struct.pack("<f", rsc[row]) != struct.pack("<f", binv):
                fails.append("expert smooth: copy (%d, %d) differs from brute force" % (t, j))
                return fails
    same = np.tile(smooth[:1], (E, 1))
    rx2, rsc2 = oracle.dispatch_expert_smooth(cfg, x, same, idx, lay["dst_pos"], rows, lib=lib)
    q, ts = oracle.quantize(cfg, x, smooth[0], lib=lib)
    rx3, rsc3 = oracle.dispatch(cfg, q, ts, lay["dst_pos"], rows, lib=lib)
    if not (np.array_equal(rx2, rx3) and np.array_equal(rsc2.view(np.uint32), rsc3.view(np.uint32))):
        fails.append("expert smooth with identical rows differs from the per-token scale")
    return fails


# ----------------------------------------------------------------------------- scatter


def pin_dispatch_brute(lib):
    fails = []
    rng = np.random.default_rng(6)
    B, d, k, P, M, E = 12, 16, 3, 2, 7, 4
    idx = np.stack([rng.permutation(E)[:k] for _ in range(B)]).astype(np.int32)
    idx[2, 1] = -1
    x = _torch_bf16(rng.standard_normal((B, d)).astype(np.float32))
    ec, rc, dp, rs, err = brute.layout(idx.tolist(), B, k, P, M, E, 0)
    rows = E * P * M
    for qm in (0, 2):
        cfg = oracle.make_cfg(B, d, k, P, M, E, 0, 0, 0, qm)
        lay = oracle.layout(cfg, idx, lib=lib)
        q, sc = oracle.quantize(cfg, x, None, lib=lib)
        rx, rsc = oracle.dispatch(cfg, q, sc, lay["dst_pos"], rows, lib=lib)
        for row in range(rows):
            if row in rs:
                t = rs[row]
                if qm == 0:
                    want, wsc = x[t].tolist(), None
                else:
                    want, wsc = brute.quantize_row(x[t].tolist())
                if rx[row].tolist() != want or (qm == 2 and rsc[row] != wsc):
                    fails.append("scatter mode %d: row %d differs from brute force" % (qm, row))
                    break
            elif np.any(rx[row] != 0):
                fails.append("scatter mode %d: row %d written but no pick maps there" % (qm, row))
                break
    return fails


# ----------------------------------------------------------------------------- combine


def pin_combine_brute(lib):
    fails = []
    rng = np.random.default_rng(8)
    for trial in range(4):
        B, d, k, P, M = 8, 12, 4, 2, 5
        E, Z, C, K = 6, 1, 1, 2
        E_tot = E + Z + C + K
        idx = np.stack([rng.permutation(E_tot)[:k] for _ in range(B)]).astype(np.int32)
        idx[0, 1] = -1
        if trial == 3:
            idx[1, 2] = idx[1, 0] if idx[1, 0] < E else 0   # a duplicate routed id
            idx[2, 0] = E_tot + 3                            # not an expert id
        wts = rng.standard_normal((B, k)).astype(np.float32)
        rows = E * P * M
        eo = _torch_bf16(rng.standard_normal((rows, d)).astype(np.float32))
        x = _torch_bf16(rng.standard_normal((B, d)).astype(np.float32))
        a1 = _torch_bf16(rng.random((K, d)).astype(np.float32))
        a2 = _torch_bf16(rng.random((K, d)).astype(np.float32))
        v = _torch_bf16(rng.standard_normal((K, d)).astype(np.float32))
        cfg = oracle.make_cfg(B, d, k, P, M, E, Z, C, K, 0)
        lay = oracle.layout(cfg, idx, lib=lib)
        y = oracle.combine(cfg, eo, idx, wts, lay["dst_pos"], x, a1, a2, v, lib=lib)
        _, _, dp, _, _ = brute.layout(idx.tolist(), B, k, P, M, E, Z + C + K)
        for t in range(B):
            picks = [(int(idx[t, j]), dp[t][j]) for j in range(k)]
            want = brute.combine_token(d, picks, wts[t].tolist(), E, Z, C, K,
                                       lambda r: eo[r].tolist(), x[t].tolist(),
                                       a1.tolist(), a2.tolist(), v.tolist())
            if y[t].tolist() != want:
                fails.append("combine trial %d token %d differs from brute force" % (trial, t))
                break
    return fails


def pin_combine_closed_forms(lib):
    from combine_ep_layout_12_b200 import workloads as wl
    fails = []
    rng = np.random.default_rng(9)
    B, d, k, P, E = 64, 48, 4, 4, 16
    M = B // P
    Z, C, K = 1, 1, 1
    zero_id, copy_id, const_id = E, E + 1, E + 2
    x = wl.gen_x(rng, B, d)
    x[0, :3] = 0x8000   # negative zeros, as the normal sampler can produce
    rows = E * P * M
    # 1. every pick is the copy expert, dyadic weights summing to 1 -> y == x
    cfg = oracle.make_cfg(B, d, k, P, M, E, Z, C, K, 0)
    idx = np.full((B, k), copy_id, np.int32)
    wts = np.tile(np.array([0.5, 0.25, 0.125, 0.125], np.float32), (B, 1))
    a1 = a2 = v = np.zeros((K, d), np.uint16)
    lay = oracle.layout(cfg, idx, lib=lib)
    y = oracle.combine(cfg, None, idx, wts, lay["dst_pos"], x, a1, a2, v, lib=lib)
    # an exact sum of zeros is +0 (round to nearest), so -0 in x comes back as +0
    x_pz = np.where(x == 0x8000, np.uint16(0), x)
    if not np.array_equal(y, x_pz):
        fails.append("copy experts with weights summing to 1 do not return x (-0 as +0)")
    # 2. identity expert, mode 0, one-hot weights -> combine(dispatch(x)) == x
    idx = wl.gen_topk_uniform(rng, B, E, k)
    wts = np.zeros((B, k), np.float32)
    wts[np.arange(B), rng.integers(0, k, B)] = 1.0
    lay = oracle.layout(cfg, idx, lib=lib)
    q, sc = oracle.quantize(cfg, x, None, lib=lib)
    rx, _ = oracle.dispatch(cfg, q, sc, lay["dst_pos"], rows, lib=lib)
    y = oracle.combine(cfg, rx, idx, wts, lay["dst_pos"], x, a1, a2, v, lib=lib)
    if not np.array_equal(y, x_pz):
        fails.append("identity expert with one-hot weights does not return x (-0 as +0)")
    # 3. weights summing to 1 with identity experts -> y close to x
    wts = wl.gen_weights(rng, B, k)
    y = oracle.combine(cfg, rx, idx, wts, lay["dst_pos"], x, a1, a2, v, lib=lib)
    xf, yf = _bf16_to_f32(x), _bf16_to_f32(y)
    if np.any(np.abs(xf - yf) > 2.0**-7 * np.abs(xf) + 1e-30):
        fails.append("identity experts with softmax weights do not return about x")
    # 4. every pick is the zero expert (or masked) -> y == +0
    idx = np.full((B, k), zero_id, np.int32)
    idx[:, 1] = -1
    y = oracle.combine(cfg, rx, idx, wts, np.full((B, k), -1, np.int32), x, a1, a2, v, lib=lib)
    if np.any(y != 0):
        fails.append("zero experts do not give y == 0")
    # 5. a single constant pick with weight 1 -> bf16(a1*x + a2*v), fp32 ops
    a1 = wl.f32_to_bf16_bits(rng.random((K, d), dtype=np.float32))
    a2 = wl.f32_to_bf16_bits(rng.random((K, d), dtype=np.float32))
    v = wl.gen_x(rng, K, d)
    idx = np.full((B, k), -1, np.int32)
    idx[:, 2] = const_id
    wts = np.zeros((B, k), np.float32)
    wts[:, 2] = 1.0
    y = oracle.combine(cfg, None, idx, wts, np.full((B, k), -1, np.int32), x, a1, a2, v, lib=lib)
    e = (_bf16_to_f32(a1[0])[None, :] * _bf16_to_f32(x)).astype(np.float32) + \
        (_bf16_to_f32(a2[0]) * _bf16_to_f32(v[0])).astype(np.float32)[None, :]
    if not np.array_equal(y, _torch_bf16(e.astype(np.float32))):
        fails.append("single constant pick does not give bf16(a1*x + a2*v)")
    # 6. the accumulation is one fused multiply-add per pick.  Pick 0 gives
    # acc = -(1 + 2^-7 + 2^-23) (weight, expert value 1.0); pick 1 has weight
    # 1 + 2^-23 and expert value 1 + 2^-7, whose exact product is
    # 1 + 2^-7 + 2^-23 + 2^-30: fused, acc becomes exactly 2^-30; a separately
    # rounded product would lose the 2^-30 and give 0.
    B1, k1, P1, E1 = 1, 2, 1, 2
    cfg1 = oracle.make_cfg(B1, 8, k1, P1, 1, E1, 0, 0, 0, 0)
    idx1 = np.array([[0, 1]], np.int32)
    lay1 = oracle.layout(cfg1, idx1, lib=lib)
    eo1 = np.zeros((E1 * P1 * 1, 8), np.uint16)
    eo1[lay1["dst_pos"][0, 0]] = 0x3F80            # 1.0
    eo1[lay1["dst_pos"][0, 1]] = 0x3F81            # 1 + 2^-7
    w1 = np.array([[-(1 + 2.0**-7 + 2.0**-23), 1 + 2.0**-23]], np.float32)
    y1 = oracle.combine(cfg1, eo1, idx1, w1, lay1["dst_pos"], lib=lib)
    if not np.all(y1 == _torch_bf16(np.array([2.0**-30], np.float32))[0]):
        fails.append("accumulation is not a fused multiply-add per pick")
    return fails


# ----------------------------------------------------------------------------- x_active_mask


def pin_active_mask(lib):
    """x_active_mask: brute force (inactive tokens not looked at, in low-latency and
    packed rows), the all-ones mask equals no mask, the all-zeros mask routes and
    counts nothing and flags no bad id, and combine gives +0 for inactive tokens
    and, for active ones, what it gives without the mask."""
    fails = []
    rng = np.random.default_rng(31)
    for trial in range(8):
        P = int(rng.integers(1, 4))
        T = int(rng.integers(2, 7))
        B, M = P * T, T + int(rng.integers(0, 2))
        L = int(rng.integers(1, 4))
        E = L * P
        Z, C, K = (int(v) for v in rng.integers(0, 2, 3))
        E_tot = E + Z + C + K
        k = int(rng.integers(1, min(5, E_tot) + 1))
        idx = np.stack([rng.permutation(E_tot)[:k] for _ in range(B)]).astype(np.int32)
        if trial % 2:
            idx[rng.integers(0, B), 0] = E_tot + 1       # a bad id (flagged only if active)
        act = (rng.random(B) < 0.6).astype(np.uint8)
        packed = trial % 4 >= 2
        cfg = oracle.make_cfg(B, 16, k, P, M, E, Z, C, K, 0, layout=int(packed))
        out = oracle.layout(cfg, idx, lib=lib, active=act)
        ref = brute.layout(idx.tolist(), B, k, P, M, E, Z + C + K, packed=packed, active=act.tolist())
        rows = oracle.receive_rows(cfg, lib)
        fails += _compare_layout("active mask trial %d" % trial, out, ref, B, k, P, M, E, rows=rows)
        full = oracle.layout(cfg, idx, lib=lib, active=np.ones(B, np.uint8))
        plain = oracle.layout(cfg, idx, lib=lib)
        if any(not np.array_equal(full[n], plain[n]) for n in ("expert_count", "dst_pos", "recv_src")) \
                or full["err"] != plain["err"]:
            fails.append("active mask of ones differs from no mask (trial %d)" % trial)
        none = oracle.layout(cfg, idx, lib=lib, active=np.zeros(B, np.uint8))
        if none["expert_count"].any() or (none["dst_pos"] != -1).any() or none["err"]:
            fails.append("active mask of zeros still routes, counts or flags (trial %d)" % trial)
        if fails:
            return fails
    # combine
    B, d, k, P, M, E, Z, C, K = 12, 16, 3, 2, 6, 6, 1, 1, 1
    E_tot = E + Z + C + K
    idx = np.stack([rng.permutation(E_tot)[:k] for _ in range(B)]).astype(np.int32)
    act = np.array([1, 0, 1, 1, 0, 1, 0, 1, 1, 0, 1, 1], np.uint8)
    cfg = oracle.make_cfg(B, d, k, P, M, E, Z, C, K, 0)
    lay = oracle.layout(cfg, idx, lib=lib, active=act)
    eo = _torch_bf16(rng.standard_normal((E * P * M, d)).astype(np.float32))
    x = _torch_bf16(rng.standard_normal((B, d)).astype(np.float32))
    a1 = _torch_bf16(rng.random((K, d)).astype(np.float32))
    a2 = _torch_bf16(rng.random((K, d)).astype(np.float32))
    v = _torch_bf16(rng.standard_normal((K, d)).astype(np.float32))
    wts = rng.standard_normal((B, k)).astype(np.float32)
    y = oracle.combine(cfg, eo, idx, wts, lay["dst_pos"], x, a1, a2, v, lib=lib, active=act)
    y0 = oracle.combine(cfg, eo, idx, wts, lay["dst_pos"], x, a1, a2, v, lib=lib)
    if np.any(y[act == 0] != 0):
        fails.append("combine: inactive tokens are not +0")
    if not np.array_equal(y[act == 1], y0[act == 1]):
        fails.append("combine: active tokens differ from the unmasked combine")
    for t in np.nonzero(act)[0][:3]:
        picks = [(int(idx[t, j]), int(lay["dst_pos"][t, j])) for j in range(k)]
        want = brute.combine_token(d, picks, wts[t].tolist(), E, Z, C, K, lambda r: eo[r].tolist(),
                                   x[t].tolist(), a1.tolist(), a2.tolist(), v.tolist())
        if y[t].tolist() != want:
            fails.append("combine: active token %d differs from brute force" % t)
    return fails


# ----------------------------------------------------------------------------- static quantization


def pin_static_quant(lib):
    """quant_mode 1, CastToInt8(CastToFp32(x) * scales): brute force with and
    without scales, exact closed forms (integers, ties, saturation), the per-copy
    form with an [E, d] scale, and the scatter carrying no scale."""
    fails = []
    rng = np.random.default_rng(41)
    B, d = 6, 40
    x = _torch_bf16((rng.standard_normal((B, d)) * 40).astype(np.float32))
    for smooth in (None, rng.uniform(0.25, 4.0, d).astype(np.float32)):
        cfg = oracle.make_cfg(B, d, 1, 1, B, 1, 0, 0, 0, 1)
        q, sc = oracle.quantize(cfg, x, smooth, lib=lib)
        if sc is not None:
            fails.append("static cast returned a scale")
        for t in range(B):
            want = brute.cast_static_row(x[t].tolist(), None if smooth is None else smooth.tolist())
            if q[t].tolist() != want:
                fails.append("static cast row %d (scales %s) differs from brute force"
                             % (t, "none" if smooth is None else "set"))
                return fails
    # integers pass through, x.5 ties go to even, beyond the int8 range saturates
    vals = np.array([0, 1, -1, 2.5, 3.5, -2.5, -0.5, 0.5, 126, 127, 127.5, 128, 300,
                     -128, -128.5, -129, -300, 1.5, -1.5, 64.25], np.float32)
    want = [0, 1, -1, 2, 4, -2, 0, 0, 126, 127, 127, 127, 127, -128, -128, -128, -128, 2, -2, 64]
    cfg = oracle.make_cfg(1, 32, 1, 1, 1, 1, 0, 0, 0, 1)
    xv = np.zeros((1, 32), np.float32)
    xv[0, :vals.size] = vals
    q, _ = oracle.quantize(cfg, _torch_bf16(xv), None, lib=lib)
    if q[0, :vals.size].tolist() != want:
        fails.append("static cast closed forms: got %s, want %s" % (q[0, :vals.size].tolist(), want))
    # a power-of-two scale is exact: q(x, 2^-3) = q(x / 8)
    q8, _ = oracle.quantize(cfg, _torch_bf16(xv), np.full(32, 0.125, np.float32), lib=lib)
    qd, _ = oracle.quantize(cfg, _torch_bf16(xv / 8), None, lib=lib)
    if not np.array_equal(q8, qd):
        fails.append("static cast with scale 2^-3 differs from the cast of x / 8")
    # per-copy with an [E, d] scale, scattered; the scatter carries no scale
    Bp, k, P, E = 8, 3, 2, 6
    M = Bp // P
    idx = np.stack([rng.permutation(E)[:k] for _ in range(Bp)]).astype(np.int32)
    xs = _torch_bf16((rng.standard_normal((Bp, d)) * 30).astype(np.float32))
    sm = rng.uniform(0.25, 4.0, (E, d)).astype(np.float32)
    cfg = oracle.make_cfg(Bp, d, k, P, M, E, 0, 0, 0, 1)
    lay = oracle.layout(cfg, idx, lib=lib)
    rows = E * P * M
    rx, rsc = oracle.dispatch_expert_smooth(cfg, xs, sm, idx, lay["dst_pos"], rows, lib=lib)
    if rsc is not None:
        fails.append("static per-copy dispatch returned scales")
    for t in range(Bp):
        for j in range(k):
            row = lay["dst_pos"][t, j]
            if rx[row].tolist() != brute.cast_static_row(xs[t].tolist(), sm[idx[t, j]].tolist()):
                fails.append("static per-copy row (%d, %d) differs from brute force" % (t, j))
                return fails
    q, _ = oracle.quantize(cfg, xs, sm[2], lib=lib)
    rx2, rs2 = oracle.dispatch(cfg, q, None, lay["dst_pos"], rows, lib=lib)
    if rs2 is not None or rx2.dtype != np.int8:
        fails.append("static scatter: wrong payload type or a scale")
    for t in range(Bp):
        for j in range(k):
            if rx2[lay["dst_pos"][t, j]].tolist() != q[t].tolist():
                fails.append("static scatter: row (%d, %d) is not the token's cast" % (t, j))
                return fails
    return fails


ALL_PINS = [
    pin_bf16_format,
    pin_layout_golden,
    pin_layout_random_brute,
    pin_layout_invariants,
    pin_layout_packed_brute,
    pin_layout_packed_invariants,
    pin_mask_experiment,
    pin_quant_brute,
    pin_quant_properties,
    pin_quant_ties,
    pin_quant_inv_order,
    pin_expert_smooth,
    pin_dispatch_brute,
    pin_combine_brute,
    pin_combine_closed_forms,
    pin_active_mask,
    pin_static_quant,
]
