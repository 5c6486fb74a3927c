"""Multi-GPU form (ep_shard_* through combine_ep_layout_12_b200/shard.py) on one GPU:
the P logical ranks run in one process, each with its own receive slab in a
separate allocation, reached through the same pointer table a multi-GPU run fills
with CUDA-IPC-mapped peer slabs.  Every rank's layout, dispatch into the owners'
slabs, the count exchange, and every rank's combine reading the owners' slabs are
compared with the CPU oracle's single-GPU definition of the same routing: integer
results and payloads bit for bit, and combine bit for bit (within 8e-3 relative as
the stated bound).  The dual-batch overlap of two micro-batches on two streams must
give exactly the results of the two steps run one after the other."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_12_b200 import runner, shard
from combine_ep_layout_12_b200 import build as ep_build
from combine_ep_layout_12_b200 import workloads as wl
from tests import gpu_parity as gp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ep_build.build()
    torch.cuda.set_device(0)
    return torch.device("cuda", 0)


CASES = {
    "decode": wl.get("decode"),
    "skewed": wl.get("skewed"),  # 1024 tokens per rank: the chunked layout; specials
    "tiny_q0": wl.get("tiny_q0"),
    "static": wl.get("decode_static").with_(B=8 * 96, M=96),
    "active": wl.get("decode_active").with_(B=8 * 64, M=64, d=2048),
    "ragged": wl.Workload("ragged", B=3 * 37, d=272, k=3, P=3, M=40, E=9, n_zero=1, n_copy=1, n_const=1,
                          quant_mode=2, smooth="rand", seed=5),
}


def _per_rank(w, dev_inp):
    return shard.split_inputs(w, dev_inp)


def _expert_rows(w, ref, seed_offset=0):
    """Seeded expert outputs for every routed pick, and per owner rank the slab rows
    and values to place (what an expert computation would write)."""
    dp = ref["dst_pos"]
    routed = dp >= 0
    n = int(routed.sum())
    vals = wl.gen_expert_rows(w, max(n, 1), seed_offset)[:n]
    compact = np.full(dp.shape, -1, np.int32)
    compact[routed] = np.arange(n, dtype=np.int32)
    rows = dp[routed].astype(np.int64)
    per_owner = []
    nrow = shard.slab_rows(w)
    for q in range(w.P):
        sel = (rows // nrow) == q
        per_owner.append((rows[sel] - q * nrow, vals[sel]))
    return vals, compact, per_owner


def _run(w, dev, seed_offset=0, shards=None, stream=None):
    inp = wl.generate(w)
    dev_inp = runner.to_device(inp, dev)
    cfg = gp.ocfg(w)
    ref = oracle.layout(cfg, inp["topk_idx"], active=inp.get("active"))
    vals, compact, per_owner = _expert_rows(w, ref, seed_offset)
    placed = [(torch.from_numpy(r).to(dev), runner.bf16_tensor(v, dev) if len(v) else None) for r, v in per_owner]

    def expert_fn(slab, q):
        rows, v = placed[q]
        if v is not None:
            slab.expert_out[rows] = v

    sh = shards or shard.LocalShards(w, dev)
    ys = sh.step(_per_rank(w, dev_inp), expert_fn, stream)
    return sh, inp, ref, vals, compact, ys


def _check(w, sh, inp, ref, vals, compact, ys):
    rep = gp.Report()
    T = w.B // w.P
    L = w.E // w.P
    nrow = shard.slab_rows(w)
    cfg = gp.ocfg(w)
    q_ref, ts_ref = oracle.quantize(cfg, inp["x"], inp["smooth"])
    torch.cuda.synchronize()
    for r, rk in enumerate(sh.ranks):
        sl = slice(r * T, (r + 1) * T)
        err = rk.check()
        ref_err = oracle.layout(gp.ocfg(w, B=T, P=1, M=w.M), inp["topk_idx"][sl],
                                active=None if inp.get("active") is None else inp["active"][sl])["err"]
        rep.check(err == ref_err, "rank %d: error bits %#x, oracle %#x" % (r, err, ref_err))
        rep.check(np.array_equal(rk.dst_pos.cpu().numpy(), ref["dst_pos"][sl]), "rank %d: dst_pos" % r)
        rep.check(np.array_equal(rk.send_count.cpu().numpy(), ref["recv_count"][:, r]), "rank %d: send_count" % r)
        if w.quant_mode == 2:
            rep.check(np.array_equal(rk.token_scale.cpu().numpy().view(np.uint32), ts_ref[sl].view(np.uint32)),
                      "rank %d: token_scale" % r)
    for q, slab in enumerate(sh.slabs):
        rep.check(np.array_equal(slab.recv_count.cpu().numpy(), ref["recv_count"][q * L:(q + 1) * L]),
                  "slab %d: recv_count" % q)
        rows = np.nonzero(ref["recv_src"][q * nrow:(q + 1) * nrow] >= 0)[0]
        src = ref["recv_src"][q * nrow + rows]
        rows_d = torch.from_numpy(rows.astype(np.int64)).to(slab.recv_x.device)
        rep.check(np.array_equal(slab.recv_src[rows_d].cpu().numpy(), src), "slab %d: recv_src" % q)
        got = slab.recv_x[rows_d]
        got = runner.bf16_bits(got) if w.quant_mode == 0 else got.cpu().numpy()
        rep.check(np.array_equal(got, q_ref[src]), "slab %d: payload" % q)
        if w.quant_mode == 2:
            rep.check(np.array_equal(slab.recv_scale[rows_d].cpu().numpy().view(np.uint32),
                                     ts_ref[src].view(np.uint32)), "slab %d: recv_scale" % q)
    for r, y in enumerate(ys):
        sl = slice(r * T, (r + 1) * T)
        tokens = np.arange(r * T, (r + 1) * T)
        sub = gp.ocfg(w, B=T, P=1, M=max(T, 1), layout=0)
        cr = compact[sl]
        act = None if inp.get("active") is None else inp["active"][sl]
        y_ref = oracle.combine(sub, vals if vals.shape[0] else None, inp["topk_idx"][sl], inp["topk_weights"][sl],
                               cr, inp["x"][sl], inp["a1"], inp["a2"], inp["v"], active=act)
        gp.compare_combine(rep, "%s rank %d" % (w.name, r), runner.bf16_bits(y), y_ref, inp["topk_idx"][sl],
                           inp["topk_weights"][sl], cr, vals, inp["x"][tokens], w)
    rep.assert_ok()


@pytest.mark.parametrize("fused", [True, False], ids=["one_call", "separate_calls"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_shard_step_matches_oracle(dev, name, fused):
    """Layout and dispatch as ep_shard_layout_dispatch (one grid for T <= 128, with the
    count exchange in the layout CTAs) or as ep_shard_layout + ep_shard_dispatch."""
    w = CASES[name]
    if gp.need_bytes(w, True) > gp.free_bytes() - (4 << 30):
        pytest.skip("needs %.1f GB" % (gp.need_bytes(w, True) / 1e9))
    _check(w, *_run(w, dev, shards=shard.LocalShards(w, dev, fused=fused)))


def test_shard_rank_streams(dev):
    """Each rank's kernels on a stream of its own (as P GPUs run them), joined where
    ranks meet: the same results as the ranks in turn."""
    w = CASES["skewed"]
    _check(w, *_run(w, dev, shards=shard.LocalShards(w, dev, rank_streams=True)))


def test_shard_dbo_two_microbatches(dev):
    """Micro-batches A and B (different routing and tokens) on two streams with the
    dual-batch overlap give exactly the results of two sequential steps."""
    wa = wl.get("decode").with_(name="mb_a", B=8 * 64, M=64, seed=31)
    wb = wl.get("decode").with_(name="mb_b", B=8 * 64, M=64, seed=32)
    dev_a = runner.to_device(wl.generate(wa), dev)
    dev_b = runner.to_device(wl.generate(wb), dev)

    def identity_expert(slab, q):
        # expert output = the dequantized received row (rows past the counts are
        # never read by combine)
        slab.expert_out.copy_((slab.recv_x.float() * slab.recv_scale[:, None]).to(torch.bfloat16))

    seq = []
    for w, d in ((wa, dev_a), (wb, dev_b)):
        sh = shard.LocalShards(w, dev)
        ys = sh.step(_per_rank(w, d), identity_expert)
        torch.cuda.synchronize()
        seq.append([y.clone() for y in ys])
    sa, sb = shard.LocalShards(wa, dev), shard.LocalShards(wb, dev)
    ya, yb = shard.dbo(sa, sb, _per_rank(wa, dev_a), _per_rank(wb, dev_b), identity_expert)
    torch.cuda.synchronize()
    for got, want in ((ya, seq[0]), (yb, seq[1])):
        for g, s in zip(got, want):
            assert torch.equal(g, s)


def test_shard_counts_with_empty_batch(dev):
    """Ranks without tokens still perform the count exchange: every owner's recv_count
    column is overwritten with zeros (no stale counts survive), and nothing else runs."""
    w = wl.get("decode").with_(name="empty_shards", B=0, M=16, d=256)
    sh = shard.LocalShards(w, dev)
    for slab in sh.slabs:
        slab.recv_count.fill_(-7)
    k = w.k
    inputs = [{"topk_idx": torch.empty((0, k), dtype=torch.int32, device=dev),
               "topk_weights": torch.empty((0, k), dtype=torch.float32, device=dev),
               "x": torch.empty((0, w.d), dtype=torch.bfloat16, device=dev)} for _ in range(w.P)]
    ys = sh.step(inputs)
    torch.cuda.synchronize()
    for slab in sh.slabs:
        assert int(slab.recv_count.abs().sum()) == 0
    for rk, y in zip(sh.ranks, ys):
        assert rk.check() == 0 and y.shape == (0, w.d)
