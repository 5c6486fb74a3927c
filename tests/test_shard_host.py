"""Host-side logic of the multi-GPU form (combine_ep_layout_12_b200/shard.py), on CPU:
the rank-to-slab mapping of receive rows and the count exchange, against the CPU
oracle's single-GPU layout of the same routing.  The exchange also runs over
torch.distributed with the gloo backend at world size 2 (one process per rank), as
it would over NCCL between GPUs."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_12_b200 import shard
from combine_ep_layout_12_b200 import workloads as wl

CASES = {
    "two_ranks": wl.Workload("two_ranks", B=2 * 48, d=16, k=4, P=2, M=48, E=16, quant_mode=0, seed=21),
    "eight_ranks_specials": wl.Workload("eight_ranks_specials", B=8 * 40, d=16, k=6, P=8, M=64, E=32, n_zero=1,
                                        n_copy=1, n_const=1, routing="zipf", seed=22),
}


def _ref(w):
    inp = wl.generate(w, with_x=False)
    cfg = oracle.make_cfg(w.B, w.d, w.k, w.P, w.M, w.E, w.n_zero, w.n_copy, w.n_const, w.quant_mode)
    return inp["topk_idx"], oracle.layout(cfg, inp["topk_idx"])


@pytest.mark.parametrize("name", sorted(CASES))
def test_rows_land_in_the_owner_slab(name):
    """Every routed pick's global row belongs to the slab of the rank that owns its
    expert; slab rows of different ranks never collide; the slabs tile the buffer."""
    w = CASES[name]
    idx, ref = _ref(w)
    n = shard.slab_rows(w)
    assert n * w.P == w.E * w.P * w.M
    seen = set()
    for t in range(w.B):
        for j in range(w.k):
            row = int(ref["dst_pos"][t, j])
            if row < 0:
                continue
            g = int(idx[t, j])
            q, local = shard.owner_of_row(w, row)
            assert q == shard.owner_of_expert(w, g) == g // (w.E // w.P)
            assert 0 <= local < n
            # the local row is (local expert, source rank, slot) in the owner's slab
            le, rest = divmod(local, w.P * w.M)
            assert le == g % (w.E // w.P) and rest // w.M == t // (w.B // w.P)
            assert (q, local) not in seen
            seen.add((q, local))


def _send_counts(w, ref):
    """Rank s's send_count [E]: its routed picks per expert = column s of recv_count."""
    return [torch.from_numpy(np.ascontiguousarray(ref["recv_count"][:, s])) for s in range(w.P)]


@pytest.mark.parametrize("name", sorted(CASES))
def test_local_count_exchange(name):
    w = CASES[name]
    _, ref = _ref(w)
    got = shard.LocalGroup(w.P).exchange_counts(_send_counts(w, ref))
    L = w.E // w.P
    for q in range(w.P):
        assert torch.equal(got[q], torch.from_numpy(ref["recv_count"][q * L:(q + 1) * L, :]))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, name, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w = CASES[name].with_(P=world, B=world * 48, M=48)
        _, ref = _ref(w)
        g = shard.DistGroup()
        assert g.rank == rank and g.world == world
        recv = g.exchange_count(_send_counts(w, ref)[rank], w.P)
        g.barrier()
        L = w.E // w.P
        ok = torch.equal(recv, torch.from_numpy(ref["recv_count"][rank * L:(rank + 1) * L, :]))
        with open(os.path.join(out_dir, "rank%d" % rank), "w") as f:
            f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", sorted(CASES))
def test_gloo_count_exchange_world2(tmp_path, name):
    import torch.multiprocessing as mp
    mp.start_processes(_gloo_worker, args=(2, _free_port(), name, str(tmp_path)), nprocs=2,
                       start_method="spawn", join=True)
    for r in range(2):
        assert (tmp_path / ("rank%d" % r)).read_text() == "ok"
