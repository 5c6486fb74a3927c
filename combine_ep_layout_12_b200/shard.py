"""Expert parallelism across GPUs: one process per GPU, through the ep_shard_* entry
points of include/ep.h (the wide expert parallelism of the Wide-EP blog, getimpala.ai;
the low-latency receive layout of DeepEP issue #84).

Logical rank r holds its own T = B / P tokens and receive slab r: the low-latency
rows of its experts r*L .. r*L+L-1, [L*P*M, d], slab row = global row - r*L*P*M,
where the global row of (expert g, source rank s, slot) is g*P*M + s*M + slot as on
one GPU.  One step of rank r:

  layout     ep_shard_layout: dst_pos [T, k] (global rows) and send_count [E]
  dispatch   ep_shard_dispatch: every routed copy stored straight into the owning
             rank's slab (plain stores over NVLink), with its scale and source token;
             the same kernel performs the count exchange: send_count[q*L:(q+1)*L]
             stored into column r of rank q's recv_count [L, P] (rows of each local
             expert from each source rank)
             (ep_shard_layout_dispatch does layout and dispatch as one call, one grid
             for T <= 128, the way ep_layout_dispatch does on one GPU)
  barrier    every rank's dispatch (rows and counts) is complete before any rank's
             experts read their slab
  experts    the caller's function over this rank's slab (not part of this library)
  barrier    every rank's expert outputs are complete before any rank reads them
  combine    ep_shard_combine: each pick's expert output read from the owner's slab,
             reduced into y [T, d]

Groups: LocalGroup runs the P logical ranks in one process on one GPU (P separate
slab allocations; a barrier is stream order), and DistGroup runs one rank per
process over torch.distributed (the barrier is a one-integer all-reduce, NCCL
between GPUs, gloo on CPU for the host-side tests), mapping the peers' slabs
through CUDA IPC.  exchange_count(s) are the same count exchange as a collective
(all-to-all), for callers whose tables carry no recv_count addresses.  torch
supplies memory, streams and the barriers; every step of the data path runs in
libep's kernels.

dbo(): the Wide-EP blog's dual-batch overlap, two micro-batches on two streams so
that one micro-batch's dispatch runs while the other's experts and combine do.
"""
import torch

from . import _binding as abi


# ----------------------------------------------------------------------------- row arithmetic


def local_experts(cfg):
    return cfg.E // cfg.P


def slab_rows(cfg):
    """Receive rows per rank: L experts x P source ranks x M slots."""
    return local_experts(cfg) * cfg.P * cfg.M


def owner_of_expert(cfg, g):
    """The rank that holds expert g (expert g lives on rank g / L)."""
    return g // local_experts(cfg)


def owner_of_row(cfg, row):
    """(rank, slab row) of a global low-latency receive row."""
    n = slab_rows(cfg)
    return row // n, row - (row // n) * n


def send_slices(cfg, send_count):
    """send_count [E] -> [P, L]: row q is what this rank sends rank q (its picks of
    rank q's experts)."""
    return send_count.reshape(cfg.P, local_experts(cfg))


def split_inputs(cfg, inputs):
    """Device inputs of the whole batch (dict: topk_idx [B, k], topk_weights, x, and the
    optional smooth, a1, a2, v, active) -> a list over ranks of the dicts that
    LocalShards.step takes: rank r's tokens r*T .. r*T+T-1, the shared tables as they are."""
    T = cfg.B // cfg.P
    out = []
    for r in range(cfg.P):
        sl = slice(r * T, (r + 1) * T)
        d = {"topk_idx": inputs["topk_idx"][sl].contiguous(), "topk_weights": inputs["topk_weights"][sl].contiguous(),
             "x": inputs["x"][sl].contiguous(), "smooth": inputs.get("smooth"), "a1": inputs.get("a1"),
             "a2": inputs.get("a2"), "v": inputs.get("v")}
        if inputs.get("active") is not None:
            d["x_active_mask"] = inputs["active"][sl].contiguous()
        out.append(d)
    return out


# ----------------------------------------------------------------------------- groups


class LocalGroup:
    """The P logical ranks of a configuration as objects in one process (one GPU)."""

    def __init__(self, world):
        self.world = world

    def exchange_counts(self, send_counts):
        """send_counts: list over ranks of [E] tensors; returns, per rank q, recv_count
        [L, P] whose column s is rank s's picks of q's experts."""
        P = self.world
        parts = [sc.reshape(P, -1) for sc in send_counts]  # [P(dest), L]
        return [torch.stack([parts[s][q] for s in range(P)], dim=1).contiguous() for q in range(P)]

    def barrier(self, device=None):
        """Stream order already orders every logical rank's work in one process."""


class DistGroup:
    """One rank per process over torch.distributed (backend nccl between GPUs, gloo on
    CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def exchange_count(self, send_count, P):
        """This rank's send_count [E] -> its recv_count [L, P] (one all-to-all)."""
        inp = send_count.reshape(P, -1).contiguous()
        out = torch.empty_like(inp)
        self.dist.all_to_all_single(out, inp, group=self.group)  # out[s] = rank s's row for me
        return out.t().contiguous()

    def barrier(self, device=None):
        t = torch.zeros(1, dtype=torch.int32, device=device)
        self.dist.all_reduce(t, group=self.group)

    def map_peers(self, arrays):
        """Every rank's device arrays (a dict of tensors) as tensors in this process:
        its own, and the peers' mapped through CUDA IPC (same node)."""
        from torch.multiprocessing.reductions import reduce_tensor
        mine = {n: reduce_tensor(t) for n, t in arrays.items() if t is not None}
        everyone = [None] * self.world
        self.dist.all_gather_object(everyone, mine, group=self.group)
        out = []
        for q, h in enumerate(everyone):
            if q == self.rank:
                out.append(dict(arrays))
            else:
                out.append({n: fn(*args) for n, (fn, args) in h.items()})
        return out


# ----------------------------------------------------------------------------- one rank


class Slab:
    """Receive slab of one rank: recv_x [L*P*M, d] (int8, or bf16 in quant_mode 0),
    recv_scale [L*P*M] (quant_mode 2), recv_src [L*P*M] and the bf16 expert outputs
    of the same rows."""

    def __init__(self, cfg, device, expert_out=True):
        n = slab_rows(cfg)
        xdt = torch.int8 if cfg.quant_mode != 0 else torch.bfloat16
        self.recv_x = torch.empty((n, cfg.d), dtype=xdt, device=device)
        self.recv_scale = torch.empty((n,), dtype=torch.float32, device=device) if cfg.quant_mode == 2 else None
        self.recv_src = torch.full((n,), -1, dtype=torch.int32, device=device)
        self.recv_count = torch.zeros((local_experts(cfg), cfg.P), dtype=torch.int32, device=device)
        self.expert_out = torch.empty((n, cfg.d), dtype=torch.bfloat16, device=device) if expert_out else None

    def arrays(self):
        return {"recv_x": self.recv_x, "recv_scale": self.recv_scale, "recv_src": self.recv_src,
                "recv_count": self.recv_count, "expert_out": self.expert_out}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream


class ShardRank:
    """Rank `rank` of a sharded run: its local arrays and the table of every rank's
    slab (`slabs`: a list over ranks of dicts of tensors, from LocalGroup slabs or
    DistGroup.map_peers)."""

    def __init__(self, cfg, rank, slabs, device):
        if not isinstance(cfg, abi.ep_config):
            cfg = abi.make_config(cfg.B, cfg.d, cfg.k, cfg.P, cfg.M, cfg.E, cfg.n_zero, cfg.n_copy,
                                  cfg.n_const, cfg.quant_mode, getattr(cfg, "smooth_rows", 1), 0)
        self.cfg, self.rank, self.device = cfg, rank, torch.device(device)
        T = cfg.B // cfg.P
        self.T = T
        self.dst_pos = torch.empty((T, cfg.k), dtype=torch.int32, device=self.device)
        self.send_count = torch.empty((cfg.E,), dtype=torch.int32, device=self.device)
        self.token_scale = torch.empty((T,), dtype=torch.float32, device=self.device) if cfg.quant_mode == 2 else None
        self.y = torch.empty((T, cfg.d), dtype=torch.bfloat16, device=self.device)
        nbytes = abi.ep_shard_workspace_size(cfg)
        self.workspace = torch.zeros((nbytes,), dtype=torch.uint8, device=self.device)
        self.dispatch_table = abi.make_shard_table(
            rank, [_ptr(s["recv_x"]) for s in slabs], [_ptr(s.get("recv_scale")) for s in slabs],
            [_ptr(s.get("recv_src")) for s in slabs], [_ptr(s.get("recv_count")) for s in slabs])
        self.combine_table = abi.make_shard_table(rank, [_ptr(s["expert_out"]) for s in slabs])
        self._keep = slabs  # the mapped peer tensors must outlive the tables

    def layout(self, topk_idx, x_active_mask=None, stream=None):
        abi.ep_shard_layout(self.cfg, self.rank, _ptr(topk_idx), _ptr(x_active_mask), _ptr(self.dst_pos),
                            _ptr(self.send_count), _ptr(self.workspace), _stream(stream))

    def dispatch(self, x, smooth_scale=None, stream=None):
        """Rows, scales and source tokens into the owners' slabs, and this rank's
        send_count into column `rank` of every owner's recv_count."""
        abi.ep_shard_dispatch(self.cfg, self.dispatch_table, _ptr(x), _ptr(smooth_scale), _ptr(self.dst_pos),
                              _ptr(self.send_count), _ptr(self.token_scale), _ptr(self.workspace),
                              _stream(stream))

    def layout_dispatch(self, topk_idx, x, x_active_mask=None, smooth_scale=None, stream=None):
        """layout and dispatch (with the count exchange) as one call: one grid when
        T <= 128 and k <= 8."""
        abi.ep_shard_layout_dispatch(self.cfg, self.dispatch_table, _ptr(topk_idx), _ptr(x_active_mask), _ptr(x),
                                     _ptr(smooth_scale), _ptr(self.dst_pos), _ptr(self.send_count),
                                     _ptr(self.token_scale), _ptr(self.workspace), _stream(stream))

    def combine(self, topk_idx, topk_weights, x_active_mask=None, ori_x=None, a1=None, a2=None, v=None,
                stream=None):
        abi.ep_shard_combine(self.cfg, self.combine_table, _ptr(topk_idx), _ptr(topk_weights),
                             _ptr(x_active_mask), _ptr(self.dst_pos), _ptr(ori_x), _ptr(a1), _ptr(a2), _ptr(v),
                             _ptr(self.y), _ptr(self.workspace), _stream(stream))
        return self.y

    def check(self, stream=None):
        return abi.ep_shard_check(_ptr(self.workspace), _stream(stream))


class LocalShards:
    """All P logical ranks of one micro-batch in one process on one GPU: P separate
    slab allocations and one ShardRank per rank.  With rank_streams each rank's
    kernels go to a stream of its own, forked from and joined back to the step's
    stream at the two points where ranks meet (after every dispatch, after every
    combine), as P GPUs would run them; otherwise the ranks run in turn."""

    def __init__(self, cfg, device, rank_streams=False, fused=True):
        self.cfg = cfg
        self.fused = fused  # layout and dispatch as one call (ep_shard_layout_dispatch)
        self.group = LocalGroup(cfg.P)
        self.slabs = [Slab(cfg, device) for _ in range(cfg.P)]
        tabs = [s.arrays() for s in self.slabs]
        self.ranks = [ShardRank(cfg, r, tabs, device) for r in range(cfg.P)]
        self.streams = [torch.cuda.Stream(device) for _ in range(cfg.P)] if rank_streams else None

    def _per_rank(self, main, fn):
        """fn(r, stream) for every rank: on `main` in turn, or forked onto the ranks'
        streams and joined back to `main`."""
        if self.streams is None:
            return [fn(r, main) for r in range(self.cfg.P)]
        start = torch.cuda.Event()
        start.record(main)
        out = []
        for r, st in enumerate(self.streams):
            st.wait_event(start)
            with torch.cuda.stream(st):
                out.append(fn(r, st))
            done = torch.cuda.Event()
            done.record(st)
            main.wait_event(done)
        return out

    def step(self, inputs, expert_fn=None, stream=None):
        """One step over per-rank inputs (a list over ranks of dicts with topk_idx,
        topk_weights, x and optional x_active_mask, smooth, a1, a2, v).  expert_fn(slab,
        rank) fills slab.expert_out from the received rows (default: leave it as is).
        Everything, the count exchange and expert_fn included, runs on `stream`
        (default: the current stream)."""
        with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream()):
            return self._step(inputs, expert_fn, stream)

    def _step(self, inputs, expert_fn, stream):
        main = torch.cuda.current_stream()

        def send(r, st):  # rows and counts into the owners' slabs
            rk, inp = self.ranks[r], inputs[r]
            if self.fused:
                rk.layout_dispatch(inp["topk_idx"], inp["x"], inp.get("x_active_mask"), inp.get("smooth"), st)
            else:
                rk.layout(inp["topk_idx"], inp.get("x_active_mask"), st)
                rk.dispatch(inp["x"], inp.get("smooth"), st)

        def receive(r, st):
            rk, inp = self.ranks[r], inputs[r]
            return rk.combine(inp["topk_idx"], inp["topk_weights"], inp.get("x_active_mask"), inp["x"],
                              inp.get("a1"), inp.get("a2"), inp.get("v"), st)

        self._per_rank(main, send)
        self.group.barrier()
        if expert_fn is not None:
            for r, slab in enumerate(self.slabs):
                expert_fn(slab, r)
        self.group.barrier()
        return self._per_rank(main, receive)


class DistShard:
    """This process's rank of a multi-GPU run (one process per GPU): its slab, the
    peers' slabs mapped through CUDA IPC, and its ShardRank."""

    def __init__(self, cfg, device, group=None):
        self.cfg = cfg
        self.group = DistGroup(group)
        self.slab = Slab(cfg, device)
        peers = self.group.map_peers(self.slab.arrays())
        self.rank = ShardRank(cfg, self.group.rank, peers, device)
        self.device = torch.device(device)

    def step(self, inp, expert_fn=None, stream=None):
        """One step over this rank's inputs (dict as in LocalShards.step).  The library
        calls, the collectives and expert_fn all run on `stream` (default: the current
        stream), so each collective is ordered after the kernels it depends on."""
        with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream()):
            return self._step(inp, expert_fn, stream)

    def _step(self, inp, expert_fn, stream):
        rk = self.rank
        rk.layout_dispatch(inp["topk_idx"], inp["x"], inp.get("x_active_mask"), inp.get("smooth"), stream)
        self.group.barrier(self.device)  # every rank's dispatch is complete before the experts read
        if expert_fn is not None:
            expert_fn(self.slab, self.group.rank)
        self.group.barrier(self.device)  # every rank's expert outputs are complete
        return rk.combine(inp["topk_idx"], inp["topk_weights"], inp.get("x_active_mask"), inp["x"],
                          inp.get("a1"), inp.get("a2"), inp.get("v"), stream)


def dbo(shards_a, shards_b, inputs_a, inputs_b, expert_fn=None, streams=None):
    """Two micro-batches with the dual-batch overlap of the Wide-EP blog: micro-batch
    A on streams[0] and B on streams[1], each with its own buffers, so B's layout and
    dispatch run while A's experts and combine run.  Returns (y_a, y_b), lists over
    ranks; the caller synchronizes."""
    if streams is None:
        streams = (torch.cuda.Stream(), torch.cuda.Stream())
    start = torch.cuda.Event()
    start.record(torch.cuda.current_stream())
    out = []
    for sh, inp, st in ((shards_a, inputs_a, streams[0]), (shards_b, inputs_b, streams[1])):
        st.wait_event(start)
        with torch.cuda.stream(st):
            out.append(sh.step(inp, expert_fn, st))
    done = [torch.cuda.Event(), torch.cuda.Event()]
    for ev, st in zip(done, streams):
        ev.record(st)
        torch.cuda.current_stream().wait_event(ev)
    return out[0], out[1]
