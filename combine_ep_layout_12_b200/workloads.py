"""Seeded synthetic inputs for MoE dispatch/combine, and the named workloads.

This module only draws inputs: hidden states x, routing ids topk_idx, routing
weights, constant-expert tables and smooth scales.  It holds none of the
dispatch/combine arithmetic, so both the CPU oracle (through the tests) and the
CUDA library can be fed from it without sharing any of the method.

Recipe (all from numpy.random.default_rng streams spawned from one seed):
  x           fp32 N(0, 1), rounded to bf16 (nearest even, by torch's cast)
  topk_idx    "uniform": the k smallest of U(0,1) keys over the E routed experts,
              pick order = ascending key (k distinct experts per token);
              "zipf": k distinct draws without replacement over all E+Z+C+K ids
              with P(id i) proportional to (i+1)^-s (Gumbel top-k), pick order =
              draw order; expert 0 is the hottest.
  weights     softmax (fp64, cast to fp32) of N(0, 1) logits, [B, k]
  a1, a2      U(0, 1) per element, [n_const, d] bf16;  v  N(0, 1), [n_const, d] bf16
  smooth      "none" (absent), "ones" ([d] of 1.0), "rand" (U(0.5, 2) per channel) or
              "expert" (U(0.5, 2) per expert and channel, [E, d])
  active      x_active_mask: absent when active_frac is None, else uint8 [B] with
              each token active with probability active_frac
"""
from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    d: int
    k: int
    P: int
    M: int
    E: int
    n_zero: int = 0
    n_copy: int = 0
    n_const: int = 0
    quant_mode: int = 0
    routing: str = "uniform"
    zipf_s: float = 1.2
    smooth: str = "none"
    seed: int = 0
    layout: int = 0  # 0: low-latency receive rows [E][P*M]; 1: packed rows [B*k]
    active_frac: float = None  # x_active_mask: None = no mask

    @property
    def T(self):
        return self.B // self.P

    @property
    def L(self):
        return self.E // self.P

    @property
    def E_tot(self):
        return self.E + self.n_zero + self.n_copy + self.n_const

    @property
    def smooth_rows(self):
        """Rows of the smooth scale: E for a per-expert scale, else 1."""
        return self.E if self.smooth == "expert" else 1

    @property
    def rows(self):
        """Receive rows: E * P * M (low-latency layout) or B * k (packed layout)."""
        return self.B * self.k if self.layout == 1 else self.E * self.P * self.M

    def with_(self, **kw):
        return replace(self, **kw)


def _sweep(T, qm):
    return Workload(f"sweep_T{T}_q{qm}", B=16 * T, d=7168, k=8, P=16, M=T, E=256, quant_mode=qm)


WORKLOADS = {
    # correctness-only case: one logical rank, 8 experts, top-2
    "tiny_q0": Workload("tiny_q0", B=128, d=256, k=2, P=1, M=128, E=8, quant_mode=0),
    "tiny_q2": Workload("tiny_q2", B=128, d=256, k=2, P=1, M=128, E=8, quant_mode=2,
                        smooth="ones"),
    # DeepSeek-V3-shaped low-latency decode: 8 ranks x 128 tokens, 256 experts, top-8, int8
    "decode": Workload("decode", B=1024, d=7168, k=8, P=8, M=128, E=256, quant_mode=2),
    # the decode kernels on a smaller receive buffer (64 experts: 1.4 GB instead of
    # 5.6 GB of device buffers; same B, d, k and routed rows per launch), used for
    # multi-pass profiler captures
    "decode_e64": Workload("decode_e64", B=1024, d=7168, k=8, P=8, M=128, E=64, quant_mode=2),
    # high-throughput prefill: 8 ranks x 4096 tokens, bf16 payload
    "prefill": Workload("prefill", B=32768, d=7168, k=8, P=8, M=4096, E=256, quant_mode=0),
    # skewed Zipf(1.2) routing over 64 routed + 1 zero + 1 copy + 1 const experts, top-6
    "skewed": Workload("skewed", B=8192, d=4096, k=6, P=8, M=1024, E=64, n_zero=1, n_copy=1,
                       n_const=1, quant_mode=2, routing="zipf", zipf_s=1.2),
}
# per-expert smooth scale [E, d] (one quantization per routed copy), decode shape
WORKLOADS["decode_expert_smooth"] = replace(WORKLOADS["decode"], name="decode_expert_smooth",
                                            smooth="expert")
# the same on the 64-expert receive buffer (1.4 GB), for multi-pass profiler captures
WORKLOADS["decode_e64_expert_smooth"] = replace(WORKLOADS["decode_e64"], name="decode_e64_expert_smooth",
                                                smooth="expert")
# static int8 (quant_mode 1) with a [d] scale, decode shape
WORKLOADS["decode_static"] = replace(WORKLOADS["decode"], name="decode_static", quant_mode=1,
                                     smooth="rand")
# decode with an x_active_mask of 3/4 of the tokens active
WORKLOADS["decode_active"] = replace(WORKLOADS["decode"], name="decode_active", active_frac=0.75)
SWEEP_T = (1, 4, 16, 64, 256, 1024, 4096)
for _T in SWEEP_T:
    for _qm in (0, 2):
        WORKLOADS[f"sweep_T{_T}_q{_qm}"] = _sweep(_T, _qm)
# the same workloads with the packed receive layout (rows contiguous per expert,
# no per-(expert, rank) padding)
for _name in list(WORKLOADS):
    if not _name.startswith("tiny_q0"):
        WORKLOADS[_name + "_packed"] = replace(WORKLOADS[_name], name=_name + "_packed", layout=1)
WORKLOADS["tiny_q0_packed"] = replace(WORKLOADS["tiny_q0"], name="tiny_q0_packed", layout=1)


def get(name):
    return WORKLOADS[name]


def f32_to_bf16_bits(a):
    """Round an fp32 array to bf16 with torch's cast; return the uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _streams(seed):
    ss = np.random.SeedSequence(seed)
    names = ("x", "idx", "w", "const", "smooth", "expert", "active")
    return {n: np.random.default_rng(s) for n, s in zip(names, ss.spawn(len(names)))}


def gen_x(rng, B, d, chunk=4096):
    out = np.empty((B, d), np.uint16)
    for r0 in range(0, B, chunk):
        r1 = min(B, r0 + chunk)
        out[r0:r1] = f32_to_bf16_bits(rng.standard_normal((r1 - r0, d), dtype=np.float32))
    return out


def gen_topk_uniform(rng, B, E, k, chunk=8192):
    out = np.empty((B, k), np.int32)
    for r0 in range(0, B, chunk):
        r1 = min(B, r0 + chunk)
        keys = rng.random((r1 - r0, E))
        part = np.argpartition(keys, k - 1, axis=1)[:, :k]
        order = np.argsort(np.take_along_axis(keys, part, axis=1), axis=1, kind="stable")
        out[r0:r1] = np.take_along_axis(part, order, axis=1)
    return out


def gen_topk_zipf(rng, B, n_ids, k, s):
    logp = -s * np.log(np.arange(1, n_ids + 1, dtype=np.float64))
    u = rng.random((B, n_ids))
    gumbel = -np.log(-np.log(np.clip(u, 1e-300, 1.0)))
    keys = logp[None, :] + gumbel
    order = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    return order.astype(np.int32)


def gen_weights(rng, B, k):
    logits = rng.standard_normal((B, k))
    z = np.exp(logits - logits.max(axis=1, keepdims=True))
    return (z / z.sum(axis=1, keepdims=True)).astype(np.float32)


def generate(w: Workload, with_x=True):
    """All inputs of one workload as numpy arrays (bf16 as uint16 bits)."""
    rs = _streams(w.seed)
    inp = {}
    inp["x"] = gen_x(rs["x"], w.B, w.d) if with_x else None
    if w.routing == "uniform":
        inp["topk_idx"] = gen_topk_uniform(rs["idx"], w.B, w.E, w.k)
    elif w.routing == "zipf":
        inp["topk_idx"] = gen_topk_zipf(rs["idx"], w.B, w.E_tot, w.k, w.zipf_s)
    else:
        raise ValueError(w.routing)
    inp["topk_weights"] = gen_weights(rs["w"], w.B, w.k)
    if w.n_const:
        rc = rs["const"]
        inp["a1"] = f32_to_bf16_bits(rc.random((w.n_const, w.d), dtype=np.float32))
        inp["a2"] = f32_to_bf16_bits(rc.random((w.n_const, w.d), dtype=np.float32))
        inp["v"] = f32_to_bf16_bits(rc.standard_normal((w.n_const, w.d), dtype=np.float32))
    else:
        inp["a1"] = inp["a2"] = inp["v"] = None
    if w.smooth == "none":
        inp["smooth"] = None
    elif w.smooth == "ones":
        inp["smooth"] = np.ones(w.d, np.float32)
    elif w.smooth == "rand":
        inp["smooth"] = rs["smooth"].uniform(0.5, 2.0, w.d).astype(np.float32)
    elif w.smooth == "expert":
        inp["smooth"] = rs["smooth"].uniform(0.5, 2.0, (w.E, w.d)).astype(np.float32)
    else:
        raise ValueError(w.smooth)
    if w.active_frac is None:
        inp["active"] = None
    else:
        inp["active"] = (rs["active"].random(w.B) < w.active_frac).astype(np.uint8)
    return inp


def gen_expert_rows(w: Workload, n_rows, seed_offset=0):
    """Synthetic expert outputs: n_rows rows of d bf16 values, N(0, 1)."""
    rng = np.random.default_rng(np.random.SeedSequence([w.seed, 7919 + seed_offset]))
    return gen_x(rng, n_rows, w.d)
