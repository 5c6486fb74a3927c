"""Host-side pieces of bench.py (CPU only): the latency/bandwidth fit, the
recorded-traffic lookup and its staleness rule, and the seeded inputs the
measurements are taken on."""
import json
import os

import numpy as np

import bench
from combine_ep_layout_12_b200 import workloads as wl


def test_fit_recovers_latency_and_bandwidth():
    L, bw = 7.5e-6, 6.2e12
    pts = [(v, L + v / bw) for v in (1e5, 1e6, 1e7, 1e8, 1e9)]
    f = bench.fit_latency_bandwidth(pts)
    assert abs(f["L_us"] - 7.5) < 1e-6
    assert abs(f["BW_eff_gbs"] - 6200.0) < 1e-6


def test_recorded_traffic_follows_the_source(tmp_path, monkeypatch):
    doc = {"w": {"combine": {"dram_bytes_per_launch": 123.0, "source_sha": bench.source_hash("combine")},
                 "dispatch": {"dram_bytes_per_launch": 45.0, "source_sha": "0" * 16}}}
    (tmp_path / "traffic.json").write_text(json.dumps(doc))
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    assert bench.recorded_traffic("w", "combine") == 123.0
    assert bench.recorded_traffic("w", "dispatch") is None      # taken on other kernel source
    assert bench.recorded_traffic("other", "combine") is None
    assert bench.recorded_traffic("w", "combine", with_shape=True) == (123.0, "w")
    assert bench.recorded_traffic("w", "dispatch", with_shape=True) == (None, None)


def test_committed_traffic_records_name_known_kernels():
    """Every record of the committed traffic file belongs to a kernel whose sources
    the benchmark hashes, with the bytes, the hash and the workload it was taken on."""
    with open(os.path.join(bench.PROFILES, "traffic.json")) as f:
        doc = json.load(f)
    n = 0
    for wname, recs in doc.items():
        if wname.startswith("_"):
            continue
        for kern, rec in recs.items():
            assert kern in bench.KERNEL_SOURCES, (wname, kern)
            assert rec["dram_bytes_per_launch"] > 0
            assert len(rec["source_sha"]) == 16 and rec["captured_on"]
            n += 1
    assert "layout_dispatch" in doc["decode"]
    assert n >= 10


def test_source_hash_ignores_comments_only():
    """The recorded traffic stays valid across comment edits, not across code edits."""
    base = "int f(int a) {\n  // twice a\n  return 2 * a; /* doubled */\n}\n"
    comment_edit = "int f(int a) {\n  // two times a, reworded\n  return 2 * a;\n}\n"
    code_edit = "int f(int a) {\n  // twice a\n  return 3 * a; /* doubled */\n}\n"
    assert bench.code_text(base) == bench.code_text(comment_edit) == "int f(int a) { return 2 * a; }"
    assert bench.code_text(base) != bench.code_text(code_edit)
    files = {rel: base for rel in bench.KERNEL_SOURCES["combine"]}
    h = bench.source_hash("combine", read=files.__getitem__)
    assert h == bench.source_hash("combine", read={k: comment_edit for k in files}.__getitem__)
    assert h != bench.source_hash("combine", read={k: code_edit for k in files}.__getitem__)


def test_seeded_inputs_are_fixed():
    """The decode inputs every measurement and parity case uses do not drift."""
    inp = wl.generate(wl.get("decode"))
    again = wl.generate(wl.get("decode"))
    assert np.array_equal(inp["x"], again["x"]) and np.array_equal(inp["topk_idx"], again["topk_idx"])
    # every token has k distinct routed experts
    idx = inp["topk_idx"]
    assert idx.min() >= 0 and idx.max() < 256
    assert all(len(set(r)) == 8 for r in idx[:64].tolist())
    w = inp["topk_weights"]
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6) and (w > 0).all()
