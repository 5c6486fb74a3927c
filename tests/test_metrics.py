"""The algorithmic byte counts behind every roofline fraction (CPU only), against
counts worked out by hand for the decode shape and its variants."""
import numpy as np

from combine_ep_layout_12_b200 import metrics
from combine_ep_layout_12_b200 import workloads as wl


def test_decode_bytes():
    w = wl.get("decode")                       # B=1024, d=7168, k=8, P=8, E=256, int8
    b = metrics.kernel_bytes(w, n_routed=8192, b_sp=0, smooth=False)
    B, d, k, E, P, Nr = 1024, 7168, 8, 256, 8, 8192
    assert b["layout"] == B * k * 4 * 2 + Nr * 4 + (2 * E + 1 + E * P) * 4 == 108548
    # x once, dst_pos, int8 rows, a scale per row and per token
    assert b["dispatch"] == B * d * 2 + B * k * 4 + Nr * d + Nr * 4 + B * 4 == 73469952
    # bf16 expert rows, routing (ids, weights, rows), y
    assert b["combine"] == Nr * d * 2 + B * k * 12 + B * d * 2 == 132218880


def test_bf16_and_static_and_smooth_bytes():
    w = wl.get("decode")
    b0 = metrics.kernel_bytes(w.with_(quant_mode=0), 8192, 0)
    assert b0["dispatch"] == 1024 * 7168 * 2 + 1024 * 8 * 4 + 8192 * 7168 * 2
    b1 = metrics.kernel_bytes(w.with_(quant_mode=1, smooth="rand"), 8192, 0, smooth=True)
    assert b1["dispatch"] == 1024 * 7168 * 2 + 1024 * 8 * 4 + 8192 * 7168 + 7168 * 4  # no scales
    be = metrics.kernel_bytes(w.with_(smooth="expert"), 8192, 0, smooth=True)
    # one scale per copy, none per token, the whole [E, d] table read once
    assert be["dispatch"] == 1024 * 7168 * 2 + 1024 * 8 * 4 + 8192 * 7168 + 8192 * 4 + 256 * 7168 * 4


def test_specials_and_mask_bytes():
    w = wl.get("skewed")                       # E=64, Z=C=K=1, k=6, d=4096
    idx = np.array([[0, 1, 2, 3, 64, 65], [66, 1, 2, 3, 4, 5], [-1, 1, 2, 3, 4, 65]], np.int32)
    w3 = w.with_(B=3)
    n_r, b_sp = metrics.routing_counts(w3, idx)
    assert n_r == 4 + 5 + 4 and b_sp == 3        # copy (65) in rows 0 and 2, const (66) in row 1
    n_r, b_sp = metrics.routing_counts(w3, idx, active=np.array([1, 0, 1], np.uint8))
    assert n_r == 8 and b_sp == 2
    b = metrics.kernel_bytes(w3, n_r, b_sp, masked=True)
    d, k = 4096, 6
    assert b["combine"] == n_r * d * 2 + 3 * k * 12 + b_sp * d * 2 + 3 * 1 * d * 2 + 3 * d * 2 + 3
    assert b["layout"] == 3 * k * 8 + n_r * 4 + (2 * 67 + 1 + 64 * 8) * 4 + 3
