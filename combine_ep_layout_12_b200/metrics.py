"""Algorithmic byte counts of the three kernels: the minimal traffic the method
must move for one call, not the padded receive buffer.

  layout   : read topk_idx (B*k*4); write dst_pos (B*k*4), recv_src of the routed
             rows (N_r*4), expert_count + expert_offset + recv_count
             ((2*E_tot + 1 + E*P)*4)
  dispatch : read x once (B*d*2) and dst_pos (B*k*4) [+ smooth d*4, or E*d*4 for
             a per-expert smooth scale]; write every routed row (N_r*d*s, s = 1
             int8 / 2 bf16) [+ recv_scale N_r*4, and token_scale B*4 with a
             per-token scale, for dynamic int8 only]
  combine  : read every routed expert row (N_r*d*2), topk_idx + weights + dst_pos
             (B*k*12), ori_x of tokens with a copy/const pick (B_sp*d*2) and the
             const tables (3*K*d*2); write y (B*d*2)

N_r = routed picks that got a receive row; B_sp = tokens with >= 1 copy or const pick.
With an x_active_mask, layout and combine also read it (B bytes each), and N_r and
B_sp count active tokens only.
"""
import numpy as np


def routing_counts(w, topk_idx, n_routed=None, active=None):
    idx = np.asarray(topk_idx)
    if active is not None:
        idx = idx[np.asarray(active) != 0]
    if n_routed is None:
        n_routed = int(((idx >= 0) & (idx < w.E)).sum())
    sp = (idx >= w.E + w.n_zero) & (idx < w.E_tot)
    b_sp = int(sp.any(axis=1).sum()) if idx.size else 0
    return n_routed, b_sp


def kernel_bytes(w, n_routed, b_sp, smooth=False, masked=False):
    B, d, k, E, P = w.B, w.d, w.k, w.E, w.P
    s = 1 if w.quant_mode != 0 else 2
    layout = B * k * 4 + B * k * 4 + n_routed * 4 + (2 * w.E_tot + 1 + E * P) * 4
    dispatch = B * d * 2 + B * k * 4 + n_routed * d * s
    expert = getattr(w, "smooth", "none") == "expert"
    if w.quant_mode == 2:
        dispatch += n_routed * 4 + (0 if (expert and smooth) else B * 4)
    if w.quant_mode != 0 and smooth:
        dispatch += (E if expert else 1) * d * 4
    combine = n_routed * d * 2 + B * k * 12 + b_sp * d * 2 + 3 * w.n_const * d * 2 + B * d * 2
    if masked:
        layout += B
        combine += B
    return {"layout": layout, "dispatch": dispatch, "combine": combine}
