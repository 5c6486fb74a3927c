"""Mutation check of the oracle's pins.

Each mutant is the oracle source with one plausible mistake planted in it (a
dropped term, a wrong sign, index, operand, rounding or order), compiled on the
CPU into a scratch directory.  The pins must reject every mutant: a pin set that
let one through would not have caught that mistake in the oracle itself.
Mutants run in child processes, so one that crashes counts as caught.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

from oracle import build as obuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, exact source text, replacement)
MUTANTS = [
    ("scale_amax_over_127", "return 1.0f / s;", "return amax / 127.0f;"),
    ("round_half_away", "float y = nearbyintf(xf[i] * s);", "float y = roundf(xf[i] * s);"),
    ("round_truncate", "float y = nearbyintf(xf[i] * s);", "float y = truncf(xf[i] * s);"),
    ("signed_max_not_abs", "if (a > amax) amax = a;", "if (v > amax) amax = v;"),
    ("smooth_dropped", "if (smooth) v = v * smooth[i];", "(void)smooth;"),
    ("zero_row_scale_one", "return 0.0f;\n    }\n    for", "return 1.0f;\n    }\n    for"),
    ("unfused_accumulate", "acc = fmaf(w, e, acc);", "acc = acc + w * e;"),
    ("const_sign", "e = p1 + p2;", "e = p1 - p2;"),
    ("const_operand", "float p2 = bf16_to_f32(a2[ci * d + i]) * bf16_to_f32(v[ci * d + i]);",
     "float p2 = bf16_to_f32(a1[ci * d + i]) * bf16_to_f32(v[ci * d + i]);"),
    ("const_index", "int64_t ci = g - E - Z - C;", "int64_t ci = g - E - Z - C + (K > 1);"),
    ("zero_copy_swapped", "} else if (g >= E + Z && g < E + Z + C) {",
     "} else if (g >= E && g < E + C) {"),
    ("weights_transposed", "float w = topk_weights[t * k + j];",
     "float w = topk_weights[(j * B + t) % (B * k)];"),
    ("row_rank_expert_swapped", "int64_t row = g * P * M + r * M + slot;",
     "int64_t row = (r * (E / P) + g % (E / P)) * P * M + (g / (E / P)) * M + slot;"),
    ("slot_descending", "int64_t row = g * P * M + r * M + slot;",
     "int64_t row = g * P * M + r * M + (T - 1 - slot);"),
    ("dup_check_off", "for (int64_t jj = 0; jj < j; ++jj)", "for (int64_t jj = 0; jj < 0; ++jj)"),
    ("minus_one_is_bad", "if (g == -1) continue;", "if (g == -7) continue;"),
    ("inclusive_prefix", "expert_offset[g] = (int32_t)run;\n        run += expert_count[g];",
     "run += expert_count[g];\n        expert_offset[g] = (int32_t)run;"),
    ("specials_not_counted", "expert_count[g] += 1;\n                    continue;",
     "continue;"),
    ("bf16_ties_away", "u = u + 0x7fffu + keep_lsb;", "u = u + 0x8000u + 0 * keep_lsb;"),
    ("bf16_truncate", "u = u + 0x7fffu + keep_lsb;", "u = u + 0 * keep_lsb;"),
    ("last_pick_dropped", "for (int64_t j = 0; j < k_t; ++j) {", "for (int64_t j = 0; j < k_t - 1; ++j) {"),
    ("scatter_scale_dropped", "if (c->quant_mode == 2) recv_scale[row] = token_scale[t];",
     "(void)recv_scale;"),
    ("expert_smooth_wrong_row", "smooth + g * d, d, xf", "smooth + ((g + 1) % E) * d, d, xf"),
    ("expert_smooth_token_row", "quantize_row(x + t * d, smooth + g", "quantize_row(x + (t ^ 1) % B * d, smooth + g"),
    ("active_ignored_in_layout", "if (active && !active[t]) {", "if (0 && active && !active[t]) {"),
    ("active_inverted_in_layout", "if (active && !active[t]) {", "if (active && active[t]) {"),
    ("active_slot_counts_inactive", "for (int64_t j = 0; j < k; ++j) dst_pos[t * k + j] = -1;\n                continue;",
     "for (int64_t j = 0; j < k; ++j) dst_pos[t * k + j] = -1;"),
    ("active_ignored_in_combine", "(active && !active[t]) ? 0 : k;", "k;"),
    ("static_round_away", "float y = nearbyintf(v);", "float y = roundf(v);"),
    ("static_scale_dropped", "if (scales) v = v * scales[i];", "(void)scales;"),
    ("static_wraps", "if (y > 127.0f) y = 127.0f;\n        else", "if (y > 127.0f) y = y - 256.0f;\n        else"),
    ("static_copy_first_row", "cast_row_static(x + t * d, smooth + g * d", "cast_row_static(x + t * d, smooth + 0 * g * d"),
    ("packed_rank_prefix_dropped", "for (int64_t rr = 0; rr < r; ++rr) base += recv_count[g * P + rr];",
     "for (int64_t rr = 0; rr < 0; ++rr) base += recv_count[g * P + rr];"),
    ("packed_rank_prefix_inclusive", "for (int64_t rr = 0; rr < r; ++rr) base += recv_count[g * P + rr];",
     "for (int64_t rr = 0; rr < r && rr < P - 1; ++rr) base += recv_count[g * P + rr + (r > 1)];"),
]

RUNNER = r"""
import sys
sys.path.insert(0, {root!r})
import oracle
from tests import oracle_pins
lib = oracle.load({lib!r})
for pin in oracle_pins.ALL_PINS:
    try:
        fails = pin(lib)
    except Exception as exc:  # an exception inside a pin also rejects the mutant
        fails = ["raised %r" % (exc,)]
    if fails:
        print("CAUGHT", pin.__name__, fails[0])
        sys.exit(0)
print("SURVIVED")
sys.exit(1)
"""


def _run_mutant(tmpdir, name, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, "mutation site for %s not found exactly once" % name
    msrc = os.path.join(tmpdir, name + ".c")
    with open(msrc, "w") as f:
        f.write(src.replace(old, new))
    mlib = os.path.join(tmpdir, name + ".so")
    obuild.build(src=msrc, out=mlib, force=True)
    res = subprocess.run([sys.executable, "-c", RUNNER.format(root=ROOT, lib=mlib)],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    return name, res.returncode, (res.stdout + res.stderr)[-400:]


def test_every_mutant_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda m: _run_mutant(tmp, *m), MUTANTS))
    survived = [(n, out) for n, rc, out in results if rc == 1 and "SURVIVED" in out]
    assert not survived, "mutants not caught by any pin: %s" % survived
