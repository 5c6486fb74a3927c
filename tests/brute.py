"""Pure-Python brute force for tiny inputs: an implementation of MoE dispatch and
combine that is independent of the C oracle (no shared code, different language,
exact rational arithmetic where rounding matters).  Used only to pin the oracle.

Rounding model (IEEE binary32 / bf16, round to nearest, ties to even):
  * products, sums and quotients of two fp32 numbers are formed in Python floats
    (binary64) and then rounded to binary32 with struct: binary64 carries
    53 >= 2*24 + 2 bits, so this double rounding equals one correct binary32
    rounding for +, -, *, / (Figueroa's bound);
  * a fused multiply-add is evaluated exactly with Fractions and rounded once;
  * fp32 -> bf16 rounds the exact value once with ties to even.

Sources: Ascend CANN "low_latency_dispatch" (Function / Formula, special experts,
Constraints, Example ids) and DeepEP issue #84 (rank of expert g is g // (E / P);
-1 masks a pick).
"""
import math
import struct
from fractions import Fraction

ERR_BAD_ID = 0x1
ERR_DUP_ID = 0x2


def f32(x):
    """Round a Python float (binary64) to the nearest binary32, ties to even."""
    return struct.unpack("<f", struct.pack("<f", x))[0]


def round_binary(x: Fraction, p, emin, emax):
    """Correctly round an exact rational to a binary format with p significand bits."""
    if x == 0:
        return 0.0
    sign = -1.0 if x < 0 else 1.0
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    q = Fraction(2) ** (e - (p - 1))
    m = a / q
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = n * q
    if r >= Fraction(2) ** (emax + 1):
        return sign * math.inf
    if r == 0:
        return math.copysign(0.0, sign)
    return sign * float(r)


def fma32(a, b, c):
    """binary32 fused multiply-add: a*b + c exact, rounded once."""
    exact = Fraction(a) * Fraction(b) + Fraction(c)
    if exact == 0:
        prod_neg = (math.copysign(1.0, a) * math.copysign(1.0, b)) < 0
        both_neg_zero = prod_neg and math.copysign(1.0, c) < 0
        return -0.0 if both_neg_zero else 0.0
    return round_binary(exact, 24, -126, 127)


def bf16_bits_to_float(h):
    return struct.unpack("<f", struct.pack("<I", (int(h) & 0xFFFF) << 16))[0]


def float_to_bf16_bits(f):
    """Round a binary32 value to bf16 (ties to even) and return the bit pattern."""
    if math.isnan(f):
        return 0x7FC0
    if math.isinf(f):
        return 0x7F80 if f > 0 else 0xFF80
    r = round_binary(Fraction(f), 8, -126, 127) if f != 0 else f
    bits = struct.unpack("<I", struct.pack("<f", r))[0]
    return bits >> 16


def layout(topk_idx, B, k, P, M, E, n_special, packed=False, active=None):
    """Returns (expert_count, recv_count[g][r], dst_pos[t][j], recv_src dict row->t, err).
    packed: rows of expert g come after every pick of a lower expert id, and within
    g the rows of rank r after those of lower ranks (contiguous per expert, then
    per rank); otherwise row = g*P*M + r*M + slot.  active: optional per-token
    flags; a token whose flag is false is not looked at."""
    E_tot = E + n_special
    T = B // P
    expert_count = [0] * E_tot
    recv_count = [[0] * P for _ in range(E)]
    dst_pos = [[-1] * k for _ in range(B)]
    recv_src = {}
    err = 0
    def on(t):
        return active is None or bool(active[t])

    for t in range(B):
        r = t // T
        seen = set()
        if not on(t):
            continue
        for j in range(k):
            g = int(topk_idx[t][j])
            if g == -1:
                continue
            if g < -1 or g >= E_tot:
                err |= ERR_BAD_ID
                continue
            if g >= E:
                expert_count[g] += 1
                continue
            if g in seen:
                err |= ERR_DUP_ID
                continue
            seen.add(g)
            # slot = number of earlier tokens of rank r that routed to g
            slot = 0
            for t2 in range(r * T, t):
                row_ids = [int(v) for v in topk_idx[t2]]
                if on(t2) and g in row_ids:
                    slot += 1
            if packed:
                dst_pos[t][j] = (g, r, slot)  # resolved below, once all counts are known
            else:
                row = g * P * M + r * M + slot
                dst_pos[t][j] = row
                recv_src[row] = t
            recv_count[g][r] += 1
            expert_count[g] += 1
    if packed:
        for t in range(B):
            for j in range(k):
                if dst_pos[t][j] == -1:
                    continue
                g, r, slot = dst_pos[t][j]
                lower_experts = sum(expert_count[h] for h in range(g))
                lower_ranks = sum(recv_count[g][q] for q in range(r))
                row = lower_experts + lower_ranks + slot
                dst_pos[t][j] = row
                recv_src[row] = t
    return expert_count, recv_count, dst_pos, recv_src, err


def quantize_row(xbits, smooth=None):
    """Dynamic int8 quantization of one token row; returns (q list, inv)."""
    xf = []
    for i, h in enumerate(xbits):
        v = bf16_bits_to_float(h)
        if smooth is not None:
            v = f32(v * float(smooth[i]))
        xf.append(v)
    amax = max(abs(v) for v in xf)
    if amax == 0.0:
        return [0] * len(xf), 0.0
    s = 127.0 / amax
    if s > 3.4028234663852886e38:
        return [0] * len(xf), 0.0
    s = f32(s)
    if math.isinf(s):
        return [0] * len(xf), 0.0
    q = []
    for v in xf:
        z = round(f32(v * s))  # Python round(): half to even
        q.append(max(-128, min(127, z)))
    return q, f32(1.0 / s)


def cast_static_row(xbits, scales=None):
    """Static int8 cast of one row (quant_mode 1): q = clamp(round_half_even(x * scale))."""
    q = []
    for i, h in enumerate(xbits):
        v = bf16_bits_to_float(h)
        if scales is not None:
            v = f32(v * float(scales[i]))
        q.append(max(-128, min(127, round(v))))
    return q


def combine_token(d, picks, weights, E, Z, C, K, expert_row, ori_row, a1, a2, v):
    """y row (bf16 bits) for one token.  picks = [(g, dst)]; expert_row(dst) -> bf16 bits."""
    out = []
    for i in range(d):
        acc = 0.0
        for (g, dst), w in zip(picks, weights):
            w = float(w)
            if 0 <= g < E:
                if dst < 0:
                    continue
                e = bf16_bits_to_float(expert_row(dst)[i])
            elif E + Z <= g < E + Z + C:
                e = bf16_bits_to_float(ori_row[i])
            elif E + Z + C <= g < E + Z + C + K:
                c = g - E - Z - C
                p1 = f32(bf16_bits_to_float(a1[c][i]) * bf16_bits_to_float(ori_row[i]))
                p2 = f32(bf16_bits_to_float(a2[c][i]) * bf16_bits_to_float(v[c][i]))
                e = f32(p1 + p2)
            else:
                continue
            acc = fma32(w, e, acc)
        out.append(float_to_bf16_bits(acc))
    return out
