"""Loop-level brute force of the same format, for tiny sizes only.

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

An independent restatement of the definitions in ``tq_oracle`` (it imports
nothing from it): the Hadamard matrix is built element by element from the
Sylvester recursion and applied as a dense product, fp16 rounding goes
through Python's ``struct`` half-precision codec, rounding through Python's
``round`` (ties to even), softmax through explicit sums.  Used by
``tests/test_oracle_brute.py`` to catch a slip in either implementation.
"""
from __future__ import annotations

import math
import struct


def sylvester(d):
    """H_d as a list of lists, from H_1 = [1], H_2n = [[H, H], [H, -H]]."""
    h = [[1]]
    while len(h) < d:
        n = len(h)
        nh = [[0] * (2 * n) for _ in range(2 * n)]
        for i in range(n):
            for j in range(n):
                nh[i][j] = h[i][j]
                nh[i][j + n] = h[i][j]
                nh[i + n][j] = h[i][j]
                nh[i + n][j + n] = -h[i][j]
        h = nh
    return h


def to_half(x):
    """Nearest IEEE binary16 value (ties to even) as a Python float."""
    try:
        return struct.unpack("<e", struct.pack("<e", x))[0]
    except OverflowError:
        return math.inf


def rotate(x, signs):
    d = len(signs)
    xs = list(x) + [0.0] * (d - len(x))
    h = sylvester(d)
    c = 1.0 / math.sqrt(d)
    return [sum(h[i][j] * signs[j] * xs[j] for j in range(d)) * c for i in range(d)]


def rotate_inverse(y, signs):
    d = len(signs)
    h = sylvester(d)
    c = 1.0 / math.sqrt(d)
    return [signs[i] * sum(h[i][j] * y[j] for j in range(d)) * c for i in range(d)]


def encode_one(x, signs, S, b_r, b_theta):
    """Returns dict(s16, cr, ct, rn16, bits) for one vector."""
    L = 2 ** b_r - 1
    nt = 2 ** b_theta
    y = rotate(x, signs)
    p = len(y) // 2
    rho = [math.sqrt(y[2 * j] * y[2 * j] + y[2 * j + 1] * y[2 * j + 1]) for j in range(p)]
    th = [math.atan2(y[2 * j + 1], y[2 * j]) for j in range(p)]
    s16 = to_half(max(rho))
    cr, ct = [], []
    for j in range(p):
        if s16 == 0.0:
            cr.append(0)
            ct.append(0)
            continue
        cr.append(min(max(round((rho[j] / s16) * L), 0), L))
        ct.append(round((th[j] * nt) / (2.0 * math.pi)) % nt)
    out = {"s16": s16, "cr": cr, "ct": ct}
    if S is not None:
        r = []
        for j in range(p):
            rh = (cr[j] * s16) / L
            a = (ct[j] * (2.0 * math.pi)) / nt
            r.append(y[2 * j] - rh * math.cos(a))
            r.append(y[2 * j + 1] - rh * math.sin(a))
        out["rn16"] = to_half(math.sqrt(sum(v * v for v in r)))
        out["bits"] = [1 if sum(float(S[i][k]) * r[k] for k in range(len(r))) >= 0.0 else 0
                       for i in range(len(S))]
        out["residual"] = r
    return out


def key_ip(q, signs, S, rec, b_r, b_theta):
    """Estimated <q, k> of one key record."""
    L = 2 ** b_r - 1
    nt = 2 ** b_theta
    qr = rotate(q, signs)
    p = len(rec["cr"])
    acc = 0.0
    for j in range(p):
        a = (rec["ct"][j] * (2.0 * math.pi)) / nt
        acc += qr[2 * j] * rec["cr"][j] * math.cos(a) + qr[2 * j + 1] * rec["cr"][j] * math.sin(a)
    ip = acc * rec["s16"] / L
    if S is not None and "bits" in rec:
        m = len(S)
        corr = 0.0
        for i in range(m):
            sq = sum(float(S[i][k]) * qr[k] for k in range(len(qr)))
            corr += sq * (1.0 if rec["bits"][i] else -1.0)
        ip += rec["rn16"] * math.sqrt(math.pi / 2.0) / m * corr
    return ip


def decode_one_head(q, hot_k, hot_v, cold_k, cold_v, signs, S, b_r, b_theta, sigma):
    """One query head over hot lists of vectors and cold lists of records."""
    d = len(q)
    logits = [sigma * sum(q[i] * k[i] for i in range(d)) for k in hot_k]
    logits += [sigma * key_ip(q, signs, S, rec, b_r, b_theta) for rec in cold_k]
    mx = max(logits)
    e = [math.exp(v - mx) for v in logits]
    tot = sum(e)
    p = [v / tot for v in e]
    nh = len(hot_k)
    o = [0.0] * d
    for t, v in enumerate(hot_v):
        for i in range(d):
            o[i] += p[t] * v[i]
    L = 2 ** b_r - 1
    nt = 2 ** b_theta
    acc = [0.0] * len(signs)
    for t, rec in enumerate(cold_v):
        w = p[nh + t] * rec["s16"] / L
        for j in range(len(rec["cr"])):
            a = (rec["ct"][j] * (2.0 * math.pi)) / nt
            acc[2 * j] += w * rec["cr"][j] * math.cos(a)
            acc[2 * j + 1] += w * rec["cr"][j] * math.sin(a)
    back = rotate_inverse(acc, signs)
    return [o[i] + back[i] for i in range(d)]


def decode_one_head_gated(q, hot_k, hot_v, cold_k, cold_v, signs, S, b_r, b_theta, sigma,
                          threshold):
    """The cold tier is read only when the hot window is empty or its largest
    plain score q.k is below ``threshold``; otherwise one softmax over the
    hot tokens alone.  Returns (output, skipped)."""
    d = len(q)
    best = None
    for k in hot_k:
        sc = 0.0
        for i in range(d):
            sc += q[i] * k[i]
        if best is None or sc > best:
            best = sc
    skipped = best is not None and best >= threshold
    if skipped:
        return decode_one_head(q, hot_k, hot_v, [], [], signs, S, b_r, b_theta, sigma), True
    return decode_one_head(q, hot_k, hot_v, cold_k, cold_v, signs, S, b_r, b_theta, sigma), False


def tc_write_loops(A, k, v, lam, eta):
    """A <- lambda A + eta k v^T, element by element (lists of lists)."""
    d = len(A)
    return [[lam * A[i][j] + eta * k[i] * v[j] for j in range(d)] for i in range(d)]


def tc_read_loops(q, A):
    """r_j = sum_i q_i A_ij."""
    d = len(A)
    return [sum(q[i] * A[i][j] for i in range(d)) for j in range(d)]


def value_estimate_loops(rec, S, b_r, b_theta):
    """One value record with QJL bits, rotated domain: s16/L * c_r (cos, sin)
    per pair plus sqrt(pi/2)/m * rn16 * sum_i S_i (+1 or -1)."""
    L = 2 ** b_r - 1
    nt = 2 ** b_theta
    d = 2 * len(rec["cr"])
    y = [0.0] * d
    for j in range(len(rec["cr"])):
        a = (rec["ct"][j] * (2.0 * math.pi)) / nt
        y[2 * j] = rec["s16"] / L * rec["cr"][j] * math.cos(a)
        y[2 * j + 1] = rec["s16"] / L * rec["cr"][j] * math.sin(a)
    m = len(S)
    c = rec["rn16"] * math.sqrt(math.pi / 2.0) / m
    for i in range(m):
        sgn = 1.0 if rec["bits"][i] else -1.0
        for k in range(d):
            y[k] += c * sgn * float(S[i][k])
    return y
