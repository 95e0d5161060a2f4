"""fp64 CPU oracle: TurboQuant-style KV compression and decode attention.

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.  The product path
never imports this module.

What it computes, and where each step comes from
------------------------------------------------
Sources are the pages' titles and sections:

* "TurboQuant: kompresja KV-cache w LLM 6 razy bez utraty dokładności",
  section "Zasada działania PolarQuant": rotate the vector at random, map it
  to radius/angle, quantize both.  Section "Kompensacja błędów przez QJL":
  the residual left by PolarQuant is coded with 1 bit per value by a quantized
  Johnson-Lindenstrauss map that preserves inner products.
* "TurboQuant: optimización de memoria para KV caches en inferencia de LLMs",
  section "Flujo de Cuantificación de KV Cache con TurboQuant", steps 2-6:
  polar mapping, polar quantization, QJL error correction, compressed store,
  attention logits computed from the compressed cache.
* "Monarch v3: Paginación KV Inspirada en NES ...", sections "Cómo funciona"
  and "Bucle de Decodificación Simplificado": recent tokens stay in a
  full-precision hot region, older ones are evicted to a compressed cold
  region, attention aggregates both with one softmax.
* "Compresión del caché KV de los LLM a 3 bits: TurboQuant de Google
  Research", section "Aplicaciones más allá de los LLMs": the same codes rank
  database vectors by estimated inner product (vector search).

The pages give an outline only.  The concrete format (randomized Hadamard
rotation from a seed, 2-D pairs coded as uniform radius / angle codes with an
fp16 per-vector scale, m sign bits of S.r for a seeded Gaussian S with an fp16
residual norm, and the logit estimator
``<q, k_hat> + ||r|| * sqrt(pi/2) / m * <S q, sign(S r)>``) is the one the
library implements; every point the pages leave open is a stated reading
(see the READING notes below).

Everything here is float64 NumPy, vectorised only along batch axes, with no
blocking, fusion or reordering beyond what the definitions state.

Parity status: every public function is pinned by ``tests/test_oracle_*.py``
against closed forms, library routines (scipy's Sylvester Hadamard, textbook
softmax attention), invariants, published generator outputs or the
independent loop implementation in ``oracle/brute.py``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

# ---------------------------------------------------------------------------
# Seeded randomness of the method (rotation signs D and QJL matrix S).
#
# READING: the pages only say "random rotation" / "random projection".  Both
# sides draw from one counter-based generator with a published definition:
# the SplitMix64 finalizer (Steele, Lea & Flood, "Fast splittable pseudorandom
# number generators", OOPSLA 2014) applied to a Weyl sequence.
#   rand64(seed, stream, i) = mix64(mix64(seed + stream) + (i + 1) * GAMMA)
# Stream 0 -> rotation signs, stream 1 -> Gaussian QJL entries (Box-Muller,
# first output only, evaluated with the C library's log/cos/sqrt in float64,
# then rounded to float32: the float32 matrix is the canonical S).
# ---------------------------------------------------------------------------

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
STREAM_SIGNS = 0
STREAM_QJL = 1


def mix64(z: int) -> int:
    """SplitMix64 output function (variant 13 constants) on a 64-bit int."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def rand64(seed: int, stream: int, i: int) -> int:
    """i-th 64-bit draw of a stream; counter based, so any draw is direct."""
    base = mix64((seed + stream) & MASK64)
    return mix64((base + (i + 1) * GAMMA) & MASK64)


def rotation_signs(seed: int, d: int) -> np.ndarray:
    """Diagonal of D: +1 when the top bit of draw i (stream 0) is 0, else -1."""
    out = np.empty(d, dtype=np.float64)
    for i in range(d):
        out[i] = -1.0 if (rand64(seed, STREAM_SIGNS, i) >> 63) else 1.0
    return out


def qjl_matrix(seed: int, m: int, d: int) -> np.ndarray:
    """m x d Gaussian QJL matrix S (float32 values, returned as float32).

    Entry k = row * d + col uses draws 2k and 2k+1 of stream 1:
    u1 = ((a >> 11) + 1) * 2^-53 in (0, 1], u2 = (b >> 11) * 2^-53 in [0, 1),
    S_k = float32(sqrt(-2 ln u1) * cos(2 pi u2)).
    """
    out = np.empty(m * d, dtype=np.float32)
    two_pi = 2.0 * math.pi
    scale = 2.0 ** -53
    for k in range(m * d):
        a = rand64(seed, STREAM_QJL, 2 * k)
        b = rand64(seed, STREAM_QJL, 2 * k + 1)
        u1 = ((a >> 11) + 1) * scale
        u2 = (b >> 11) * scale
        out[k] = np.float32(math.sqrt(-2.0 * math.log(u1)) * math.cos(two_pi * u2))
    return out.reshape(m, d)


# ---------------------------------------------------------------------------
# Rotation.  READING: one randomized Sylvester-Hadamard round,
#   R = (1/sqrt(d)) H_d D,  H_1 = [1],  H_2n = [[H_n, H_n], [H_n, -H_n]].
# A vector whose length is not a power of two is zero-padded to the next one.
# ---------------------------------------------------------------------------

def padded_dim(d_in: int) -> int:
    d = 1
    while d < d_in:
        d *= 2
    return d


def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalised Sylvester-ordered Walsh-Hadamard transform, last axis."""
    y = np.array(x, dtype=np.float64, copy=True)
    d = y.shape[-1]
    lead = y.shape[:-1]
    h = 1
    while h < d:
        y = y.reshape(lead + (d // (2 * h), 2, h))
        a = y[..., 0, :]
        b = y[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2)
        h *= 2
    return y.reshape(lead + (d,))


def rotate(x: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """y = (1/sqrt(d)) H_d (signs * x), x zero-padded to len(signs)."""
    d = signs.shape[0]
    x = np.asarray(x, dtype=np.float64)
    if x.shape[-1] < d:
        pad = np.zeros(x.shape[:-1] + (d - x.shape[-1],), dtype=np.float64)
        x = np.concatenate([x, pad], axis=-1)
    return fwht(signs * x) * (1.0 / math.sqrt(d))


def rotate_inverse(y: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """R^T y = (1/sqrt(d)) D H_d y  (H symmetric, D diagonal)."""
    d = signs.shape[0]
    return signs * (fwht(y) * (1.0 / math.sqrt(d)))


# ---------------------------------------------------------------------------
# Encode.  Per vector (K and V alike), in the order the PolarQuant pseudocode
# gives: rotate -> polar -> quantize; then, for keys, QJL on the residual.
# ---------------------------------------------------------------------------

TWO_PI = 2.0 * math.pi
TIE_EPS = 1e-6
# residual norms below this fraction of ||y|| are float64 noise
DEGENERATE_RESIDUAL = 1e-9


def fp16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 to the nearest fp16 (ties to even), returned as float64."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def fp16_margin(x: np.ndarray) -> np.ndarray:
    """Relative distance of x from the nearest fp16 rounding midpoint.

    A value within TIE_EPS of a midpoint may legitimately round either way
    in another precision; such decisions are ties.
    """
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
        h = x.astype(np.float16)
        v = h.astype(np.float64)
        toward = np.where(v > x, np.float16(-np.inf), np.float16(np.inf)).astype(np.float16)
        other = np.nextafter(h, toward).astype(np.float64)
        mid = 0.5 * (v + other)
        m = np.abs(x - mid) / np.abs(x)
    m = np.where(v == x, np.inf, m)
    m = np.where(np.isfinite(v), m, np.inf)
    return m


def half_margin(t: np.ndarray) -> np.ndarray:
    """Distance of t from the nearest half-integer (a rounding boundary)."""
    return np.abs(t - np.floor(t) - 0.5)


@dataclass
class Codes:
    """Canonical (unpacked) record of N encoded vectors of padded length d.

    s16, rn16 are the fp16 values as float64; cr/ct are int64 [N, d/2];
    bits is uint8 [N, m] (1 means (S r)_i >= 0).  ``tie_*`` flag decisions
    that fell within TIE_EPS of a boundary; ``vec_tie`` marks vectors whose
    scale or any code was a tie, so that their residual-derived fields
    (rn16, bits) are exempt from bit-exact comparison.
    """
    b_r: int
    b_theta: int
    s16: np.ndarray
    cr: np.ndarray
    ct: np.ndarray
    rn16: Optional[np.ndarray] = None
    bits: Optional[np.ndarray] = None
    range_error: Optional[np.ndarray] = None
    tie_s16: Optional[np.ndarray] = None
    tie_cr: Optional[np.ndarray] = None
    tie_ct: Optional[np.ndarray] = None
    tie_rn16: Optional[np.ndarray] = None
    tie_bits: Optional[np.ndarray] = None
    vec_tie: Optional[np.ndarray] = None
    residual: Optional[np.ndarray] = None
    rotated: Optional[np.ndarray] = None


def dequant_unit(cr: np.ndarray, ct: np.ndarray, b_theta: int) -> np.ndarray:
    """'Unit' reconstruction c_r * (cos th_hat, sin th_hat), pairs interleaved.

    th_hat = c_theta * 2 pi / 2^b_theta.  The scale s16 / (2^b_r - 1) is left
    out; callers apply it (the logit estimator factors it per token).
    """
    n_t = 1 << b_theta
    th = (np.asarray(ct, dtype=np.float64) * TWO_PI) / n_t
    c = np.asarray(cr, dtype=np.float64)
    out = np.empty(c.shape[:-1] + (2 * c.shape[-1],), dtype=np.float64)
    out[..., 0::2] = c * np.cos(th)
    out[..., 1::2] = c * np.sin(th)
    return out


def dequant(cr: np.ndarray, ct: np.ndarray, s16: np.ndarray, b_r: int,
            b_theta: int) -> np.ndarray:
    """Rotated-domain reconstruction y_hat: rho_hat (cos th_hat, sin th_hat).

    rho_hat = c_r * s16 / (2^b_r - 1) (evaluated as (c_r * s16) / L).
    """
    L = (1 << b_r) - 1
    n_t = 1 << b_theta
    rho_hat = (np.asarray(cr, dtype=np.float64) * np.asarray(s16, dtype=np.float64)[..., None]) / L
    th = (np.asarray(ct, dtype=np.float64) * TWO_PI) / n_t
    out = np.empty(rho_hat.shape[:-1] + (2 * rho_hat.shape[-1],), dtype=np.float64)
    out[..., 0::2] = rho_hat * np.cos(th)
    out[..., 1::2] = rho_hat * np.sin(th)
    return out


def encode(x: np.ndarray, signs: np.ndarray, S: Optional[np.ndarray], b_r: int,
           b_theta: int, keep_intermediates: bool = False) -> Codes:
    """Encode vectors x [N, d_in] (any float dtype, widened exactly to fp64).

    Steps (PolarQuant pseudocode, then QJL on the residual):
      1. y = R x (randomized Hadamard, zero padding to d = len(signs)).
      2. pairs (y_2j, y_2j+1) -> rho_j = sqrt(y_2j^2 + y_2j+1^2),
         theta_j = atan2(y_2j+1, y_2j) in (-pi, pi].
      3. s = max_j rho_j, s16 = fp16(s).  fp16 overflow -> range_error.
      4. radius code (endpoint grid, READING): t = rho / s16 * (2^b_r - 1),
         c_r = clamp(round_half_even(t), 0, 2^b_r - 1).
      5. angle code (periodic grid through 0, READING):
         t = theta * 2^b_theta / (2 pi), c_theta = round_half_even(t) mod 2^b_theta.
         When s16 == 0 both codes are 0 (the radius grid is degenerate).
      6. residual r = y - y_hat, rn16 = fp16(||r||_2),
         bit_i = [(S r)_i >= 0]  (a zero projection gives bit 1).   (S given)
    """
    x = np.asarray(x, dtype=np.float64)
    if x.ndim != 2:
        raise ValueError("x must be [N, d_in]")
    d = signs.shape[0]
    if x.shape[1] > d:
        raise ValueError("d_in larger than the rotation size")
    L = (1 << b_r) - 1
    n_t = 1 << b_theta

    y = rotate(x, signs)
    y0 = y[:, 0::2]
    y1 = y[:, 1::2]
    rho = np.sqrt(y0 * y0 + y1 * y1)
    theta = np.arctan2(y1, y0)

    s = rho.max(axis=1)
    s16 = fp16_round(s)
    range_error = ~np.isfinite(s16)
    s16 = np.where(range_error, 0.0, s16)
    zero = s16 == 0.0

    safe = np.where(zero, 1.0, s16)
    t_r = (rho / safe[:, None]) * L
    cr = np.clip(np.rint(t_r), 0, L).astype(np.int64)
    t_t = (theta * n_t) / TWO_PI
    ct = np.mod(np.rint(t_t).astype(np.int64), n_t)
    cr[zero] = 0
    ct[zero] = 0

    tie_s16 = fp16_margin(s) < TIE_EPS
    tie_cr = (half_margin(t_r) < TIE_EPS) & ~zero[:, None]
    tie_ct = (half_margin(t_t) < TIE_EPS) & ~zero[:, None]
    vec_tie = tie_s16 | tie_cr.any(axis=1) | tie_ct.any(axis=1)

    codes = Codes(b_r=b_r, b_theta=b_theta, s16=s16, cr=cr, ct=ct,
                  range_error=range_error, tie_s16=tie_s16, tie_cr=tie_cr,
                  tie_ct=tie_ct, vec_tie=vec_tie)
    if keep_intermediates:
        codes.rotated = y

    if S is not None:
        S64 = np.asarray(S, dtype=np.float32).astype(np.float64)
        if S64.shape[1] != d:
            raise ValueError("S must be [m, d]")
        r = y - dequant(cr, ct, s16, b_r, b_theta)
        rn = np.sqrt(np.sum(r * r, axis=1))
        rn16 = fp16_round(rn)
        proj = r @ S64.T
        bits = (proj >= 0.0).astype(np.uint8)
        row_norm = np.sqrt(np.sum(S64 * S64, axis=1))
        with np.errstate(divide="ignore", invalid="ignore"):
            marg = np.abs(proj) / (row_norm[None, :] * rn[:, None])
        # A residual at the level of float64 rounding noise of y carries no
        # decision at all: every sign and its norm are ties (READING).
        ynorm = np.sqrt(np.sum(y * y, axis=1))
        degenerate = (rn <= DEGENERATE_RESIDUAL * ynorm) & (rn > 0)
        marg = np.where(rn[:, None] > 0, marg, 0.0)
        marg = np.where(degenerate[:, None], 0.0, marg)
        codes.rn16 = rn16
        codes.bits = bits
        codes.tie_rn16 = (fp16_margin(rn) < TIE_EPS) | degenerate
        codes.tie_bits = marg < TIE_EPS
        if keep_intermediates:
            codes.residual = r
    return codes


# ---------------------------------------------------------------------------
# Canonical byte packing (for byte-for-byte comparison with the library's
# export): pair j's word w_j = (c_r << b_theta) | c_theta sits LSB-first at
# bit offset j * (b_r + b_theta) of a little-endian bit stream; sign bit i at
# bit offset i of its own stream; s16 / rn16 as raw IEEE fp16 bits.
# ---------------------------------------------------------------------------

def pack_codes(cr: np.ndarray, ct: np.ndarray, b_theta: int, b_r: int) -> np.ndarray:
    """[N, P] codes -> [N, ceil(P * bw / 8)] uint8 canonical bit stream."""
    bw = b_r + b_theta
    cr = np.asarray(cr, dtype=np.int64)
    ct = np.asarray(ct, dtype=np.int64)
    n, p = cr.shape
    words = (cr << b_theta) | ct
    bits = np.zeros((n, p * bw), dtype=np.uint8)
    for b in range(bw):
        bits[:, b::bw] = (words >> b) & 1
    return np.packbits(bits, axis=1, bitorder="little")


def unpack_codes(packed: np.ndarray, p: int, b_r: int, b_theta: int):
    """Inverse of pack_codes: returns (cr, ct) int64 [N, P]."""
    bw = b_r + b_theta
    bits = np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=1,
                         bitorder="little")[:, : p * bw].astype(np.int64)
    words = np.zeros((bits.shape[0], p), dtype=np.int64)
    for b in range(bw):
        words |= bits[:, b::bw] << b
    return words >> b_theta, words & ((1 << b_theta) - 1)


def pack_bits(bits: np.ndarray) -> np.ndarray:
    return np.packbits(np.asarray(bits, dtype=np.uint8), axis=1, bitorder="little")


def unpack_bits(packed: np.ndarray, m: int) -> np.ndarray:
    return np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=1,
                         bitorder="little")[:, :m]


# ---------------------------------------------------------------------------
# Estimators.
# ---------------------------------------------------------------------------

QJL_CONST = math.sqrt(math.pi / 2.0)


def qjl_estimate(q_rot: np.ndarray, S: np.ndarray, bits: np.ndarray, rn: np.ndarray) -> np.ndarray:
    """rn * sqrt(pi/2) / m * <S q', 2 bits - 1>  (estimates <q', r>).

    q_rot: [..., d]; bits [N, m]; rn [N].  Returns [..., N].
    """
    S64 = np.asarray(S, dtype=np.float32).astype(np.float64)
    m = S64.shape[0]
    qq = np.asarray(q_rot, dtype=np.float64) @ S64.T            # [..., m]
    sg = 2.0 * np.asarray(bits, dtype=np.float64) - 1.0          # [N, m]
    return (qq @ sg.T) * (np.asarray(rn, dtype=np.float64) * (QJL_CONST / m))


def key_inner_products(q: np.ndarray, signs: np.ndarray, S: Optional[np.ndarray],
                       codes: Codes) -> np.ndarray:
    """Estimated <q, k> for every encoded key (no softmax scale).

    <q, k_hat> is computed in the rotated domain, where R is orthogonal:
    <q, R^T y_hat> = <R q, y_hat> = s16 / (2^b_r - 1) * <q', y_hat_unit>;
    the QJL term is added when the record carries sign bits.
    """
    L = (1 << codes.b_r) - 1
    q_rot = rotate(q, signs)                                   # [..., d]
    unit = dequant_unit(codes.cr, codes.ct, codes.b_theta)     # [N, d]
    ip = (q_rot @ unit.T) * (codes.s16 / L)
    if S is not None and codes.bits is not None:
        ip = ip + qjl_estimate(q_rot, S, codes.bits, codes.rn16)
    return ip


# ---------------------------------------------------------------------------
# Decode attention over hot (fp16, exact) and cold (compressed) tokens.
# ---------------------------------------------------------------------------

def decode_attention(q: np.ndarray, hot_k: np.ndarray, hot_v: np.ndarray,
                     cold_k: Optional[Codes], cold_v: Optional[Codes],
                     signs: np.ndarray, S: Optional[np.ndarray],
                     num_kv_heads: int, softmax_scale: Optional[float] = None) -> np.ndarray:
    """Single-token decode attention for one batch row.

    q      [Hq, d]            query of the new token
    hot_k  [Hkv, W, d]        hot (full precision) keys   (W may be 0)
    hot_v  [Hkv, W, d]        hot values
    cold_k list-like per kv head of Codes (keys, with QJL) or None
    cold_v list-like per kv head of Codes (values) or None
    Query head h reads kv head h // (Hq / Hkv).  softmax_scale defaults to
    1/sqrt(d) (READING: the pages never state it).

    Logits: hot  l = sigma <q, k>;
            cold l = sigma [ s16/(2^b_r-1) <q', y_hat_unit>
                             + rn16 sqrt(pi/2)/m <S q', 2 bits - 1> ].
    p = softmax over hot U cold (one softmax, max-subtracted);
    o = sum_hot p v + R^T ( sum_cold p * s16_v/(2^b_r-1) * v_hat_unit ).
    """
    q = np.asarray(q, dtype=np.float64)
    hq, d = q.shape
    g = hq // num_kv_heads
    sigma = (1.0 / math.sqrt(d)) if softmax_scale is None else float(softmax_scale)
    out = np.zeros((hq, d), dtype=np.float64)
    for h in range(hq):
        kvh = h // g
        logits = []
        if hot_k is not None and hot_k.shape[1] > 0:
            kh = np.asarray(hot_k[kvh], dtype=np.float64)
            logits.append(sigma * (kh @ q[h]))
        n_cold = 0
        if cold_k is not None and cold_k[kvh] is not None and cold_k[kvh].s16.shape[0] > 0:
            ck = cold_k[kvh]
            n_cold = ck.s16.shape[0]
            logits.append(sigma * key_inner_products(q[h], signs, S, ck))
        lg = np.concatenate(logits) if logits else np.zeros(0)
        if lg.size == 0:
            continue
        mx = lg.max()
        p = np.exp(lg - mx)
        p = p / p.sum()
        n_hot = lg.size - n_cold
        o = np.zeros(d, dtype=np.float64)
        if n_hot:
            o += p[:n_hot] @ np.asarray(hot_v[kvh], dtype=np.float64)
        if n_cold:
            cv = cold_v[kvh]
            L = (1 << cv.b_r) - 1
            unit = dequant_unit(cv.cr, cv.ct, cv.b_theta)
            acc = (p[n_hot:] * (cv.s16 / L)) @ unit
            o += rotate_inverse(acc, signs)
        out[h] = o
    return out


def hot_gate(q: np.ndarray, hot_k: np.ndarray, num_kv_heads: int, threshold: float) -> np.ndarray:
    """Which query heads skip the cold tier (Monarch v3 page, section "Bucle
    de Decodificación Simplificado": the cold pages are read only while the
    largest hot score q.k stays below a threshold).

    READINGS: the score is the plain product q.k over the hot window (the
    loop computes it before any softmax scale); a head with an empty hot
    window always reads the cold tier.  Returns a bool per query head, True
    where max_t q.k_t >= threshold over a non-empty hot window.
    """
    q = np.asarray(q, dtype=np.float64)
    hq = q.shape[0]
    g = hq // num_kv_heads
    skip = np.zeros(hq, dtype=bool)
    if hot_k is None or hot_k.shape[1] == 0:
        return skip
    for h in range(hq):
        scores = np.asarray(hot_k[h // g], dtype=np.float64) @ q[h]
        skip[h] = scores.max() >= threshold
    return skip


def decode_attention_gated(q: np.ndarray, hot_k: np.ndarray, hot_v: np.ndarray,
                           cold_k: Optional[Codes], cold_v: Optional[Codes],
                           signs: np.ndarray, S: Optional[np.ndarray], num_kv_heads: int,
                           threshold: float, softmax_scale: Optional[float] = None):
    """Decode attention with the threshold-gated cold tier (Monarch v3 page,
    "Bucle de Decodificación Simplificado").  A head that ``hot_gate`` marks
    attends to its hot window alone (one softmax over the hot tokens); every
    other head is ``decode_attention`` over hot and cold.  Returns
    (out [Hq, d], skip [Hq])."""
    skip = hot_gate(q, hot_k, num_kv_heads, threshold)
    full = decode_attention(q, hot_k, hot_v, cold_k, cold_v, signs, S, num_kv_heads, softmax_scale)
    hot_only = decode_attention(q, hot_k, hot_v, None, None, signs, S, num_kv_heads, softmax_scale)
    return np.where(skip[:, None], hot_only, full), skip


# ---------------------------------------------------------------------------
# Value-side QJL ("TurboQuant: kompresja KV-cache ...", section "Kompensacja
# błędów przez QJL": the residual is coded with one bit per projection; here
# applied to values as well as keys).  A value's record then also carries its
# m sign bits and rn16, and the cold part of the output uses the residual's
# QJL reconstruction sqrt(pi/2)/m * rn16 * S^T (2 bits - 1), whose expectation
# over S is the residual itself.  READING: the same S as the keys; the
# correction is added in the rotated domain before R^T, as c S^T (sum_t p_t
# rn_t (2 bits_t - 1)) per query head with c = sqrt(pi/2)/m.
# ---------------------------------------------------------------------------

def qjl_vector_estimate(S: np.ndarray, bits: np.ndarray, rn: np.ndarray) -> np.ndarray:
    """Per record the estimate of its residual vector r (rotated domain):
    sqrt(pi/2)/m * rn * S^T (2 bits - 1).  bits [N, m], rn [N] -> [N, d]."""
    S64 = np.asarray(S, dtype=np.float32).astype(np.float64)
    m = S64.shape[0]
    sg = 2.0 * np.asarray(bits, dtype=np.float64) - 1.0
    return (sg @ S64) * (np.asarray(rn, dtype=np.float64) * (QJL_CONST / m))[:, None]


def decode_attention_vqjl(q: np.ndarray, hot_k: np.ndarray, hot_v: np.ndarray,
                          cold_k: Optional[Codes], cold_v: Optional[Codes],
                          signs: np.ndarray, S: np.ndarray, num_kv_heads: int,
                          softmax_scale: Optional[float] = None) -> np.ndarray:
    """``decode_attention`` whose cold values also carry QJL bits: the cold
    sum becomes sum_t p_t (s16_t/(2^b_r-1) v_hat_unit_t + r_hat_t) with
    r_hat from ``qjl_vector_estimate``, then R^T.  cold_v entries need
    ``bits`` and ``rn16``."""
    q = np.asarray(q, dtype=np.float64)
    hq, d = q.shape
    g = hq // num_kv_heads
    sigma = (1.0 / math.sqrt(d)) if softmax_scale is None else float(softmax_scale)
    out = np.zeros((hq, d), dtype=np.float64)
    for h in range(hq):
        kvh = h // g
        logits = []
        if hot_k is not None and hot_k.shape[1] > 0:
            logits.append(sigma * (np.asarray(hot_k[kvh], dtype=np.float64) @ q[h]))
        n_cold = 0
        if cold_k is not None and cold_k[kvh] is not None and cold_k[kvh].s16.shape[0] > 0:
            n_cold = cold_k[kvh].s16.shape[0]
            logits.append(sigma * key_inner_products(q[h], signs, S, cold_k[kvh]))
        lg = np.concatenate(logits) if logits else np.zeros(0)
        if lg.size == 0:
            continue
        p = np.exp(lg - lg.max())
        p = p / p.sum()
        n_hot = lg.size - n_cold
        o = np.zeros(d, dtype=np.float64)
        if n_hot:
            o += p[:n_hot] @ np.asarray(hot_v[kvh], dtype=np.float64)
        if n_cold:
            cv = cold_v[kvh]
            L = (1 << cv.b_r) - 1
            y_hat = (cv.s16 / L)[:, None] * dequant_unit(cv.cr, cv.ct, cv.b_theta)
            r_hat = qjl_vector_estimate(S, cv.bits, cv.rn16)
            o += rotate_inverse(p[n_hot:] @ (y_hat + r_hat), signs)
        out[h] = o
    return out


# ---------------------------------------------------------------------------
# Attention-weighted promotion ("Monarch v3 ...", section "Cómo funciona",
# item "Promoción Ponderada por Atención": cold tokens that receive high
# attention return to the hot region, with a persistence mechanism against
# thrashing; the benchmark command's --promotion-threshold 0.15 and
# --sticky-threshold 3).
# READINGS: a cold token's attention mass at a step is the mean, over the
# query heads of its kv head, of its softmax weight in that step's decode;
# its counter rises by one at every step where the mass is at least the
# threshold and returns to 0 at any step where it is not; the token is
# promoted at the step its counter reaches the sticky threshold, and its
# counter is cleared.  A promoted token leaves the cold store and enters the
# ring with its dequantized K and V, R^T (s16/(2^b_r-1) * unit pairs)
# rounded to fp16; the ring's oldest token is then evicted to cold as usual.
# ``PromotingUnit`` replays a unit step by step.
# ---------------------------------------------------------------------------

def cold_attention_mass(p_cold: np.ndarray, num_kv_heads: int) -> np.ndarray:
    """p_cold [Hq, n_cold] softmax weights of the cold tokens -> [Hkv, n_cold],
    the mean over each kv head's query heads."""
    p = np.asarray(p_cold, dtype=np.float64)
    g = p.shape[0] // num_kv_heads
    return p.reshape(num_kv_heads, g, -1).mean(axis=1)


def promotion_step(counters: np.ndarray, mass: np.ndarray, threshold: float, sticky: int):
    """One decode step of the sticky counters: returns (new counters, the
    tokens promoted now).  counters and mass have the same shape."""
    hit = np.asarray(mass, dtype=np.float64) >= threshold
    c = np.where(hit, np.asarray(counters) + 1, 0)
    promote = c >= sticky
    return np.where(promote, 0, c), promote


def cold_softmax_weights(q: np.ndarray, hot_k: np.ndarray, cold_k, signs: np.ndarray,
                         S: Optional[np.ndarray], num_kv_heads: int,
                         softmax_scale: Optional[float] = None) -> np.ndarray:
    """The softmax weights ``decode_attention`` gives the cold tokens of each
    query head (one softmax over hot and cold): [Hq, n_cold]."""
    q = np.asarray(q, dtype=np.float64)
    hq, d = q.shape
    g = hq // num_kv_heads
    sigma = (1.0 / math.sqrt(d)) if softmax_scale is None else float(softmax_scale)
    n_cold = cold_k[0].s16.shape[0]
    out = np.zeros((hq, n_cold))
    for h in range(hq):
        kvh = h // g
        lc = sigma * key_inner_products(q[h], signs, S, cold_k[kvh])
        lh = (sigma * (np.asarray(hot_k[kvh], dtype=np.float64) @ q[h])
              if hot_k is not None and hot_k.shape[1] > 0 else np.zeros(0))
        mx = max(lc.max(), lh.max() if lh.size else -np.inf)
        den = np.exp(lc - mx).sum() + np.exp(lh - mx).sum()
        out[h] = np.exp(lc - mx) / den
    return out


def dequant_vectors(codes: Codes, signs: np.ndarray) -> np.ndarray:
    """fp16 reconstruction of coded vectors in the original basis:
    R^T (s16/(2^b_r-1) * c_r (cos, sin)), rounded to fp16 (the hot ring's
    format)."""
    L = (1 << codes.b_r) - 1
    y_hat = (np.asarray(codes.s16, dtype=np.float64) / L)[:, None] * dequant_unit(
        codes.cr, codes.ct, codes.b_theta)
    return fp16_round(rotate_inverse(y_hat, signs))


class PromotingUnit:
    """One (batch row, kv head) of a cache with attention-weighted promotion:
    a hot ring of W tokens, a cold list indexed by cold position, the sticky
    counters and the tokens promoted by the last decode.

    READINGS (beyond those of ``promotion_step`` above): a decode decides the
    promotions from its own masses; they are applied at the next insert,
    where the promoted tokens (their dequantized fp16 K and V, oldest cold
    index first) enter the ring before the new tokens, so that a new token
    is the newest; every insert into a full ring evicts the oldest ring
    token, and an evicted token takes the cold index of the earliest still
    open promoted position (ascending), or is appended when none is left.
    So each unit's cold list grows by exactly the number of new tokens.  A
    promotion decided while the ring is not full is dropped (the token stays
    cold; its counter was cleared).  The vectors held here are whatever the
    caller inserts: fp16 values for the ring, raw vectors for the cold list
    (the caller encodes them)."""

    def __init__(self, W: int, d: int, threshold: float, sticky: int):
        self.W, self.d = W, d
        self.threshold, self.sticky = float(threshold), int(sticky)
        self.ring_k = np.zeros((W, d))
        self.ring_v = np.zeros((W, d))
        self.ring_pos = 0
        self.n_hot = 0
        self.cold_k: list = []           # cold position -> raw key vector
        self.cold_v: list = []
        self.counters = np.zeros(0, dtype=np.int64)
        self.pending: list = []          # cold positions promoted by the last decode

    def append_cold(self, k: np.ndarray, v: np.ndarray) -> None:
        """Prefill: tokens encoded straight into the cold list."""
        for kk, vv in zip(np.asarray(k, dtype=np.float64), np.asarray(v, dtype=np.float64)):
            self.cold_k.append(kk.copy())
            self.cold_v.append(vv.copy())
        self.counters = np.concatenate([self.counters, np.zeros(len(k), dtype=np.int64)])

    def insert(self, k_new: np.ndarray, v_new: np.ndarray, promoted_k: np.ndarray,
               promoted_v: np.ndarray) -> list:
        """Insert the pending promoted tokens (given as their fp16
        dequantization, in ``pending`` order) and then the new tokens;
        returns the cold positions written, in eviction order."""
        holes = list(self.pending)
        self.pending = []
        assert len(promoted_k) == len(holes)
        seq_k = list(np.asarray(promoted_k, dtype=np.float64)) + list(np.asarray(k_new, dtype=np.float64))
        seq_v = list(np.asarray(promoted_v, dtype=np.float64)) + list(np.asarray(v_new, dtype=np.float64))
        written = []
        for kk, vv in zip(seq_k, seq_v):
            if self.n_hot == self.W:
                old_k = self.ring_k[self.ring_pos].copy()
                old_v = self.ring_v[self.ring_pos].copy()
                if holes:
                    i = holes.pop(0)
                    self.cold_k[i], self.cold_v[i] = old_k, old_v
                    self.counters[i] = 0
                else:
                    i = len(self.cold_k)
                    self.cold_k.append(old_k)
                    self.cold_v.append(old_v)
                    self.counters = np.append(self.counters, 0)
                written.append(i)
            else:
                self.n_hot += 1
            self.ring_k[self.ring_pos] = kk
            self.ring_v[self.ring_pos] = vv
            self.ring_pos = (self.ring_pos + 1) % self.W
        assert not holes, "promotions are only kept while the ring is full"
        return written

    def after_decode(self, mass: np.ndarray) -> np.ndarray:
        """Counters after a decode whose cold tokens got ``mass``; returns the
        promoted positions (ascending), which become ``pending``."""
        self.counters, promote = promotion_step(self.counters, mass, self.threshold, self.sticky)
        if self.n_hot < self.W:
            promote = np.zeros_like(promote)
        self.pending = [int(i) for i in np.nonzero(promote)[0]]
        return np.array(self.pending, dtype=np.int64)

    def hot_slots(self):
        return self.ring_k, self.ring_v


# ---------------------------------------------------------------------------
# Tensor Cache second tier ("Tensor Cache: Eviction-conditioned Associative
# Memory for Transformers", section "Metodología", items "Mecanismo de
# Escritura", "Mecanismo de Lectura" and "Fusión").  The ring of W tokens is
# the first level; every token the ring displaces is written into a d x d
# outer-product matrix A per kv head, and queries read A back.
# READINGS: lambda and eta are one scalar pair per kv head (the page learns
# them per head; here they are given); the gate g is one scalar per query
# head; A starts at zero; the local output y_local is the exact softmax
# attention over the ring (the same as ``decode_attention`` with no cold
# tokens).
# ---------------------------------------------------------------------------

def tc_write(A: np.ndarray, k: np.ndarray, v: np.ndarray, lam: float, eta: float) -> np.ndarray:
    """One eviction: A <- lambda A + eta (k outer v)."""
    return lam * np.asarray(A, dtype=np.float64) + eta * np.outer(
        np.asarray(k, dtype=np.float64), np.asarray(v, dtype=np.float64))


def tc_write_sequence(A: np.ndarray, ks: np.ndarray, vs: np.ndarray, lam: float,
                      eta: float) -> np.ndarray:
    """Evictions in order (oldest first), one ``tc_write`` each."""
    for k, v in zip(ks, vs):
        A = tc_write(A, k, v, lam, eta)
    return A


def tc_decode(q: np.ndarray, hot_k: np.ndarray, hot_v: np.ndarray, A: np.ndarray,
              gate: np.ndarray, num_kv_heads: int,
              softmax_scale: Optional[float] = None) -> np.ndarray:
    """y = y_local + sigmoid(g) (q A) per query head h, with y_local the
    softmax attention over h's ring and A = A[kv head of h] ([Hkv, d, d])."""
    q = np.asarray(q, dtype=np.float64)
    hq = q.shape[0]
    g = hq // num_kv_heads
    y_local = decode_attention(q, hot_k, hot_v, None, None, None, None, num_kv_heads,
                               softmax_scale)
    out = np.empty_like(y_local)
    for h in range(hq):
        m = q[h] @ np.asarray(A[h // g], dtype=np.float64)
        gh = float(gate[h])          # logistic sigmoid, evaluated without overflow
        sig = 1.0 / (1.0 + math.exp(-gh)) if gh >= 0 else math.exp(gh) / (1.0 + math.exp(gh))
        out[h] = y_local[h] + sig * m
    return out


def attention_reference(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                        num_kv_heads: int, softmax_scale: Optional[float] = None) -> np.ndarray:
    """Textbook softmax(q K^T * sigma) V per query head, fp64 (GQA mapping)."""
    q = np.asarray(q, dtype=np.float64)
    hq, d = q.shape
    g = hq // num_kv_heads
    sigma = (1.0 / math.sqrt(d)) if softmax_scale is None else float(softmax_scale)
    out = np.zeros((hq, d))
    for h in range(hq):
        kk = np.asarray(k[h // g], dtype=np.float64)
        vv = np.asarray(v[h // g], dtype=np.float64)
        lg = sigma * (kk @ q[h])
        p = np.exp(lg - lg.max())
        out[h] = (p / p.sum()) @ vv
    return out


# ---------------------------------------------------------------------------
# Hot/cold ring (Monarch's sliding-window eviction, a ring buffer as in the
# Tensor Cache page's first-level cache).  READING: the ring holds exactly W
# tokens; the (W+1)-th insert evicts the oldest, which is encoded and appended
# to the cold store in age order.
# ---------------------------------------------------------------------------

@dataclass
class RingState:
    """Per (batch row, kv head) state of the hot ring and cold list."""
    W: int
    d: int
    ring: np.ndarray = None          # [W, d] float64 (fp16 values)
    ring_pos: int = 0                # next slot to write
    n_hot: int = 0
    cold_vectors: list = field(default_factory=list)   # evicted raw vectors

    def __post_init__(self):
        if self.ring is None:
            self.ring = np.zeros((self.W, self.d), dtype=np.float64)

    def insert(self, vecs: np.ndarray) -> None:
        """Insert new tokens one at a time, in order."""
        for v in np.asarray(vecs, dtype=np.float64):
            if self.n_hot == self.W:
                self.cold_vectors.append(self.ring[self.ring_pos].copy())
            else:
                self.n_hot += 1
            self.ring[self.ring_pos] = v
            self.ring_pos = (self.ring_pos + 1) % self.W

    def hot_tokens(self) -> np.ndarray:
        """Valid hot tokens in age order (oldest first)."""
        start = (self.ring_pos - self.n_hot) % self.W
        idx = [(start + i) % self.W for i in range(self.n_hot)]
        return self.ring[idx]

    def slots(self) -> np.ndarray:
        """The raw ring, slot order (what a device ring holds)."""
        return self.ring


# ---------------------------------------------------------------------------
# Vector inner-product search over the same codes.
# ---------------------------------------------------------------------------

def ip_scores(queries: np.ndarray, signs: np.ndarray, S: np.ndarray, codes: Codes) -> np.ndarray:
    """Estimated inner products [nq, N]: s16/(2^b_r-1) <q', x_hat_unit>
    + rn16 sqrt(pi/2)/m <S q', 2 bits - 1>  (q' = R q, zero padded)."""
    return key_inner_products(np.asarray(queries, dtype=np.float64), signs, S, codes)


def top_k(scores: np.ndarray, k: int):
    """Per row: k largest scores, descending; equal scores -> lower index."""
    scores = np.asarray(scores, dtype=np.float64)
    nq, n = scores.shape
    idx = np.empty((nq, k), dtype=np.int64)
    val = np.empty((nq, k), dtype=np.float64)
    cols = np.arange(n)
    for i in range(nq):
        order = np.lexsort((cols, -scores[i]))[:k]
        idx[i] = order
        val[i] = scores[i, order]
    return val, idx
