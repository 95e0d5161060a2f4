"""The vectorised oracle against the loop-level brute force on tiny sizes:
codes identical (except decisions the oracle flags as ties), floats to 1e-12.
"""
import math

import numpy as np
import pytest

from oracle import brute as B
from oracle import tq_oracle as O


@pytest.mark.parametrize("d,m,b_r,b_t", [(4, 4, 2, 3), (8, 8, 3, 3), (8, 8, 4, 4), (8, 5, 1, 2)])
def test_encode_matches_brute(d, m, b_r, b_t):
    rng = np.random.default_rng(d * 100 + m)
    n = 16
    x = rng.standard_normal((n, d)).astype(np.float16).astype(np.float64)
    signs = O.rotation_signs(d + m, d)
    S = O.qjl_matrix(d + m, m, d)
    c = O.encode(x, signs, S, b_r, b_t, keep_intermediates=True)
    for i in range(n):
        ref = B.encode_one(list(x[i]), list(signs), S.astype(np.float64).tolist(), b_r, b_t)
        assert ref["s16"] == c.s16[i]
        if c.vec_tie[i]:
            continue
        assert ref["cr"] == list(c.cr[i])
        assert ref["ct"] == list(c.ct[i])
        np.testing.assert_allclose(ref["residual"], c.residual[i], rtol=0, atol=1e-12)
        if not c.tie_rn16[i]:
            assert ref["rn16"] == c.rn16[i]
        for j in range(m):
            if not c.tie_bits[i, j]:
                assert ref["bits"][j] == c.bits[i, j]


def test_rotation_matches_brute():
    rng = np.random.default_rng(0)
    for d in (2, 4, 8, 16):
        signs = O.rotation_signs(d, d)
        x = rng.standard_normal(d)
        np.testing.assert_allclose(O.rotate(x[None], signs)[0], B.rotate(list(x), list(signs)), atol=1e-12)
        np.testing.assert_allclose(O.rotate_inverse(x[None], signs)[0],
                                   B.rotate_inverse(list(x), list(signs)), atol=1e-12)


@pytest.mark.parametrize("d,m,b", [(4, 4, 3), (8, 8, 4), (8, 8, 2)])
def test_decode_attention_matches_brute(d, m, b):
    rng = np.random.default_rng(d + 10 * b)
    hq, hkv, nh, nc = 4, 2, 3, 9
    q = rng.standard_normal((hq, d))
    hk = rng.standard_normal((hkv, nh, d))
    hv = rng.standard_normal((hkv, nh, d))
    ck_raw = rng.standard_normal((hkv, nc, d))
    cv_raw = rng.standard_normal((hkv, nc, d))
    signs = O.rotation_signs(1, d)
    S = O.qjl_matrix(1, m, d)
    ck = [O.encode(ck_raw[h], signs, S, b, b) for h in range(hkv)]
    cv = [O.encode(cv_raw[h], signs, None, b, b) for h in range(hkv)]
    sigma = 1 / math.sqrt(d)
    out = O.decode_attention(q, hk, hv, ck, cv, signs, S, hkv)
    Sl = S.astype(np.float64).tolist()
    for h in range(hq):
        g = h // (hq // hkv)
        recs_k = [dict(s16=ck[g].s16[t], cr=list(ck[g].cr[t]), ct=list(ck[g].ct[t]),
                       rn16=ck[g].rn16[t], bits=list(ck[g].bits[t])) for t in range(nc)]
        recs_v = [dict(s16=cv[g].s16[t], cr=list(cv[g].cr[t]), ct=list(cv[g].ct[t])) for t in range(nc)]
        ref = B.decode_one_head(list(q[h]), hk[g].tolist(), hv[g].tolist(), recs_k, recs_v,
                                list(signs), Sl, b, b, sigma)
        np.testing.assert_allclose(out[h], ref, rtol=1e-12, atol=1e-12)


def test_inner_products_match_brute():
    rng = np.random.default_rng(4)
    d, m, b_r, b_t = 8, 8, 4, 4
    signs = O.rotation_signs(2, d)
    S = O.qjl_matrix(2, m, d)
    x = rng.standard_normal((10, d))
    q = rng.standard_normal((3, d))
    c = O.encode(x, signs, S, b_r, b_t)
    sc = O.ip_scores(q, signs, S, c)
    for i in range(3):
        for t in range(10):
            rec = dict(s16=c.s16[t], cr=list(c.cr[t]), ct=list(c.ct[t]), rn16=c.rn16[t], bits=list(c.bits[t]))
            assert abs(sc[i, t] - B.key_ip(list(q[i]), list(signs), S.astype(np.float64).tolist(),
                                            rec, b_r, b_t)) < 1e-12


@pytest.mark.parametrize("d,m,b", [(4, 4, 3), (8, 8, 4)])
def test_gated_decode_matches_brute(d, m, b):
    """Threshold-gated cold tier: per-head skip decisions and outputs of the
    oracle against the loop-level restatement, at thresholds that split the
    heads both ways."""
    rng = np.random.default_rng(7 * d + b)
    hq, hkv, nh, nc = 6, 2, 5, 7
    q = rng.standard_normal((hq, d))
    hk = rng.standard_normal((hkv, nh, d))
    hv = rng.standard_normal((hkv, nh, d))
    signs = O.rotation_signs(3, d)
    S = O.qjl_matrix(3, m, d)
    ck = [O.encode(rng.standard_normal((nc, d)), signs, S, b, b) for _ in range(hkv)]
    cv = [O.encode(rng.standard_normal((nc, d)), signs, None, b, b) for _ in range(hkv)]
    gmax = np.array([(hk[h // (hq // hkv)] @ q[h]).max() for h in range(hq)])
    order = np.sort(gmax)
    sigma = 0.7 / math.sqrt(d)
    Sl = S.astype(np.float64).tolist()
    for thr in (order[0] - 1.0, 0.5 * (order[2] + order[3]), order[-1] + 1.0, order[1]):
        out, skip = O.decode_attention_gated(q, hk, hv, ck, cv, signs, S, hkv, thr, sigma)
        for h in range(hq):
            g = h // (hq // hkv)
            recs_k = [dict(s16=ck[g].s16[t], cr=list(ck[g].cr[t]), ct=list(ck[g].ct[t]),
                           rn16=ck[g].rn16[t], bits=list(ck[g].bits[t])) for t in range(nc)]
            recs_v = [dict(s16=cv[g].s16[t], cr=list(cv[g].cr[t]), ct=list(cv[g].ct[t]))
                      for t in range(nc)]
            ref, ref_skip = B.decode_one_head_gated(list(q[h]), hk[g].tolist(), hv[g].tolist(),
                                                    recs_k, recs_v, list(signs), Sl, b, b, sigma, thr)
            assert ref_skip == skip[h]
            np.testing.assert_allclose(out[h], ref, rtol=1e-12, atol=1e-12)
        assert skip.sum() == (gmax >= thr).sum()


def test_tc_write_and_read_match_loops():
    rng = np.random.default_rng(31)
    d = 6
    A = rng.standard_normal((d, d))
    Al = A.tolist()
    for _ in range(5):
        k, v, q = rng.standard_normal((3, d))
        A = O.tc_write(A, k, v, 0.8, 0.3)
        Al = B.tc_write_loops(Al, list(k), list(v), 0.8, 0.3)
        np.testing.assert_allclose(A, Al, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(q @ A, B.tc_read_loops(list(q), Al), rtol=1e-12, atol=1e-12)


def test_value_qjl_estimate_matches_loops():
    rng = np.random.default_rng(43)
    d, m, b_r, b_t = 8, 8, 3, 3
    signs = O.rotation_signs(4, d)
    S = O.qjl_matrix(4, m, d)
    x = rng.standard_normal((6, d))
    c = O.encode(x, signs, S, b_r, b_t)
    L = (1 << b_r) - 1
    est = (c.s16 / L)[:, None] * O.dequant_unit(c.cr, c.ct, b_t) + O.qjl_vector_estimate(S, c.bits, c.rn16)
    Sl = S.astype(np.float64).tolist()
    for t in range(6):
        rec = dict(s16=c.s16[t], cr=list(c.cr[t]), ct=list(c.ct[t]), rn16=c.rn16[t], bits=list(c.bits[t]))
        np.testing.assert_allclose(est[t], B.value_estimate_loops(rec, Sl, b_r, b_t), rtol=1e-12, atol=1e-12)


def test_promoted_vectors_match_loops():
    """A promoted token's fp16 K / V: the polar reconstruction rotated back,
    against the loop restatement (dense Sylvester matrix, struct halves)."""
    rng = np.random.default_rng(52)
    d, b_r, b_t = 8, 4, 3
    signs = O.rotation_signs(6, d)
    c = O.encode(rng.standard_normal((5, d)), signs, None, b_r, b_t)
    got = O.dequant_vectors(c, signs)
    L = 2 ** b_r - 1
    for t in range(5):
        y = []
        for j in range(d // 2):
            a = c.ct[t][j] * 2.0 * math.pi / 2 ** b_t
            y += [c.s16[t] / L * c.cr[t][j] * math.cos(a), c.s16[t] / L * c.cr[t][j] * math.sin(a)]
        ref = [B.to_half(x) for x in B.rotate_inverse(y, list(signs))]
        np.testing.assert_allclose(got[t], ref, rtol=0, atol=1e-6 * max(1.0, max(abs(x) for x in ref)))
