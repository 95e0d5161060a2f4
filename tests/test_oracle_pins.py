"""Pins for the fp64 oracle: each test checks it against something other than
itself -- published generator outputs, a library routine, a hand-derived
worked example, a closed form, an invariant or a statistical law.
"""
import math
import os
import struct

import numpy as np
import pytest
import scipy.linalg
import scipy.stats
import torch

from oracle import tq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_examples():
    vals = {}
    with open(os.path.join(GOLDEN, "worked_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split("=", 1)
            vals[k.strip()] = v.strip()
    return vals


def _ints(s):
    return [int(t, 0) for t in s.split()]


def _floats(s):
    return [float(t) for t in s.split()]


def _half_bits(x):
    return struct.unpack("<H", struct.pack("<e", float(x)))[0]


# --------------------------------------------------------------------------
# Generator
# --------------------------------------------------------------------------

def test_splitmix64_published_outputs():
    with open(os.path.join(GOLDEN, "splitmix64_seed0.txt")) as f:
        ref = [int(l, 16) for l in f if l.strip() and not l.startswith("#")]
    state = 0
    got = []
    for _ in range(len(ref)):
        state = (state + O.GAMMA) & O.MASK64
        got.append(O.mix64(state))
    assert got == ref
    # rand64 with base mix64(seed + stream) == 0 reproduces the same Weyl
    # sequence; check the counter form separately against the loop form.
    seed, stream = 12345, 1
    base = O.mix64(seed + stream)
    for i in range(5):
        assert O.rand64(seed, stream, i) == O.mix64((base + (i + 1) * O.GAMMA) & O.MASK64)


def test_rotation_signs_balanced_and_seeded():
    s = O.rotation_signs(7, 4096)
    assert set(np.unique(s)) == {-1.0, 1.0}
    # Binomial(4096, 1/2): 5 sigma band
    assert abs(s.sum()) < 5 * math.sqrt(4096)
    assert not np.array_equal(s[:64], O.rotation_signs(8, 64))
    np.testing.assert_array_equal(s[:64], O.rotation_signs(7, 64))


def test_qjl_matrix_is_standard_normal():
    S = O.qjl_matrix(3, 64, 128).astype(np.float64).ravel()
    assert S.dtype == np.float64
    ks = scipy.stats.kstest(S, "norm")
    assert ks.pvalue > 1e-3, ks
    assert abs(S.mean()) < 5 / math.sqrt(S.size)
    assert abs(S.var() - 1.0) < 5 * math.sqrt(2.0 / S.size)
    # rows are not copies of one another (draw index covers row and column)
    S2 = S.reshape(64, 128)
    assert np.abs(np.corrcoef(S2[:8])[np.triu_indices(8, 1)]).max() < 0.5


# --------------------------------------------------------------------------
# Rotation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 64, 128, 256])
def test_fwht_equals_sylvester_hadamard(d):
    rng = np.random.default_rng(d)
    x = rng.standard_normal((5, d))
    H = scipy.linalg.hadamard(d).astype(np.float64)   # Sylvester construction
    np.testing.assert_allclose(O.fwht(x), x @ H.T, rtol=0, atol=1e-12 * d)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rotation_orthogonal_and_norm_preserving(d):
    signs = O.rotation_signs(11, d)
    R = O.rotate(np.eye(d), signs).T          # column j = R e_j
    np.testing.assert_allclose(R.T @ R, np.eye(d), atol=1e-12)
    x = np.random.default_rng(0).standard_normal((10, d))
    y = O.rotate(x, signs)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    np.testing.assert_allclose(O.rotate_inverse(y, signs), x, atol=1e-12)


def test_zero_padding_to_power_of_two():
    assert O.padded_dim(200) == 256 and O.padded_dim(128) == 128 and O.padded_dim(1) == 1
    signs = O.rotation_signs(5, 256)
    x = np.random.default_rng(1).standard_normal((3, 200))
    y = O.rotate(x, signs)
    assert y.shape == (3, 256)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


# --------------------------------------------------------------------------
# Worked examples (hand-derived; tests/golden/worked_examples.txt)
# --------------------------------------------------------------------------

def test_worked_example_B_all_fields():
    ex = _load_examples()
    x = np.array([_floats(ex["B.x"])])
    signs = np.array(_floats(ex["B.signs"]))
    S = np.array([_floats(r) for r in ex["B.S"].split(";")], dtype=np.float32)
    b_r, b_t = int(ex["B.b_r"]), int(ex["B.b_theta"])
    c = O.encode(x, signs, S, b_r, b_t)
    assert _half_bits(c.s16[0]) == int(ex["B.s16_bits"], 0)
    assert list(c.cr[0]) == _ints(ex["B.cr"])
    assert list(c.ct[0]) == _ints(ex["B.ct"])
    assert _half_bits(c.rn16[0]) == int(ex["B.rn16_bits"], 0)
    assert list(c.bits[0]) == _ints(ex["B.bits"])
    assert not c.vec_tie[0] and not c.tie_bits.any() and not c.tie_rn16.any()
    assert list(O.pack_codes(c.cr, c.ct, b_t, b_r)[0]) == _ints(ex["B.packed_codes"])
    assert list(O.pack_bits(c.bits)[0]) == _ints(ex["B.packed_bits"])


def test_worked_example_A_unit_vector():
    ex = _load_examples()
    x = np.array([_floats(ex["A.x"])])
    S = np.random.default_rng(0).standard_normal((16, 8)).astype(np.float32)
    for sk, ctk in (("A.signs", "A.ct"), ("A2.signs", "A2.ct")):
        signs = np.array(_floats(ex[sk]))
        c = O.encode(x, signs, S, int(ex["A.b_r"]), int(ex["A.b_theta"]))
        assert _half_bits(c.s16[0]) == int(ex["A.s16_bits"], 0)
        assert list(c.cr[0]) == _ints(ex["A.cr"])
        assert list(c.ct[0]) == _ints(ex[ctk])
        assert _half_bits(c.rn16[0]) == int(ex["A.rn16_bits"], 0)
        # residual is float64 noise -> every sign decision is a tie
        assert c.tie_bits.all()
    # A3: angle exactly on a rounding boundary -> tie flagged, ties to even
    c = O.encode(x, np.array(_floats(ex["A.signs"])), S, int(ex["A.b_r"]), int(ex["A3.b_theta"]))
    assert list(c.ct[0]) == _ints(ex["A3.ct"])
    assert c.tie_ct.all() and c.vec_tie[0]


# --------------------------------------------------------------------------
# Format invariants and closed-form bounds
# --------------------------------------------------------------------------

def _gauss(n, d, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal((n, d)) * scale


@pytest.mark.parametrize("b_r,b_t", [(2, 3), (3, 3), (4, 4), (1, 7)])
def test_decode_then_reencode_is_idempotent(b_r, b_t):
    d = 128
    signs = O.rotation_signs(1, d)
    x = _gauss(200, d, 2)
    c = O.encode(x, signs, None, b_r, b_t)
    xh = O.rotate_inverse(O.dequant(c.cr, c.ct, c.s16, b_r, b_t), signs)
    c2 = O.encode(xh, signs, None, b_r, b_t)
    np.testing.assert_array_equal(c2.s16, c.s16)
    np.testing.assert_array_equal(c2.cr, c.cr)
    live = c.cr > 0          # the angle of a zero-radius pair carries nothing
    np.testing.assert_array_equal(c2.ct[live], c.ct[live])


@pytest.mark.parametrize("b_r,b_t", [(2, 3), (3, 3), (4, 4), (6, 2)])
def test_per_pair_error_bounds(b_r, b_t):
    d = 128
    L = (1 << b_r) - 1
    signs = O.rotation_signs(4, d)
    x = _gauss(300, d, 5, scale=3.0)
    c = O.encode(x, signs, None, b_r, b_t, keep_intermediates=True)
    y = c.rotated
    rho = np.hypot(y[:, 0::2], y[:, 1::2])
    s = rho.max(axis=1)
    rho_hat = c.cr * c.s16[:, None] / L
    bound_r = c.s16[:, None] / (2 * L) + np.abs(s - c.s16)[:, None]
    assert np.all(np.abs(rho_hat - rho) <= bound_r * (1 + 1e-12) + 1e-15)
    th = np.arctan2(y[:, 1::2], y[:, 0::2])
    th_hat = c.ct * 2 * np.pi / (1 << b_t)
    dth = np.abs(np.angle(np.exp(1j * (th - th_hat))))
    assert np.all(dth <= np.pi / (1 << b_t) + 1e-12)
    yh = O.dequant(c.cr, c.ct, c.s16, b_r, b_t)
    err = np.hypot((y - yh)[:, 0::2], (y - yh)[:, 1::2])
    assert np.all(err <= bound_r + rho_hat * dth + 1e-12)


def test_zero_vector_and_scale_overflow():
    d = 64
    signs = O.rotation_signs(1, d)
    S = O.qjl_matrix(1, 16, d)
    x = np.zeros((2, d))
    x[1, 0] = 1e6                    # rotated max radius ~ 1.8e5 > fp16 max
    c = O.encode(x, signs, S, 3, 3)
    assert c.s16[0] == 0 and (c.cr[0] == 0).all() and (c.ct[0] == 0).all()
    assert c.rn16[0] == 0 and (c.bits[0] == 1).all()
    assert c.range_error[1] and not c.range_error[0]


def test_rounding_is_half_even_and_codes_in_range():
    d = 64
    signs = O.rotation_signs(9, d)
    x = _gauss(500, d, 9)
    for b_r, b_t in ((1, 1), (2, 2), (5, 3), (8, 8)):
        c = O.encode(x, signs, None, b_r, b_t)
        assert c.cr.min() >= 0 and c.cr.max() <= (1 << b_r) - 1
        assert c.ct.min() >= 0 and c.ct.max() <= (1 << b_t) - 1
        # the largest pair always takes the top radius code
        assert np.all(c.cr.max(axis=1) == (1 << b_r) - 1)


def test_fp16_margin_against_struct_rounding():
    rng = np.random.default_rng(3)
    x = np.exp(rng.uniform(-10, 10, 2000))
    m = O.fp16_margin(x)
    # a value nudged across a midpoint by less than its margin must not
    # change its fp16 rounding
    for xi, mi in zip(x[:300], m[:300]):
        h = struct.unpack("<e", struct.pack("<e", xi))[0]
        nudge = xi * (1 + 0.5 * min(mi, 1e-3))
        h2 = struct.unpack("<e", struct.pack("<e", nudge))[0]
        assert h == h2
    # exact midpoint between 1 and 1 + 2^-10 has margin 0
    assert O.fp16_margin(np.array([1 + 2.0 ** -11]))[0] == 0.0


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(0)
    for b_r, b_t in ((2, 3), (3, 3), (4, 4), (1, 1), (7, 1)):
        cr = rng.integers(0, 1 << b_r, size=(7, 64))
        ct = rng.integers(0, 1 << b_t, size=(7, 64))
        p = O.pack_codes(cr, ct, b_t, b_r)
        assert p.shape == (7, 64 * (b_r + b_t) // 8)
        cr2, ct2 = O.unpack_codes(p, 64, b_r, b_t)
        np.testing.assert_array_equal(cr2, cr)
        np.testing.assert_array_equal(ct2, ct)
    bits = rng.integers(0, 2, size=(5, 200)).astype(np.uint8)
    np.testing.assert_array_equal(O.unpack_bits(O.pack_bits(bits), 200), bits)
    # LSB-first: bit 0 of the stream is the low bit of byte 0
    assert O.pack_bits(np.array([[1, 0, 0, 0, 0, 0, 0, 0, 0, 1]], dtype=np.uint8)).tolist() == [[1, 2]]


# --------------------------------------------------------------------------
# QJL estimator: unbiased, variance ~ 1/m (quantized Johnson-Lindenstrauss)
# --------------------------------------------------------------------------

def test_qjl_estimator_unbiased():
    d, m, trials = 64, 64, 4000
    rng = np.random.default_rng(42)
    q = rng.standard_normal(d)
    r = rng.standard_normal(d) * 0.1
    exact = q @ r
    est = np.empty(trials)
    for t in range(trials):
        S = rng.standard_normal((m, d)).astype(np.float32)
        bits = ((r @ S.astype(np.float64).T) >= 0).astype(np.uint8)[None]
        est[t] = O.qjl_estimate(q, S, bits, np.array([np.linalg.norm(r)]))[0]
    se = est.std(ddof=1) / math.sqrt(trials)
    assert abs(est.mean() - exact) <= 4 * se, (est.mean(), exact, se)


def test_qjl_variance_falls_with_m():
    d, trials = 64, 1500
    rng = np.random.default_rng(7)
    q = rng.standard_normal(d)
    r = rng.standard_normal(d)
    var = {}
    for m in (32, 128):
        est = np.empty(trials)
        for t in range(trials):
            S = rng.standard_normal((m, d)).astype(np.float32)
            bits = ((r @ S.astype(np.float64).T) >= 0).astype(np.uint8)[None]
            est[t] = O.qjl_estimate(q, S, bits, np.array([np.linalg.norm(r)]))[0]
        var[m] = est.var()
    ratio = var[32] / var[128]
    assert 2.5 < ratio < 6.0, ratio     # ~4 for a 4x larger m


# --------------------------------------------------------------------------
# Attention: reductions to textbook softmax attention
# --------------------------------------------------------------------------

def _sdpa(q, k, v, hkv):
    """torch's scaled_dot_product_attention on CPU in float64 (library)."""
    hq, d = q.shape
    g = hq // hkv
    kk = torch.from_numpy(np.repeat(k, g, axis=0))
    vv = torch.from_numpy(np.repeat(v, g, axis=0))
    qq = torch.from_numpy(q)[:, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)
    return o[:, 0, :].numpy()


def test_hot_only_equals_textbook_attention():
    rng = np.random.default_rng(0)
    hq, hkv, d, w = 8, 2, 64, 37
    q = rng.standard_normal((hq, d))
    k = rng.standard_normal((hkv, w, d))
    v = rng.standard_normal((hkv, w, d))
    signs = O.rotation_signs(0, d)
    o = O.decode_attention(q, k, v, None, None, signs, None, hkv)
    np.testing.assert_allclose(o, _sdpa(q, k, v, hkv), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(o, O.attention_reference(q, k, v, hkv), rtol=1e-12, atol=1e-12)


def _cold_attention(q, k, v, hkv, b, m, seed):
    d = q.shape[1]
    signs = O.rotation_signs(seed, d)
    S = O.qjl_matrix(seed, m, d) if m else None
    ck = [O.encode(k[h], signs, S, b, b) for h in range(hkv)]
    cv = [O.encode(v[h], signs, None, b, b) for h in range(hkv)]
    empty = np.zeros((hkv, 0, d))
    return O.decode_attention(q, empty, empty, ck, cv, signs, S, hkv), ck, cv, signs, S


def test_error_bound_and_infinite_bit_limit():
    """|logit error| <= sigma (|q'| |r| + QJL term bound); softmax is
    2-Lipschitz in l_inf -> l_1, so the output error is bounded by a
    quantity that vanishes as the bits grow; at 20 bits it is ~1e-5."""
    rng = np.random.default_rng(1)
    hq, hkv, d, n, m = 4, 1, 64, 50, 64
    q = rng.standard_normal((hq, d))
    k = rng.standard_normal((hkv, n, d))
    v = rng.standard_normal((hkv, n, d))
    ref = O.attention_reference(q, k, v, hkv)
    prev = None
    for b in (4, 8, 12, 16, 20):
        o, ck, cv, signs, S = _cold_attention(q, k, v, hkv, b, m, 3)
        c = O.encode(k[0], signs, S, b, b, keep_intermediates=True)
        rn = np.linalg.norm(c.residual, axis=1)
        qr = O.rotate(q, signs)
        sq = np.abs(qr @ S.astype(np.float64).T).sum(axis=1)
        sigma = 1 / math.sqrt(d)
        dl = sigma * (np.linalg.norm(qr, axis=1)[:, None] * rn[None]
                      + c.rn16[None] * O.QJL_CONST / m * sq[:, None])
        vh = O.rotate_inverse(O.dequant(cv[0].cr, cv[0].ct, cv[0].s16, b, b), signs)
        dv = np.linalg.norm(vh - v[0], axis=1).max()
        vmax = np.linalg.norm(v[0], axis=1).max()
        bound = 2 * dl.max(axis=1) * (vmax + dv) + dv
        err = np.linalg.norm(o - ref, axis=1)
        assert np.all(err <= bound + 1e-12), (b, err, bound)
        if prev is not None:
            assert bound.max() < prev
        prev = bound.max()
    rel = np.linalg.norm(o - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert rel.max() < 1e-4


def test_error_falls_as_bits_rise():
    """Monotonicity averaged over 16 seeds: more bits -> lower logit MSE and
    lower attention error (the pages: quality degrades only at very low
    precision)."""
    rng = np.random.default_rng(5)
    hq, hkv, d, n = 4, 1, 64, 64
    errs = []
    for b in (2, 3, 4, 5, 6):
        e = []
        for seed in range(16):
            q = rng.standard_normal((hq, d))
            k = rng.standard_normal((hkv, n, d))
            v = rng.standard_normal((hkv, n, d))
            o, *_ = _cold_attention(q, k, v, hkv, b, 64, seed)
            ref = O.attention_reference(q, k, v, hkv)
            e.append(np.mean(np.linalg.norm(o - ref, axis=1) / np.linalg.norm(ref, axis=1)))
        errs.append(np.mean(e))
    assert all(a > b for a, b in zip(errs, errs[1:])), errs


def test_logit_mse_falls_with_bits_and_qjl_is_unbiased_on_codes():
    d, n = 128, 400
    rng = np.random.default_rng(8)
    q = rng.standard_normal(d)
    k = rng.standard_normal((n, d))
    exact = k @ q
    mse = []
    for b in (2, 3, 4, 5, 6):
        signs = O.rotation_signs(b, d)
        S = O.qjl_matrix(b, 128, d)
        c = O.encode(k, signs, S, b, b)
        mse.append(np.mean((O.key_inner_products(q, signs, S, c) - exact) ** 2))
    assert all(a > b for a, b in zip(mse, mse[1:])), mse


# --------------------------------------------------------------------------
# Ring and top-k
# --------------------------------------------------------------------------

def test_ring_eviction_order():
    st = O.RingState(W=3, d=1)
    st.insert(np.arange(2, dtype=float)[:, None])        # tokens 0, 1
    assert st.n_hot == 2 and st.cold_vectors == []
    st.insert(np.arange(2, 6, dtype=float)[:, None])     # tokens 2..5
    # inserts 2 (fills), then 3 evicts 0, 4 evicts 1, 5 evicts 2
    assert [float(v[0]) for v in st.cold_vectors] == [0.0, 1.0, 2.0]
    assert [float(v[0]) for v in st.hot_tokens()] == [3.0, 4.0, 5.0]
    assert st.ring_pos == 0
    assert [float(v[0]) for v in st.slots()] == [3.0, 4.0, 5.0]


def test_top_k_matches_full_sort_with_index_tiebreak():
    rng = np.random.default_rng(0)
    sc = np.round(rng.standard_normal((6, 500)), 1)       # many exact ties
    val, idx = O.top_k(sc, 10)
    for i in range(6):
        order = sorted(range(500), key=lambda j: (-sc[i, j], j))[:10]
        assert list(idx[i]) == order
        np.testing.assert_array_equal(val[i], sc[i, order])


# ---- threshold-gated cold tier (Monarch v3, simplified decode loop) ------

def _gated_case(seed=11, d=16, m=16, b=3, hq=4, hkv=2, nh=6, nc=20):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((hq, d))
    hk = rng.standard_normal((hkv, nh, d))
    hv = rng.standard_normal((hkv, nh, d))
    signs = O.rotation_signs(5, d)
    S = O.qjl_matrix(5, m, d)
    ck = [O.encode(rng.standard_normal((nc, d)), signs, S, b, b) for _ in range(hkv)]
    cv = [O.encode(rng.standard_normal((nc, d)), signs, None, b, b) for _ in range(hkv)]
    return q, hk, hv, ck, cv, signs, S, hkv


def test_gate_closed_is_plain_decode():
    """A threshold above every hot score reads the cold tier for every head:
    the gated output is the ungated one."""
    q, hk, hv, ck, cv, signs, S, hkv = _gated_case()
    out, skip = O.decode_attention_gated(q, hk, hv, ck, cv, signs, S, hkv, math.inf)
    assert not skip.any()
    np.testing.assert_array_equal(out, O.decode_attention(q, hk, hv, ck, cv, signs, S, hkv))


def test_gate_open_is_textbook_hot_attention():
    """A threshold of -inf skips the cold tier of every head with a hot
    window: the output is textbook softmax attention over the hot tokens,
    here written out with scipy's softmax."""
    from scipy.special import softmax
    q, hk, hv, ck, cv, signs, S, hkv = _gated_case()
    out, skip = O.decode_attention_gated(q, hk, hv, ck, cv, signs, S, hkv, -math.inf)
    assert skip.all()
    d = q.shape[1]
    for h in range(q.shape[0]):
        g = h // (q.shape[0] // hkv)
        p = softmax(hk[g] @ q[h] / math.sqrt(d))
        np.testing.assert_allclose(out[h], p @ hv[g], rtol=1e-12, atol=1e-14)


def test_gate_boundary_and_empty_hot_window():
    """Equality with the threshold skips (the cold tier is read only below
    it); an empty hot window always reads the cold tier."""
    q, hk, hv, ck, cv, signs, S, hkv = _gated_case()
    g = q.shape[0] // hkv
    best = [float((hk[h // g] @ q[h]).max()) for h in range(q.shape[0])]
    skip = O.hot_gate(q, hk, hkv, best[0])
    assert skip[0]
    assert list(skip) == [b >= best[0] for b in best]
    empty = hk[:, :0]
    out, skip = O.decode_attention_gated(q, empty, hv[:, :0], ck, cv, signs, S, hkv, -math.inf)
    assert not skip.any()
    np.testing.assert_array_equal(out, O.decode_attention(q, empty, hv[:, :0], ck, cv, signs, S, hkv))


# ---- Tensor Cache second tier (outer-product memory of evicted tokens) ----

def test_tc_sequence_equals_weighted_closed_form():
    """Sequential writes equal the weighted sum the page's parallel scan
    computes: A_E = lambda^E A_0 + eta sum_e lambda^(E-1-e) k_e v_e^T,
    written here as one matrix product K^T diag(w) V."""
    rng = np.random.default_rng(21)
    d, E, lam, eta = 8, 37, 0.93, 0.4
    A0 = rng.standard_normal((d, d))
    K = rng.standard_normal((E, d))
    V = rng.standard_normal((E, d))
    seq = O.tc_write_sequence(A0, K, V, lam, eta)
    w = eta * lam ** (E - 1 - np.arange(E))
    closed = lam ** E * A0 + K.T @ (w[:, None] * V)
    np.testing.assert_allclose(seq, closed, rtol=1e-12, atol=1e-12)
    # lambda = eta = 1: the plain sum of outer products K^T V
    np.testing.assert_allclose(O.tc_write_sequence(np.zeros((d, d)), K, V, 1.0, 1.0), K.T @ V,
                               rtol=1e-12, atol=1e-12)


def test_tc_read_is_linear_attention_identity():
    """q (k outer v) = <q, k> v: one write into an empty memory returns the
    value scaled by eta times the key's inner product with the query."""
    rng = np.random.default_rng(22)
    d = 16
    q, k, v = rng.standard_normal((3, d))
    A = O.tc_write(np.zeros((d, d)), k, v, 0.5, 0.25)
    np.testing.assert_allclose(q @ A, 0.25 * (q @ k) * v, rtol=1e-12, atol=1e-14)


def test_tc_decode_gate_limits():
    """A closed gate (g -> -inf) leaves textbook softmax attention over the
    ring (scipy's softmax); g = 0 adds half the memory read; with an empty
    memory the gate has no effect."""
    from scipy.special import softmax
    rng = np.random.default_rng(23)
    hq, hkv, W, d = 4, 2, 6, 8
    q = rng.standard_normal((hq, d))
    hk = rng.standard_normal((hkv, W, d))
    hv = rng.standard_normal((hkv, W, d))
    A = rng.standard_normal((hkv, d, d))
    closed = O.tc_decode(q, hk, hv, A, np.full(hq, -800.0), hkv)
    half = O.tc_decode(q, hk, hv, A, np.zeros(hq), hkv)
    empty = O.tc_decode(q, hk, hv, np.zeros((hkv, d, d)), rng.standard_normal(hq), hkv)
    for h in range(hq):
        g = h // (hq // hkv)
        local = softmax(hk[g] @ q[h] / math.sqrt(d)) @ hv[g]
        np.testing.assert_allclose(closed[h], local, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(empty[h], local, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(half[h], local + 0.5 * (q[h] @ A[g]), rtol=1e-12, atol=1e-12)


# ---- value-side QJL (the residual's sign sketch reconstructs the vector) ---

def test_qjl_vector_estimate_unbiased_and_variance():
    """For s ~ N(0, I), E[sign(<s, r>) s] = sqrt(2/pi) r/|r|, so the
    estimate sqrt(pi/2)/m |r| S^T sign(S r) has mean r; its variance falls
    as 1/m."""
    rng = np.random.default_rng(41)
    d, N = 16, 6000
    r = rng.standard_normal(d)
    nr = np.linalg.norm(r)

    def draws(m):
        est = np.empty((N, d))
        for t in range(N):
            S = rng.standard_normal((m, d)).astype(np.float32)
            bits = (S.astype(np.float64) @ r >= 0)[None]
            est[t] = O.qjl_vector_estimate(S, bits, np.array([nr]))[0]
        return est

    e4 = draws(4)
    e16 = draws(16)
    for e in (e4, e16):
        se = e.std(axis=0) / math.sqrt(N)
        assert np.all(np.abs(e.mean(axis=0) - r) < 4.5 * se)
    ratio = e4.var(axis=0).sum() / e16.var(axis=0).sum()
    assert 3.0 < ratio < 5.0


def test_value_qjl_attention_converges_to_exact_values():
    """With the values' residual sketched by m bits, the cold part of the
    output tends to the one with exact (rotated) values as m grows: the
    error at m = 4096 is far below the error of the codes alone."""
    rng = np.random.default_rng(42)
    hq, hkv, d, nc, b = 2, 1, 16, 12, 2
    q = rng.standard_normal((hq, d))
    kx = rng.standard_normal((nc, d))
    vx = rng.standard_normal((nc, d))
    signs = O.rotation_signs(9, d)
    errs = []
    for m in (0, 64, 4096):
        S = O.qjl_matrix(9, max(m, 8), d)
        ck = [O.encode(kx, signs, S, b, b)]
        cv = [O.encode(vx, signs, S, b, b)]
        if m == 0:
            out = O.decode_attention(q, None, None, ck, cv, signs, S, hkv)
        else:
            out = O.decode_attention_vqjl(q, None, None, ck, cv, signs, S, hkv)
        # the same logits with exact values: p from the cold logits
        exact = np.zeros((hq, d))
        for h in range(hq):
            lg = O.key_inner_products(q[h], signs, S, ck[0]) / math.sqrt(d)
            p = np.exp(lg - lg.max())
            exact[h] = (p / p.sum()) @ vx
        errs.append(np.abs(out - exact).max())
    assert errs[2] < 0.25 * errs[0] and errs[2] < errs[1]


# ---- attention-weighted promotion with sticky counters (Monarch) ----------

def test_promotion_counters_worked_sequence():
    """Threshold 0.15, sticky 3, worked by hand: a miss resets the count,
    equality counts as a hit, the third hit in a row promotes and clears."""
    masses = [0.2, 0.15, 0.1, 0.3, 0.16, 0.9, 0.9, 0.0]
    want_c = [1, 2, 0, 1, 2, 0, 1, 0]
    want_p = [False, False, False, False, False, True, False, False]
    c = np.zeros(1, dtype=np.int64)
    for m, wc, wp in zip(masses, want_c, want_p):
        c, p = O.promotion_step(c, np.array([m]), 0.15, 3)
        assert c[0] == wc and p[0] == wp


def test_cold_mass_and_weights():
    """With no hot window each kv head's cold masses sum to 1; with one, the
    cold weights and the hot weights of every head sum to 1 (recomputed
    here from the hot logits with scipy's logsumexp)."""
    from scipy.special import logsumexp
    rng = np.random.default_rng(51)
    hq, hkv, d, nc, nh = 4, 2, 8, 10, 3
    q = rng.standard_normal((hq, d))
    signs = O.rotation_signs(2, d)
    S = O.qjl_matrix(2, 8, d)
    ck = [O.encode(rng.standard_normal((nc, d)), signs, S, 3, 3) for _ in range(hkv)]
    hk = rng.standard_normal((hkv, nh, d))
    w0 = O.cold_softmax_weights(q, None, ck, signs, S, hkv)
    np.testing.assert_allclose(O.cold_attention_mass(w0, hkv).sum(axis=1), 1.0, rtol=1e-12)
    w = O.cold_softmax_weights(q, hk, ck, signs, S, hkv)
    for h in range(hq):
        g = h // (hq // hkv)
        lc = O.key_inner_products(q[h], signs, S, ck[g]) / math.sqrt(d)
        lh = hk[g] @ q[h] / math.sqrt(d)
        lse = logsumexp(np.concatenate([lc, lh]))
        np.testing.assert_allclose(w[h], np.exp(lc - lse), rtol=1e-12)
    m = O.cold_attention_mass(w, hkv)
    np.testing.assert_allclose(m[0], w[:2].mean(axis=0), rtol=1e-15)


def test_qjl_vector_estimate_error_closed_form():
    """E|r_hat - r|^2 = |r|^2 (pi d / (2 m) - 1 / m) for the sign-sketch
    estimate of a vector (from E|s|^2 = d and E[sign(<s, r>) s] =
    sqrt(2/pi) r/|r| for s ~ N(0, I)); so the sketch lowers a value's error
    only when m > pi d / 2."""
    rng = np.random.default_rng(44)
    d, N = 16, 4000
    r = rng.standard_normal(d)
    nr2 = float(r @ r)
    for m in (8, 32):
        errs = np.empty(N)
        for t in range(N):
            S = rng.standard_normal((m, d)).astype(np.float32)
            bits = (S.astype(np.float64) @ r >= 0)[None]
            e = O.qjl_vector_estimate(S, bits, np.array([math.sqrt(nr2)]))[0] - r
            errs[t] = e @ e
        want = nr2 * (math.pi * d / (2 * m) - 1.0 / m)
        assert abs(errs.mean() - want) < 4 * errs.std() / math.sqrt(N), (m, errs.mean(), want)


def _tags(xs):
    return [int(round(float(x[0]))) for x in xs]


def test_promoting_unit_hand_worked_trace():
    """W = 2, threshold 0.15, sticky 2, tokens tagged by value; worked by
    hand: a promoted token re-enters the ring before the new token, the
    eviction it causes takes the promoted cold position, the next one is
    appended."""
    u = O.PromotingUnit(W=2, d=1, threshold=0.15, sticky=2)
    a, b, c, d, e, f, g = ([[float(t)]] for t in (1, 2, 3, 4, 5, 6, 7))
    u.append_cold(np.array(a + b + c), np.array(a + b + c))
    assert u.insert(np.array(d + e), np.array(d + e), np.zeros((0, 1)), np.zeros((0, 1))) == []
    assert list(u.after_decode(np.array([0.1, 0.5, 0.0]))) == []
    assert list(u.counters) == [0, 1, 0]
    assert u.insert(np.array(f), np.array(f), np.zeros((0, 1)), np.zeros((0, 1))) == [3]   # d appended
    assert list(u.after_decode(np.array([0.2, 0.6, 0.0, 0.3]))) == [1]                    # b promoted
    assert list(u.counters) == [1, 0, 0, 1]
    b_deq = np.array([[1002.0]])           # stands in for b's fp16 dequantization
    assert u.insert(np.array(g), np.array(g), b_deq, b_deq) == [1, 4]   # e takes b's place, f appended
    assert _tags(u.cold_k) == [1, 5, 3, 4, 6]
    assert list(u.counters) == [1, 0, 0, 1, 0]
    assert _tags(u.ring_k) == [7, 1002] and u.ring_pos == 1
    assert list(u.after_decode(np.array([0.0, 0.0, 0.0, 0.0, 0.9]))) == []
    assert list(u.counters) == [0, 0, 0, 0, 1]


def test_promoting_unit_drops_promotions_before_the_ring_is_full():
    u = O.PromotingUnit(W=3, d=1, threshold=0.15, sticky=1)
    u.append_cold(np.array([[1.0]]), np.array([[1.0]]))
    u.insert(np.array([[2.0]]), np.array([[2.0]]), np.zeros((0, 1)), np.zeros((0, 1)))
    assert list(u.after_decode(np.array([0.9]))) == [] and u.pending == []
    assert list(u.counters) == [0]


def test_promoting_unit_conserves_tokens():
    """Random masses over many steps: every inserted token is in the ring or
    the cold list exactly once (a promoted one as its stand-in), the cold
    list grows by one per inserted token once the ring is full, and no step
    promotes more than floor(1 / threshold) tokens."""
    rng = np.random.default_rng(61)
    W, thr = 4, 0.15
    u = O.PromotingUnit(W=W, d=1, threshold=thr, sticky=2)
    u.append_cold(np.arange(100, 110, dtype=np.float64)[:, None], np.zeros((10, 1)))
    u.insert(np.arange(200, 204, dtype=np.float64)[:, None], np.zeros((4, 1)), np.zeros((0, 1)),
             np.zeros((0, 1)))
    alive = set(range(100, 110)) | set(range(200, 204))
    nxt = 300
    for step in range(200):
        n_before = len(u.cold_k)
        # a promoted token t re-enters as a stand-in tagged 10 t + 5
        old = [int(round(u.cold_k[i][0])) for i in u.pending]
        for t in old:
            alive.remove(t)
            alive.add(10 * t + 5)
        prom_tags = np.array([[10.0 * t + 5] for t in old]).reshape(-1, 1)
        u.insert(np.array([[float(nxt)]]), np.zeros((1, 1)), prom_tags, np.zeros_like(prom_tags))
        alive.add(nxt)
        nxt += 1
        assert len(u.cold_k) == n_before + 1
        have = sorted(_tags(u.cold_k) + _tags(u.ring_k))
        assert have == sorted(alive)
        n = len(u.cold_k)
        raw = rng.dirichlet(np.full(n, 0.05))          # a peaked mass vector summing to 1
        p = u.after_decode(raw * rng.uniform(0.5, 1.0))
        assert len(p) <= int(1 / thr)
