"""GPU parity of the threshold-gated cold tier (tq_decode_attention_gated):
the per-head skip decisions equal the oracle's exactly, and every output
row is within 2e-3 (relative L2 per query head) of the fp64 oracle's gated
attention fed the GPU's own cold records.

Thresholds are placed inside gaps of the heads' hot maxima (computed here
in fp64 from the same fp16 inputs), so no decision sits within rounding of
the threshold; the kernel's fp32 maxima decide the same way."""
import math

import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import WORKLOADS, Workload, kv_block, queries
from oracle import tq_oracle as O
from tests.tq_testutil import (ATTN_RTOL, codes_from_export, config_for, oracle_signs_S, rel_err)

pytestmark = pytest.mark.gpu


def _cache(wl, batch, n_cold, n_hot, W, seed=0, spare=0):
    cfg = config_for(wl, batch=batch, hot_window=W, cold_capacity=max(n_cold + spare, 1), seed=seed)
    cache = tq.TQCache(cfg)
    total = n_cold + n_hot
    k = kv_block(wl, 0, seed, 0, 0, total)[:batch]
    v = kv_block(wl, 0, seed, 1, 0, total)[:batch]
    if n_cold:
        cache.encode_append(torch.from_numpy(np.ascontiguousarray(k[:, :, :n_cold])).cuda(),
                            torch.from_numpy(np.ascontiguousarray(v[:, :, :n_cold])).cuda())
    if n_hot:
        cache.evict_window(torch.from_numpy(np.ascontiguousarray(k[:, :, n_cold:])).cuda(),
                           torch.from_numpy(np.ascontiguousarray(v[:, :, n_cold:])).cuda())
    return cache, cfg, k, v


def _hot_max(q, k, n_cold, hkv):
    """fp64 max_t q.k_t over the hot tokens, [B, Hq] (empty window: -inf)."""
    B, hq, _ = q.shape
    g = hq // hkv
    out = np.full((B, hq), -np.inf)
    hot = k[:, :, n_cold:].astype(np.float64)
    if hot.shape[2]:
        for b in range(B):
            for h in range(hq):
                out[b, h] = (hot[b, h // g] @ q[b, h].astype(np.float64)).max()
    return out


def _threshold_in_gap(values, quantile):
    """A threshold near the given quantile of ``values``, in the middle of
    the widest nearby gap (so that no value is within rounding of it)."""
    v = np.sort(values.ravel())
    i = int(np.clip(round(quantile * (v.size - 1)), 1, v.size - 1))
    lo, hi = max(1, i - 4), min(v.size - 1, i + 4)
    j = max(range(lo, hi + 1), key=lambda t: v[t] - v[t - 1])
    gap = v[j] - v[j - 1]
    assert gap > 1e-3 * np.abs(v).max(), "no usable gap"
    return 0.5 * (v[j] + v[j - 1])


def _check(cache, cfg, q, k, v, n_cold, threshold, scale=None, user_skip=True):
    B = q.shape[0]
    hs = torch.full((B, cfg.num_q_heads), -7, dtype=torch.int32, device="cuda") if user_skip else None
    out = cache.decode_attention_gated(torch.from_numpy(q).cuda(), threshold, head_skip=hs,
                                       softmax_scale=0.0 if scale is None else scale)
    assert cache.get_status() == 0
    got = out.cpu().numpy().astype(np.float64)
    signs, S = oracle_signs_S(cfg)
    nc = cache.counts()[0]
    skips = []
    for b in range(B):
        ck, cv = [], []
        for h in range(cfg.num_kv_heads):
            if nc:
                exp = cache.export_cold(b, h, 0, nc)
                ck.append(codes_from_export(exp, cfg, True))
                cv.append(codes_from_export(exp, cfg, False))
            else:
                ck.append(None)
                cv.append(None)
        ref, skip = O.decode_attention_gated(q[b].astype(np.float64),
                                             k[b, :, n_cold:].astype(np.float64),
                                             v[b, :, n_cold:].astype(np.float64), ck, cv, signs, S,
                                             cfg.num_kv_heads, threshold, scale)
        e = rel_err(got[b], ref)
        assert np.all(e <= ATTN_RTOL), (b, e.max(), np.argmax(e))
        skips.append(skip)
    skips = np.array(skips)
    if hs is not None:
        np.testing.assert_array_equal(hs.cpu().numpy(), skips.astype(np.int32))
    return skips


@pytest.mark.parametrize("name,batch,n_cold,n_hot", [
    ("llama8b", 2, 1500, 512),       # G = 4 (packed columns), ragged cold tail
    ("tinyllama", 1, 1024, 512),     # G = 8
    ("tiny", 1, 192, 64),
])
@pytest.mark.parametrize("quantile", [0.2, 0.5, 0.85])
def test_gated_parity_mixed(name, batch, n_cold, n_hot, quantile):
    wl = WORKLOADS[name]
    cache, cfg, k, v = _cache(wl, batch, n_cold, n_hot, wl.hot)
    q = queries(wl, 0, 0)[:batch]
    thr = _threshold_in_gap(_hot_max(q, k, n_cold, cfg.num_kv_heads), quantile)
    skips = _check(cache, cfg, q, k, v, n_cold, thr)
    G = cfg.num_q_heads // cfg.num_kv_heads
    whole = skips.reshape(batch, cfg.num_kv_heads, G).all(axis=2)
    print(name, quantile, "heads skipped", int(skips.sum()), "of", skips.size,
          "units skipped", int(whole.sum()), "of", whole.size)
    assert 0 < skips.sum() < skips.size
    cache.close()


def test_gated_whole_units_skip():
    """Raise the queries of every other kv head's group so that whole units
    skip while their neighbours read the cold tier (the compacted split)."""
    wl = WORKLOADS["llama8b"]
    batch = 2
    cache, cfg, k, v = _cache(wl, batch, 2100, 300, 512, seed=3)
    q = queries(wl, 0, 3)[:batch].astype(np.float64)
    G = cfg.num_q_heads // cfg.num_kv_heads
    for h in range(cfg.num_q_heads):
        if (h // G) % 2 == 0:
            q[:, h] *= 4.0
    q = q.astype(np.float16)
    hm = _hot_max(q, k, 2100, cfg.num_kv_heads)
    lifted = np.array([[(h // G) % 2 == 0 for h in range(cfg.num_q_heads)]] * batch)
    thr = 0.5 * (hm[lifted].min() + hm[~lifted].max())
    if not hm[lifted].min() > hm[~lifted].max() * 1.001:
        thr = _threshold_in_gap(hm, 0.5)
    skips = _check(cache, cfg, q, k, v, 2100, thr)
    whole = skips.reshape(batch, cfg.num_kv_heads, G).all(axis=2)
    assert whole.any() and not whole.all()
    cache.close()


@pytest.mark.parametrize("thr", [math.inf, -math.inf])
def test_gated_extremes(thr):
    """+inf reads every cold tier (the ungated result); -inf skips every
    head with a hot window (attention over the hot window alone)."""
    wl = WORKLOADS["llama8b"]
    cache, cfg, k, v = _cache(wl, 2, 900, 200, 256)
    q = queries(wl, 0, 0)[:2]
    skips = _check(cache, cfg, q, k, v, 900, thr, user_skip=(thr > 0))
    assert skips.all() == (thr < 0) and skips.any() == (thr < 0)
    if thr > 0:     # same output as the ungated call, up to the partials' summation order
        a = cache.decode_attention(torch.from_numpy(q).cuda()).cpu().numpy()
        b = cache.decode_attention_gated(torch.from_numpy(q).cuda(), thr).cpu().numpy()
        np.testing.assert_allclose(b, a, rtol=1e-5, atol=1e-6)
    cache.close()


@pytest.mark.parametrize("n_cold,n_hot", [(700, 0), (0, 130), (0, 0), (65, 1)])
def test_gated_edge_windows(n_cold, n_hot):
    """An empty hot window never skips; a cache without cold tokens or
    without anything at all still gives the oracle's result."""
    wl = WORKLOADS["llama8b"]
    cache, cfg, k, v = _cache(wl, 1, n_cold, n_hot, 256)
    q = queries(wl, 0, 0)[:1]
    skips = _check(cache, cfg, q, k, v, n_cold, -math.inf)
    assert skips.all() == (n_hot > 0)
    cache.close()


def test_gated_shapes_and_scale():
    wl = Workload("grid", 1, 2, 16, 2, 64, 64, 300, 2, 3, 64, "lognormal")
    cache, cfg, k, v = _cache(wl, 2, 300, 64, 64, seed=5)
    q = queries(wl, 0, 5)[:2]
    thr = _threshold_in_gap(_hot_max(q, k, 300, cfg.num_kv_heads), 0.4)
    _check(cache, cfg, q, k, v, 300, thr, scale=3.0 / math.sqrt(64))
    cache.close()


def test_gated_argument_checks():
    wl = WORKLOADS["llama8b"]
    cache, cfg, _, _ = _cache(wl, 1, 64, 8, 64)
    q = torch.from_numpy(queries(wl, 0, 0)[:1]).cuda()
    with pytest.raises(tq.TQError):
        cache.decode_attention_gated(q, float("nan"))
    with pytest.raises(ValueError):
        cache.decode_attention_gated(q, 0.0, head_skip=torch.zeros(32, dtype=torch.int64, device="cuda"))
    # queries must start on a 16-byte boundary (ungated and gated calls)
    buf = torch.zeros(q.numel() + 8, dtype=torch.float16, device="cuda")
    q_off = buf[1:1 + q.numel()].view(q.shape)
    with pytest.raises(tq.TQError):
        cache.decode_attention(q_off)
    with pytest.raises(tq.TQError):
        cache.decode_attention_gated(q_off, 0.0)
    cache.close()


@pytest.mark.parametrize("name", ["llama8b", "tinyllama"])
def test_gated_after_single_token_eviction(name):
    """The decode step: one new token evicts into a full window, then the
    gated call.  The gate reads the new token's ring slot only after the
    eviction has finished; the token is built so that it alone lifts some
    heads' hot maxima past the threshold."""
    wl = WORKLOADS[name]
    W, n_cold = 64, 300
    cache, cfg, k, v = _cache(wl, 1, n_cold, W, W, seed=9, spare=8)
    G = cfg.num_q_heads // cfg.num_kv_heads
    q = queries(wl, 0, 9)[:1]
    old = _hot_max(q, k, n_cold, cfg.num_kv_heads)[0]
    # new token: in kv head 0, K = 4 q of query head 0 (q.k = 4 |q|^2, far above the window)
    k_new = np.zeros((1, cfg.num_kv_heads, 1, cfg.head_dim), dtype=np.float16)
    v_new = (np.arange(cfg.num_kv_heads * cfg.head_dim, dtype=np.float64)
             .reshape(1, cfg.num_kv_heads, 1, cfg.head_dim) % 7 - 3).astype(np.float16)
    k_new[0, 0, 0] = (4.0 * q[0, 0].astype(np.float64)).astype(np.float16)
    for h in range(1, cfg.num_kv_heads):
        k_new[0, h, 0] = k[0, h, n_cold]        # elsewhere a copy of an existing hot key
    cache.evict_window(torch.from_numpy(k_new).cuda(), torch.from_numpy(v_new).cuda())
    hk, hv = cache.hot_ring()
    hk = hk.cpu().numpy().astype(np.float64)[0]
    hv = hv.cpu().numpy().astype(np.float64)[0]
    new = np.array([(hk[h // G] @ q[0, h].astype(np.float64)).max() for h in range(cfg.num_q_heads)])
    assert new[0] > old.max() * 1.5
    thr = 0.5 * (old.max() + new[0])           # only head 0's new maximum reaches it
    hs = torch.zeros((1, cfg.num_q_heads), dtype=torch.int32, device="cuda")
    out = cache.decode_attention_gated(torch.from_numpy(q).cuda(), thr, head_skip=hs)
    assert cache.get_status() == 0
    skip_gpu = hs.cpu().numpy()[0]
    assert skip_gpu[0] == 1 and skip_gpu[1:].sum() == (new[1:] >= thr).sum()
    nc = cache.counts()[0]
    signs, S = oracle_signs_S(cfg)
    ck, cv = [], []
    for h in range(cfg.num_kv_heads):
        exp = cache.export_cold(0, h, 0, nc)
        ck.append(codes_from_export(exp, cfg, True))
        cv.append(codes_from_export(exp, cfg, False))
    ref, skip = O.decode_attention_gated(q[0].astype(np.float64), hk, hv, ck, cv, signs, S,
                                         cfg.num_kv_heads, thr)
    np.testing.assert_array_equal(skip_gpu, skip.astype(np.int32))
    e = rel_err(out.cpu().numpy()[0].astype(np.float64), ref)
    assert np.all(e <= ATTN_RTOL), e.max()
    cache.close()
