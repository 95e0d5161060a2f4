"""GPU parity of the Tensor Cache second tier: after a sequence of
evictions the device matrices A equal the oracle's sequential writes
(float32 against float64: |A_gpu - A_ref| <= 1e-5 max|A_ref| + 1e-6), and
every decode output row is within 2e-3 (relative L2 per query head) of the
oracle's ring attention plus sigmoid(g) q A."""
import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import WORKLOADS, Workload, gaussian_fp16, queries
from oracle import tq_oracle as O
from tests.tq_testutil import ATTN_RTOL, config_for, rel_err

pytestmark = pytest.mark.gpu


def _params(hkv, hq, seed):
    rng = np.random.default_rng(seed)
    lam = rng.uniform(0.85, 0.999, hkv)
    eta = rng.uniform(0.02, 0.2, hkv)
    gate = rng.uniform(-2.0, 2.0, hq)
    return lam.astype(np.float32), eta.astype(np.float32), gate.astype(np.float32)


class _Model:
    """Host bookkeeping of every token inserted per (row, kv head): the last
    W are the ring, all earlier ones have been evicted (oldest first)."""

    def __init__(self, B, hkv, d):
        self.k = np.zeros((B, hkv, 0, d))
        self.v = np.zeros((B, hkv, 0, d))

    def insert(self, k, v):
        self.k = np.concatenate([self.k, k.astype(np.float64)], axis=2)
        self.v = np.concatenate([self.v, v.astype(np.float64)], axis=2)


def _check(cache, cfg, model, A_dev, lam, eta, gate, q, W):
    B, hkv, d = cfg.batch, cfg.num_kv_heads, cfg.head_dim
    n = model.k.shape[2]
    ne = max(0, n - W)
    A_ref = np.zeros((B, hkv, d, d))
    for b in range(B):
        for h in range(hkv):
            A_ref[b, h] = O.tc_write_sequence(np.zeros((d, d)), model.k[b, h, :ne], model.v[b, h, :ne],
                                              float(lam[h]), float(eta[h]))
    got_A = A_dev.cpu().numpy().astype(np.float64)
    tol = 1e-5 * max(np.abs(A_ref).max(), 1e-30) + 1e-6
    assert np.abs(got_A - A_ref).max() <= tol, (np.abs(got_A - A_ref).max(), tol)
    out = cache.decode_attention(torch.from_numpy(q).cuda())
    assert cache.get_status() == 0
    got = out.cpu().numpy().astype(np.float64)
    errs = []
    for b in range(B):
        ref = O.tc_decode(q[b].astype(np.float64), model.k[b, :, ne:], model.v[b, :, ne:], A_ref[b],
                          gate.astype(np.float64), hkv)
        e = rel_err(got[b], ref)
        assert np.all(e <= ATTN_RTOL), (b, e.max())
        errs.append(e)
    return np.concatenate(errs)


@pytest.mark.parametrize("name,batch,W", [("llama8b", 2, 64), ("tinyllama", 1, 128), ("tiny", 1, 32)])
def test_tensor_cache_parity(name, batch, W):
    wl = WORKLOADS[name]
    cfg = config_for(wl, batch=batch, hot_window=W, cold_capacity=0)
    cache = tq.TQCache(cfg)
    lam, eta, gate = _params(cfg.num_kv_heads, cfg.num_q_heads, 5)
    A = cache.enable_tensor_cache(lam, eta, gate)
    model = _Model(batch, cfg.num_kv_heads, cfg.head_dim)
    step = [0]

    def feed(n):
        shape = (batch, cfg.num_kv_heads, n, cfg.head_dim)
        k = gaussian_fp16(shape, 40, step[0], 0)
        v = gaussian_fp16(shape, 40, step[0], 1)
        step[0] += 1
        cache.evict_window(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
        model.insert(k, v)

    q = queries(wl, 0, 3)[:batch]
    feed(W // 2)                      # ring not full: no eviction, A stays 0
    _check(cache, cfg, model, A, lam, eta, gate, q, W)
    feed(W)                           # W/2 ring tokens evicted in one run
    feed(W + 37)                      # the whole ring plus 37 new tokens that never enter it
    for _ in range(5):                # decode steps: one eviction each
        feed(1)
    e = _check(cache, cfg, model, A, lam, eta, gate, q, W)
    print(name, "evicted", model.k.shape[2] - W, "max rel err", float(e.max()))
    cache.close()


def test_tensor_cache_long_run_and_scale():
    """Many evictions through the run path (4096 tokens at once) and the
    decay over them, then decode with another softmax scale."""
    wl = Workload("tc", 1, 2, 8, 2, 128, 64, 0, 3, 3, 128, "lognormal")
    cfg = config_for(wl, batch=2, hot_window=64, cold_capacity=0)
    cache = tq.TQCache(cfg)
    lam, eta, gate = _params(2, 8, 6)
    A = cache.enable_tensor_cache(lam, eta, gate)
    model = _Model(2, 2, 128)
    k = gaussian_fp16((2, 2, 4096, 128), 41, 0)
    v = gaussian_fp16((2, 2, 4096, 128), 41, 1)
    cache.evict_window(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    model.insert(k, v)
    _check(cache, cfg, model, A, lam, eta, gate, queries(wl, 0, 1)[:2], 64)
    cache.close()


def test_tensor_cache_argument_checks():
    wl = WORKLOADS["llama8b"]
    cfg = config_for(wl, batch=1, hot_window=64, cold_capacity=0)
    cache = tq.TQCache(cfg)
    lam, eta, gate = _params(8, 32, 7)
    bad = lam.copy()
    bad[3] = np.nan
    with pytest.raises(tq.TQError):
        cache.enable_tensor_cache(bad, eta, gate)
    cache.enable_tensor_cache(lam, eta, gate)
    with pytest.raises(tq.TQError):                 # already enabled
        cache.enable_tensor_cache(lam, eta, gate)
    cache.close()
