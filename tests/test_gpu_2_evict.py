"""GPU ring eviction: tq_evict_window replayed against the oracle's ring.
Hot slots must hold the same fp16 bits; evicted tokens must be encoded
bit-exactly (ties excepted) in age order; decode over the result must
match the oracle."""
import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import WORKLOADS, Workload, kv_block, queries
from oracle import tq_oracle as O
from tests.tq_testutil import (ATTN_RTOL, CodeReport, compare_codes, config_for,
                               oracle_decode_row, oracle_signs_S, rel_err)

pytestmark = pytest.mark.gpu


def _replay(wl: Workload, batch: int, W: int, prefix: int, inserts, seed=0):
    total = prefix + sum(inserts)
    cap = total
    cfg = config_for(wl, batch=batch, hot_window=W, cold_capacity=cap, seed=seed)
    cache = tq.TQCache(cfg)
    k = kv_block(wl, 0, seed, 0, 0, total)[:batch]
    v = kv_block(wl, 0, seed, 1, 0, total)[:batch]
    rings_k = [[O.RingState(W=W, d=wl.head_dim) for _ in range(wl.num_kv_heads)] for _ in range(batch)]
    rings_v = [[O.RingState(W=W, d=wl.head_dim) for _ in range(wl.num_kv_heads)] for _ in range(batch)]
    if prefix:
        cache.encode_append(torch.from_numpy(np.ascontiguousarray(k[:, :, :prefix])).cuda(),
                            torch.from_numpy(np.ascontiguousarray(v[:, :, :prefix])).cuda())
    pos = prefix
    for n in inserts:
        cache.evict_window(torch.from_numpy(np.ascontiguousarray(k[:, :, pos:pos + n])).cuda(),
                           torch.from_numpy(np.ascontiguousarray(v[:, :, pos:pos + n])).cuda())
        for b in range(batch):
            for h in range(wl.num_kv_heads):
                rings_k[b][h].insert(k[b, h, pos:pos + n])
                rings_v[b][h].insert(v[b, h, pos:pos + n])
        pos += n
    assert cache.get_status() == 0
    r0 = rings_k[0][0]
    n_cold = prefix + len(r0.cold_vectors)
    assert cache.counts() == (n_cold, r0.n_hot, r0.ring_pos)
    hk, hv = cache.hot_ring()
    hk, hv = hk.cpu().numpy(), hv.cpu().numpy()
    signs, S = oracle_signs_S(cfg)
    rep = CodeReport()
    for b in range(batch):
        for h in range(wl.num_kv_heads):
            valid = r0.n_hot
            np.testing.assert_array_equal(hk[b, h, :valid].view(np.uint16),
                                          rings_k[b][h].slots()[:valid].astype(np.float16).view(np.uint16))
            np.testing.assert_array_equal(hv[b, h, :valid].view(np.uint16),
                                          rings_v[b][h].slots()[:valid].astype(np.float16).view(np.uint16))
            ev_k = np.array(rings_k[b][h].cold_vectors).reshape(-1, wl.head_dim)
            ev_v = np.array(rings_v[b][h].cold_vectors).reshape(-1, wl.head_dim)
            all_k = np.concatenate([k[b, h, :prefix].astype(np.float64), ev_k])
            all_v = np.concatenate([v[b, h, :prefix].astype(np.float64), ev_v])
            exp = cache.export_cold(b, h, 0, n_cold)
            rep.add(compare_codes(exp, O.encode(all_k, signs, S, cfg.b_r, cfg.b_theta), cfg, True))
            rep.add(compare_codes(exp, O.encode(all_v, signs, None, cfg.b_r, cfg.b_theta), cfg, False))
    print(rep)
    # decode over the evolved cache
    q = queries(wl, 0, seed, step=5)[:batch]
    out = cache.decode_attention(torch.from_numpy(q).cuda()).cpu().numpy().astype(np.float64)
    for b in range(batch):
        hot_k = np.stack([rings_k[b][h].hot_tokens() for h in range(wl.num_kv_heads)])
        hot_v = np.stack([rings_v[b][h].hot_tokens() for h in range(wl.num_kv_heads)])
        ref = oracle_decode_row(cache, b, q[b], hot_k, hot_v, signs, S)
        assert np.all(rel_err(out[b], ref) <= ATTN_RTOL)
    cache.close()


def test_ring_fill_then_single_token_steps():
    # the long-context pattern in miniature: a cold prefix, the hot ring
    # filled in one call, then one-token decode steps that each evict
    _replay(WORKLOADS["longctx"], 1, 64, 256, [64] + [1] * 20)


def test_ring_multi_token_inserts_and_wraparound():
    _replay(WORKLOADS["llama8b"], 2, 32, 0, [5, 30, 7, 1, 33, 64, 2])


def test_ring_insert_larger_than_window():
    # tokens displaced inside the same call go straight to the cold store
    _replay(WORKLOADS["tiny"], 1, 16, 10, [3, 50, 1, 17])
