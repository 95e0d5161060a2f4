"""tq_decode_attention_static: decode attention for callers that may not
allocate device memory while they run (an allocator-free serving loop, a
plugin whose host framework owns every allocation).  It keeps its per-call
scratch in a fixed array inside the library, so, call after call, with
nothing left over from the previous call, it must give the fp64 oracle's
answer (fed the GPU's own records) and agree with tq_decode_attention.

This file is collected last on purpose: a failure here cannot hide the
results of the other GPU tests.  It also passes when run alone.
"""
import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import WORKLOADS, kv_block, queries
from tests.tq_testutil import (ATTN_RTOL, cold_blocks_per_cta_lower_bound, config_for,
                               oracle_decode_row, oracle_decode_unit, oracle_signs_S, rel_err)

pytestmark = pytest.mark.gpu


def _filled_cache(name, batch, n_cold, n_hot, seed=0):
    wl = WORKLOADS[name]
    cfg = config_for(wl, batch=batch, cold_capacity=max(n_cold, 1), seed=seed)
    cache = tq.TQCache(cfg)
    k = kv_block(wl, 0, seed, 0, 0, n_cold + n_hot)[:batch]
    v = kv_block(wl, 0, seed, 1, 0, n_cold + n_hot)[:batch]
    if n_cold:
        cache.encode_append(torch.from_numpy(np.ascontiguousarray(k[:, :, :n_cold])).cuda(),
                            torch.from_numpy(np.ascontiguousarray(v[:, :, :n_cold])).cuda())
    if n_hot:
        cache.evict_window(torch.from_numpy(np.ascontiguousarray(k[:, :, n_cold:])).cuda(),
                           torch.from_numpy(np.ascontiguousarray(v[:, :, n_cold:])).cuda())
    return wl, cache, k, v


def _static(cache, q):
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device=q.device)
    tq.tq_decode_attention_static(cache.handle, q.data_ptr(), out.data_ptr(), 0.0,
                                  torch.cuda.current_stream().cuda_stream)
    return out


@pytest.mark.parametrize("name,batch,n_cold,n_hot", [
    ("llama8b", 2, 3000, 512),     # Llama-8B heads, ragged cold tail
    ("tinyllama", 1, 1024, 512),   # G = 8, d = 64
    ("llama8b", 8, 0, 512),        # batch 8 before the first eviction: hot tokens only
])
def test_static_scratch_matches_oracle_twice(name, batch, n_cold, n_hot):
    wl, cache, k, v = _filled_cache(name, batch, n_cold, n_hot)
    signs, S = oracle_signs_S(cache.cfg)
    for step in (1, 2):            # two calls in a row, different queries
        q_np = queries(wl, 0, 0, step=step)[:batch]
        q = torch.from_numpy(q_np).cuda()
        got = _static(cache, q)
        ref_ws = cache.decode_attention(q)
        assert cache.get_status() == 0
        got = got.cpu().numpy().astype(np.float64)
        err_ws = rel_err(got, ref_ws.cpu().numpy().astype(np.float64))
        assert np.all(err_ws <= ATTN_RTOL), (step, err_ws.max())
        for b in range(batch):
            ref = oracle_decode_row(cache, b, q_np[b], k[b, :, n_cold:].astype(np.float64),
                                    v[b, :, n_cold:].astype(np.float64), signs, S)
            e = rel_err(got[b], ref)
            assert np.all(e <= ATTN_RTOL), (step, b, e.max())
    cache.close()


def test_static_scratch_many_blocks_per_cta():
    """Batch 8 of Llama-8B heads with 8000 cold tokens: every attention CTA
    streams many cold blocks and several units' runs meet inside one CTA;
    sampled units against the oracle, on two calls in a row."""
    batch, n_cold, n_hot = 8, 8000, 512
    wl, cache, k, v = _filled_cache("llama8b", batch, n_cold, n_hot)
    assert cold_blocks_per_cta_lower_bound(batch * wl.num_kv_heads, n_cold) >= 4
    signs, S = oracle_signs_S(cache.cfg)
    G = wl.group
    for step in (3, 4):
        q_np = queries(wl, 0, 0, step=step)
        got = _static(cache, torch.from_numpy(q_np).cuda()).cpu().numpy().astype(np.float64)
        assert cache.get_status() == 0
        for u in (0, 1, 33, 63):
            b, h = divmod(u, wl.num_kv_heads)
            ref = oracle_decode_unit(cache, b, h, q_np[b], k[b, h, n_cold:], v[b, h, n_cold:],
                                     signs, S)
            e = rel_err(got[b, h * G:(h + 1) * G], ref)
            assert np.all(e <= ATTN_RTOL), (step, u, e.max())
    cache.close()


def test_static_scratch_empty_cache_gives_zeros():
    wl = WORKLOADS["llama8b"]
    cache = tq.TQCache(config_for(wl, batch=8, cold_capacity=64))
    q = torch.from_numpy(queries(wl, 0, 0)).cuda()
    for _ in range(2):
        out = _static(cache, q)
        assert cache.get_status() == 0
        assert torch.count_nonzero(out).item() == 0
    cache.close()


def test_static_scratch_rejects_configurations_that_do_not_fit():
    # 2048 (row, kv head) units of d = 128 need far more than the 4 MiB
    # static scratch even with hot tokens only: the call must refuse before
    # launching anything.
    cfg = tq.make_config(batch=256, num_q_heads=64, num_kv_heads=8, head_dim=128, hot_window=16,
                         cold_capacity=64, b_r=3, b_theta=3, qjl_bits=128, seed=0)
    cache = tq.TQCache(cfg)
    k = torch.zeros((256, 8, 16, 128), dtype=torch.float16, device="cuda")
    cache.evict_window(k, k)
    q = torch.zeros((256, 64, 128), dtype=torch.float16, device="cuda")
    with pytest.raises(tq.TQError) as e:
        _static(cache, q)
    assert e.value.code == 3        # TQ_ERR_CAPACITY
    assert cache.get_status() == 0
    cache.close()
