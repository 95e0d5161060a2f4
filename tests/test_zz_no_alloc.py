"""tq_decode_attention_static: decode attention for callers that may not
allocate device memory while they run (an allocator-free serving loop, a
plugin whose host framework owns every allocation).  It keeps its per-call
scratch in a fixed array inside the library, so it must give the same
answer as tq_decode_attention, call after call, with nothing left over from
the previous call.

This file is collected last on purpose: a failure here cannot hide the
results of the other GPU tests.  It also passes when run alone.
"""
import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import WORKLOADS, kv_block, queries
from tests.tq_testutil import ATTN_RTOL, config_for, rel_err

pytestmark = pytest.mark.gpu


def _filled_cache(name, batch, n_cold, n_hot, seed=0):
    wl = WORKLOADS[name]
    cfg = config_for(wl, batch=batch, cold_capacity=n_cold, seed=seed)
    cache = tq.TQCache(cfg)
    k = kv_block(wl, 0, seed, 0, 0, n_cold + n_hot)[:batch]
    v = kv_block(wl, 0, seed, 1, 0, n_cold + n_hot)[:batch]
    cache.encode_append(torch.from_numpy(np.ascontiguousarray(k[:, :, :n_cold])).cuda(),
                        torch.from_numpy(np.ascontiguousarray(v[:, :, :n_cold])).cuda())
    cache.evict_window(torch.from_numpy(np.ascontiguousarray(k[:, :, n_cold:])).cuda(),
                       torch.from_numpy(np.ascontiguousarray(v[:, :, n_cold:])).cuda())
    return wl, cache


def _static(cache, q):
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    tq.tq_decode_attention_static(cache.handle, q.data_ptr(), out.data_ptr(), 0.0,
                                  torch.cuda.current_stream().cuda_stream)
    return out


@pytest.mark.parametrize("name,batch,n_cold,n_hot", [
    ("llama8b", 2, 3000, 512),     # Llama-8B heads, ragged cold tail
    ("tinyllama", 1, 1024, 512),   # G = 8, d = 64
])
def test_static_scratch_matches_workspace_entry_point_twice(name, batch, n_cold, n_hot):
    wl, cache = _filled_cache(name, batch, n_cold, n_hot)
    for step in (1, 2):            # two calls in a row, different queries
        q = torch.from_numpy(queries(wl, 0, 0, step=step)[:batch]).cuda()
        ref = cache.decode_attention(q)
        got = _static(cache, q)
        assert cache.get_status() == 0
        err = rel_err(got.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64))
        assert np.all(err <= ATTN_RTOL), (step, err.max())
    cache.close()


def test_static_scratch_rejects_configurations_that_do_not_fit():
    # 2048 (row, kv head) units of d = 128 need far more than the 4 MiB
    # static scratch: the call must refuse before launching anything.
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
