"""Failure detection of the attention kernel's bounded waits, without a GPU
fault: a wait limit of 0 makes every wait for a cold tile's bulk copy give
up at once.  The call must latch TQ_ERR_TIMEOUT (read by tq_get_status),
write NaN rather than stale partials while the error is latched, drain the
copies it issued, and leave the context usable: the next call with the
default limit is oracle-correct."""
import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import WORKLOADS, kv_block, queries
from tests.tq_testutil import ATTN_RTOL, config_for, oracle_decode_row, oracle_signs_S, rel_err

pytestmark = pytest.mark.gpu
TQ_ERR_TIMEOUT = 5


def _cache(batch, n_cold, n_hot):
    wl = WORKLOADS["llama8b"]
    cache = tq.TQCache(config_for(wl, batch=batch, hot_window=max(n_hot, 1), cold_capacity=n_cold))
    k = kv_block(wl, 0, 0, 0, 0, n_cold + n_hot)[:batch]
    v = kv_block(wl, 0, 0, 1, 0, n_cold + n_hot)[:batch]
    cache.encode_append(torch.from_numpy(np.ascontiguousarray(k[:, :, :n_cold])).cuda(),
                        torch.from_numpy(np.ascontiguousarray(v[:, :, :n_cold])).cuda())
    if n_hot:
        cache.evict_window(torch.from_numpy(np.ascontiguousarray(k[:, :, n_cold:])).cuda(),
                           torch.from_numpy(np.ascontiguousarray(v[:, :, n_cold:])).cuda())
    return wl, cache, k, v


@pytest.mark.parametrize("batch,n_cold,n_hot", [(1, 2000, 64), (2, 9000, 512)])
def test_forced_timeout_is_reported_and_context_stays_usable(batch, n_cold, n_hot):
    wl, cache, k, v = _cache(batch, n_cold, n_hot)
    q_np = queries(wl, 0, 0)[:batch]
    q = torch.from_numpy(q_np).cuda()
    good = cache.decode_attention(q).clone()
    assert cache.get_status() == 0

    cache.set_wait_limit(0)
    out = cache.decode_attention(q)
    torch.cuda.synchronize()
    assert torch.isnan(out).all().item()          # no stale partials merged
    out2 = cache.decode_attention(q)              # still latched: NaN again
    assert torch.isnan(out2).all().item()
    assert cache.get_status() == TQ_ERR_TIMEOUT   # read and cleared
    assert cache.get_status() == 0

    cache.set_wait_limit(-1)                      # default limit again
    out = cache.decode_attention(q)
    assert cache.get_status() == 0
    np.testing.assert_array_equal(out.cpu().numpy(), good.cpu().numpy())
    signs, S = oracle_signs_S(cache.cfg)
    got = out.cpu().numpy().astype(np.float64)
    for b in range(batch):
        ref = oracle_decode_row(cache, b, q_np[b], k[b, :, n_cold:].astype(np.float64),
                                v[b, :, n_cold:].astype(np.float64), signs, S)
        assert np.all(rel_err(got[b], ref) <= ATTN_RTOL)
    cache.close()

