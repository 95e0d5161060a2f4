"""GPU decode-attention parity: tq_decode_attention (fp32 accumulation,
tensor-core products) against the fp64 oracle fed the GPU's own cold
records, per (row, query head): ||o_gpu - o_ref|| <= 2e-3 ||o_ref||."""
import math

import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import (WORKLOADS, Workload, gaussian_fp16,
                                                            kv_block, queries)
from oracle import tq_oracle as O
from tests.tq_testutil import ATTN_RTOL, config_for, oracle_decode_row, oracle_signs_S, rel_err

pytestmark = pytest.mark.gpu


def _run(wl: Workload, batch: int, n_cold: int, n_hot: int, W: int, seed=0, scale=0.0,
         layer=0, q=None, kv=None):
    cfg = config_for(wl, batch=batch, hot_window=W, cold_capacity=max(n_cold, 1), seed=seed)
    cache = tq.TQCache(cfg)
    total = n_cold + n_hot
    if kv is None:
        k = kv_block(wl, layer, seed, 0, 0, total)[:batch]
        v = kv_block(wl, layer, seed, 1, 0, total)[:batch]
    else:
        k, v = kv
    if n_cold:
        cache.encode_append(torch.from_numpy(np.ascontiguousarray(k[:, :, :n_cold])).cuda(),
                            torch.from_numpy(np.ascontiguousarray(v[:, :, :n_cold])).cuda())
    if n_hot:
        cache.evict_window(torch.from_numpy(np.ascontiguousarray(k[:, :, n_cold:])).cuda(),
                           torch.from_numpy(np.ascontiguousarray(v[:, :, n_cold:])).cuda())
    if q is None:
        q = queries(wl, layer, seed)[:batch]
    out = cache.decode_attention(torch.from_numpy(q).cuda(), softmax_scale=scale)
    assert cache.get_status() == 0
    got = out.cpu().numpy().astype(np.float64)
    signs, S = oracle_signs_S(cfg)
    errs = []
    for b in range(batch):
        ref = oracle_decode_row(cache, b, q[b], k[b, :, n_cold:].astype(np.float64),
                                v[b, :, n_cold:].astype(np.float64), signs, S,
                                None if scale == 0.0 else scale)
        e = rel_err(got[b], ref)
        errs.append(e)
        assert np.all(e <= ATTN_RTOL), (b, e.max(), np.argmax(e))
    cache.close()
    return np.concatenate(errs)


@pytest.mark.parametrize("name,batch,n_cold,n_hot", [
    ("tiny", 1, 192, 64),              # the tiny workload exactly
    ("tinyllama", 1, 1024, 512),       # TinyLlama-shaped layer (G = 8)
    ("llama8b", 2, 2000, 512),         # Llama-8B heads, ragged cold tail
    ("longctx", 1, 4096, 512),         # 2/3-bit codes
])
def test_decode_parity_workloads(name, batch, n_cold, n_hot):
    wl = WORKLOADS[name]
    e = _run(wl, batch, n_cold, n_hot, wl.hot)
    print(name, "max rel err", float(e.max()))


@pytest.mark.parametrize("n_cold,n_hot,W", [
    (0, 37, 64),        # hot only, ragged
    (1, 0, 64),         # a single cold token, no hot
    (65, 1, 64),        # one token past a block boundary
    (127, 63, 64),
    (640, 0, 64),       # cold only, several blocks
    (0, 0, 64),         # nothing cached: output is zero
])
def test_decode_edge_sizes(n_cold, n_hot, W):
    wl = WORKLOADS["llama8b"]
    if n_cold + n_hot == 0:
        cfg = config_for(wl, batch=1, hot_window=W, cold_capacity=1)
        cache = tq.TQCache(cfg)
        q = torch.from_numpy(queries(wl, 0, 0)[:1]).cuda()
        out = cache.decode_attention(q)
        assert cache.get_status() == 0
        assert torch.count_nonzero(out).item() == 0
        return
    _run(wl, 1, n_cold, n_hot, W)


@pytest.mark.parametrize("hq,hkv,d,m,br,bt", [
    (4, 4, 64, 64, 4, 4),      # G = 1
    (8, 1, 128, 64, 3, 3),     # G = 8, d = 128, m = 64
    (6, 2, 64, 128, 2, 2),     # G = 3, m = 128 on d = 64
    (16, 2, 128, 128, 1, 7),   # 1-bit radius, 7-bit angle
    (4, 1, 64, 64, 6, 2),
])
def test_decode_shapes_and_bit_widths(hq, hkv, d, m, br, bt):
    wl = Workload("grid", 1, 2, hq, hkv, d, 64, 300, br, bt, m, "lognormal")
    _run(wl, 2, 300, 40, 64, seed=7)


def test_decode_custom_scale_and_peaked_logits():
    wl = WORKLOADS["llama8b"]
    # large logits: scale x4 makes the softmax sharply peaked
    _run(wl, 1, 700, 100, 128, scale=4.0 / math.sqrt(128))


def test_decode_zero_value_vectors():
    wl = Workload("z", 1, 1, 4, 1, 64, 64, 200, 3, 3, 64, "lognormal")
    k = gaussian_fp16((1, 1, 260, 64), 1)
    v = gaussian_fp16((1, 1, 260, 64), 2)
    v[:, :, 10:150] = 0                      # scale 0 -> excluded from V, kept in softmax
    _run(wl, 1, 200, 60, 64, kv=(k, v))
