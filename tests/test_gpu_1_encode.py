"""GPU encode parity: tq_encode_append records are bit-exact against the
fp64 oracle (decisions within 1e-6 of a rounding boundary excepted, counted
and reported)."""
import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import WORKLOADS, Workload, kv_block
from oracle import tq_oracle as O
from tests.tq_testutil import CodeReport, compare_codes, config_for, oracle_signs_S

pytestmark = pytest.mark.gpu


def _encode_and_compare(wl: Workload, batch: int, n: int, seed: int, chunks=(None,), layer=0):
    cfg = config_for(wl, batch=batch, cold_capacity=n, seed=seed)
    cache = tq.TQCache(cfg)
    k = kv_block(wl, layer, seed, 0, 0, n)[:batch]
    v = kv_block(wl, layer, seed, 1, 0, n)[:batch]
    pos = 0
    sizes = [n] if chunks == (None,) else list(chunks)
    for c in sizes:
        kt = torch.from_numpy(np.ascontiguousarray(k[:, :, pos:pos + c])).cuda()
        vt = torch.from_numpy(np.ascontiguousarray(v[:, :, pos:pos + c])).cuda()
        cache.encode_append(kt, vt)
        pos += c
    assert pos == n
    assert cache.get_status() == 0
    assert cache.counts()[0] == n
    signs, S = oracle_signs_S(cfg)
    rep = CodeReport()
    for b in range(batch):
        for h in range(cfg.num_kv_heads):
            exp = cache.export_cold(b, h, 0, n)
            ck = O.encode(k[b, h].astype(np.float64), signs, S, cfg.b_r, cfg.b_theta)
            cv = O.encode(v[b, h].astype(np.float64), signs, None, cfg.b_r, cfg.b_theta)
            rep.add(compare_codes(exp, ck, cfg, True))
            rep.add(compare_codes(exp, cv, cfg, False))
    print(f"{wl.name}: {rep}")
    cache.close()
    return rep


@pytest.mark.parametrize("name,batch,n", [
    ("tiny", 1, 192),           # the tiny workload's whole cold store
    ("tinyllama", 1, 1024),     # TinyLlama-shaped layer, 4/4 bits, m = 64
    ("llama8b", 2, 300),        # Llama-8B heads, 3/3 bits, m = 128, ragged tail
    ("longctx", 1, 257),        # 2/3 bits (5-bit pairs), m = 128
])
def test_encode_bit_exact(name, batch, n):
    _encode_and_compare(WORKLOADS[name], batch, n, seed=0)


def test_encode_chunked_appends_equal_one_append():
    wl = WORKLOADS["llama8b"]
    # 4 appends of uneven sizes crossing 64-token block boundaries
    _encode_and_compare(wl, 1, 200, seed=3, chunks=(1, 63, 70, 66))


@pytest.mark.parametrize("name,batch,chunks", [
    ("llama8b", 2, (3, 8, 1, 5, 64, 2, 7, 30, 1, 1)),    # appends of <= 8 tokens take the
    ("tinyllama", 1, (1, 2, 3, 4, 5, 6, 7, 8, 60, 8)),   # per-token path, others the group path
])
def test_encode_small_appends_interleaved(name, batch, chunks):
    # neighbouring tokens of one 32-bit word arrive in different appends
    _encode_and_compare(WORKLOADS[name], batch, sum(chunks), seed=4, chunks=chunks)


def test_encode_small_append_zero_and_overflow():
    cfg = tq.make_config(1, 4, 1, 128, 64, 16, 3, 3, 128, seed=6)
    cache = tq.TQCache(cfg)
    z = torch.zeros((1, 1, 1, 128), dtype=torch.float16, device="cuda")
    cache.encode_append(z, z)                                  # zero vector, alone
    big = torch.full((1, 1, 1, 128), 60000.0, dtype=torch.float16, device="cuda")
    cache.encode_append(big, z)                                # overflowing key, alone
    assert cache.get_status() == 4
    exp = cache.export_cold(0, 0, 0, 2)
    assert exp["k_s16"][0] == 0 and exp["v_s16"][0] == 0 and exp["k_s16"][1] == 0
    assert (exp["k_bits"][0] == 0xFF).all()
    cache.close()


@pytest.mark.parametrize("b_r,b_t,m,d", [(1, 1, 64, 64), (1, 7, 128, 128), (7, 1, 64, 128),
                                         (5, 3, 128, 64), (2, 2, 64, 64)])
def test_encode_bit_widths(b_r, b_t, m, d):
    wl = Workload("grid", 1, 1, 2, 1, d, 64, 130, b_r, b_t, m, "lognormal")
    _encode_and_compare(wl, 1, 130, seed=11)


def test_encode_zero_and_tiny_vectors():
    cfg = tq.make_config(1, 4, 1, 64, 64, 64, 3, 3, 64, seed=5)
    cache = tq.TQCache(cfg)
    k = np.zeros((1, 1, 64, 64), np.float16)
    k[0, 0, 1, 0] = np.float16(6e-8)          # smallest subnormal: scale underflows to 0
    k[0, 0, 2] = np.float16(1.0)
    v = k.copy()
    cache.encode_append(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    assert cache.get_status() == 0
    exp = cache.export_cold(0, 0, 0, 64)
    signs, S = oracle_signs_S(cfg)
    compare_codes(exp, O.encode(k[0, 0].astype(np.float64), signs, S, 3, 3), cfg, True)
    compare_codes(exp, O.encode(v[0, 0].astype(np.float64), signs, None, 3, 3), cfg, False)
    assert exp["k_s16"][0] == 0 and (exp["k_bits"][0] == 0xFF).all()
    cache.close()


def test_encode_range_error_is_latched_not_fatal():
    cfg = tq.make_config(1, 1, 1, 64, 64, 64, 3, 3, 64, seed=5)
    cache = tq.TQCache(cfg)
    k = np.full((1, 1, 1, 64), 60000.0, np.float16)   # rotated max radius > fp16 max
    cache.encode_append(torch.from_numpy(k).cuda(), torch.from_numpy(k).cuda())
    assert cache.get_status() == 4          # TQ_ERR_RANGE, then cleared
    assert cache.get_status() == 0
    cache.close()


def test_capacity_error_launches_nothing():
    cfg = tq.make_config(1, 1, 1, 64, 64, 100, 3, 3, 64, seed=5)
    cache = tq.TQCache(cfg)
    k = torch.zeros((1, 1, 101, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(tq.TQError) as e:
        cache.encode_append(k, k)
    assert e.value.code == 3
    assert cache.counts()[0] == 0
    cache.close()
