"""C-ABI checks that need no GPU: the library loads, exports every function
include/tq.h declares, generates the method randomness bit-for-bit like the
oracle's independent generator, sizes buffers as documented and rejects bad
arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

from compressed_decode_attention_encode_b200 import build as B
from compressed_decode_attention_encode_b200 import tq
from oracle import tq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return tq.lib()


def _declared_functions():
    txt = open(os.path.join(ROOT, "include", "tq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", txt)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(n for n, _, _ in tq.SIGNATURES) == names


def test_abi_version_and_status_strings(lib):
    assert tq.tq_abi_version() == 1
    for code, name in tq.STATUS_NAMES.items():
        assert tq.tq_status_string(code) == name


@pytest.mark.parametrize("seed,d", [(0, 64), (123456789, 128), (2**64 - 1, 256)])
def test_rotation_signs_bitwise_equal_oracle(lib, seed, d):
    np.testing.assert_array_equal(tq.tq_rotation_signs(seed, d).astype(np.float64),
                                  O.rotation_signs(seed, d))


@pytest.mark.parametrize("seed,m,d", [(0, 64, 64), (42, 128, 128), (7, 200, 256)])
def test_qjl_matrix_bitwise_equal_oracle(lib, seed, m, d):
    a = tq.tq_qjl_matrix(seed, m, d)
    b = O.qjl_matrix(seed, m, d)
    assert a.dtype == b.dtype == np.float32
    np.testing.assert_array_equal(a.view(np.uint32), b.view(np.uint32))


def _cfg(**kw):
    base = dict(batch=8, num_q_heads=32, num_kv_heads=8, head_dim=128, hot_window=512,
                cold_capacity=32256, b_r=3, b_theta=3, qjl_bits=128, seed=0)
    base.update(kw)
    return tq.make_config(**base)


def test_cache_bytes_match_documented_layout(lib):
    # K: d/2*bw/8 + m/8 + 4 bytes, V: d/2*bw/8 + 2 bytes per cold token and kv head
    for d, br, bt, m, per_tok in ((128, 3, 3, 128, 118), (128, 2, 3, 128, 102), (64, 4, 4, 64, 78)):
        cap = 32256
        hot, cold, ws = tq.tq_cache_bytes(_cfg(head_dim=d, b_r=br, b_theta=bt, qjl_bits=m,
                                               cold_capacity=cap))
        units = 8 * 8
        assert hot == 2 * units * 512 * d * 2
        blocks = -(-cap // tq.TOKENS_PER_BLOCK)
        assert cold == units * blocks * tq.TOKENS_PER_BLOCK * per_tok
        assert ws > 0 and ws % 256 == 0


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), 1),            # not a power of two
    (dict(head_dim=256), 2),           # power of two, not implemented
    (dict(b_r=5, b_theta=4), 1),       # bw > 8
    (dict(b_r=0), 1),
    (dict(qjl_bits=60), 1),            # not a multiple of 8
    (dict(qjl_bits=200), 2),
    (dict(num_q_heads=30), 1),         # not a multiple of Hkv
    (dict(num_q_heads=72), 2),         # G = 9 > 8
    (dict(batch=0), 1),
    (dict(hot_window=0), 1),
    (dict(cold_capacity=-1), 1),
])
def test_config_validation(lib, kw, code):
    with pytest.raises(tq.TQError) as e:
        tq.tq_cache_bytes(_cfg(**kw))
    assert e.value.code == code


def test_null_arguments_rejected_before_device(lib):
    cfg = _cfg()
    out = ctypes.c_void_p()
    assert lib.tq_cache_create(ctypes.byref(cfg), None, None, None, None, ctypes.byref(out)) == 1
    assert lib.tq_cache_create(ctypes.byref(cfg), 256, 512, 768, None, None) == 1
    # misaligned buffers
    assert lib.tq_cache_create(ctypes.byref(cfg), 257, 512, 768, None, ctypes.byref(out)) == 1
    assert lib.tq_encode_append(None, None, None, 1, None) == 1
    assert lib.tq_evict_window(None, None, None, 1, None) == 1
    assert lib.tq_decode_attention(None, None, None, 0.0, None) == 1
    assert lib.tq_get_status(None, None) == 1
    assert lib.tq_set_wait_limit(None, 0) == 1
    assert lib.tq_cache_destroy(None) == 0
    assert lib.tq_rotation_signs(0, 0, None) == 1


@pytest.mark.parametrize("d,m", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("b_r,b_t", [(1, 1), (2, 2), (3, 3), (2, 3), (4, 4), (1, 7), (5, 3)])
def test_cold_store_holds_exactly_the_algorithmic_bytes(lib, d, m, b_r, b_t):
    """The fragment-major tile layout adds no padding: a 64-token block is
    64 x (2 * d/2*bw/8 + m/8 + 6) bytes, except that d = 64 with an odd bit
    width rounds each lane's 16*bw-bit chunk up to whole words."""
    bw = b_r + b_t
    cfg = _cfg(batch=1, num_q_heads=4, num_kv_heads=1, head_dim=d, qjl_bits=m, b_r=b_r,
               b_theta=b_t, cold_capacity=64)
    _, cold, _ = tq.tq_cache_bytes(cfg)
    per_token = 2 * (d // 2 * bw // 8) + m // 8 + 6
    if d == 64 and bw % 2:
        words = -(-16 * bw // 32)
        per_token = 2 * (words * 4 * 32 // 16) + m // 8 + 6
    assert cold == 64 * per_token


@pytest.mark.parametrize("kw,code", [
    (dict(b_r=3, b_theta=3), 2),      # the search kernel reads one byte per pair
    (dict(dim=300), 2),
    (dict(qjl_bits=20), 1),
    (dict(qjl_bits=264), 2),
    (dict(dim=0), 1),
])
def test_vector_config_validation(lib, kw, code):
    base = dict(dim=200, b_r=4, b_theta=4, qjl_bits=200, seed=0)
    base.update(kw)
    cfg = tq.tq_vec_config(base["dim"], base["b_r"], base["b_theta"], base["qjl_bits"], base["seed"])
    with pytest.raises(tq.TQError) as e:
        tq.tq_vec_bytes(cfg, 1000, 16)
    assert e.value.code == code


def test_vector_codes_bytes():
    """codes [n][d/2] + signs [n][32] + s16 [n] + rn16 [n], each section
    rounded up to 256 bytes (d = 200 pads to 256)."""
    tq.lib()
    cfg = tq.tq_vec_config(200, 4, 4, 200, 0)
    n = 1_000_000
    cb, wb = tq.tq_vec_bytes(cfg, n, 1024)
    r = lambda x: -(-x // 256) * 256
    assert cb == r(n * 128) + r(n * 32) + 2 * r(n * 2)
    assert wb > 0


def test_tensor_cache_bytes():
    """The Tensor Cache tier's buffer: A as [B, Hkv, d, d] float32, then
    lambda, eta [Hkv] and sigmoid(g) [Hq], each part 256-byte aligned."""
    cfg = tq.make_config(8, 32, 8, 128, 512, 1000, 3, 3, 128)
    assert tq.tq_tc_bytes(cfg) == 8 * 8 * 128 * 128 * 4 + 256
    cfg = tq.make_config(1, 6, 2, 64, 64, 0, 2, 2, 64)
    assert tq.tq_tc_bytes(cfg) == 2 * 64 * 64 * 4 + 256
    with pytest.raises(tq.TQError):
        tq.tq_tc_bytes(tq.make_config(1, 6, 4, 64, 64, 0, 2, 2, 64))   # Hq not a multiple of Hkv
