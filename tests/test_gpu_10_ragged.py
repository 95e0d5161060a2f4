"""GPU parity of ragged batches (per-row lengths): rows that hold different
numbers of cold and hot tokens -- including rows with none -- are attended
row by row exactly as the fp64 oracle attends each row's own tokens (fed
the GPU's records, relative L2 per query head <= 2e-3), and per-row
insertions replay the oracle's ring per (row, kv head): hot slots fp16-equal,
evicted records bit-exact in age order."""
import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import gaussian_fp16
from oracle import tq_oracle as O
from tests.tq_testutil import (ATTN_RTOL, CodeReport, cold_blocks_per_cta_lower_bound, codes_from_export,
                               compare_codes, oracle_signs_S, rel_err)

pytestmark = pytest.mark.gpu


def _up(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _cfg(B, W, cap, Hq=32, Hkv=8, d=128, br=3, bt=3, m=128, seed=0):
    return tq.make_config(B, Hq, Hkv, d, W, cap, br, bt, m, seed=seed)


def _row_oracle(cache, cfg, b, q_row, hot_k, hot_v, signs, S, units=None):
    """Oracle output of row b ([Hq, d]) from its own cold records and the
    given hot tokens hot_k, hot_v [Hkv, n_hot, d]; `units` limits the kv
    heads (others are None)."""
    nc = cache.row_counts(b)[0]
    ck, cv = [], []
    for h in range(cfg.num_kv_heads):
        if nc and (units is None or h in units):
            exp = cache.export_cold(b, h, 0, nc)
            ck.append(codes_from_export(exp, cfg, True))
            cv.append(codes_from_export(exp, cfg, False))
        else:
            ck.append(None)
            cv.append(None)
    return O.decode_attention(q_row.astype(np.float64), hot_k.astype(np.float64),
                              hot_v.astype(np.float64), ck, cv, signs, S, cfg.num_kv_heads)


@pytest.mark.parametrize("static", [False, True])
def test_ragged_prefill_and_ring_fill(static):
    B, W = 5, 64
    n_cold = [3000, 0, 777, 1500, 0]
    n_hot = [64, 20, 0, 64, 0]
    cfg = _cfg(B, W, 3100)
    cache = tq.TQCache(cfg)
    k = gaussian_fp16((B, 8, 3000, 128), 21, 0)
    v = gaussian_fp16((B, 8, 3000, 128), 21, 1)
    kh = gaussian_fp16((B, 8, W, 128), 21, 2)
    vh = gaussian_fp16((B, 8, W, 128), 21, 3)
    cache.encode_append_rows(_up(k), _up(v), n_cold)
    cache.evict_window_rows(_up(kh), _up(vh), n_hot)
    for b in range(B):
        assert cache.row_counts(b) == (n_cold[b], n_hot[b], n_hot[b] % W)
    signs, S = oracle_signs_S(cfg)
    rep = CodeReport()
    for b, h in [(0, 0), (0, 7), (2, 3), (3, 5)]:     # each row's records, bit for bit
        exp = cache.export_cold(b, h, 0, n_cold[b])
        rep.add(compare_codes(exp, O.encode(k[b, h, :n_cold[b]].astype(np.float64), signs, S, 3, 3),
                              cfg, True))
        rep.add(compare_codes(exp, O.encode(v[b, h, :n_cold[b]].astype(np.float64), signs, None, 3, 3),
                              cfg, False))
    q = gaussian_fp16((B, 32, 128), 21, 4)
    qt = _up(q)
    if static:
        out = torch.full(qt.shape, float("nan"), dtype=torch.float32, device="cuda")
        tq.tq_decode_attention_static(cache.handle, qt.data_ptr(), out.data_ptr(), 0.0,
                                      torch.cuda.current_stream().cuda_stream)
    else:
        out = cache.decode_attention(qt)
    assert cache.get_status() == 0
    got = out.cpu().numpy().astype(np.float64)
    for b in range(B):
        if n_cold[b] + n_hot[b] == 0:
            assert np.all(got[b] == 0.0)
            continue
        ref = _row_oracle(cache, cfg, b, q[b], kh[b, :, :n_hot[b]], vh[b, :, :n_hot[b]], signs, S)
        e = rel_err(got[b], ref)
        assert np.all(e <= ATTN_RTOL), (b, e.max())
    cache.close()


def test_ragged_decode_steps_replay_the_rings():
    """Rows insert different numbers of tokens per step (0 to 3), so some
    rows evict and others are still filling; after each step the hot rings,
    the evicted records and the attention match the oracle row by row."""
    B, Hq, Hkv, d, W = 3, 8, 2, 64, 16
    cfg = _cfg(B, W, 400, Hq=Hq, Hkv=Hkv, d=d, br=4, bt=4, m=64, seed=3)
    cache = tq.TQCache(cfg)
    prefix = [40, 0, 13]
    steps = [[1, 3, 0], [2, 0, 1], [3, 3, 3], [0, 1, 2], [1, 1, 1], [3, 2, 0]] * 3
    total = 64 + 3 * len(steps)
    k = gaussian_fp16((B, Hkv, total, d), 31, 0)
    v = gaussian_fp16((B, Hkv, total, d), 31, 1)
    cache.encode_append_rows(_up(k[:, :, :64]), _up(v[:, :, :64]), prefix)
    rings = [[O.RingState(W=W, d=d) for _ in range(Hkv)] for _ in range(B)]
    vrings = [[O.RingState(W=W, d=d) for _ in range(Hkv)] for _ in range(B)]
    pos = list(prefix)
    signs, S = oracle_signs_S(cfg)
    rep = CodeReport()
    for si, n_rows in enumerate(steps):
        kn = np.zeros((B, Hkv, 3, d), np.float16)
        vn = np.zeros((B, Hkv, 3, d), np.float16)
        for b in range(B):
            kn[b, :, :n_rows[b]] = k[b, :, pos[b]:pos[b] + n_rows[b]]
            vn[b, :, :n_rows[b]] = v[b, :, pos[b]:pos[b] + n_rows[b]]
            for h in range(Hkv):
                rings[b][h].insert(kn[b, h, :n_rows[b]])
                vrings[b][h].insert(vn[b, h, :n_rows[b]])
            pos[b] += n_rows[b]
        cache.evict_window_rows(_up(kn), _up(vn), n_rows)
        hk, hv = cache.hot_ring()
        hk, hv = hk.cpu().numpy(), hv.cpu().numpy()
        q = gaussian_fp16((B, Hq, d), 31, 100 + si)
        out = cache.decode_attention(_up(q)).cpu().numpy().astype(np.float64)
        assert cache.get_status() == 0
        for b in range(B):
            r0 = rings[b][0]
            nc = prefix[b] + len(r0.cold_vectors)
            assert cache.row_counts(b) == (nc, r0.n_hot, r0.ring_pos), (si, b)
            for h in range(Hkv):
                nh = rings[b][h].n_hot
                np.testing.assert_array_equal(hk[b, h, :nh].view(np.uint16),
                                              rings[b][h].slots()[:nh].astype(np.float16).view(np.uint16))
                np.testing.assert_array_equal(hv[b, h, :nh].view(np.uint16),
                                              vrings[b][h].slots()[:nh].astype(np.float16).view(np.uint16))
                ev = len(rings[b][h].cold_vectors)
                if ev:
                    exp = cache.export_cold(b, h, prefix[b], ev)
                    xk = np.array(rings[b][h].cold_vectors)
                    xv = np.array(vrings[b][h].cold_vectors)
                    rep.add(compare_codes(exp, O.encode(xk, signs, S, 4, 4), cfg, True))
                    rep.add(compare_codes(exp, O.encode(xv, signs, None, 4, 4), cfg, False))
            hot_k = np.stack([rings[b][h].hot_tokens() for h in range(Hkv)])
            hot_v = np.stack([vrings[b][h].hot_tokens() for h in range(Hkv)])
            if nc + r0.n_hot == 0:
                assert np.all(out[b] == 0.0)
                continue
            ref = _row_oracle(cache, cfg, b, q[b], hot_k, hot_v, signs, S)
            e = rel_err(out[b], ref)
            assert np.all(e <= ATTN_RTOL), (si, b, e.max())
    print(rep)
    cache.close()


def test_ragged_batch_many_blocks_per_cta():
    """Batch 8 of Llama-8B heads with cold lengths from 0 to 8000 tokens: the
    flattened split gives every CTA several blocks and runs cross from one
    row's units into another's; sampled units against the oracle."""
    B, W = 8, 512
    n_cold = [8000, 6100, 0, 7777, 3000, 65, 8000, 4500]
    n_hot = [512, 512, 300, 512, 100, 512, 0, 512]
    cfg = _cfg(B, W, 8000)
    cache = tq.TQCache(cfg)
    k = gaussian_fp16((B, 8, 8000, 128), 41, 0)
    v = gaussian_fp16((B, 8, 8000, 128), 41, 1)
    kh = gaussian_fp16((B, 8, W, 128), 41, 2)
    vh = gaussian_fp16((B, 8, W, 128), 41, 3)
    cache.encode_append_rows(_up(k), _up(v), n_cold)
    cache.evict_window_rows(_up(kh), _up(vh), n_hot)
    assert cold_blocks_per_cta_lower_bound(8 * 8, 5000) >= 4
    q = gaussian_fp16((B, 32, 128), 41, 4)
    out = cache.decode_attention(_up(q)).cpu().numpy().astype(np.float64)
    assert cache.get_status() == 0
    signs, S = oracle_signs_S(cfg)
    G = 4
    for (b, h) in [(0, 0), (0, 7), (1, 3), (2, 5), (3, 0), (5, 2), (6, 6), (7, 7)]:
        ref = _row_oracle(cache, cfg, b, q[b], kh[b, :, :n_hot[b]], vh[b, :, :n_hot[b]], signs, S,
                          units={h})
        e = rel_err(out[b, h * G:(h + 1) * G], ref[h * G:(h + 1) * G])
        assert np.all(e <= ATTN_RTOL), (b, h, e.max())
    cache.close()


def test_ragged_argument_checks():
    cfg = _cfg(2, 16, 32, Hq=4, Hkv=1, d=64, m=64)
    cache = tq.TQCache(cfg)
    x = torch.zeros((2, 1, 40, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(tq.TQError) as e:            # row 0 over capacity
        cache.encode_append_rows(x, x, [33, 1])
    assert e.value.code == 3
    x4, x8 = x[:, :, :4].contiguous(), x[:, :, :8].contiguous()
    with pytest.raises(tq.TQError):                 # more than n_max
        cache.encode_append_rows(x4, x4, [5, 1])
    cache.encode_append_rows(x8, x8, [8, 3])
    assert cache.row_counts(0)[0] == 8 and cache.row_counts(1)[0] == 3
    q = torch.zeros((2, 4, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(tq.TQError):                 # gated decode needs a uniform batch
        cache.decode_attention_gated(q, 0.0)
    cache.close()
