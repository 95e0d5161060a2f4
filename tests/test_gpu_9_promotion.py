"""GPU parity of attention-weighted promotion with sticky counters ("Monarch
v3 ...", section "Cómo funciona", item "Promoción Ponderada por Atención";
threshold 0.15, sticky count 3 as in the page's benchmark command).

A cache of Llama-8B-shaped heads (G = 4, d = 128, 3/3 bits, m = 128) is
driven step by step -- one new token into a full 16-token window, then a
decode with promotion -- next to the oracle's ``PromotingUnit`` replay, fed
the GPU's own cold records.  After every step: the sticky counts and the
pending promotions are equal, each unit's ring position is equal, the ring
holds the same fp16 values (a promoted token as its float64
dequantization), the records written by the evictions are bit-exact at the
positions the readings give, and every output head is within 2e-3.

The inputs plant two cold "magnet" tokens per unit along the unit's query
direction, so that they draw most of the attention and are promoted, and a
token along a second direction that the queries favour only on odd steps,
so that its count rises and resets."""
import math

import numpy as np
import pytest
import torch

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import Workload, gaussian_fp16
from oracle import tq_oracle as O
from tests.tq_testutil import (ATTN_RTOL, CodeReport, codes_from_export, compare_codes,
                               oracle_signs_S, rel_err)

pytestmark = pytest.mark.gpu

THR, STICKY = 0.15, 3


def _unit_dirs(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def test_promotion_replay_against_oracle():
    B, Hq, Hkv, d, W, NC, steps = 2, 8, 2, 128, 16, 200, 14
    G = Hq // Hkv
    wl = Workload("promo", 1, B, Hq, Hkv, d, W, NC, 3, 3, 128, "lognormal")
    cfg = tq.make_config(B, Hq, Hkv, d, W, NC + W + steps + 8, 3, 3, 128, seed=11)
    cache = tq.TQCache(cfg)
    rng = np.random.default_rng(5)
    units = B * Hkv
    u_dir = _unit_dirs(rng, units, d)          # each unit's query direction
    f_dir = _unit_dirs(rng, units, d)          # the flicker token's direction
    total = NC + W + steps
    k = gaussian_fp16((B, Hkv, total, d), 3, 0).astype(np.float64)
    v = gaussian_fp16((B, Hkv, total, d), 3, 1).astype(np.float64)
    magnets, flicker = (37, 150), 90
    for u in range(units):
        b, h = divmod(u, Hkv)
        for m in magnets:
            k[b, h, m] = 13.0 * u_dir[u]
        k[b, h, flicker] = 11.5 * f_dir[u]
    k, v = k.astype(np.float16), v.astype(np.float16)

    def queries(step):
        q = np.empty((B, Hq, d))
        for u in range(units):
            b, h = divmod(u, Hkv)
            for g in range(G):
                q[b, h * G + g] = (5.0 * u_dir[u] + (5.5 if step % 2 else 0.0) * f_dir[u]
                                   + 0.15 * rng.standard_normal(d))
        return q.astype(np.float16)

    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    cache.enable_promotion(THR, STICKY)
    cache.encode_append(up(k[:, :, :NC]), up(v[:, :, :NC]))
    cache.evict_window(up(k[:, :, NC:NC + W]), up(v[:, :, NC:NC + W]))
    signs, S = oracle_signs_S(cfg)
    ref = [O.PromotingUnit(W, d, THR, STICKY) for _ in range(units)]
    for u in range(units):
        b, h = divmod(u, Hkv)
        ref[u].append_cold(k[b, h, :NC], v[b, h, :NC])
        ref[u].insert(k[b, h, NC:NC + W], v[b, h, NC:NC + W], np.zeros((0, d)), np.zeros((0, d)))

    promoted_total, resets, rep = 0, 0, CodeReport()
    prev_counts = [dict() for _ in range(units)]
    for s in range(steps):
        p = NC + W + s
        # ---- insert: the oracle takes the promoted tokens' fp16 dequantization
        # from the GPU's records (read before the eviction overwrites them)
        deq = []
        for u in range(units):
            b, h = divmod(u, Hkv)
            pk, pv = [], []
            for i in ref[u].pending:
                exp = cache.export_cold(b, h, i, 1)
                pk.append(O.dequant_vectors(codes_from_export(exp, cfg, True), signs)[0])
                pv.append(O.dequant_vectors(codes_from_export(exp, cfg, False), signs)[0])
            deq.append((np.array(pk).reshape(-1, d), np.array(pv).reshape(-1, d)))
        cache.evict_window(up(k[:, :, p:p + 1]), up(v[:, :, p:p + 1]))
        written = []
        for u in range(units):
            b, h = divmod(u, Hkv)
            written.append(ref[u].insert(k[b, h, p:p + 1], v[b, h, p:p + 1], *deq[u]))
        st = cache.promotion_state()
        hk, hv = cache.hot_ring()
        hk, hv = hk.cpu().numpy(), hv.cpu().numpy()
        for u in range(units):
            b, h = divmod(u, Hkv)
            assert st[u]["ring_pos"] == ref[u].ring_pos, (s, u)
            np.testing.assert_array_equal(hk[b, h].view(np.uint16),
                                          ref[u].ring_k.astype(np.float16).view(np.uint16))
            np.testing.assert_array_equal(hv[b, h].view(np.uint16),
                                          ref[u].ring_v.astype(np.float16).view(np.uint16))
            for i in written[u]:
                exp = cache.export_cold(b, h, i, 1)
                rep.add(compare_codes(exp, O.encode(ref[u].cold_k[i][None], signs, S, 3, 3), cfg, True))
                rep.add(compare_codes(exp, O.encode(ref[u].cold_v[i][None], signs, None, 3, 3), cfg, False))
        # ---- decode with promotion
        q = queries(s)
        out = cache.decode_attention(up(q)).cpu().numpy().astype(np.float64)
        assert cache.get_status() == 0
        st = cache.promotion_state()
        nc = cache.counts()[0]
        for u in range(units):
            b, h = divmod(u, Hkv)
            exp = cache.export_cold(b, h, 0, nc)
            ck, cv = codes_from_export(exp, cfg, True), codes_from_export(exp, cfg, False)
            qu = q[b, h * G:(h + 1) * G].astype(np.float64)
            w = O.cold_softmax_weights(qu, ref[u].ring_k[None], [ck], signs, S, 1)
            mass = O.cold_attention_mass(w, 1)[0]
            near = np.abs(mass - THR) < 1e-2 * THR
            assert not near.any(), f"a mass sits at the threshold (step {s}, unit {u})"
            pend = ref[u].after_decode(mass)
            counts = {int(i): int(ref[u].counters[i]) for i in np.nonzero(ref[u].counters)[0]}
            assert st[u]["counts"] == counts, (s, u, st[u]["counts"], counts)
            assert st[u]["pending"] == [int(x) for x in pend], (s, u)
            promoted_total += len(pend)
            resets += sum(1 for i in prev_counts[u] if i not in counts and i not in pend)
            prev_counts[u] = counts
            refo = O.decode_attention(qu, ref[u].ring_k[None], ref[u].ring_v[None], [ck], [cv],
                                      signs, S, 1)
            e = rel_err(out[b, h * G:(h + 1) * G], refo)
            assert np.all(e <= ATTN_RTOL), (s, u, e.max())
    print(f"promotions {promoted_total}, counter resets {resets}; {rep}")
    assert promoted_total >= 2 * units and resets >= 1
    cache.close()


def test_promotion_argument_checks():
    cfg = tq.make_config(1, 4, 1, 64, 16, 64, 3, 3, 64, seed=0)
    cache = tq.TQCache(cfg)
    mem = torch.empty(tq.tq_promotion_bytes(cfg), dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    for thr, sticky in ((0.1, 3), (1.5, 3), (0.2, 0)):
        with pytest.raises(tq.TQError):
            tq.tq_promotion_enable(cache.handle, mem.data_ptr(), thr, sticky, s)
    tq.tq_promotion_enable(cache.handle, mem.data_ptr(), 0.2, 2, s)
    with pytest.raises(tq.TQError):                       # already on
        tq.tq_promotion_enable(cache.handle, mem.data_ptr(), 0.2, 2, s)
    q = torch.zeros((1, 4, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(tq.TQError):                       # gated decode is not combined with it
        cache.decode_attention_gated(q, 0.0)
    x = torch.zeros((1, 1, 16, 64), dtype=torch.float16, device="cuda")
    cache.evict_window(x, x)                              # fills the window
    y = torch.zeros((1, 1, 9, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(tq.TQError):                       # n > W - 8 once the window is full
        cache.evict_window(y, y)
    cache.close()
    # a small window cannot hold a step's promotions
    small = tq.TQCache(tq.make_config(1, 4, 1, 64, 8, 64, 3, 3, 64, seed=0))
    with pytest.raises(tq.TQError):
        small.enable_promotion(0.2, 2)
    small.close()
