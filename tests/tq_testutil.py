"""Helpers for the GPU parity tests: build caches from the seeded workloads,
turn the library's exported records into oracle ``Codes`` and compare."""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from compressed_decode_attention_encode_b200 import tq
from compressed_decode_attention_encode_b200.inputs import Workload
from oracle import tq_oracle as O

ATTN_RTOL = 2e-3      # relative L2 per (row, query head), fp32 GPU vs fp64 oracle


def config_for(wl: Workload, batch=None, hot_window=None, cold_capacity=None, seed=0):
    return tq.make_config(batch=batch or wl.batch, num_q_heads=wl.num_q_heads,
                          num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim,
                          hot_window=hot_window or wl.hot,
                          cold_capacity=wl.cold if cold_capacity is None else cold_capacity,
                          b_r=wl.b_r, b_theta=wl.b_theta, qjl_bits=wl.qjl_bits, seed=seed)


def half_from_bits(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def half_bits(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def codes_from_export(exp: dict, cfg, key: bool) -> O.Codes:
    p = cfg.head_dim // 2
    pre = "k_" if key else "v_"
    cr, ct = O.unpack_codes(exp[pre + "codes"], p, cfg.b_r, cfg.b_theta)
    c = O.Codes(b_r=cfg.b_r, b_theta=cfg.b_theta, s16=half_from_bits(exp[pre + "s16"]),
                cr=cr, ct=ct)
    if key:
        c.rn16 = half_from_bits(exp["k_rn16"])
        c.bits = O.unpack_bits(exp["k_bits"], cfg.qjl_bits)
    return c


@dataclass
class CodeReport:
    vectors: int = 0
    tie_vectors: int = 0
    tie_fields: int = 0
    mismatched_ties: int = 0

    def add(self, other: "CodeReport"):
        for f in ("vectors", "tie_vectors", "tie_fields", "mismatched_ties"):
            setattr(self, f, getattr(self, f) + getattr(other, f))


def compare_codes(exp: dict, ref: O.Codes, cfg, key: bool) -> CodeReport:
    """Asserts bit-exact records except decisions the oracle flags as ties
    (within 1e-6 of a boundary); returns the tie counts."""
    rep = CodeReport(vectors=len(ref.s16))
    pre = "k_" if key else "v_"
    got = codes_from_export(exp, cfg, key)
    vt = ref.vec_tie
    rep.tie_vectors = int(vt.sum())
    # scale
    s_ok = (exp[pre + "s16"] == half_bits(ref.s16)) | ref.tie_s16
    assert s_ok.all(), f"s16 mismatch at {np.nonzero(~s_ok)[0][:10]}"
    # codes: a tie in the scale exempts the whole vector, a code tie itself
    cr_ok = (got.cr == ref.cr) | ref.tie_cr | ref.tie_s16[:, None]
    ct_ok = (got.ct == ref.ct) | ref.tie_ct | ref.tie_s16[:, None]
    assert cr_ok.all(), f"radius code mismatch at {np.argwhere(~cr_ok)[:10]}"
    assert ct_ok.all(), f"angle code mismatch at {np.argwhere(~ct_ok)[:10]}"
    clean = ~vt
    packed = O.pack_codes(ref.cr, ref.ct, cfg.b_theta, cfg.b_r)
    assert np.array_equal(exp[pre + "codes"][clean], packed[clean]), "packed code bytes differ"
    rep.tie_fields += int(ref.tie_cr.sum() + ref.tie_ct.sum() + ref.tie_s16.sum())
    rep.mismatched_ties += int((got.cr != ref.cr).sum() + (got.ct != ref.ct).sum())
    if key:
        rn_ok = (exp["k_rn16"] == half_bits(ref.rn16)) | ref.tie_rn16 | vt
        assert rn_ok.all(), f"rn16 mismatch at {np.nonzero(~rn_ok)[0][:10]}"
        b_ok = (got.bits == ref.bits) | ref.tie_bits | vt[:, None]
        assert b_ok.all(), f"sign bit mismatch at {np.argwhere(~b_ok)[:10]}"
        rep.tie_fields += int(ref.tie_rn16.sum() + ref.tie_bits.sum())
        rep.mismatched_ties += int((got.bits != ref.bits).sum())
    return rep


def oracle_signs_S(cfg):
    return O.rotation_signs(cfg.seed, cfg.head_dim), O.qjl_matrix(cfg.seed, cfg.qjl_bits, cfg.head_dim)


def oracle_decode_row(cache: tq.TQCache, row: int, q_row: np.ndarray, hot_k_row, hot_v_row,
                      signs, S, scale=None, n_cold=None):
    """fp64 oracle attention for one batch row, fed the GPU's cold records."""
    cfg = cache.cfg
    nc = cache.counts()[0] if n_cold is None else n_cold
    ck, cv = [], []
    for h in range(cfg.num_kv_heads):
        if nc:
            exp = cache.export_cold(row, h, 0, nc)
            ck.append(codes_from_export(exp, cfg, True))
            cv.append(codes_from_export(exp, cfg, False))
        else:
            ck.append(None)
            cv.append(None)
    return O.decode_attention(q_row.astype(np.float64), hot_k_row, hot_v_row, ck, cv, signs, S,
                              cfg.num_kv_heads, scale)


def rel_err(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    num = np.linalg.norm(got - ref, axis=-1)
    den = np.linalg.norm(ref, axis=-1)
    return num / np.maximum(den, 1e-30)


def oracle_decode_unit(cache: tq.TQCache, row: int, kv_head: int, q_row: np.ndarray,
                       hot_k_unit: np.ndarray, hot_v_unit: np.ndarray, signs, S, scale=None):
    """fp64 oracle attention for the query heads of one (row, kv head) unit,
    fed the GPU's cold records of that unit only; [G, d]."""
    cfg = cache.cfg
    G = cfg.num_q_heads // cfg.num_kv_heads
    nc = cache.counts()[0]
    ck = cv = None
    if nc:
        exp = cache.export_cold(row, kv_head, 0, nc)
        ck = [codes_from_export(exp, cfg, True)]
        cv = [codes_from_export(exp, cfg, False)]
    q = q_row[kv_head * G:(kv_head + 1) * G].astype(np.float64)
    return O.decode_attention(q, hot_k_unit[None].astype(np.float64),
                              hot_v_unit[None].astype(np.float64), ck, cv, signs, S, 1, scale)


def cold_blocks_per_cta_lower_bound(units: int, n_cold: int) -> int:
    """A lower bound on the cold blocks each attention CTA streams for this
    cache, whatever the occupancy (at most 8 CTAs per SM): the plan gives a
    CTA ceil(units * blocks / CTAs) blocks."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    blocks = units * ((n_cold + tq.TOKENS_PER_BLOCK - 1) // tq.TOKENS_PER_BLOCK)
    return blocks // (sms * 8)
