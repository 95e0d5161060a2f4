"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds workload shapes and random-number recipes only -- none of
the compression or attention arithmetic -- so that the CPU oracle tests and
the CUDA path can be fed identical inputs without sharing method code.

Workloads (the pages' model shapes; no weights or datasets are used):

* ``tiny``         batch 1, 1 KV head / 4 query heads, head_dim 64,
                   64 hot + 192 cold tokens, b_r = b_theta = 4, m = 64.
                   K, V, Q ~ N(0, 1) with 2 outlier channels scaled x8 (the
                   same two channels in K, V and Q, picked by the seed).
* ``tinyllama``    TinyLlama-1.1B shape: 22 layers, 32 q / 4 kv heads,
                   head_dim 64, batch 1, 512 hot + 1024 cold, 4/4 bits,
                   m = 64.  K, V = N(0,1) * exp(0.5 n_c) with n_c ~ N(0,1)
                   per (layer, head, channel); Q ~ N(0, 1).
* ``llama8b``      Llama-3.1-8B shape: 32 layers, 32 q / 8 kv heads,
                   head_dim 128, batch 8, 32768 tokens = 512 hot + 32256
                   cold, b_r = b_theta = 3, m = 128.  K, V channel scales
                   lognormal(0, 0.5) and 1 % outlier channels (Bernoulli 0.01
                   per layer/head/channel) x10; Q ~ N(0, 1).
* ``longctx``      Llama-3.1-8B heads, batch 1, 131072 cold tokens appended
                   in 4096-token chunks, 512 hot, 64 decode steps with ring
                   eviction, b_r = 2, b_theta = 3, m = 128; values as llama8b.
* ``vsearch``      1,000,000 unit-norm float32 vectors of dimension 200 from
                   a 64-component Gaussian mixture (centres ~ N(0, I),
                   x = normalize(centre + N(0, I))), 1024 queries from the
                   same mixture; 4/4 bits, m = 200, top-10.

Every draw comes from NumPy's PCG64 keyed by a SeedSequence over
(seed, purpose, layer, batch row, head), so any one (layer, row, head) slice
can be regenerated alone.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    hot: int                 # hot window W (and initial hot tokens)
    cold: int                # tokens in the cold store before decoding
    b_r: int
    b_theta: int
    qjl_bits: int
    recipe: str              # "outlier8" | "lognormal" | "lognormal_outlier10"
    decode_steps: int = 1
    prefill_chunk: int = 0   # 0: one append of all cold tokens

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def tokens(self) -> int:
        """Tokens per (row, kv head) stream, decode-step tokens included."""
        return self.cold + self.hot + self.decode_steps


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 4, 1, 64, 64, 192, 4, 4, 64, "outlier8"),
    "tinyllama": Workload("tinyllama", 22, 1, 32, 4, 64, 512, 1024, 4, 4, 64, "lognormal"),
    "llama8b": Workload("llama8b", 32, 8, 32, 8, 128, 512, 32256, 3, 3, 128,
                        "lognormal_outlier10"),
    "longctx": Workload("longctx", 32, 1, 32, 8, 128, 512, 131072, 2, 3, 128,
                        "lognormal_outlier10", decode_steps=64, prefill_chunk=4096),
}

# purposes (first SeedSequence words after the seed)
_P_SCALE, _P_K, _P_V, _P_Q, _P_OUT, _P_VEC, _P_CENTRE, _P_QUERY = range(8)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def outlier_channels(wl: Workload, seed: int) -> np.ndarray:
    """For the outlier8 recipe: the two channels scaled x8 (same in K, V, Q)."""
    return _rng(seed, _P_OUT).choice(wl.head_dim, size=2, replace=False)


def channel_scales(wl: Workload, layer: int, seed: int, which: int) -> np.ndarray:
    """Per (kv head, channel) multiplicative scales, float64 [Hkv, d].

    which: 0 for K, 1 for V.
    """
    hk, d = wl.num_kv_heads, wl.head_dim
    if wl.recipe == "outlier8":
        sc = np.ones((hk, d))
        sc[:, outlier_channels(wl, seed)] = 8.0
        return sc
    g = _rng(seed, _P_SCALE, layer, which)
    if wl.recipe == "lognormal":
        return np.exp(0.5 * g.standard_normal((hk, d)))
    if wl.recipe == "lognormal_outlier10":
        sc = g.lognormal(0.0, 0.5, size=(hk, d))
        out = g.random((hk, d)) < 0.01
        return np.where(out, sc * 10.0, sc)
    raise ValueError(wl.recipe)


def kv_stream(wl: Workload, layer: int, seed: int, which: int, b: int, h: int,
              start: int = 0, count: Optional[int] = None) -> np.ndarray:
    """fp16 [count, d] tokens start..start+count of one (row, kv head) stream.

    The whole stream of ``wl.tokens`` tokens is drawn from one generator, so
    slices are consistent whatever the slicing.
    """
    if count is None:
        count = wl.tokens - start
    g = _rng(seed, _P_K if which == 0 else _P_V, layer, b, h)
    z = g.standard_normal((wl.tokens, wl.head_dim))[start:start + count]
    sc = channel_scales(wl, layer, seed, which)[h]
    return (z * sc).astype(np.float16)


def kv_block(wl: Workload, layer: int, seed: int, which: int, start: int,
             count: int) -> np.ndarray:
    """fp16 [B, Hkv, count, d]: the same slice for every (row, kv head)."""
    out = np.empty((wl.batch, wl.num_kv_heads, count, wl.head_dim), dtype=np.float16)
    for b in range(wl.batch):
        for h in range(wl.num_kv_heads):
            out[b, h] = kv_stream(wl, layer, seed, which, b, h, start, count)
    return out


def queries(wl: Workload, layer: int, seed: int, step: int = 0) -> np.ndarray:
    """fp16 [B, Hq, d] query of decode step ``step``."""
    g = _rng(seed, _P_Q, layer, step)
    q = g.standard_normal((wl.batch, wl.num_q_heads, wl.head_dim))
    if wl.recipe == "outlier8":
        q[..., outlier_channels(wl, seed)] *= 8.0
    return q.astype(np.float16)


def gaussian_fp16(shape, seed: int, *key: int, scale: float = 1.0) -> np.ndarray:
    """Plain N(0, scale^2) fp16 tensor (edge-case and small parity inputs)."""
    return (_rng(seed, 99, *key).standard_normal(shape) * scale).astype(np.float16)


# ---------------------------------------------------------------------------
# Vector search workload.
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class SearchWorkload:
    name: str
    n: int
    dim: int
    n_queries: int
    components: int
    b_r: int
    b_theta: int
    qjl_bits: int
    k: int


SEARCH_WORKLOADS = {
    "vsearch": SearchWorkload("vsearch", 1_000_000, 200, 1024, 64, 4, 4, 200, 10),
}


def mixture_centres(sw: SearchWorkload, seed: int) -> np.ndarray:
    return _rng(seed, _P_CENTRE).standard_normal((sw.components, sw.dim))


def mixture_vectors(sw: SearchWorkload, seed: int, start: int, count: int,
                    chunk: int = 65536) -> np.ndarray:
    """float32 [count, dim] unit-norm database vectors start..start+count.

    Vectors are drawn in fixed chunks of ``chunk`` rows (one generator per
    chunk) so that any range can be regenerated without the others.
    """
    centres = mixture_centres(sw, seed)
    out = np.empty((count, sw.dim), dtype=np.float32)
    pos = start
    while pos < start + count:
        c = pos // chunk
        lo = c * chunk
        hi = min(lo + chunk, sw.n)
        g = _rng(seed, _P_VEC, c)
        comp = g.integers(0, sw.components, size=hi - lo)
        x = centres[comp] + g.standard_normal((hi - lo, sw.dim))
        x /= np.linalg.norm(x, axis=1, keepdims=True)
        a = pos - lo
        b = min(hi, start + count) - lo
        out[pos - start: pos - start + (b - a)] = x[a:b]
        pos += b - a
    return out


def mixture_queries(sw: SearchWorkload, seed: int, count: Optional[int] = None) -> np.ndarray:
    count = sw.n_queries if count is None else count
    centres = mixture_centres(sw, seed)
    g = _rng(seed, _P_QUERY)
    comp = g.integers(0, sw.components, size=count)
    x = centres[comp] + g.standard_normal((count, sw.dim))
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    return x.astype(np.float32)
