"""Thin ctypes binding of ``libtq.so`` (the C ABI declared in include/tq.h).

The functions below carry the C names and only marshal arguments; every
step of the compressed-cache path runs in the library's CUDA kernels.
PyTorch is used for device memory and streams only (``TQCache``).  There is
no fallback: if the library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import (POINTER, Structure, c_char_p, c_float, c_int8, c_int32, c_int64,
                    c_size_t, c_uint8, c_uint16, c_uint64, c_void_p)

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtq.so")

TQ_OK = 0
STATUS_NAMES = {0: "TQ_OK", 1: "TQ_ERR_INVALID_ARG", 2: "TQ_ERR_UNSUPPORTED",
                3: "TQ_ERR_CAPACITY", 4: "TQ_ERR_RANGE", 5: "TQ_ERR_TIMEOUT",
                6: "TQ_ERR_CUDA"}
TOKENS_PER_BLOCK = 64


class TQError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")
        self.code = code


class tq_config(Structure):
    _fields_ = [("batch", c_int32), ("num_q_heads", c_int32), ("num_kv_heads", c_int32),
                ("head_dim", c_int32), ("hot_window", c_int32), ("cold_capacity", c_int64),
                ("b_r", c_int32), ("b_theta", c_int32), ("qjl_bits", c_int32),
                ("seed", c_uint64)]


class tq_vec_config(Structure):
    _fields_ = [("dim", c_int32), ("b_r", c_int32), ("b_theta", c_int32), ("qjl_bits", c_int32),
                ("seed", c_uint64)]


_lib = None

# (name, restype, argtypes) of every exported symbol
SIGNATURES = [
    ("tq_status_string", c_char_p, [c_int32]),
    ("tq_abi_version", c_int32, []),
    ("tq_cache_bytes", c_int32, [POINTER(tq_config), POINTER(c_size_t), POINTER(c_size_t),
                                 POINTER(c_size_t)]),
    ("tq_cache_create", c_int32, [POINTER(tq_config), c_void_p, c_void_p, c_void_p, c_void_p,
                                  POINTER(c_void_p)]),
    ("tq_cache_destroy", c_int32, [c_void_p]),
    ("tq_cache_counts", c_int32, [c_void_p, POINTER(c_int64), POINTER(c_int32), POINTER(c_int32)]),
    ("tq_encode_append", c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_void_p]),
    ("tq_encode_append_rows", c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_void_p]),
    ("tq_evict_window_rows", c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_void_p]),
    ("tq_cache_row_counts", c_int32, [c_void_p, c_int32, POINTER(c_int64), POINTER(c_int32),
                                      POINTER(c_int32)]),
    ("tq_evict_window", c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_void_p]),
    ("tq_decode_attention", c_int32, [c_void_p, c_void_p, c_void_p, c_float, c_void_p]),
    ("tq_decode_attention_static", c_int32, [c_void_p, c_void_p, c_void_p, c_float, c_void_p]),
    ("tq_decode_attention_gated", c_int32, [c_void_p, c_void_p, c_void_p, c_float, c_float, c_void_p,
                                            c_void_p]),
    ("tq_tc_bytes", c_int32, [POINTER(tq_config), POINTER(c_size_t)]),
    ("tq_tc_enable", c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    ("tq_get_status", c_int32, [c_void_p, c_void_p]),
    ("tq_set_attend_events", c_int32, [c_void_p, c_void_p, c_void_p]),
    ("tq_set_wait_limit", c_int32, [c_void_p, c_int64]),
    ("tq_promotion_bytes", c_int32, [POINTER(tq_config), POINTER(c_size_t)]),
    ("tq_promotion_enable", c_int32, [c_void_p, c_void_p, c_float, c_int32, c_void_p]),
    ("tq_promotion_state", c_int32, [c_void_p, c_void_p, c_void_p]),
    ("tq_export_cold", c_int32, [c_void_p, c_int32, c_int32, c_int64, c_int64, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    ("tq_vec_bytes", c_int32, [POINTER(tq_vec_config), c_int64, c_int32, POINTER(c_size_t),
                               POINTER(c_size_t)]),
    ("tq_vec_create", c_int32, [POINTER(tq_vec_config), c_int64, c_int32, c_void_p, c_void_p,
                                POINTER(c_void_p)]),
    ("tq_vec_destroy", c_int32, [c_void_p]),
    ("tq_encode_vectors", c_int32, [c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_void_p]),
    ("tq_ip_search", c_int32, [c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p,
                               c_void_p]),
    ("tq_vec_get_status", c_int32, [c_void_p, c_void_p]),
    ("tq_export_vectors", c_int32, [c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_void_p,
                                    c_void_p, c_void_p, c_void_p]),
    ("tq_rotation_signs", c_int32, [c_uint64, c_int32, POINTER(c_int8)]),
    ("tq_qjl_matrix", c_int32, [c_uint64, c_int32, c_int32, POINTER(c_float)]),
]


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m compressed_decode_attention_encode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code: int, what: str) -> None:
    if code != TQ_OK:
        raise TQError(code, what)


def make_config(batch, num_q_heads, num_kv_heads, head_dim, hot_window, cold_capacity,
                b_r, b_theta, qjl_bits, seed=0) -> tq_config:
    return tq_config(batch, num_q_heads, num_kv_heads, head_dim, hot_window, cold_capacity,
                     b_r, b_theta, qjl_bits, seed)


# ---- functions with the C names -------------------------------------------

def tq_status_string(code: int) -> str:
    return lib().tq_status_string(code).decode()


def tq_abi_version() -> int:
    return lib().tq_abi_version()


def tq_cache_bytes(cfg: tq_config):
    h, c, w = c_size_t(), c_size_t(), c_size_t()
    _check(lib().tq_cache_bytes(ctypes.byref(cfg), ctypes.byref(h), ctypes.byref(c),
                                ctypes.byref(w)), "tq_cache_bytes")
    return h.value, c.value, w.value


def tq_cache_create(cfg: tq_config, hot_ptr: int, cold_ptr: int, ws_ptr: int, stream: int) -> int:
    out = c_void_p()
    _check(lib().tq_cache_create(ctypes.byref(cfg), hot_ptr, cold_ptr, ws_ptr, stream,
                                 ctypes.byref(out)), "tq_cache_create")
    return out.value


def tq_cache_destroy(handle: int) -> None:
    _check(lib().tq_cache_destroy(handle), "tq_cache_destroy")


def tq_cache_counts(handle: int):
    nc, nh, rp = c_int64(), c_int32(), c_int32()
    _check(lib().tq_cache_counts(handle, ctypes.byref(nc), ctypes.byref(nh), ctypes.byref(rp)),
           "tq_cache_counts")
    return nc.value, nh.value, rp.value


def tq_encode_append(handle: int, k_ptr: int, v_ptr: int, n: int, stream: int) -> None:
    _check(lib().tq_encode_append(handle, k_ptr, v_ptr, n, stream), "tq_encode_append")


def tq_evict_window(handle: int, k_ptr: int, v_ptr: int, n: int, stream: int) -> None:
    _check(lib().tq_evict_window(handle, k_ptr, v_ptr, n, stream), "tq_evict_window")


def tq_decode_attention(handle: int, q_ptr: int, out_ptr: int, scale: float, stream: int) -> None:
    _check(lib().tq_decode_attention(handle, q_ptr, out_ptr, scale, stream), "tq_decode_attention")


def tq_decode_attention_static(handle: int, q_ptr: int, out_ptr: int, scale: float,
                               stream: int) -> None:
    _check(lib().tq_decode_attention_static(handle, q_ptr, out_ptr, scale, stream),
           "tq_decode_attention_static")


def tq_decode_attention_gated(handle: int, q_ptr: int, out_ptr: int, scale: float, threshold: float,
                              head_skip_ptr, stream: int) -> None:
    _check(lib().tq_decode_attention_gated(handle, q_ptr, out_ptr, scale, threshold, head_skip_ptr,
                                           stream), "tq_decode_attention_gated")


def tq_tc_bytes(cfg: tq_config) -> int:
    n = c_size_t()
    _check(lib().tq_tc_bytes(ctypes.byref(cfg), ctypes.byref(n)), "tq_tc_bytes")
    return n.value


def tq_tc_enable(handle: int, tc_ptr: int, lam, eta, gate, stream: int) -> None:
    def arr(x):
        a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
        return a, a.ctypes.data_as(c_void_p)
    la, lp = arr(lam)
    ea, ep = arr(eta)
    ga, gp = arr(gate)
    _check(lib().tq_tc_enable(handle, tc_ptr, lp, ep, gp, stream), "tq_tc_enable")


def tq_get_status(handle: int, stream: int) -> int:
    return lib().tq_get_status(handle, stream)


def tq_set_attend_events(handle: int, start: int, stop: int) -> None:
    _check(lib().tq_set_attend_events(handle, start, stop), "tq_set_attend_events")


def tq_promotion_bytes(cfg: tq_config) -> int:
    n = c_size_t()
    _check(lib().tq_promotion_bytes(ctypes.byref(cfg), ctypes.byref(n)), "tq_promotion_bytes")
    return n.value


def tq_promotion_enable(handle: int, mem_ptr: int, threshold: float, sticky: int, stream: int) -> None:
    _check(lib().tq_promotion_enable(handle, mem_ptr, threshold, sticky, stream), "tq_promotion_enable")


def tq_set_wait_limit(handle: int, limit_ns: int) -> None:
    _check(lib().tq_set_wait_limit(handle, limit_ns), "tq_set_wait_limit")


def tq_rotation_signs(seed: int, d: int) -> np.ndarray:
    out = np.empty(d, dtype=np.int8)
    _check(lib().tq_rotation_signs(seed, d, out.ctypes.data_as(POINTER(c_int8))),
           "tq_rotation_signs")
    return out


def tq_qjl_matrix(seed: int, m: int, d: int) -> np.ndarray:
    out = np.empty((m, d), dtype=np.float32)
    _check(lib().tq_qjl_matrix(seed, m, d, out.ctypes.data_as(POINTER(c_float))), "tq_qjl_matrix")
    return out


# ---- device-memory plumbing (PyTorch) --------------------------------------

def _stream_handle(stream=None) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t) -> int:
    return t.data_ptr()


class TQCache:
    """A per-layer compressed cache: PyTorch-allocated device buffers bound to
    a library handle.  Every method is a direct call into libtq.so."""

    def __init__(self, cfg: tq_config, device="cuda", stream=None):
        import torch
        self.cfg = cfg
        self.device = torch.device(device)
        hot, cold, ws = tq_cache_bytes(cfg)
        self.hot = torch.empty(max(hot, 256), dtype=torch.uint8, device=self.device)
        self.cold = torch.empty(max(cold, 256), dtype=torch.uint8, device=self.device)
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=self.device)
        self.bytes = dict(hot=hot, cold=cold, workspace=ws)
        self.handle = tq_cache_create(cfg, _ptr(self.hot), _ptr(self.cold), _ptr(self.ws),
                                      _stream_handle(stream))

    def close(self):
        if getattr(self, "handle", None):
            tq_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # shape checks are the library's; these only guard the Python objects
    @staticmethod
    def _dev16(t):
        import torch
        if t.dtype != torch.float16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("expected a contiguous CUDA float16 tensor")
        return _ptr(t)

    def encode_append(self, k, v, stream=None):
        n = k.shape[2]
        tq_encode_append(self.handle, self._dev16(k), self._dev16(v), n, _stream_handle(stream))

    def evict_window(self, k_new, v_new, stream=None):
        tq_evict_window(self.handle, self._dev16(k_new), self._dev16(v_new), k_new.shape[2],
                        _stream_handle(stream))

    def decode_attention(self, q, out=None, softmax_scale=0.0, stream=None):
        import torch
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        if out.dtype != torch.float32 or not out.is_contiguous():
            raise ValueError("out must be contiguous float32")
        tq_decode_attention(self.handle, self._dev16(q), _ptr(out), softmax_scale,
                            _stream_handle(stream))
        return out

    def decode_attention_gated(self, q, threshold, out=None, head_skip=None, softmax_scale=0.0,
                               stream=None):
        """Decode attention whose cold tier is read only by the query heads
        whose largest hot score q.k is below ``threshold``; ``head_skip``
        (int32 [B, Hq] on the device) receives 1 for the heads that skipped."""
        import torch
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        if out.dtype != torch.float32 or not out.is_contiguous():
            raise ValueError("out must be contiguous float32")
        hs = None
        if head_skip is not None:
            if head_skip.dtype != torch.int32 or not head_skip.is_cuda or not head_skip.is_contiguous():
                raise ValueError("head_skip must be a contiguous CUDA int32 tensor")
            hs = _ptr(head_skip)
        tq_decode_attention_gated(self.handle, self._dev16(q), _ptr(out), softmax_scale,
                                  float(threshold), hs, _stream_handle(stream))
        return out

    def enable_tensor_cache(self, lam, eta, gate, stream=None):
        """Switch evictions to the Tensor Cache tier: lam, eta per kv head,
        gate (g, before the sigmoid) per query head.  Returns the view of A
        [B, Hkv, d, d] (float32, on the device)."""
        import torch
        c = self.cfg
        if len(lam) != c.num_kv_heads or len(eta) != c.num_kv_heads or len(gate) != c.num_q_heads:
            raise ValueError("lam, eta: one per kv head; gate: one per query head")
        self.tc_mem = torch.empty(tq_tc_bytes(c), dtype=torch.uint8, device=self.device)
        tq_tc_enable(self.handle, _ptr(self.tc_mem), lam, eta, gate, _stream_handle(stream))
        n = c.batch * c.num_kv_heads * c.head_dim * c.head_dim
        return self.tc_mem[: 4 * n].view(torch.float32).view(c.batch, c.num_kv_heads, c.head_dim,
                                                             c.head_dim)

    def get_status(self, stream=None) -> int:
        return tq_get_status(self.handle, _stream_handle(stream))

    def set_attend_events(self, start=None, stop=None):
        """Record torch.cuda.Events around the attention kernel of the next
        decode calls (None, None stops recording)."""
        tq_set_attend_events(self.handle, start.cuda_event if start is not None else None,
                             stop.cuda_event if stop is not None else None)

    def enable_promotion(self, threshold=0.15, sticky=3, stream=None):
        """Attention-weighted promotion (sticky counters) on this handle;
        the library's buffer comes from PyTorch."""
        import torch
        self.promo_mem = torch.empty(tq_promotion_bytes(self.cfg), dtype=torch.uint8, device=self.device)
        tq_promotion_enable(self.handle, _ptr(self.promo_mem), float(threshold), int(sticky),
                            _stream_handle(stream))

    def promotion_state(self, stream=None):
        """Per (row, kv head): dict of counted positions -> counts, the
        promoted positions not yet moved, and the ring position."""
        units = self.cfg.batch * self.cfg.num_kv_heads
        out = np.zeros((units, 28), dtype=np.int32)
        _check(lib().tq_promotion_state(self.handle, out.ctypes.data, _stream_handle(stream)),
               "tq_promotion_state")
        res = []
        for u in range(units):
            o = out[u]
            res.append(dict(counts={int(o[4 + i]): int(o[12 + i]) for i in range(o[0])},
                            pending=[int(x) for x in o[20:20 + o[1]]], ring_pos=int(o[2])))
        return res

    def set_wait_limit(self, limit_ns: int):
        """Bounded-wait limit of the attention kernel (ns; 0 forces a
        timeout at the first wait, < 0 restores the default)."""
        tq_set_wait_limit(self.handle, limit_ns)

    def counts(self):
        return tq_cache_counts(self.handle)

    def row_counts(self, row: int):
        nc, nh, rp = c_int64(), c_int32(), c_int32()
        _check(lib().tq_cache_row_counts(self.handle, row, ctypes.byref(nc), ctypes.byref(nh),
                                         ctypes.byref(rp)), "tq_cache_row_counts")
        return nc.value, nh.value, rp.value

    def encode_append_rows(self, k, v, n_rows, stream=None):
        """Row b appends its first n_rows[b] tokens of k, v [B, Hkv, n_max, d]."""
        rows = np.ascontiguousarray(np.asarray(n_rows, dtype=np.int32))
        _check(lib().tq_encode_append_rows(self.handle, self._dev16(k), self._dev16(v), k.shape[2],
                                           rows.ctypes.data, _stream_handle(stream)),
               "tq_encode_append_rows")

    def evict_window_rows(self, k_new, v_new, n_rows, stream=None):
        """Row b inserts its first n_rows[b] tokens of k_new, v_new [B, Hkv, n_max, d]."""
        rows = np.ascontiguousarray(np.asarray(n_rows, dtype=np.int32))
        _check(lib().tq_evict_window_rows(self.handle, self._dev16(k_new), self._dev16(v_new),
                                          k_new.shape[2], rows.ctypes.data, _stream_handle(stream)),
               "tq_evict_window_rows")

    def hot_ring(self):
        """Views of the fp16 hot rings K, V: [B, Hkv, W, d] (slot order)."""
        import torch
        c = self.cfg
        n = c.batch * c.num_kv_heads * c.hot_window * c.head_dim
        h = self.hot[: 4 * n].view(torch.float16)
        shape = (c.batch, c.num_kv_heads, c.hot_window, c.head_dim)
        return h[:n].view(shape), h[n:].view(shape)

    def export_cold(self, row: int, kv_head: int, start: int, count: int, stream=None):
        """Canonical records of cold tokens start..start+count (host numpy)."""
        c = self.cfg
        kc = c.head_dim // 2 * (c.b_r + c.b_theta) // 8
        sg = c.qjl_bits // 8
        out = dict(k_codes=np.zeros((count, kc), np.uint8), k_bits=np.zeros((count, sg), np.uint8),
                   k_s16=np.zeros(count, np.uint16), k_rn16=np.zeros(count, np.uint16),
                   v_codes=np.zeros((count, kc), np.uint8), v_s16=np.zeros(count, np.uint16))
        p = {k: v.ctypes.data for k, v in out.items()}
        _check(lib().tq_export_cold(self.handle, row, kv_head, start, count, p["k_codes"],
                                    p["k_bits"], p["k_s16"], p["k_rn16"], p["v_codes"], p["v_s16"],
                                    _stream_handle(stream)), "tq_export_cold")
        return out


# ---- vector search ----------------------------------------------------------

def tq_vec_bytes(cfg: tq_vec_config, n: int, max_queries: int):
    c, w = c_size_t(), c_size_t()
    _check(lib().tq_vec_bytes(ctypes.byref(cfg), n, max_queries, ctypes.byref(c), ctypes.byref(w)),
           "tq_vec_bytes")
    return c.value, w.value


class TQVecIndex:
    """Compressed vector database + search handle (device memory from
    PyTorch; every method is a direct call into libtq.so)."""

    def __init__(self, dim, n, b_r=4, b_theta=4, qjl_bits=200, seed=0, max_queries=1024,
                 device="cuda", stream=None):
        import torch
        self.cfg = tq_vec_config(dim, b_r, b_theta, qjl_bits, seed)
        self.n = n
        cb, wb = tq_vec_bytes(self.cfg, n, max_queries)
        self.codes = torch.empty(max(cb, 256), dtype=torch.uint8, device=device)
        self.ws = torch.empty(max(wb, 256), dtype=torch.uint8, device=device)
        out = c_void_p()
        _check(lib().tq_vec_create(ctypes.byref(self.cfg), n, max_queries, self.ws.data_ptr(),
                                   _stream_handle(stream), ctypes.byref(out)), "tq_vec_create")
        self.handle = out.value

    def close(self):
        if getattr(self, "handle", None):
            _check(lib().tq_vec_destroy(self.handle), "tq_vec_destroy")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def encode(self, x, start=0, stream=None):
        """x: contiguous CUDA float32 [count, dim] -> database rows start.."""
        import torch
        if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
            raise ValueError("expected a contiguous CUDA float32 tensor")
        _check(lib().tq_encode_vectors(self.handle, x.data_ptr(), start, x.shape[0],
                                       self.codes.data_ptr(), _stream_handle(stream)),
               "tq_encode_vectors")

    def search(self, q, k=10, stream=None):
        """q: contiguous CUDA float32 [nq, dim] -> (scores [nq, k], idx [nq, k])."""
        import torch
        if q.dtype != torch.float32 or not q.is_cuda or not q.is_contiguous():
            raise ValueError("expected a contiguous CUDA float32 tensor")
        nq = q.shape[0]
        scores = torch.empty((nq, k), dtype=torch.float32, device=q.device)
        idx = torch.empty((nq, k), dtype=torch.int32, device=q.device)
        _check(lib().tq_ip_search(self.handle, self.codes.data_ptr(), q.data_ptr(), nq, k,
                                  scores.data_ptr(), idx.data_ptr(), _stream_handle(stream)),
               "tq_ip_search")
        return scores, idx

    def get_status(self, stream=None):
        """Latched device status of the searches (0 = TQ_OK); clears it."""
        return lib().tq_vec_get_status(self.handle, _stream_handle(stream))

    def export(self, start, count, stream=None):
        d = 64
        while d < self.cfg.dim:
            d *= 2
        kc = d // 2 * (self.cfg.b_r + self.cfg.b_theta) // 8
        mb = self.cfg.qjl_bits // 8
        out = dict(codes=np.zeros((count, kc), np.uint8), bits=np.zeros((count, mb), np.uint8),
                   s16=np.zeros(count, np.uint16), rn16=np.zeros(count, np.uint16))
        p = {k: v.ctypes.data for k, v in out.items()}
        _check(lib().tq_export_vectors(self.handle, self.codes.data_ptr(), start, count, p["codes"],
                                       p["bits"], p["s16"], p["rn16"], _stream_handle(stream)),
               "tq_export_vectors")
        return out
