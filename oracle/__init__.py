"""ORACLE — test infrastructure only.

ctypes wrapper around ``oracle.c``, the plain fp64 CPU implementation of the
ExpertsInt8 mixture-of-experts layer (Jamba-1.5 paper, §3.1 "ExpertsInt8" and
"Model Architecture"), of the same layer with unquantized bf16 weights and with FP8 (E4M3)
weights and activations, and of the dense ExpertsInt8 MLP of the layers without MoE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA path (``int8_expert_weight_b200``), and the two never import
each other; the only common dependency is the input generator ``synth``.

``Oracle(path)`` binds one compiled copy of ``oracle.c``; the module-level
functions use the default build.  Tests bind deliberately broken copies too,
to show that the pins catch plausible mistakes.
"""
import ctypes
from typing import Optional, Tuple

import numpy as np

from . import build as _build


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


class Oracle:
    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        vp, i64, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.oracle_quantize_rows.restype = c_int
        lib.oracle_quantize_rows.argtypes = [vp, i64, i64, vp, vp, c_int]
        lib.oracle_route.restype = c_int
        lib.oracle_route.argtypes = [vp, i64, i64, vp, vp, c_int, c_int, vp, vp, vp, c_int]
        lib.oracle_moe_forward.restype = c_int
        lib.oracle_moe_forward.argtypes = [vp, i64, i64, i64, c_int, c_int, vp, vp, vp, vp, vp, vp, vp, vp,
                                           vp, i64, vp, vp, vp, vp, c_int]
        lib.oracle_moe_forward_bf16w.restype = c_int
        lib.oracle_moe_forward_bf16w.argtypes = [vp, i64, i64, i64, c_int, c_int, vp, vp, vp, vp, vp, vp, i64, vp,
                                                 vp, vp, vp, c_int]
        lib.oracle_quantize_rows_fp8.restype = c_int
        lib.oracle_quantize_rows_fp8.argtypes = [vp, i64, i64, vp, vp, c_int]
        lib.oracle_e4m3_round.restype = c_int
        lib.oracle_e4m3_round.argtypes = [vp, i64, vp, vp]
        lib.oracle_moe_forward_fp8.restype = c_int
        lib.oracle_moe_forward_fp8.argtypes = lib.oracle_moe_forward.argtypes
        lib.oracle_mlp_forward.restype = c_int
        lib.oracle_mlp_forward.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, i64, vp, vp, c_int]
        lib.oracle_default_threads.restype = c_int
        lib.oracle_default_threads.argtypes = []
        self.lib = lib
        self.path = path

    def default_threads(self) -> int:
        return int(self.lib.oracle_default_threads())

    def quantize(self, w_bits: np.ndarray, threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
        """ExpertsInt8 quantization of bf16 weights (uint16 bit patterns), one scale per row of the
        last dim.  Returns (q int8, same shape; s fp32, shape[:-1])."""
        w = _c(w_bits, np.uint16)
        cols = w.shape[-1]
        rows = w.size // cols
        q = np.empty(w.shape, dtype=np.int8)
        s = np.empty(w.shape[:-1], dtype=np.float32)
        rc = self.lib.oracle_quantize_rows(w.ctypes.data, rows, cols, q.ctypes.data, s.ctypes.data, threads)
        if rc != 0:
            raise ValueError("oracle_quantize_rows rejected its arguments")
        return q, s

    def quantize_fp8(self, w_bits: np.ndarray, threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
        """FP8 (E4M3) quantization of bf16 weights (uint16 bit patterns), one scale per row of the last
        dim.  Returns (codes uint8, same shape; s fp32, shape[:-1])."""
        w = _c(w_bits, np.uint16)
        cols = w.shape[-1]
        rows = w.size // cols
        q = np.empty(w.shape, dtype=np.uint8)
        s = np.empty(w.shape[:-1], dtype=np.float32)
        rc = self.lib.oracle_quantize_rows_fp8(w.ctypes.data, rows, cols, q.ctypes.data, s.ctypes.data, threads)
        if rc != 0:
            raise ValueError("oracle_quantize_rows_fp8 rejected its arguments")
        return q, s

    def e4m3_round(self, v) -> Tuple[np.ndarray, np.ndarray]:
        """(E4M3 codes, their values) of the nearest E4M3 numbers to v (fp64), ties to even."""
        v = np.ascontiguousarray(v, dtype=np.float64)
        codes = np.empty(v.shape, dtype=np.uint8)
        vals = np.empty(v.shape, dtype=np.float64)
        rc = self.lib.oracle_e4m3_round(v.ctypes.data, v.size, codes.ctypes.data, vals.ctypes.data)
        if rc != 0:
            raise ValueError("oracle_e4m3_round rejected its arguments")
        return codes, vals

    def route(self, x_bits: np.ndarray, router_w: np.ndarray, bias: Optional[np.ndarray] = None,
              top_k: int = 2, threads: int = 0, want_logits: bool = False):
        """Router: (ids int32 [T][K], weights fp64 [T][K]) and, if asked, logits fp64 [T][E]."""
        x = _c(x_bits, np.uint16)
        wr = _c(router_w, np.float32)
        b = _c(bias, np.float32)
        T, d = x.shape
        E = wr.shape[0]
        ids = np.empty((T, top_k), dtype=np.int32)
        wts = np.empty((T, top_k), dtype=np.float64)
        logits = np.empty((T, E), dtype=np.float64) if want_logits else None
        rc = self.lib.oracle_route(x.ctypes.data, T, d, wr.ctypes.data, _ptr(b), E, top_k, ids.ctypes.data,
                                   wts.ctypes.data, _ptr(logits), threads)
        if rc != 0:
            raise ValueError("oracle_route rejected its arguments")
        return (ids, wts, logits) if want_logits else (ids, wts)

    def moe_forward(self, x_bits, router_w, bias, q1, s1, q3, s3, q2, s2, tokens=None, top_k: int = 2,
                    threads: int = 0, want_hidden: bool = False):
        """The layer in fp64 on the listed tokens (all if None).

        x [T][d] bf16 bits; router_w [E][d] fp32; bias [E] fp32 or None; q1, q3 [E][F][d] int8 with
        s1, s3 [E][F] fp32; q2 [E][d][F] int8 with s2 [E][d] fp32.  Returns a dict with y fp64 [n][d],
        ids int32 [n][K], w fp64 [n][K] and, if asked, h fp64 [n][K][F] (SwiGLU hidden of each slot).
        """
        x = _c(x_bits, np.uint16)
        wr = _c(router_w, np.float32)
        b = _c(bias, np.float32)
        q1, q3, q2 = (_c(a, np.int8) for a in (q1, q3, q2))
        s1, s3, s2 = (_c(a, np.float32) for a in (s1, s3, s2))
        T, d = x.shape
        E, F = q1.shape[0], q1.shape[1]
        assert q1.shape == (E, F, d) and q3.shape == (E, F, d) and q2.shape == (E, d, F)
        assert s1.shape == (E, F) and s3.shape == (E, F) and s2.shape == (E, d) and wr.shape == (E, d)
        tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
        n = T if tok is None else tok.size
        y = np.empty((n, d), dtype=np.float64)
        ids = np.empty((n, top_k), dtype=np.int32)
        wts = np.empty((n, top_k), dtype=np.float64)
        h = np.empty((n, top_k, F), dtype=np.float64) if want_hidden else None
        rc = self.lib.oracle_moe_forward(x.ctypes.data, T, d, F, E, top_k, wr.ctypes.data, _ptr(b),
                                         q1.ctypes.data, s1.ctypes.data, q3.ctypes.data, s3.ctypes.data,
                                         q2.ctypes.data, s2.ctypes.data, _ptr(tok), n, y.ctypes.data,
                                         ids.ctypes.data, wts.ctypes.data, _ptr(h), threads)
        if rc != 0:
            raise ValueError("oracle_moe_forward rejected its arguments")
        out = {"y": y, "ids": ids, "w": wts}
        if want_hidden:
            out["h"] = h
        return out

    def moe_forward_fp8(self, x_bits, router_W, bias, q1, s1, q3, s3, q2, s2, tokens=None, top_k: int = 2,
                        threads: int = 0, want_hidden: bool = False):
        """The FP8 layer in fp64: as moe_forward with E4M3 codes (uint8) q1, q3, q2 and their scales;
        x and the SwiGLU intermediate are quantized per row inside.  h (if asked) is the intermediate
        before its quantization."""
        x = _c(x_bits, np.uint16)
        wr = _c(router_W, np.float32)
        b = _c(bias, np.float32)
        q1, q3, q2 = (_c(a, np.uint8) for a in (q1, q3, q2))
        s1, s3, s2 = (_c(a, np.float32) for a in (s1, s3, s2))
        T, d = x.shape
        E, F = q1.shape[0], q1.shape[1]
        assert q1.shape == (E, F, d) and q3.shape == (E, F, d) and q2.shape == (E, d, F)
        assert s1.shape == (E, F) and s3.shape == (E, F) and s2.shape == (E, d) and wr.shape == (E, d)
        tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
        n = T if tok is None else tok.size
        y = np.empty((n, d), dtype=np.float64)
        ids = np.empty((n, top_k), dtype=np.int32)
        wts = np.empty((n, top_k), dtype=np.float64)
        h = np.empty((n, top_k, F), dtype=np.float64) if want_hidden else None
        rc = self.lib.oracle_moe_forward_fp8(x.ctypes.data, T, d, F, E, top_k, wr.ctypes.data, _ptr(b),
                                             q1.ctypes.data, s1.ctypes.data, q3.ctypes.data, s3.ctypes.data,
                                             q2.ctypes.data, s2.ctypes.data, _ptr(tok), n, y.ctypes.data,
                                             ids.ctypes.data, wts.ctypes.data, _ptr(h), threads)
        if rc != 0:
            raise ValueError("oracle_moe_forward_fp8 rejected its arguments")
        out = {"y": y, "ids": ids, "w": wts}
        if want_hidden:
            out["h"] = h
        return out

    def moe_forward_bf16w(self, x_bits, router_w, bias, w1, w3, w2, tokens=None, top_k: int = 2,
                          threads: int = 0, want_hidden: bool = False):
        """The layer in fp64 with unquantized bf16 weights (uint16 bit patterns): w1, w3 [E][F][d],
        w2 [E][d][F]; other arguments and the result as in moe_forward."""
        x = _c(x_bits, np.uint16)
        wr = _c(router_w, np.float32)
        b = _c(bias, np.float32)
        w1, w3, w2 = (_c(a, np.uint16) for a in (w1, w3, w2))
        T, d = x.shape
        E, F = w1.shape[0], w1.shape[1]
        assert w1.shape == (E, F, d) and w3.shape == (E, F, d) and w2.shape == (E, d, F) and wr.shape == (E, d)
        tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
        n = T if tok is None else tok.size
        y = np.empty((n, d), dtype=np.float64)
        ids = np.empty((n, top_k), dtype=np.int32)
        wts = np.empty((n, top_k), dtype=np.float64)
        h = np.empty((n, top_k, F), dtype=np.float64) if want_hidden else None
        rc = self.lib.oracle_moe_forward_bf16w(x.ctypes.data, T, d, F, E, top_k, wr.ctypes.data, _ptr(b),
                                               w1.ctypes.data, w3.ctypes.data, w2.ctypes.data, _ptr(tok), n,
                                               y.ctypes.data, ids.ctypes.data, wts.ctypes.data, _ptr(h), threads)
        if rc != 0:
            raise ValueError("oracle_moe_forward_bf16w rejected its arguments")
        out = {"y": y, "ids": ids, "w": wts}
        if want_hidden:
            out["h"] = h
        return out

    def mlp_forward(self, x_bits, q1, s1, q3, s3, q2, s2, tokens=None, threads: int = 0,
                    want_hidden: bool = False):
        """The dense ExpertsInt8 MLP in fp64 on the listed tokens (all if None).

        x [T][d] bf16 bits; q1, q3 [F][d] int8 with s1, s3 [F] fp32; q2 [d][F] int8 with s2 [d] fp32.
        Returns a dict with y fp64 [n][d] and, if asked, h fp64 [n][F].
        """
        x = _c(x_bits, np.uint16)
        q1, q3, q2 = (_c(a, np.int8) for a in (q1, q3, q2))
        s1, s3, s2 = (_c(a, np.float32) for a in (s1, s3, s2))
        T, d = x.shape
        F = q1.shape[0]
        assert q1.shape == (F, d) and q3.shape == (F, d) and q2.shape == (d, F)
        assert s1.shape == (F,) and s3.shape == (F,) and s2.shape == (d,)
        tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
        n = T if tok is None else tok.size
        y = np.empty((n, d), dtype=np.float64)
        h = np.empty((n, F), dtype=np.float64) if want_hidden else None
        rc = self.lib.oracle_mlp_forward(x.ctypes.data, T, d, F, q1.ctypes.data, s1.ctypes.data, q3.ctypes.data,
                                         s3.ctypes.data, q2.ctypes.data, s2.ctypes.data, _ptr(tok), n,
                                         y.ctypes.data, _ptr(h), threads)
        if rc != 0:
            raise ValueError("oracle_mlp_forward rejected its arguments")
        out = {"y": y}
        if want_hidden:
            out["h"] = h
        return out


_default: Optional[Oracle] = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def default_threads() -> int:
    return get().default_threads()


def quantize(w_bits, threads: int = 0):
    return get().quantize(w_bits, threads)


def route(x_bits, router_w, bias=None, top_k: int = 2, threads: int = 0, want_logits: bool = False):
    return get().route(x_bits, router_w, bias, top_k, threads, want_logits)


def moe_forward(*args, **kwargs):
    return get().moe_forward(*args, **kwargs)


def moe_forward_bf16w(*args, **kwargs):
    return get().moe_forward_bf16w(*args, **kwargs)


def mlp_forward(*args, **kwargs):
    return get().mlp_forward(*args, **kwargs)


def quantize_fp8(w_bits, threads: int = 0):
    return get().quantize_fp8(w_bits, threads)


def e4m3_round(v):
    return get().e4m3_round(v)


def moe_forward_fp8(*args, **kwargs):
    return get().moe_forward_fp8(*args, **kwargs)
