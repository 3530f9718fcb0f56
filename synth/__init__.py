"""Seeded synthetic inputs for the ExpertsInt8 MoE layer, shared by the oracle and the CUDA path.

Holds no arithmetic of the layer itself: only the counter-based normal generator
(SplitMix64 + Box-Muller, defined in ``synth.c``) and the workload shapes and
distributions.  Every tensor is a pure function of (seed, stream, attempt, index),
so the oracle and the GPU see bit-identical bf16 / fp32 inputs, and any slice
(one expert, one row) can be drawn on its own.

Workloads (Jamba-1.5 paper, "Model Architecture": n=16 experts, top K=2,
hidden 8192 for 1.5-Large; Jamba v0.1 summary page: 16 experts, two per token):
shapes, standard deviations and the router bias of the skewed case are the
synthetic stand-ins described in the design notes; no dataset or trained weight
is involved anywhere.
"""
import ctypes
import os
from dataclasses import dataclass, field
from typing import Dict, Optional

import numpy as np

from . import build as _build

STREAM_X = 1
STREAM_ROUTER = 2
STREAM_W1 = 3
STREAM_W3 = 4
STREAM_W2 = 5
STREAM_MLP_W1 = 6
STREAM_MLP_W3 = 7
STREAM_MLP_W2 = 8
_WEIGHT_STREAM = {"w1": STREAM_W1, "w3": STREAM_W3, "w2": STREAM_W2}
_MLP_WEIGHT_STREAM = {"w1": STREAM_MLP_W1, "w3": STREAM_MLP_W3, "w2": STREAM_MLP_W2}

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        u64 = ctypes.c_uint64
        lib.synth_stream_key.restype = u64
        lib.synth_stream_key.argtypes = [u64, u64, u64]
        lib.synth_raw.restype = u64
        lib.synth_raw.argtypes = [u64, u64]
        for name in ("synth_normal_bf16", "synth_normal_f32"):
            fn = getattr(lib, name)
            fn.restype = None
            fn.argtypes = [u64, u64, u64, u64, u64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int]
        _lib = lib
    return _lib


def stream_key(seed: int, stream: int, attempt: int = 0) -> int:
    return int(_load().synth_stream_key(seed, stream, attempt))


def raw(key: int, n: int) -> int:
    return int(_load().synth_raw(key, n))


def normal_bf16(seed: int, stream: int, attempt: int, start: int, count: int, std: float,
                out: Optional[np.ndarray] = None, threads: int = 0) -> np.ndarray:
    """bf16 bit patterns (uint16) of std * N(0,1) for stream indices [start, start+count)."""
    if out is None:
        out = np.empty(count, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == count
    if count:
        _load().synth_normal_bf16(seed, stream, attempt, start, count, float(std), out.ctypes.data, threads)
    return out


def normal_f32(seed: int, stream: int, attempt: int, start: int, count: int, std: float,
               out: Optional[np.ndarray] = None, threads: int = 0) -> np.ndarray:
    if out is None:
        out = np.empty(count, dtype=np.float32)
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size == count
    if count:
        _load().synth_normal_f32(seed, stream, attempt, start, count, float(std), out.ctypes.data, threads)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Reinterpret bf16 bit patterns as the fp32 values they denote (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); finite inputs only."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


@dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens
    d: int            # model (hidden) dimension
    F: int            # expert FFN dimension
    E: int = 16       # experts
    K: int = 2        # experts per token
    x_std: float = 1.0
    router_std: float = 0.02
    w_std: float = 0.02
    bias: Dict[int, float] = field(default_factory=dict)  # router logit bias per expert
    seed: int = 0
    note: str = ""
    layer: str = "moe"  # "moe": the routed expert layer; "mlp": the dense MLP (E = K = 1, no router)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", T=64, d=256, F=512, router_std=0.05, w_std=0.02,
                 note="tiny MoE layer, oracle-checkable in full"),
        Workload("v01_decode", T=32, d=4096, F=14336, router_std=0.02, w_std=0.02,
                 note="Jamba-v0.1-shaped decode step (int8 experts ~2.8 GB, HBM-bound)"),
        Workload("v01_prefill", T=8192, d=4096, F=14336, router_std=0.02, w_std=0.02,
                 note="Jamba-v0.1-shaped prefill (tensor-core bound)"),
        Workload("large_decode", T=64, d=8192, F=24576, router_std=0.015, w_std=0.015,
                 note="Jamba-1.5-Large-shaped decode step (int8 experts ~9.7 GB)"),
        Workload("large_prefill", T=16384, d=8192, F=24576, router_std=0.015, w_std=0.015,
                 note="Jamba-1.5-Large-shaped prefill chunk"),
        Workload("skewed", T=65536, d=4096, F=14336, router_std=0.02, w_std=0.02,
                 bias={3: 2.0, 11: 2.0}, note="skewed routing stress (+2.0 logit bias on experts 3 and 11)"),
    ]
}


# The dense MLP of the layers without MoE (Jamba-1.5 paper, "Model Architecture": one layer in e = 2 has an
# MoE block, the other an MLP; §3.1: ExpertsInt8 quantizes the MLP weights too), with the expert's shape.
MLP_WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("mlp_tiny", T=64, d=256, F=512, E=1, K=1, w_std=0.02, layer="mlp",
                 note="tiny dense MLP, oracle-checkable in full"),
        Workload("mlp_v01_decode", T=32, d=4096, F=14336, E=1, K=1, w_std=0.02, layer="mlp",
                 note="Jamba-v0.1-shaped dense MLP, decode step (int8 weights 176 MB, HBM-bound)"),
        Workload("mlp_v01_prefill", T=8192, d=4096, F=14336, E=1, K=1, w_std=0.02, layer="mlp",
                 note="Jamba-v0.1-shaped dense MLP, prefill (tensor-core bound)"),
    ]
}

ALL_WORKLOADS: Dict[str, Workload] = {**WORKLOADS, **MLP_WORKLOADS}


def _weight_stream(wl: Workload, which: str) -> int:
    return (_MLP_WEIGHT_STREAM if wl.layer == "mlp" else _WEIGHT_STREAM)[which]


def weight_shape(wl: Workload, which: str):
    """(rows, cols) of one expert's matrix, out x in as in nn.Linear: W1, W3 are [F][d], W2 is [d][F]."""
    return (wl.F, wl.d) if which in ("w1", "w3") else (wl.d, wl.F)


def gen_x(wl: Workload, seed: Optional[int] = None, attempts: Optional[np.ndarray] = None,
          rows: Optional[np.ndarray] = None) -> np.ndarray:
    """Activations x as bf16 bits [T][d].  Row t is drawn from stream (X, attempts[t]), indices
    [t*d, (t+1)*d); a row is redrawn with a larger attempt number by callers that need it."""
    seed = wl.seed if seed is None else seed
    rows = np.arange(wl.T) if rows is None else np.asarray(rows)
    att = np.zeros(wl.T, dtype=np.int64) if attempts is None else np.asarray(attempts)
    out = np.empty((len(rows), wl.d), dtype=np.uint16)
    if rows.size and np.all(att[rows] == 0) and np.all(np.diff(rows) == 1):
        normal_bf16(seed, STREAM_X, 0, int(rows[0]) * wl.d, len(rows) * wl.d, wl.x_std, out.reshape(-1))
        return out
    for i, t in enumerate(rows):
        normal_bf16(seed, STREAM_X, int(att[t]), int(t) * wl.d, wl.d, wl.x_std, out[i], threads=1)
    return out


def gen_router(wl: Workload, seed: Optional[int] = None) -> np.ndarray:
    """Router weight, fp32 [E][d]."""
    seed = wl.seed if seed is None else seed
    return normal_f32(seed, STREAM_ROUTER, 0, 0, wl.E * wl.d, wl.router_std).reshape(wl.E, wl.d)


def gen_bias(wl: Workload) -> Optional[np.ndarray]:
    """Router logit bias, fp32 [E], or None when the workload has none."""
    if not wl.bias:
        return None
    b = np.zeros(wl.E, dtype=np.float32)
    for e, v in wl.bias.items():
        b[e] = v
    return b


def gen_expert(wl: Workload, which: str, e: int, seed: Optional[int] = None,
               out: Optional[np.ndarray] = None, threads: int = 0) -> np.ndarray:
    """One expert's unquantized weight as bf16 bits [rows][cols]; index e*rows*cols + r*cols + c."""
    seed = wl.seed if seed is None else seed
    rows, cols = weight_shape(wl, which)
    n = rows * cols
    if out is None:
        out = np.empty((rows, cols), dtype=np.uint16)
    normal_bf16(seed, _weight_stream(wl, which), 0, e * n, n, wl.w_std, out.reshape(-1), threads)
    return out


def gen_experts(wl: Workload, which: str, seed: Optional[int] = None) -> np.ndarray:
    """All experts' unquantized weights, bf16 bits [E][rows][cols]."""
    rows, cols = weight_shape(wl, which)
    out = np.empty((wl.E, rows, cols), dtype=np.uint16)
    seed = wl.seed if seed is None else seed
    normal_bf16(seed, _weight_stream(wl, which), 0, 0, out.size, wl.w_std, out.reshape(-1))
    return out
