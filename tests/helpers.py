"""Test helpers: seeded layer inputs (with the router-gap rule), oracle-quantized weights, and the
parity measures.  Inputs come from ``synth``; expected values only from ``oracle``."""
import dataclasses
from typing import Optional

import numpy as np

import oracle
import synth

GAP = 1e-3          # required fp64 gap between the 2nd and 3rd router logit of every token
Y_ABS = 2e-2        # max |y - ref| <= Y_ABS * (1 + |ref|)
Y_MEAN_REL = 5e-3   # sum |y - ref| / sum |ref| <= Y_MEAN_REL
W_ABS = 1e-5        # |routing weight - ref|


def workload(name: str, **over) -> synth.Workload:
    wl = synth.WORKLOADS[name]
    return dataclasses.replace(wl, **over) if over else wl


def gap_inputs(wl: synth.Workload, gap: float = GAP, max_rounds: int = 64, router_wl: Optional[synth.Workload] = None):
    """x, router weight and bias, with every row of x redrawn (next attempt number of its own
    stream) until its 2nd-vs-3rd router logit gap in fp64 exceeds `gap`, so that the top-2 set is
    decided by the data and not by rounding.  The router comes from `router_wl` if given (ranks
    that share one router but draw their own tokens).  Returns dict(x, wr, bias, attempts, redrawn)."""
    wr = synth.gen_router(router_wl or wl)
    bias = synth.gen_bias(router_wl or wl)
    attempts = np.zeros(wl.T, dtype=np.int64)
    x = synth.gen_x(wl)
    rows = np.arange(wl.T)
    redrawn = 0
    for _ in range(max_rounds):
        _, _, z = oracle.route(x[rows], wr, bias, want_logits=True)
        zs = -np.sort(-z, axis=1)
        bad = rows[(zs[:, 1] - zs[:, 2]) <= gap]
        if bad.size == 0:
            return dict(x=x, wr=wr, bias=bias, attempts=attempts, redrawn=redrawn)
        attempts[bad] += 1
        redrawn += bad.size
        x[bad] = synth.gen_x(wl, attempts=attempts, rows=bad)
        rows = bad
    raise RuntimeError("router gap rule did not converge")


def first_gap(z: np.ndarray) -> np.ndarray:
    zs = -np.sort(-z, axis=1)
    return zs[:, 0] - zs[:, 1]


def oracle_expert_weights(wl: synth.Workload, which: str):
    """(bf16 bits [E][rows][cols], q int8, s fp32) for one of w1, w3, w2, quantized by the oracle."""
    w = synth.gen_experts(wl, which)
    q, s = oracle.quantize(w)
    return w, q, s


def y_errors(y_bf16_bits: np.ndarray, ref: np.ndarray):
    y = synth.bf16_bits_to_f32(y_bf16_bits).astype(np.float64)
    err = np.abs(y - ref)
    max_ratio = float(np.max(err / (1.0 + np.abs(ref)))) if err.size else 0.0
    mean_rel = float(err.sum() / max(np.abs(ref).sum(), 1e-300))
    return max_ratio, mean_rel


def assert_y_close(y_bf16_bits: np.ndarray, ref: np.ndarray, what: str = "y"):
    max_ratio, mean_rel = y_errors(y_bf16_bits, ref)
    assert np.all(np.isfinite(synth.bf16_bits_to_f32(y_bf16_bits))), f"{what}: non-finite output"
    assert max_ratio <= Y_ABS, f"{what}: max |y-ref|/(1+|ref|) = {max_ratio:.3e} > {Y_ABS}"
    assert mean_rel <= Y_MEAN_REL, f"{what}: mean relative error {mean_rel:.3e} > {Y_MEAN_REL}"
    return max_ratio, mean_rel


def assert_routing(ids_gpu: np.ndarray, w_gpu: np.ndarray, ids_ref: np.ndarray, w_ref: np.ndarray,
                   z_ref: Optional[np.ndarray] = None):
    """Top-2 sets bit-exact per token; order compared where the 1st-2nd logit gap exceeds GAP;
    weights within W_ABS (matched by expert id)."""
    assert ids_gpu.shape == ids_ref.shape
    assert np.array_equal(np.sort(ids_gpu, 1), np.sort(ids_ref, 1)), "top-2 expert sets differ"
    if z_ref is not None:
        sure = first_gap(z_ref) > GAP
        assert np.array_equal(ids_gpu[sure], ids_ref[sure]), "top-2 order differs where the gap is clear"
    same = ids_gpu == ids_ref
    w_ref_matched = np.where(same, w_ref, w_ref[:, ::-1])
    assert np.max(np.abs(w_gpu.astype(np.float64) - w_ref_matched)) <= W_ABS


def expert_segments(ids: np.ndarray, n_experts: int = 16):
    """Per expert, the assignment indices a = t*K + k routed to it in the order of its permuted
    segment (ascending a: the permutation is stable, so token order)."""
    flat = np.asarray(ids).reshape(-1)
    return [np.nonzero(flat == e)[0] for e in range(n_experts)]


def tile_covering_tokens(ids: np.ndarray, n_min: int = 512, tile: int = 128, seed: int = 0) -> np.ndarray:
    """Tokens to compare with the oracle on a large batch: one row drawn (seeded) from every
    `tile`-row M tile of every expert's permuted segment, the first and last row of every segment,
    then evenly strided tokens until at least `n_min` distinct tokens (or all T) are taken."""
    ids = np.asarray(ids)
    T, K = ids.shape
    rng = np.random.default_rng(seed)
    toks = set()
    for seg in expert_segments(ids):
        if seg.size == 0:
            continue
        toks.update([int(seg[0] // K), int(seg[-1] // K)])
        for m0 in range(0, seg.size, tile):
            rows = seg[m0:m0 + tile]
            toks.add(int(rows[rng.integers(rows.size)] // K))
    n = min(n_min, T)
    extra = n_min
    while len(toks) < n:
        toks.update(np.linspace(0, T - 1, extra).round().astype(int).tolist())
        extra *= 2
    return np.array(sorted(toks), dtype=np.int64)


def uncovered_tiles(ids: np.ndarray, tokens: np.ndarray, tile: int = 128):
    """(expert, M tile) pairs of the permuted order none of whose rows belongs to `tokens`."""
    ids = np.asarray(ids)
    K = ids.shape[1]
    chosen = np.zeros(ids.shape[0], bool)
    chosen[np.asarray(tokens)] = True
    missing = []
    for e, seg in enumerate(expert_segments(ids)):
        for m, m0 in enumerate(range(0, seg.size, tile)):
            if not chosen[seg[m0:m0 + tile] // K].any():
                missing.append((e, m))
    return missing
