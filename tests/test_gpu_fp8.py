"""GPU parity of the FP8 (E4M3) comparator layer: quantization bit-exact against the oracle, the
layer (jamba_moe_forward_fp8) against the fp64 oracle of the same FP8 scheme.

Tolerance: the same as the ExpertsInt8 layer's.  Only the activation codes of the SwiGLU
intermediate are not bit-exact (the GPU quantizes its fp32 h, the oracle its fp64 h); the two h
differ by ~1e-6 relatively, so a code flips only when h sits that close to a rounding boundary of
the E4M3 grid (steps of 6-12 %), i.e. for ~1e-5 of the elements, each moving y by well under the
tolerance."""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import int8_expert_weight_b200 as jm  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402
from gpu_layer import bf16_to_dev, dev_to_bf16_bits  # noqa: E402
from helpers import (Y_ABS, Y_MEAN_REL, assert_routing, assert_y_close, gap_inputs,  # noqa: E402
                     tile_covering_tokens, uncovered_tiles, workload, y_errors)
from oracle_pins import E4M3_VALUES, bf16_bits  # noqa: E402

PATHS = [pytest.param(jm.PATH_GEMV, id="gemv"), pytest.param(jm.PATH_GEMM, id="gemm")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from int8_expert_weight_b200 import build
    build.build()
    jm.load_library()


def assert_fp8_quant_equal(w_bits):
    Q, S = jm.jamba_moe_quantize_fp8(bf16_to_dev(w_bits))
    torch.cuda.synchronize()
    qo, so = oracle.quantize_fp8(w_bits)
    assert np.array_equal(S.cpu().numpy().view(np.uint32), so.view(np.uint32)), "scales differ"
    qg = Q.cpu().numpy()
    assert np.array_equal(qg, qo), f"{np.count_nonzero(qg != qo)} codes differ"
    return qg, S.cpu().numpy()


@pytest.mark.parametrize("cols", [16, 48, 256, 4096, 4112, 8192, 14336, 24576, 32768, 40000])
def test_fp8_quantize_random_rows(cols):
    rng = np.random.default_rng(cols + 7)
    rows = max(1, 300000 // cols)
    w = synth.f32_to_bf16_bits((rng.standard_normal((rows, cols)) * 0.02).astype(np.float32))
    w[0, cols // 3] = bf16_bits([0.75])[0]
    assert_fp8_quant_equal(w)


def test_fp8_quantize_ties_subnormals_and_zeros():
    # rows whose amax is 448 * 2^-8, so the scale is 2^-8 exactly and w / s is the value itself:
    # every E4M3 midpoint that bf16 holds (ties to even), subnormal-range values, -0 and a zero row
    finite = E4M3_VALUES[np.isfinite(E4M3_VALUES)]
    pos = np.unique(finite[finite >= 0])
    mids = (pos[1:] + pos[:-1]) / 2
    vals = np.concatenate([[448.0], mids, -mids, pos[:12] / 3, [-0.0, 0.0]])
    vals = vals[np.asarray(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(vals.astype(np.float32)))) == vals]
    vals = vals[: (vals.size // 16) * 16]
    row = bf16_bits((vals * 2.0 ** -8).astype(np.float32))
    w = np.stack([row, np.zeros_like(row), row[::-1].copy()])
    q, s = assert_fp8_quant_equal(w)
    assert s[0] == np.float32(2.0 ** -8) and s[1] == 1.0 and not q[1].any()


class F8Layer:
    def __init__(self, wl):
        self.wl = wl
        inp = gap_inputs(wl)
        self.x_bits, self.wr, self.bias = inp["x"], inp["wr"], inp["bias"]
        self.q, self.s, self.qd, self.sd = {}, {}, {}, {}
        for which in ("w1", "w3", "w2"):
            w = synth.gen_experts(wl, which)
            Q, S = jm.jamba_moe_quantize_fp8(bf16_to_dev(w))
            q, s = oracle.quantize_fp8(w)
            torch.cuda.synchronize()
            assert np.array_equal(Q.cpu().numpy(), q), which
            assert np.array_equal(S.cpu().numpy().view(np.uint32), s.view(np.uint32)), which
            self.q[which], self.s[which], self.qd[which], self.sd[which] = q, s, Q, S

    def forward(self, path):
        bias = None if self.bias is None else torch.from_numpy(self.bias).cuda()
        y, ids, w = jm.jamba_moe_forward_fp8(bf16_to_dev(self.x_bits), torch.from_numpy(self.wr).cuda(), bias,
                                             self.qd["w1"], self.sd["w1"], self.qd["w3"], self.sd["w3"],
                                             self.qd["w2"], self.sd["w2"], path=path)
        torch.cuda.synchronize()
        return dev_to_bf16_bits(y), ids.cpu().numpy(), w.cpu().numpy()

    def ref(self, tokens=None, want_hidden=False):
        return oracle.moe_forward_fp8(self.x_bits, self.wr, self.bias, self.q["w1"], self.s["w1"], self.q["w3"],
                                      self.s["w3"], self.q["w2"], self.s["w2"], tokens=tokens,
                                      want_hidden=want_hidden)


# The GPU's SwiGLU value before its bf16 rounding is within this relative distance of the exact
# one: its dot products add exact E4M3 x E4M3 products in fp32, whose rounding errors grow like
# sqrt(K) fp32 ulps (K <= 16384 here: 128 * 2^-24 = 2^-17), and SiLU and the product with the up
# value add a few ulps more; twice that is allowed.  It is far below a bf16 step (2^-8).
H_REL = 2.0 ** -16


def scale_ambiguous(h: np.ndarray) -> np.ndarray:
    """Per row of fp64 SwiGLU values h [..., F]: whether the row's E4M3 scale (its largest |bf16 h|
    over 448) is not decided by the exact values, because the largest |h| lies within H_REL of a
    bf16 rounding boundary, so that both neighbouring bf16 values are results a correct fp32
    computation can round to; the row's codes then follow either scale."""
    m = np.abs(h).max(-1)
    lo = synth.f32_to_bf16_bits((m * (1 - H_REL)).astype(np.float32))
    hi = synth.f32_to_bf16_bits((m * (1 + H_REL)).astype(np.float32))
    return lo != hi


def check(L, path, tokens=None):
    """Routing exact; y within the layer tolerance on every token whose two SwiGLU rows have their
    E4M3 scales decided, and within twice that on the rest (one bf16 step in a row's scale moves
    its codes by at most one E4M3 step each); the mean relative error over all tokens as usual."""
    y, ids, w = L.forward(path)
    ref = L.ref(tokens, want_hidden=True)
    sel = slice(None) if tokens is None else np.asarray(tokens)
    _, _, z = oracle.route(L.x_bits[sel], L.wr, L.bias, want_logits=True)
    assert_routing(ids[sel], w[sel], ref["ids"], ref["w"], z)
    amb = scale_ambiguous(ref["h"]).any(-1)
    ys = y[sel]
    if (~amb).any():
        assert_y_close(ys[~amb], ref["y"][~amb], "y, tokens with decided scales")
    if amb.any():
        err, _ = y_errors(ys[amb], ref["y"][amb])
        assert err <= 2 * Y_ABS, f"y, tokens with an undecided scale: {err:.3e}"
    _, mean_rel = y_errors(ys, ref["y"])
    assert mean_rel <= Y_MEAN_REL, f"mean relative error {mean_rel:.3e}"


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T,d,F", [(64, 256, 512), (3, 256, 512), (17, 384, 640), (129, 256, 1152),
                                   (40, 1024, 2048)])
def test_fp8_layer_small(T, d, F, path):
    check(F8Layer(dataclasses.replace(workload("tiny"), T=T, d=d, F=F)), path)


def test_fp8_deterministic():
    L = F8Layer(dataclasses.replace(workload("tiny"), T=200))
    for path in (jm.PATH_GEMV, jm.PATH_GEMM):
        a = L.forward(path)[0]
        assert np.array_equal(a, L.forward(path)[0]), path


def test_fp8_v01_decode_all_tokens():
    check(F8Layer(workload("v01_decode")), jm.PATH_AUTO)


def test_fp8_v01_prefill_sampled():
    L = F8Layer(workload("v01_prefill"))
    ids_o, _, _ = oracle.route(L.x_bits, L.wr, L.bias, want_logits=True)
    toks = tile_covering_tokens(ids_o)
    assert toks.size >= 512 and uncovered_tiles(ids_o, toks) == []
    check(L, jm.PATH_AUTO, toks)
