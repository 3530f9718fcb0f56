"""GPU parity of the dense ExpertsInt8 MLP (jamba_mlp_forward) against the fp64 oracle: the MLP of
the layers without MoE, whose weights ExpertsInt8 quantizes like the experts' (Jamba-1.5 paper,
§3.1).  Same y tolerances as the MoE layer; codes and scales bit-exact."""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import int8_expert_weight_b200 as jm  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402
from gpu_layer import bf16_to_dev, dev_to_bf16_bits  # noqa: E402
from helpers import assert_y_close, tile_covering_tokens, uncovered_tiles  # noqa: E402

PATHS = [pytest.param(jm.PATH_GEMV, id="gemv"), pytest.param(jm.PATH_GEMM, id="gemm")]


class Mlp:
    """x and the MLP's three matrices of one workload; quantized on the GPU and checked bit for bit
    against the oracle's quantization of the same bf16 weights."""

    def __init__(self, wl: synth.Workload):
        self.wl = wl
        self.x_bits = synth.gen_x(wl)
        self.q, self.s, self.qd, self.sd = {}, {}, {}, {}
        for which in ("w1", "w3", "w2"):
            w = synth.gen_experts(wl, which)[0]
            Q, S = jm.jamba_moe_quantize(bf16_to_dev(w))
            q, s = oracle.quantize(w)
            torch.cuda.synchronize()
            assert np.array_equal(Q.cpu().numpy(), q), f"{which}: int8 codes differ from the oracle's"
            assert np.array_equal(S.cpu().numpy().view(np.uint32), s.view(np.uint32)), f"{which}: scales differ"
            self.q[which], self.s[which], self.qd[which], self.sd[which] = q, s, Q, S

    def forward(self, path, T=None):
        x = bf16_to_dev(self.x_bits if T is None else self.x_bits[:T])
        y = jm.jamba_mlp_forward(x, self.qd["w1"], self.sd["w1"], self.qd["w3"], self.sd["w3"], self.qd["w2"],
                                 self.sd["w2"], path=path)
        torch.cuda.synchronize()
        return dev_to_bf16_bits(y)

    def ref(self, tokens=None, T=None):
        x = self.x_bits if T is None else self.x_bits[:T]
        return oracle.mlp_forward(x, self.q["w1"], self.s["w1"], self.q["w3"], self.s["w3"], self.q["w2"],
                                  self.s["w2"], tokens=tokens)["y"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from int8_expert_weight_b200 import build
    build.build()
    jm.load_library()


def mlp_workload(name, **over):
    wl = synth.MLP_WORKLOADS[name]
    return dataclasses.replace(wl, **over) if over else wl


@pytest.fixture(scope="module")
def tiny():
    return Mlp(mlp_workload("mlp_tiny", T=300))


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T", [1, 7, 8, 9, 16, 17, 32, 33, 64, 127, 128, 129, 300])
def test_mlp_tiny_ragged(tiny, T, path):
    """Token counts around the GEMV pass widths (8, 16, 32) and the 128-row GEMM tile."""
    assert_y_close(tiny.forward(path, T), tiny.ref(T=T), f"T={T}")


@pytest.mark.parametrize("T,d,F", [(40, 384, 640), (130, 512, 1152), (5, 2048, 3072), (40, 2048, 3072)])
@pytest.mark.parametrize("path", PATHS)
def test_mlp_other_shapes(T, d, F, path):
    L = Mlp(mlp_workload("mlp_tiny", T=T, d=d, F=F))
    assert_y_close(L.forward(path), L.ref())


def test_mlp_deterministic(tiny):
    for path in (jm.PATH_GEMV, jm.PATH_GEMM):
        a = tiny.forward(path, 100)
        b = tiny.forward(path, 100)
        assert np.array_equal(a, b), path


@pytest.mark.parametrize("T", [3, 24, 64])
def test_mlp_decode_repeatable(T):
    """Repeated decode calls agree bit for bit, and with the oracle."""
    L = Mlp(mlp_workload("mlp_tiny", T=T, d=2048, F=3072))
    a = L.forward(jm.PATH_GEMV)
    for _ in range(3):
        assert np.array_equal(L.forward(jm.PATH_GEMV), a)
    assert_y_close(a, L.ref())


def test_mlp_v01_decode_all_tokens():
    L = Mlp(mlp_workload("mlp_v01_decode"))
    ref = L.ref()
    for path in (jm.PATH_AUTO, jm.PATH_GEMM):
        assert_y_close(L.forward(path), ref, f"path {path}")


def test_mlp_v01_prefill_sampled():
    L = Mlp(mlp_workload("mlp_v01_prefill"))
    y = L.forward(jm.PATH_AUTO)
    one_expert = np.zeros((L.wl.T, 1), np.int32)  # the MLP's rows are its tokens, in order
    toks = tile_covering_tokens(one_expert)
    assert toks.size >= 512 and uncovered_tiles(one_expert, toks) == []
    assert_y_close(y[toks], L.ref(tokens=toks))
