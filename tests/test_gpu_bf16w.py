"""GPU parity of the BF16-weight comparator layer (jamba_moe_forward_bf16w) against the fp64 oracle
with the same bf16 weights; same tolerances as the ExpertsInt8 layer."""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import int8_expert_weight_b200 as jm  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402
from gpu_layer import bf16_to_dev, dev_to_bf16_bits  # noqa: E402
from helpers import (assert_routing, assert_y_close, gap_inputs, tile_covering_tokens,  # noqa: E402
                     uncovered_tiles, workload)

PATHS = [pytest.param(jm.PATH_GEMV, id="gemv"), pytest.param(jm.PATH_GEMM, id="gemm")]


class BLayer:
    def __init__(self, wl):
        self.wl = wl
        inp = gap_inputs(wl)
        self.x_bits, self.wr, self.bias = inp["x"], inp["wr"], inp["bias"]
        self.w = {k: synth.gen_experts(wl, k) for k in ("w1", "w3", "w2")}
        self.dev = {k: bf16_to_dev(v) for k, v in self.w.items()}

    def forward(self, path):
        bias = None if self.bias is None else torch.from_numpy(self.bias).cuda()
        y, ids, w = jm.jamba_moe_forward_bf16w(bf16_to_dev(self.x_bits), torch.from_numpy(self.wr).cuda(), bias,
                                               self.dev["w1"], self.dev["w3"], self.dev["w2"], path=path)
        torch.cuda.synchronize()
        return dev_to_bf16_bits(y), ids.cpu().numpy(), w.cpu().numpy()

    def ref(self, tokens=None):
        return oracle.moe_forward_bf16w(self.x_bits, self.wr, self.bias, self.w["w1"], self.w["w3"], self.w["w2"],
                                        tokens=tokens)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from int8_expert_weight_b200 import build
    build.build()
    jm.load_library()


def check(L, path, tokens=None):
    y, ids, w = L.forward(path)
    ref = L.ref(tokens)
    sel = slice(None) if tokens is None else np.asarray(tokens)
    _, _, z = oracle.route(L.x_bits[sel], L.wr, L.bias, want_logits=True)
    assert_routing(ids[sel], w[sel], ref["ids"], ref["w"], z)
    assert_y_close(y[sel], ref["y"])


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T,d,F", [(64, 256, 512), (3, 256, 512), (17, 384, 640), (129, 256, 1152)])
def test_bf16w_small(T, d, F, path):
    check(BLayer(dataclasses.replace(workload("tiny"), T=T, d=d, F=F)), path)


def test_bf16w_v01_decode_all_tokens():
    check(BLayer(workload("v01_decode")), jm.PATH_AUTO)


def test_bf16w_v01_prefill_sampled():
    L = BLayer(workload("v01_prefill"))
    ids_o, _, _ = oracle.route(L.x_bits, L.wr, L.bias, want_logits=True)
    toks = tile_covering_tokens(ids_o)
    assert toks.size >= 512 and uncovered_tiles(ids_o, toks) == []
    check(L, jm.PATH_AUTO, toks)
