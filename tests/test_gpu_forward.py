"""GPU parity of the whole layer against the fp64 oracle.

y within max |y - ref| <= 2e-2 (1 + |ref|) and mean relative error <= 5e-3; routing ids exact;
int8 codes and scales of every weight matrix bit-exact (checked while building each layer)."""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import int8_expert_weight_b200 as jm  # noqa: E402
from gpu_layer import Layer  # noqa: E402
from helpers import (assert_routing, assert_y_close, tile_covering_tokens, uncovered_tiles,  # noqa: E402
                     workload)
import oracle  # noqa: E402

PATHS = [pytest.param(jm.PATH_GEMV, id="gemv"), pytest.param(jm.PATH_GEMM, id="gemm")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from int8_expert_weight_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    jm.load_library()


def check_layer(L: Layer, path, tokens=None):
    assert all(v == 0 for v in L.quant_mismatch.values()), L.quant_mismatch
    y, ids, w = L.forward(path=path)
    ref = L.oracle_forward(tokens=tokens)
    sel = slice(None) if tokens is None else np.asarray(tokens)
    _, _, z = oracle.route(L.x_bits[sel], L.wr, L.bias, want_logits=True)
    assert_routing(ids[sel], w[sel], ref["ids"], ref["w"], z)
    return assert_y_close(y[sel], ref["y"])


@pytest.fixture(scope="module")
def tiny():
    return Layer(workload("tiny"))


@pytest.mark.parametrize("path", PATHS)
def test_tiny_all_tokens(tiny, path):
    check_layer(tiny, path)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T,d,F", [(1, 256, 512), (3, 256, 512), (17, 384, 640), (80, 384, 640), (96, 256, 512),
                                   (129, 256, 512), (300, 128, 128), (257, 512, 1152)])
def test_ragged_shapes(T, d, F, path):
    wl = dataclasses.replace(workload("tiny"), T=T, d=d, F=F)
    check_layer(Layer(wl), path)


@pytest.mark.parametrize("path", PATHS)
def test_deterministic_and_status(tiny, path):
    ws = torch.empty(jm.jamba_moe_workspace_size(tiny.wl.T, tiny.wl.d, tiny.wl.F), dtype=torch.uint8, device="cuda")
    a = tiny.forward(path=path, workspace=ws)
    b = tiny.forward(path=path, workspace=ws)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    assert jm.jamba_moe_read_device_status(ws) == 0


def test_paths_agree_gemm(tiny):
    a = tiny.forward(path=jm.PATH_GEMV)
    b = tiny.forward(path=jm.PATH_GEMM)
    assert np.array_equal(a[1], b[1])
    ya = a[0].astype(np.uint32) << 16
    yb = b[0].astype(np.uint32) << 16
    diff = np.abs(ya.view(np.float32).astype(np.float64) - yb.view(np.float32).astype(np.float64))
    assert diff.max() <= 2e-2


@pytest.fixture(scope="module")
def v01_decode():
    return Layer(workload("v01_decode"))


def test_v01_decode_full_size_all_tokens(v01_decode):
    """The benchmarked workload at full size, in the benchmark's launch configuration (auto path)."""
    check_layer(v01_decode, jm.PATH_AUTO)


def test_v01_decode_gemm_path(v01_decode):
    check_layer(v01_decode, jm.PATH_GEMM)


def check_sampled(L: Layer, path):
    """Routing on every token; y on tokens that cover every (expert, 128-row M tile) of the permuted
    order (at least 512), computed by the oracle one token at a time."""
    assert all(v == 0 for v in L.quant_mismatch.values()), L.quant_mismatch
    y, ids, w = L.forward(path=path)
    ids_o, w_o, z = oracle.route(L.x_bits, L.wr, L.bias, want_logits=True)
    assert_routing(ids, w, ids_o, w_o, z)  # every token
    toks = tile_covering_tokens(ids_o)
    assert toks.size >= 512 and uncovered_tiles(ids_o, toks) == []
    ref = L.oracle_forward(tokens=toks)
    return assert_y_close(y[toks], ref["y"], f"y on {toks.size} sampled tokens")


@pytest.fixture(scope="module")
def v01_prefill():
    return Layer(workload("v01_prefill"))


def test_v01_prefill_sampled(v01_prefill):
    check_sampled(v01_prefill, jm.PATH_AUTO)


def test_skewed_sampled():
    check_sampled(Layer(workload("skewed")), jm.PATH_AUTO)


@pytest.mark.slow
def test_large_prefill_sampled():
    check_sampled(Layer(workload("large_prefill")), jm.PATH_AUTO)


@pytest.mark.slow
def test_large_decode_all_paths():
    """The 1.5-Large decode shape (9.7 GB of int8 experts): every token, both expert paths."""
    L = Layer(workload("large_decode"))
    ref = L.oracle_forward()
    _, _, z = oracle.route(L.x_bits, L.wr, L.bias, want_logits=True)
    for path in (jm.PATH_AUTO, jm.PATH_GEMM):
        y, ids, w = L.forward(path=path)
        assert_routing(ids, w, ref["ids"], ref["w"], z)
        assert_y_close(y, ref["y"], f"large decode path {path}")


@pytest.mark.parametrize("path", PATHS)
def test_two_experts_take_every_token(path):
    """A router bias that sends every token to experts 5 and 9: fourteen experts get no token (their
    weights are never read) and two get all 300, in segments of three 128-row tiles each."""
    wl = dataclasses.replace(workload("tiny"), T=300, bias={5: 30.0, 9: 30.0})
    L = Layer(wl)
    check_layer(L, path)
    assert set(np.unique(L.forward(path)[1]).tolist()) == {5, 9}


def test_no_token_is_a_no_op():
    """T = 0 on every forward entry point: no error, empty outputs."""
    d, F, E = 256, 512, 16
    dev = "cuda"
    x = torch.empty((0, d), dtype=torch.bfloat16, device=dev)
    wr = torch.zeros((E, d), dtype=torch.float32, device=dev)
    q13 = torch.zeros((E, F, d), dtype=torch.int8, device=dev)
    q2 = torch.zeros((E, d, F), dtype=torch.int8, device=dev)
    s13 = torch.ones((E, F), dtype=torch.float32, device=dev)
    s2 = torch.ones((E, d), dtype=torch.float32, device=dev)
    for path in (jm.PATH_AUTO, jm.PATH_GEMV, jm.PATH_GEMM):
        y, ids, w = jm.jamba_moe_forward(x, wr, None, q13, s13, q13, s13, q2, s2, path=path)
        assert y.shape == (0, d) and ids.shape == (0, 2) and w.shape == (0, 2)
        y, _, _ = jm.jamba_moe_forward_bf16w(x, wr, None, q13.to(torch.bfloat16), q13.to(torch.bfloat16),
                                            q2.to(torch.bfloat16), path=path)
        assert y.shape == (0, d)
        y, _, _ = jm.jamba_moe_forward_fp8(x, wr, None, q13.view(torch.uint8), s13, q13.view(torch.uint8), s13,
                                          q2.view(torch.uint8), s2, path=path)
        assert y.shape == (0, d)
        y = jm.jamba_mlp_forward(x, q13[0], s13[0], q13[0], s13[0], q2[0], s2[0], path=path)
        assert y.shape == (0, d)
    torch.cuda.synchronize()
