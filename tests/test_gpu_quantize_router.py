"""GPU parity: ExpertsInt8 quantization (bit-exact) and the router (ids exact, weights 1e-5)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import int8_expert_weight_b200 as jm  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402
from gpu_layer import bf16_to_dev  # noqa: E402
from helpers import assert_routing, gap_inputs, workload  # noqa: E402
from oracle_pins import bf16_bits  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from int8_expert_weight_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    jm.load_library()


def gpu_quantize(w_bits):
    Q, S = jm.jamba_moe_quantize(bf16_to_dev(w_bits))
    torch.cuda.synchronize()
    return Q.cpu().numpy(), S.cpu().numpy()


def assert_quant_equal(w_bits):
    qg, sg = gpu_quantize(w_bits)
    qo, so = oracle.quantize(w_bits)
    assert np.array_equal(sg.view(np.uint32), so.view(np.uint32)), "scales differ"
    assert np.array_equal(qg, qo), f"{np.count_nonzero(qg != qo)} codes differ"


def test_quantize_special_rows():
    k = -6
    vals = [127, 0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 125.5, 126.5, -126.5, 0.25, 0.75, 0, 5.5, -5.5]
    halfway = bf16_bits(np.array(vals, np.float32) * np.float32(2.0 ** k))
    zero = np.zeros(16, np.uint16)
    negzero = np.full(16, 0x8000, np.uint16)
    tiny = bf16_bits(np.array(vals, np.float32) * np.float32(2.0 ** -120))  # scale < 1e-30: fp64 path
    rng = np.random.default_rng(0)
    rand = synth.f32_to_bf16_bits((rng.standard_normal(16) * 3).astype(np.float32))
    w = np.stack([halfway, zero, negzero, tiny, rand])
    assert_quant_equal(w)
    qg, sg = gpu_quantize(w)
    assert qg[0].tolist()[:14] == [127, 0, 2, 2, 4, 0, -2, -2, 126, 126, -126, 0, 1, 0]
    assert sg[1] == 1.0 and not qg[1].any()


@pytest.mark.parametrize("cols", [16, 48, 256, 4096, 4096 + 16, 8192, 14336, 16384, 16384 + 16, 24576, 32768,
                                  32768 + 16, 40000])
def test_quantize_random_rows(cols):
    rng = np.random.default_rng(cols)
    rows = max(1, 300000 // cols)
    w = synth.f32_to_bf16_bits((rng.standard_normal((rows, cols)) * 0.02).astype(np.float32))
    w[0, cols // 3] = bf16_bits([0.75])[0]  # an outlier
    assert_quant_equal(w)


def test_quantize_all_halfway_grid():
    # every (n + 1/2) * 2^k for n in 0..126, both signs, with amax = 127 * 2^k: all exact ties
    k = -10
    n = np.arange(127, dtype=np.float32)
    row = np.concatenate([[127.0], n + 0.5, -(n + 0.5), [0.0] * 1]).astype(np.float32)
    row = row[: (row.size // 16) * 16]
    assert_quant_equal(bf16_bits(row * np.float32(2.0 ** k))[None, :])


@pytest.mark.parametrize("reps", [1, 40, 300])
def test_quantize_halfway_rows_of_every_length_class(reps):
    # the halfway grid repeated: rows of 240, 9600 and 72000 weights (one warp, one CTA and the
    # two-pass kernel per row), every value an exact tie or the row's amax
    k = -7
    n = np.arange(120, dtype=np.float32)
    base = np.concatenate([[127.0], n[:119] + 0.5, -(n + 0.5)]).astype(np.float32)
    row = np.tile(base, reps)
    rows = np.stack([row, -row, row * np.float32(2.0 ** -3)])
    assert_quant_equal(bf16_bits(rows * np.float32(2.0 ** k)))


def test_quantize_full_expert_matrix():
    wl = workload("v01_decode")
    for which in ("w1", "w2"):
        assert_quant_equal(synth.gen_expert(wl, which, 5))


@pytest.mark.parametrize("name,T", [("tiny", None), ("v01_decode", None), ("v01_prefill", None),
                                    ("large_decode", None), ("skewed", 4096)])
def test_router_parity(name, T):
    wl = workload(name) if T is None else workload(name, T=T)
    inp = gap_inputs(wl)
    ids_o, w_o, z_o = oracle.route(inp["x"], inp["wr"], inp["bias"], want_logits=True)
    # the router runs as the first kernel of a forward call; zero weights keep the rest cheap
    E, d, F = wl.E, wl.d, 128
    Q1 = torch.zeros((E, F, d), dtype=torch.int8, device="cuda")
    Q2 = torch.zeros((E, d, F), dtype=torch.int8, device="cuda")
    S = torch.ones((E, F), dtype=torch.float32, device="cuda")
    S2 = torch.ones((E, d), dtype=torch.float32, device="cuda")
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).cuda()
    y, ids, w = jm.jamba_moe_forward(bf16_to_dev(inp["x"]), torch.from_numpy(inp["wr"]).cuda(), bias, Q1, S, Q1, S,
                                     Q2, S2, path=jm.PATH_GEMV)
    torch.cuda.synchronize()
    assert_routing(ids.cpu().numpy(), w.cpu().numpy(), ids_o, w_o, z_o)
    assert not torch.any(y.float() != 0)  # zero experts give exactly zero output
