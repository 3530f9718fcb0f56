"""jamba_moe_forward_noalloc (the entry point for callers that cannot allocate device memory, e.g.
code running inside a memory pool it does not own or a serving process that must not call
cudaMalloc after start-up) against the regular jamba_moe_forward, through the C ABI.

The file name makes pytest collect it last; it also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import int8_expert_weight_b200 as jm  # noqa: E402
from gpu_layer import Layer, dev_to_bf16_bits  # noqa: E402
from helpers import assert_routing, assert_y_close, workload  # noqa: E402
import oracle  # noqa: E402


@pytest.fixture(scope="module")
def lib():
    from int8_expert_weight_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return jm.load_library()


def call_noalloc(lib, L, y, ids, w):
    Q, S = L.q, L.s
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    wl = L.wl
    return lib.jamba_moe_forward_noalloc(
        L.x.data_ptr(), L.wr_dev.data_ptr(), p(L.bias_dev), Q["w1"].data_ptr(), S["w1"].data_ptr(),
        Q["w3"].data_ptr(), S["w3"].data_ptr(), Q["w2"].data_ptr(), S["w2"].data_ptr(), wl.T, wl.d, wl.F, 16, 2,
        y.data_ptr(), ids.data_ptr(), w.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,over", [("tiny", {}), ("tiny", dict(T=5, d=1024, F=2048)),
                                       ("skewed", dict(T=40, d=512, F=768))])
def test_noalloc_matches_forward_twice(lib, name, over):
    L = Layer(workload(name, **over), check_quant=False, keep_host_q=False)
    wl = L.wl
    y_ref, ids_ref, w_ref = L.forward()
    ref = y_ref.astype(np.uint32) << 16
    ref = ref.view(np.float32).astype(np.float64)
    for _ in range(2):  # two calls in a row share (and reuse) the static scratch
        y = torch.full((wl.T, wl.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        ids = torch.full((wl.T, 2), -1, dtype=torch.int32, device="cuda")
        w = torch.zeros((wl.T, 2), dtype=torch.float32, device="cuda")
        assert call_noalloc(lib, L, y, ids, w) == 0
        torch.cuda.synchronize()
        assert np.array_equal(ids.cpu().numpy(), ids_ref)
        assert np.max(np.abs(w.cpu().numpy() - w_ref)) <= 1e-5
        assert_y_close(dev_to_bf16_bits(y), ref, "noalloc y vs jamba_moe_forward")


def test_noalloc_against_oracle_and_status(lib):
    """The allocation-free call checked straight against the fp64 oracle (not only against the
    workspace call), through the Python wrapper on a side stream, and its device status word read
    back from the static scratch."""
    L = Layer(workload("tiny", T=48, d=512, F=768))
    wl = L.wl
    ref = L.oracle_forward()
    side = torch.cuda.Stream()
    y = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((wl.T, 2), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, 2), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()  # the inputs were written on the default stream
    jm.jamba_moe_forward_noalloc(L.x, L.wr_dev, L.bias_dev, L.q["w1"], L.s["w1"], L.q["w3"], L.s["w3"], L.q["w2"],
                                 L.s["w2"], y=y, topk_ids=ids, topk_w=w, stream=side)
    assert jm.jamba_moe_noalloc_read_device_status(stream=side) == 0
    _, _, z = oracle.route(L.x_bits, L.wr, L.bias, want_logits=True)
    assert_routing(ids.cpu().numpy(), w.cpu().numpy(), ref["ids"], ref["w"], z)
    assert_y_close(dev_to_bf16_bits(y), ref["y"], "noalloc y vs oracle")


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    cap = lib.jamba_moe_noalloc_scratch_capacity()
    assert cap == 64 << 20
    assert lib.jamba_moe_noalloc_scratch_needed(64, 8192, 24576) > cap
    one = torch.zeros(16, dtype=torch.uint8, device="cuda")
    fake = one.data_ptr()
    rc = lib.jamba_moe_forward_noalloc(fake, fake, None, fake, fake, fake, fake, fake, fake, 64, 8192, 24576, 16, 2,
                                       fake, None, None, None)
    assert rc == 3  # JMOE_ERR_WORKSPACE, returned before anything is launched
