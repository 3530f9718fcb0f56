"""Failure detection on the GPU without a GPU fault: a bounded pipeline wait is made to run out
(the test hook leaves one copy unissued), the kernel reports JMOE_DEV_TIMEOUT through the
workspace status word and returns, and the context stays usable for a correct forward pass."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import int8_expert_weight_b200 as jm  # noqa: E402
from gpu_layer import Layer  # noqa: E402
from helpers import assert_y_close, workload  # noqa: E402

JMOE_DEV_TIMEOUT = 5


@pytest.fixture(scope="module")
def tiny():
    from int8_expert_weight_b200 import build
    build.build()
    return Layer(workload("tiny"))


def test_wait_runs_out_and_reports_timeout(tiny):
    ws = torch.empty(jm.jamba_moe_workspace_size(64, 256, 512), dtype=torch.uint8, device="cuda")
    jm.jamba_moe_debug_skip_copy(True)
    try:
        tiny.forward(path=jm.PATH_GEMM, workspace=ws)
        assert jm.jamba_moe_read_device_status(ws) == JMOE_DEV_TIMEOUT
    finally:
        jm.jamba_moe_debug_skip_copy(False)
    # the context is still usable: the next call is correct and reports no error
    y, ids, w = tiny.forward(path=jm.PATH_GEMM, workspace=ws)
    assert jm.jamba_moe_read_device_status(ws) == 0
    ref = tiny.oracle_forward()
    assert np.array_equal(np.sort(ids, 1), np.sort(ref["ids"], 1))
    assert_y_close(y, ref["y"])
