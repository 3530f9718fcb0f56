"""Debug checks of a forward call on the GPU, tested without a GPU fault: the host corrupts one
call's routing state with in-bounds copies (an out-of-range routing id, an assignment held by two
permuted rows, an overwritten guard gap), the kernels report it through the workspace status word,
and the next call is clean and correct."""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import int8_expert_weight_b200 as jm  # noqa: E402
from gpu_layer import Layer  # noqa: E402
from helpers import assert_y_close, workload  # noqa: E402

OK, BAD_INDEX, BAD_TABLE, CANARY = 0, 6, 8, 9
PATHS = [pytest.param(jm.PATH_GEMV, id="gemv"), pytest.param(jm.PATH_GEMM, id="gemm")]


@pytest.fixture(scope="module")
def tiny():
    from int8_expert_weight_b200 import build
    build.build()
    jm.load_library()
    return Layer(workload("tiny"))


@pytest.fixture()
def checks_on():
    jm.jamba_moe_debug_checks(True)
    yield
    jm.jamba_moe_debug_checks(False)
    jm.jamba_moe_debug_corrupt(jm.CORRUPT_NONE)


def workspace(L):
    wl = L.wl
    return torch.empty(jm.jamba_moe_workspace_size(wl.T, wl.d, wl.F), dtype=torch.uint8, device="cuda")


def clean_call_is_correct(L, path, ws):
    y, ids, _ = L.forward(path=path, workspace=ws)
    assert jm.jamba_moe_read_device_status(ws) == OK
    ref = L.oracle_forward()
    assert np.array_equal(np.sort(ids, 1), np.sort(ref["ids"], 1))
    assert_y_close(y, ref["y"])


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("over", [{}, dict(T=300, d=128, F=128), dict(T=129, d=512, F=1152)])
def test_checks_pass_on_valid_calls(checks_on, path, over):
    L = Layer(dataclasses.replace(workload("tiny"), **over)) if over else Layer(workload("tiny"))
    ws = workspace(L)
    for _ in range(2):
        clean_call_is_correct(L, path, ws)


@pytest.mark.parametrize("path", PATHS)
def test_out_of_range_route_id_reported(tiny, path):
    ws = workspace(tiny)
    jm.jamba_moe_debug_corrupt(jm.CORRUPT_ROUTE_ID)
    tiny.forward(path=path, workspace=ws)
    assert jm.jamba_moe_read_device_status(ws) == BAD_INDEX
    clean_call_is_correct(tiny, path, ws)


@pytest.mark.parametrize("path", PATHS)
def test_assignment_held_twice_reported(tiny, checks_on, path):
    ws = workspace(tiny)
    jm.jamba_moe_debug_corrupt(jm.CORRUPT_PERM_ROW)
    tiny.forward(path=path, workspace=ws)
    assert jm.jamba_moe_read_device_status(ws) == BAD_TABLE
    clean_call_is_correct(tiny, path, ws)


@pytest.mark.parametrize("path", PATHS)
def test_guard_gap_overwrite_reported(tiny, checks_on, path):
    ws = workspace(tiny)
    jm.jamba_moe_debug_corrupt(jm.CORRUPT_CANARY)
    tiny.forward(path=path, workspace=ws)
    assert jm.jamba_moe_read_device_status(ws) == CANARY
    clean_call_is_correct(tiny, path, ws)


def test_corruption_without_checks_goes_unseen(tiny):
    """Without the debug checks only the permutation's own range check reports anything: a held-twice
    assignment passes silently (which is what the checks are for)."""
    ws = workspace(tiny)
    jm.jamba_moe_debug_corrupt(jm.CORRUPT_PERM_ROW)
    tiny.forward(path=jm.PATH_GEMM, workspace=ws)
    assert jm.jamba_moe_read_device_status(ws) == OK
    clean_call_is_correct(tiny, jm.PATH_GEMM, ws)
