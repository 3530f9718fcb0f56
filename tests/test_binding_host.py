"""The Python binding's marshalling, run on the CPU against a stand-in library that records its calls.

The stand-in checks every call against the argument list the real library declares through ctypes,
so a binding that passes too few or too many arguments, or sizes in the wrong slots, fails here.
The binding's device rule is checked too: every tensor of a call on one device, the call run with
that device current, and a given stream on the same device.  No GPU is needed: the dtype and CUDA
checks of individual tensors are bypassed, nothing is launched."""
import contextlib

import pytest
import torch

import int8_expert_weight_b200 as jm
from int8_expert_weight_b200 import build as jbuild


class FakeStream:
    def __init__(self, device, handle=0x5151):
        self.device = device
        self.cuda_stream = handle


class RecordingLib:
    """Returns status 0 (sizes: a fixed byte count) and records (name, args) of every call."""

    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        declared = getattr(self.real, name).argtypes

        def call(*args):
            assert len(args) == len(declared), f"{name}: {len(args)} arguments, {len(declared)} declared"
            self.calls.append((name, args))
            if "workspace_size" in name:
                return 4096
            if name == "jamba_moe_status_string":
                return b"status"
            return 0

        return call


@pytest.fixture
def fake(monkeypatch):
    jbuild.build()
    real = jm.load_library()
    rec = RecordingLib(real)
    devices = []
    monkeypatch.setattr(jm, "_lib", rec)
    monkeypatch.setattr(jm, "_check", lambda *a, **k: None)

    @contextlib.contextmanager
    def current(dev):
        devices.append(dev)
        yield

    monkeypatch.setattr(torch.cuda, "device", current)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda dev=None: FakeStream(dev))
    rec.devices = devices
    return rec


def layer(T=4, d=128, F=256, E=16, device="cpu"):
    z = lambda *s, dt=torch.float32: torch.zeros(*s, dtype=dt, device=device)  # noqa: E731
    return dict(x=z(T, d, dt=torch.bfloat16), router_W=z(E, d), router_bias=None,
                Q1=z(E, F, d, dt=torch.int8), S1=z(E, F), Q3=z(E, F, d, dt=torch.int8), S3=z(E, F),
                Q2=z(E, d, F, dt=torch.int8), S2=z(E, d))


def test_forward_passes_sizes_in_their_slots(fake):
    L = layer()
    y, ids, w = jm.jamba_moe_forward(**L, path=jm.PATH_GEMM)
    name, a = fake.calls[-1]
    assert name == "jamba_moe_forward_path"
    assert a[9:14] == (4, 128, 256, 16, 2)                     # T, d, ffn, n_experts, top_k
    assert a[2] is None                                        # no router bias
    assert a[14] == y.data_ptr() and a[15] == ids.data_ptr() and a[16] == w.data_ptr()
    assert a[18] == 4096 and a[19] == 0x5151 and a[20] == jm.PATH_GEMM  # workspace bytes, stream, path
    assert fake.devices == [torch.device("cpu")]
    assert tuple(y.shape) == (4, 128) and tuple(ids.shape) == (4, 2)


def test_every_entry_point_marshals_its_declared_arguments(fake):
    L = layer()
    jm.jamba_moe_quantize(L["x"].new_zeros(3, 16, 32))
    jm.jamba_moe_quantize_fp8(L["x"].new_zeros(16, 32))
    jm.jamba_moe_forward_fp8(**dict(L, Q1=L["Q1"].view(torch.uint8), Q3=L["Q3"].view(torch.uint8),
                                    Q2=L["Q2"].view(torch.uint8)))
    jm.jamba_moe_forward_bf16w(L["x"], L["router_W"], None, L["Q1"].to(torch.bfloat16), L["Q3"].to(torch.bfloat16),
                               L["Q2"].to(torch.bfloat16))
    jm.jamba_mlp_forward(L["x"], L["Q1"][0], L["S1"][0], L["Q3"][0], L["S3"][0], L["Q2"][0], L["S2"][0])
    y = torch.zeros_like(L["x"])
    jm.jamba_moe_forward_noalloc(**L, y=y, topk_ids=torch.zeros(4, 2, dtype=torch.int32),
                                 topk_w=torch.zeros(4, 2))
    jm.jamba_moe_read_device_status(torch.zeros(4096, dtype=torch.uint8))
    names = [n for n, _ in fake.calls if "workspace_size" not in n]
    assert names == ["jamba_moe_quantize", "jamba_moe_quantize_fp8", "jamba_moe_forward_fp8",
                     "jamba_moe_forward_bf16w", "jamba_mlp_forward_path", "jamba_moe_forward_noalloc",
                     "jamba_moe_read_device_status"]
    q = fake.calls[0][1]
    assert q[1:4] == (3, 16, 32)                               # n_mats, rows, cols
    mlp = dict(fake.calls)["jamba_mlp_forward_path"]
    assert mlp[7:10] == (4, 128, 256)                          # T, d, ffn
    assert len(fake.devices) == 7


def test_tensors_on_two_devices_are_refused(fake):
    L = layer()
    L["S2"] = torch.zeros(16, 128, device="meta")
    with pytest.raises(ValueError, match="S2 is on meta"):
        jm.jamba_moe_forward(**L)
    assert not [n for n, _ in fake.calls if n == "jamba_moe_forward_path"]


def test_a_stream_of_another_device_is_refused(fake):
    L = layer()
    with pytest.raises(ValueError, match="stream belongs to"):
        jm.jamba_moe_forward(**L, stream=FakeStream(torch.device("meta")))
