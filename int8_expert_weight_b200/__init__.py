"""ExpertsInt8 mixture-of-experts layer for NVIDIA B200 — thin Python binding of libjmoe.so.

Every step of the layer runs in the CUDA kernels of ``libjmoe.so`` (see ``include/jmoe.h`` for
the C ABI).  This module only marshals arguments: it checks dtypes, devices and shapes of torch
tensors, passes their device pointers and the current CUDA stream, and turns a non-zero status
into a ``JmoeError``.  PyTorch provides device memory and streams; there is no CPU path.

Functions keep the C names: ``jamba_moe_quantize``, ``jamba_moe_workspace_size``,
``jamba_moe_forward`` (the ExpertsInt8 MoE layer), ``jamba_moe_forward_bf16w`` (unquantized bf16
weights), ``jamba_moe_quantize_fp8`` / ``jamba_moe_workspace_size_fp8`` / ``jamba_moe_forward_fp8``
(the FP8 comparator layer), ``jamba_mlp_workspace_size`` / ``jamba_mlp_forward`` (the dense
ExpertsInt8 MLP), ``jamba_moe_forward_noalloc``, ``jamba_moe_read_device_status``,
``jamba_moe_status_string``, ``jamba_moe_timing_start``, ``jamba_moe_timing_collect``.
"""
import ctypes
import os
from typing import Dict, Optional, Tuple

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libjmoe.so")

N_EXPERTS = 16
TOP_K = 2
PATH_AUTO, PATH_GEMV, PATH_GEMM = 0, 1, 2
KERNEL_NAMES = ["quantize", "router", "permute", "gather", "gemv13", "gemv2", "gemm13", "gemm2", "combine",
                "act_quant"]


class JmoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {jamba_moe_status_string(status)} (status {status})")


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libjmoe.so; raises if it has not been built (run int8_expert_weight_b200/build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libjmoe.so not found at {path}: build it with `python int8_expert_weight_b200/build.py`")
    lib = ctypes.CDLL(path)
    vp, i64, c_int, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.jamba_moe_quantize.restype = c_int
    lib.jamba_moe_quantize.argtypes = [vp, i64, i64, i64, vp, vp, vp]
    lib.jamba_moe_workspace_size.restype = sz
    lib.jamba_moe_workspace_size.argtypes = [i64, i64, i64, c_int, c_int]
    fwd_args = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, c_int, c_int, vp, vp, vp, vp, sz, vp]
    lib.jamba_moe_forward.restype = c_int
    lib.jamba_moe_quantize_fp8.restype = c_int
    lib.jamba_moe_quantize_fp8.argtypes = [vp, i64, i64, i64, vp, vp, vp]
    lib.jamba_moe_workspace_size_fp8.restype = sz
    lib.jamba_moe_workspace_size_fp8.argtypes = [i64, i64, i64, c_int, c_int]
    lib.jamba_moe_forward_fp8.restype = c_int
    lib.jamba_moe_forward_fp8.argtypes = fwd_args + [c_int]
    lib.jamba_mlp_workspace_size.restype = sz
    lib.jamba_mlp_workspace_size.argtypes = [i64, i64, i64]
    mlp_args = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, sz, vp]
    lib.jamba_mlp_forward.restype = c_int
    lib.jamba_mlp_forward.argtypes = mlp_args
    lib.jamba_mlp_forward_path.restype = c_int
    lib.jamba_mlp_forward_path.argtypes = mlp_args + [c_int]
    lib.jamba_moe_forward.argtypes = fwd_args
    lib.jamba_moe_forward_path.restype = c_int
    lib.jamba_moe_forward_path.argtypes = fwd_args + [c_int]
    lib.jamba_moe_read_device_status.restype = c_int
    lib.jamba_moe_read_device_status.argtypes = [vp, vp]
    lib.jamba_moe_status_string.restype = ctypes.c_char_p
    lib.jamba_moe_status_string.argtypes = [c_int]
    lib.jamba_moe_timing_start.restype = c_int
    lib.jamba_moe_timing_start.argtypes = [c_int]
    lib.jamba_moe_timing_collect.restype = c_int
    lib.jamba_moe_timing_collect.argtypes = [vp, vp, c_int]
    lib.jamba_moe_forward_noalloc.restype = c_int
    lib.jamba_moe_forward_noalloc.argtypes = fwd_args[:17] + [vp]
    lib.jamba_moe_noalloc_scratch_capacity.restype = sz
    lib.jamba_moe_noalloc_scratch_capacity.argtypes = []
    lib.jamba_moe_noalloc_scratch_needed.restype = sz
    lib.jamba_moe_noalloc_scratch_needed.argtypes = [i64, i64, i64]
    lib.jamba_moe_noalloc_read_device_status.restype = c_int
    lib.jamba_moe_noalloc_read_device_status.argtypes = [vp]
    lib.jamba_moe_forward_bf16w.restype = c_int
    lib.jamba_moe_forward_bf16w.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, c_int, c_int, vp, vp, vp, vp, sz,
                                            vp, c_int]
    lib.jamba_moe_debug_skip_copy.restype = c_int
    lib.jamba_moe_debug_skip_copy.argtypes = [c_int]
    lib.jamba_moe_ep_dispatch_workspace_size.restype = sz
    lib.jamba_moe_ep_dispatch_workspace_size.argtypes = [i64, i64, c_int, c_int]
    lib.jamba_moe_ep_dispatch.restype = c_int
    lib.jamba_moe_ep_dispatch.argtypes = [vp, vp, vp, i64, i64, c_int, c_int, c_int, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                          vp]
    lib.jamba_moe_ep_experts_workspace_size.restype = sz
    lib.jamba_moe_ep_experts_workspace_size.argtypes = [i64, i64, i64]
    lib.jamba_moe_ep_experts.restype = c_int
    lib.jamba_moe_ep_experts.argtypes = [vp, vp, vp, i64, i64, i64, c_int, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                         c_int]
    lib.jamba_moe_ep_combine.restype = c_int
    lib.jamba_moe_ep_combine.argtypes = [vp, vp, i64, i64, vp, vp]
    lib.jamba_moe_debug_checks.restype = c_int
    lib.jamba_moe_debug_checks.argtypes = [c_int]
    lib.jamba_moe_debug_corrupt.restype = c_int
    lib.jamba_moe_debug_corrupt.argtypes = [c_int]
    lib.jamba_moe_kernel_name.restype = ctypes.c_char_p
    lib.jamba_moe_kernel_name.argtypes = [c_int]
    _lib = lib
    return lib


def _stream_ptr(stream: Optional[torch.cuda.Stream], device: Optional[torch.device] = None) -> int:
    """The stream to launch on: the given one, else the current stream of `device`."""
    s = torch.cuda.current_stream(device) if stream is None else stream
    if device is not None and s.device != device:
        raise ValueError(f"stream belongs to {s.device}, the tensors to {device}")
    return s.cuda_stream


def _check(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _one_device(ref: torch.Tensor, **tensors) -> torch.device:
    """The device of `ref`, after checking that every other tensor of the call is on it too.  The
    call then runs with that device current, on its stream: the library launches on the current
    device."""
    for name, t in tensors.items():
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, the call's first tensor on {ref.device}: "
                             "every tensor of a call must be on one device")
    return ref.device


def jamba_moe_status_string(status: int) -> str:
    return load_library().jamba_moe_status_string(int(status)).decode()


def jamba_moe_workspace_size(T: int, d: int, ffn: int, n_experts: int = N_EXPERTS, top_k: int = TOP_K) -> int:
    return int(load_library().jamba_moe_workspace_size(T, d, ffn, n_experts, top_k))


def jamba_moe_quantize(W: torch.Tensor, stream: Optional[torch.cuda.Stream] = None,
                       out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """ExpertsInt8 quantization of bf16 weights [..., rows, cols] (one scale per row).
    Returns (Q int8 same shape, S fp32 shape[:-1])."""
    lib = load_library()
    _check(W, "W", torch.bfloat16)
    if W.dim() < 2:
        raise ValueError("W must have at least 2 dims (rows, cols)")
    rows, cols = W.shape[-2], W.shape[-1]
    n_mats = W.numel() // (rows * cols) if W.numel() else 0
    if out is None:
        Q = torch.empty(W.shape, dtype=torch.int8, device=W.device)
        S = torch.empty(W.shape[:-1], dtype=torch.float32, device=W.device)
    else:
        Q, S = out
        _check(Q, "Q", torch.int8, W.shape)
        _check(S, "S", torch.float32, W.shape[:-1])
    dev = _one_device(W, Q=Q, S=S)
    with torch.cuda.device(dev):
        st = lib.jamba_moe_quantize(W.data_ptr(), n_mats, rows, cols, Q.data_ptr(), S.data_ptr(),
                                    _stream_ptr(stream, dev))
    if st != 0:
        raise JmoeError(st, "jamba_moe_quantize")
    return Q, S


def jamba_moe_forward(x: torch.Tensor, router_W: torch.Tensor, router_bias: Optional[torch.Tensor],
                      Q1: torch.Tensor, S1: torch.Tensor, Q3: torch.Tensor, S3: torch.Tensor,
                      Q2: torch.Tensor, S2: torch.Tensor, y: Optional[torch.Tensor] = None,
                      topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                      path: int = PATH_AUTO, want_routing: bool = True):
    """The MoE layer on x [T][d] (bf16).  Weights as produced by jamba_moe_quantize:
    Q1, Q3 int8 [16][ffn][d] with S1, S3 fp32 [16][ffn]; Q2 int8 [16][d][ffn] with S2 fp32 [16][d];
    router_W fp32 [16][d]; router_bias fp32 [16] or None.

    Returns (y bf16 [T][d], topk_ids int32 [T][2] or None, topk_w fp32 [T][2] or None).
    ``workspace`` (uint8, >= jamba_moe_workspace_size bytes) is allocated when not given.
    """
    lib = load_library()
    _check(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be [T][d]")
    T, d = x.shape
    E = router_W.shape[0]
    ffn = Q1.shape[1]
    _check(router_W, "router_W", torch.float32, (E, d))
    if router_bias is not None:
        _check(router_bias, "router_bias", torch.float32, (E,))
    _check(Q1, "Q1", torch.int8, (E, ffn, d))
    _check(Q3, "Q3", torch.int8, (E, ffn, d))
    _check(Q2, "Q2", torch.int8, (E, d, ffn))
    _check(S1, "S1", torch.float32, (E, ffn))
    _check(S3, "S3", torch.float32, (E, ffn))
    _check(S2, "S2", torch.float32, (E, d))
    if y is None:
        y = torch.empty((T, d), dtype=torch.bfloat16, device=x.device)
    _check(y, "y", torch.bfloat16, (T, d))
    if want_routing:
        if topk_ids is None:
            topk_ids = torch.empty((T, TOP_K), dtype=torch.int32, device=x.device)
        if topk_w is None:
            topk_w = torch.empty((T, TOP_K), dtype=torch.float32, device=x.device)
    if topk_ids is not None:
        _check(topk_ids, "topk_ids", torch.int32, (T, TOP_K))
    if topk_w is not None:
        _check(topk_w, "topk_w", torch.float32, (T, TOP_K))
    need = jamba_moe_workspace_size(T, d, ffn, E, TOP_K)
    if need == 0:
        raise JmoeError(2, "jamba_moe_workspace_size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(workspace, "workspace", torch.uint8)
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    dev = _one_device(x, router_W=router_W, router_bias=router_bias, Q1=Q1, S1=S1, Q3=Q3, S3=S3, Q2=Q2, S2=S2, y=y,
                      topk_ids=topk_ids, topk_w=topk_w, workspace=workspace)
    with torch.cuda.device(dev):
        st = lib.jamba_moe_forward_path(x.data_ptr(), router_W.data_ptr(), p(router_bias), Q1.data_ptr(),
                                        S1.data_ptr(), Q3.data_ptr(), S3.data_ptr(), Q2.data_ptr(), S2.data_ptr(),
                                        T, d, ffn, E, TOP_K, y.data_ptr(), p(topk_ids), p(topk_w),
                                        workspace.data_ptr(), workspace.numel(), _stream_ptr(stream, dev), int(path))
    if st != 0:
        raise JmoeError(st, "jamba_moe_forward")
    return y, topk_ids, topk_w


def jamba_moe_quantize_fp8(W: torch.Tensor, stream: Optional[torch.cuda.Stream] = None,
                           out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """FP8 (E4M3) quantization of bf16 weights [..., rows, cols] (one scale per row).
    Returns (Q uint8 E4M3 codes, same shape; S fp32, shape[:-1])."""
    lib = load_library()
    _check(W, "W", torch.bfloat16)
    if W.dim() < 2:
        raise ValueError("W must have at least 2 dims (rows, cols)")
    rows, cols = W.shape[-2], W.shape[-1]
    n_mats = W.numel() // (rows * cols) if W.numel() else 0
    if out is None:
        Q = torch.empty(W.shape, dtype=torch.uint8, device=W.device)
        S = torch.empty(W.shape[:-1], dtype=torch.float32, device=W.device)
    else:
        Q, S = out
        _check(Q, "Q", torch.uint8, W.shape)
        _check(S, "S", torch.float32, W.shape[:-1])
    dev = _one_device(W, Q=Q, S=S)
    with torch.cuda.device(dev):
        st = lib.jamba_moe_quantize_fp8(W.data_ptr(), n_mats, rows, cols, Q.data_ptr(), S.data_ptr(),
                                        _stream_ptr(stream, dev))
    if st != 0:
        raise JmoeError(st, "jamba_moe_quantize_fp8")
    return Q, S


def jamba_moe_workspace_size_fp8(T: int, d: int, ffn: int, n_experts: int = N_EXPERTS, top_k: int = TOP_K) -> int:
    return int(load_library().jamba_moe_workspace_size_fp8(T, d, ffn, n_experts, top_k))


def jamba_moe_forward_fp8(x: torch.Tensor, router_W: torch.Tensor, router_bias: Optional[torch.Tensor],
                          Q1: torch.Tensor, S1: torch.Tensor, Q3: torch.Tensor, S3: torch.Tensor,
                          Q2: torch.Tensor, S2: torch.Tensor, y: Optional[torch.Tensor] = None,
                          topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                          path: int = PATH_AUTO):
    """The FP8 (E4M3) comparator layer: as jamba_moe_forward with uint8 E4M3 codes Q1, Q3, Q2 from
    jamba_moe_quantize_fp8.  Returns (y, topk_ids, topk_w)."""
    lib = load_library()
    _check(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be [T][d]")
    T, d = x.shape
    E = router_W.shape[0]
    ffn = Q1.shape[1]
    _check(router_W, "router_W", torch.float32, (E, d))
    if router_bias is not None:
        _check(router_bias, "router_bias", torch.float32, (E,))
    _check(Q1, "Q1", torch.uint8, (E, ffn, d))
    _check(Q3, "Q3", torch.uint8, (E, ffn, d))
    _check(Q2, "Q2", torch.uint8, (E, d, ffn))
    _check(S1, "S1", torch.float32, (E, ffn))
    _check(S3, "S3", torch.float32, (E, ffn))
    _check(S2, "S2", torch.float32, (E, d))
    if y is None:
        y = torch.empty((T, d), dtype=torch.bfloat16, device=x.device)
    _check(y, "y", torch.bfloat16, (T, d))
    if topk_ids is None:
        topk_ids = torch.empty((T, TOP_K), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((T, TOP_K), dtype=torch.float32, device=x.device)
    _check(topk_ids, "topk_ids", torch.int32, (T, TOP_K))
    _check(topk_w, "topk_w", torch.float32, (T, TOP_K))
    need = jamba_moe_workspace_size_fp8(T, d, ffn, E, TOP_K)
    if need == 0:
        raise JmoeError(2, "jamba_moe_workspace_size_fp8")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(workspace, "workspace", torch.uint8)
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    dev = _one_device(x, router_W=router_W, router_bias=router_bias, Q1=Q1, S1=S1, Q3=Q3, S3=S3, Q2=Q2, S2=S2, y=y,
                      topk_ids=topk_ids, topk_w=topk_w, workspace=workspace)
    with torch.cuda.device(dev):
        st = lib.jamba_moe_forward_fp8(x.data_ptr(), router_W.data_ptr(), p(router_bias), Q1.data_ptr(),
                                       S1.data_ptr(), Q3.data_ptr(), S3.data_ptr(), Q2.data_ptr(), S2.data_ptr(), T, d,
                                       ffn, E, TOP_K, y.data_ptr(), p(topk_ids), p(topk_w), workspace.data_ptr(),
                                       workspace.numel(), _stream_ptr(stream, dev), int(path))
    if st != 0:
        raise JmoeError(st, "jamba_moe_forward_fp8")
    return y, topk_ids, topk_w


def jamba_mlp_workspace_size(T: int, d: int, ffn: int) -> int:
    return int(load_library().jamba_mlp_workspace_size(T, d, ffn))


def jamba_mlp_forward(x: torch.Tensor, Q1: torch.Tensor, S1: torch.Tensor, Q3: torch.Tensor, S3: torch.Tensor,
                      Q2: torch.Tensor, S2: torch.Tensor, y: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                      path: int = PATH_AUTO) -> torch.Tensor:
    """The dense ExpertsInt8 MLP on x [T][d] (bf16): Q1, Q3 int8 [ffn][d] with S1, S3 fp32 [ffn];
    Q2 int8 [d][ffn] with S2 fp32 [d] (from jamba_moe_quantize).  Returns y bf16 [T][d].
    ``workspace`` (uint8, >= jamba_mlp_workspace_size bytes) is allocated when not given."""
    lib = load_library()
    _check(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be [T][d]")
    T, d = x.shape
    ffn = Q1.shape[0]
    _check(Q1, "Q1", torch.int8, (ffn, d))
    _check(Q3, "Q3", torch.int8, (ffn, d))
    _check(Q2, "Q2", torch.int8, (d, ffn))
    _check(S1, "S1", torch.float32, (ffn,))
    _check(S3, "S3", torch.float32, (ffn,))
    _check(S2, "S2", torch.float32, (d,))
    if y is None:
        y = torch.empty((T, d), dtype=torch.bfloat16, device=x.device)
    _check(y, "y", torch.bfloat16, (T, d))
    need = jamba_mlp_workspace_size(T, d, ffn)
    if need == 0:
        raise JmoeError(2, "jamba_mlp_workspace_size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(workspace, "workspace", torch.uint8)
    dev = _one_device(x, Q1=Q1, S1=S1, Q3=Q3, S3=S3, Q2=Q2, S2=S2, y=y, workspace=workspace)
    with torch.cuda.device(dev):
        st = lib.jamba_mlp_forward_path(x.data_ptr(), Q1.data_ptr(), S1.data_ptr(), Q3.data_ptr(), S3.data_ptr(),
                                        Q2.data_ptr(), S2.data_ptr(), T, d, ffn, y.data_ptr(), workspace.data_ptr(),
                                        workspace.numel(), _stream_ptr(stream, dev), int(path))
    if st != 0:
        raise JmoeError(st, "jamba_mlp_forward")
    return y


def jamba_moe_forward_bf16w(x: torch.Tensor, router_W: torch.Tensor, router_bias: Optional[torch.Tensor],
                            W1: torch.Tensor, W3: torch.Tensor, W2: torch.Tensor, y: Optional[torch.Tensor] = None,
                            topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                            path: int = PATH_AUTO):
    """The same layer with unquantized bf16 expert weights W1, W3 [16][ffn][d], W2 [16][d][ffn]
    (the BF16 comparator of ExpertsInt8).  Returns (y, topk_ids, topk_w)."""
    lib = load_library()
    _check(x, "x", torch.bfloat16)
    T, d = x.shape
    E, ffn = W1.shape[0], W1.shape[1]
    _check(router_W, "router_W", torch.float32, (E, d))
    if router_bias is not None:
        _check(router_bias, "router_bias", torch.float32, (E,))
    _check(W1, "W1", torch.bfloat16, (E, ffn, d))
    _check(W3, "W3", torch.bfloat16, (E, ffn, d))
    _check(W2, "W2", torch.bfloat16, (E, d, ffn))
    y = torch.empty((T, d), dtype=torch.bfloat16, device=x.device) if y is None else y
    topk_ids = torch.empty((T, TOP_K), dtype=torch.int32, device=x.device) if topk_ids is None else topk_ids
    topk_w = torch.empty((T, TOP_K), dtype=torch.float32, device=x.device) if topk_w is None else topk_w
    _check(y, "y", torch.bfloat16, (T, d))
    _check(topk_ids, "topk_ids", torch.int32, (T, TOP_K))
    _check(topk_w, "topk_w", torch.float32, (T, TOP_K))
    need = jamba_moe_workspace_size(T, d, ffn, E, TOP_K)
    if need == 0:
        raise JmoeError(2, "jamba_moe_workspace_size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(workspace, "workspace", torch.uint8)
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    dev = _one_device(x, router_W=router_W, router_bias=router_bias, W1=W1, W3=W3, W2=W2, y=y, topk_ids=topk_ids,
                      topk_w=topk_w, workspace=workspace)
    with torch.cuda.device(dev):
        st = lib.jamba_moe_forward_bf16w(x.data_ptr(), router_W.data_ptr(), p(router_bias), W1.data_ptr(),
                                         W3.data_ptr(), W2.data_ptr(), T, d, ffn, E, TOP_K, y.data_ptr(),
                                         topk_ids.data_ptr(), topk_w.data_ptr(), workspace.data_ptr(),
                                         workspace.numel(), _stream_ptr(stream, dev), int(path))
    if st != 0:
        raise JmoeError(st, "jamba_moe_forward_bf16w")
    return y, topk_ids, topk_w


def jamba_moe_forward_noalloc(x: torch.Tensor, router_W: torch.Tensor, router_bias: Optional[torch.Tensor],
                              Q1: torch.Tensor, S1: torch.Tensor, Q3: torch.Tensor, S3: torch.Tensor,
                              Q2: torch.Tensor, S2: torch.Tensor, y: torch.Tensor, topk_ids: torch.Tensor,
                              topk_w: torch.Tensor, stream: Optional[torch.cuda.Stream] = None):
    """jamba_moe_forward without a workspace, for callers that cannot allocate device memory: the
    scratch is the library's static 64 MiB device array.  All outputs are caller-provided, so
    this wrapper allocates nothing either.  Calls that overlap on the GPU race on the array."""
    lib = load_library()
    T, d = x.shape
    E, ffn = Q1.shape[0], Q1.shape[1]
    for t, n, dt in ((x, "x", torch.bfloat16), (y, "y", torch.bfloat16), (router_W, "router_W", torch.float32),
                     (Q1, "Q1", torch.int8), (Q3, "Q3", torch.int8), (Q2, "Q2", torch.int8),
                     (S1, "S1", torch.float32), (S3, "S3", torch.float32), (S2, "S2", torch.float32),
                     (topk_ids, "topk_ids", torch.int32), (topk_w, "topk_w", torch.float32)):
        _check(t, n, dt)
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    dev = _one_device(x, router_W=router_W, router_bias=router_bias, Q1=Q1, S1=S1, Q3=Q3, S3=S3, Q2=Q2, S2=S2, y=y,
                      topk_ids=topk_ids, topk_w=topk_w)
    with torch.cuda.device(dev):
        st = lib.jamba_moe_forward_noalloc(x.data_ptr(), router_W.data_ptr(), p(router_bias), Q1.data_ptr(),
                                           S1.data_ptr(), Q3.data_ptr(), S3.data_ptr(), Q2.data_ptr(), S2.data_ptr(),
                                           T, d, ffn, E, TOP_K, y.data_ptr(), topk_ids.data_ptr(), topk_w.data_ptr(),
                                           _stream_ptr(stream, dev))
    if st != 0:
        raise JmoeError(st, "jamba_moe_forward_noalloc")
    return y, topk_ids, topk_w


def jamba_moe_noalloc_read_device_status(device=None, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise the stream and return the device status word that the last
    jamba_moe_forward_noalloc call on `device` (default: the current device) left in the static
    scratch."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(load_library().jamba_moe_noalloc_read_device_status(_stream_ptr(stream, dev)))


def jamba_moe_read_device_status(workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise the stream and return the device status word of the last forward on workspace."""
    _check(workspace, "workspace", torch.uint8)
    with torch.cuda.device(workspace.device):
        return int(load_library().jamba_moe_read_device_status(workspace.data_ptr(),
                                                               _stream_ptr(stream, workspace.device)))


def jamba_moe_debug_skip_copy(on: bool) -> None:
    """Test hook (see include/jmoe.h): make one tensor-core pipeline wait run out on purpose."""
    load_library().jamba_moe_debug_skip_copy(1 if on else 0)


def jamba_moe_ep_dispatch_workspace_size(T: int, d: int, n_experts: int = N_EXPERTS, top_k: int = TOP_K) -> int:
    return int(load_library().jamba_moe_ep_dispatch_workspace_size(T, d, n_experts, top_k))


def jamba_moe_ep_experts_workspace_size(N: int, d: int, ffn: int) -> int:
    return int(load_library().jamba_moe_ep_experts_workspace_size(N, d, ffn))


def jamba_moe_ep_dispatch(x: torch.Tensor, router_W: torch.Tensor, router_bias: Optional[torch.Tensor], n_ranks: int,
                          workspace: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """Expert-parallel step 1 (see include/jmoe.h): route this rank's tokens x [T][d] and pack
    their rows by destination rank.  Returns a dict: send_x bf16 [2T][d], send_expert int32 [2T]
    (expert index local to its rank), send_w fp32 [2T], send_counts int32 [n_ranks], pos int32
    [T][2], topk_ids int32 [T][2], topk_w fp32 [T][2], and the workspace (device status word)."""
    lib = load_library()
    _check(x, "x", torch.bfloat16)
    T, d = x.shape
    E = router_W.shape[0]
    _check(router_W, "router_W", torch.float32, (E, d))
    if router_bias is not None:
        _check(router_bias, "router_bias", torch.float32, (E,))
    dev = x.device
    out = dict(send_x=torch.empty((T * TOP_K, d), dtype=torch.bfloat16, device=dev),
               send_expert=torch.empty(T * TOP_K, dtype=torch.int32, device=dev),
               send_w=torch.empty(T * TOP_K, dtype=torch.float32, device=dev),
               send_counts=torch.empty(n_ranks, dtype=torch.int32, device=dev),
               pos=torch.empty((T, TOP_K), dtype=torch.int32, device=dev),
               topk_ids=torch.empty((T, TOP_K), dtype=torch.int32, device=dev),
               topk_w=torch.empty((T, TOP_K), dtype=torch.float32, device=dev))
    need = int(lib.jamba_moe_ep_dispatch_workspace_size(T, d, E, TOP_K))
    if need == 0:
        raise JmoeError(2, "jamba_moe_ep_dispatch_workspace_size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8)
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    _one_device(x, router_W=router_W, router_bias=router_bias, workspace=workspace)
    with torch.cuda.device(dev):
        st = lib.jamba_moe_ep_dispatch(x.data_ptr(), router_W.data_ptr(), p(router_bias), T, d, E, TOP_K, int(n_ranks),
                                       out["send_x"].data_ptr(), out["send_expert"].data_ptr(),
                                       out["send_w"].data_ptr(), out["send_counts"].data_ptr(), out["pos"].data_ptr(),
                                       out["topk_ids"].data_ptr(), out["topk_w"].data_ptr(), workspace.data_ptr(),
                                       workspace.numel(), _stream_ptr(stream, dev))
    if st != 0:
        raise JmoeError(st, "jamba_moe_ep_dispatch")
    out["workspace"] = workspace
    return out


def jamba_moe_ep_experts(xr: torch.Tensor, expert: torch.Tensor, w: torch.Tensor, Q1: torch.Tensor, S1: torch.Tensor,
                         Q3: torch.Tensor, S3: torch.Tensor, Q2: torch.Tensor, S2: torch.Tensor,
                         out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None, path: int = PATH_AUTO) -> torch.Tensor:
    """Expert-parallel step 3: this rank's experts (Q1, Q3 int8 [n_local][ffn][d], Q2 int8
    [n_local][d][ffn] and scales) on the N received rows xr [N][d] with their local expert index
    and routing weight.  Returns out fp32 [N][d] = w * E_expert(xr)."""
    lib = load_library()
    _check(xr, "xr", torch.bfloat16)
    N, d = xr.shape
    n_local, ffn = Q1.shape[0], Q1.shape[1]
    _check(expert, "expert", torch.int32, (N,))
    _check(w, "w", torch.float32, (N,))
    _check(Q1, "Q1", torch.int8, (n_local, ffn, d))
    _check(Q3, "Q3", torch.int8, (n_local, ffn, d))
    _check(Q2, "Q2", torch.int8, (n_local, d, ffn))
    _check(S1, "S1", torch.float32, (n_local, ffn))
    _check(S3, "S3", torch.float32, (n_local, ffn))
    _check(S2, "S2", torch.float32, (n_local, d))
    if out is None:
        out = torch.empty((N, d), dtype=torch.float32, device=xr.device)
    _check(out, "out", torch.float32, (N, d))
    need = int(lib.jamba_moe_ep_experts_workspace_size(N, d, ffn))
    if need == 0:
        raise JmoeError(2, "jamba_moe_ep_experts_workspace_size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=xr.device)
    _check(workspace, "workspace", torch.uint8)
    dev = _one_device(xr, expert=expert, w=w, Q1=Q1, S1=S1, Q3=Q3, S3=S3, Q2=Q2, S2=S2, out=out, workspace=workspace)
    with torch.cuda.device(dev):
        st = lib.jamba_moe_ep_experts(xr.data_ptr(), expert.data_ptr(), w.data_ptr(), N, d, ffn, n_local,
                                      Q1.data_ptr(), S1.data_ptr(), Q3.data_ptr(), S3.data_ptr(), Q2.data_ptr(),
                                      S2.data_ptr(), out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                      _stream_ptr(stream, dev), int(path))
    if st != 0:
        raise JmoeError(st, "jamba_moe_ep_experts")
    return out


def jamba_moe_ep_combine(ret: torch.Tensor, pos: torch.Tensor, y: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Expert-parallel step 5: y bf16 [T][d] = bf16(ret[pos[t][0]] + ret[pos[t][1]])."""
    lib = load_library()
    _check(ret, "ret", torch.float32)
    _check(pos, "pos", torch.int32)
    T, d = pos.shape[0], ret.shape[1]
    _check(ret, "ret", torch.float32, (T * TOP_K, d))
    _check(pos, "pos", torch.int32, (T, TOP_K))
    if y is None:
        y = torch.empty((T, d), dtype=torch.bfloat16, device=ret.device)
    _check(y, "y", torch.bfloat16, (T, d))
    dev = _one_device(ret, pos=pos, y=y)
    with torch.cuda.device(dev):
        st = lib.jamba_moe_ep_combine(ret.data_ptr(), pos.data_ptr(), T, d, y.data_ptr(), _stream_ptr(stream, dev))
    if st != 0:
        raise JmoeError(st, "jamba_moe_ep_combine")
    return y


CORRUPT_NONE, CORRUPT_ROUTE_ID, CORRUPT_PERM_ROW, CORRUPT_CANARY = 0, 1, 2, 3


def jamba_moe_debug_checks(on: bool) -> None:
    """Debug checks of every MoE forward call (see include/jmoe.h): routing tables and canaries."""
    load_library().jamba_moe_debug_checks(1 if on else 0)


def jamba_moe_debug_corrupt(what: int) -> None:
    """Test hook (see include/jmoe.h): the next MoE forward call corrupts its own state, in bounds."""
    st = load_library().jamba_moe_debug_corrupt(int(what))
    if st != 0:
        raise JmoeError(st, "jamba_moe_debug_corrupt")


def jamba_moe_timing_start(max_launches: int) -> None:
    st = load_library().jamba_moe_timing_start(int(max_launches))
    if st != 0:
        raise JmoeError(st, "jamba_moe_timing_start")


def jamba_moe_timing_collect() -> Dict[str, Tuple[float, int]]:
    """{kernel name: (total event-timed ms, launches)} for the launches recorded since timing_start."""
    n = len(KERNEL_NAMES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    r = load_library().jamba_moe_timing_collect(ctypes.addressof(ms), ctypes.addressof(cnt), n)
    if r < 0:
        raise JmoeError(-r, "jamba_moe_timing_collect")
    return {KERNEL_NAMES[k]: (ms[k], cnt[k]) for k in range(n) if cnt[k]}
