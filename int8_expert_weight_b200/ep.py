"""Expert-parallel ExpertsInt8 MoE layer over torch.distributed (one process per GPU).

With G ranks, rank g holds the int8 weights of experts [g*16/G, (g+1)*16/G) only (Jamba-1.5 paper,
"Model Architecture": ExpertsInt8 is what lets Jamba-1.5-Large be served on one machine of eight
80 GB GPUs; "Training Infrastructure": expert parallelism).  Every rank brings its own batch of
tokens.  One call:

    dispatch          router + permutation + packing of x rows by destination rank (CUDA)
    all-to-all        per-rank row counts, then rows, local expert indices, routing weights
    experts           the rank's experts on the rows it received (CUDA)
    all-to-all back   the weighted outputs, fp32, into the send order
    combine           y[t] = bf16(slot 0 + slot 1) in fixed order (CUDA)

Each row crosses the interconnect once each way; over NCCL the exchange runs over NVLink /
NVSwitch.  Every computing step is a kernel of the C library (the three ``steps``); this module
only sizes the buffers and moves them.  ``steps`` may be replaced by stand-ins with the same
contract, which is how the exchange logic is tested on CPU ranks (gloo).
"""
from typing import Optional

import torch
import torch.distributed as dist

from . import (PATH_AUTO, jamba_moe_ep_combine, jamba_moe_ep_dispatch, jamba_moe_ep_dispatch_workspace_size,
               jamba_moe_ep_experts, jamba_moe_ep_experts_workspace_size, jamba_moe_read_device_status)

N_EXPERTS = 16


def expert_range(rank: int, world: int, n_experts: int = N_EXPERTS):
    """[first, last) experts owned by `rank` of `world` ranks."""
    if n_experts % world:
        raise ValueError(f"{world} ranks do not divide {n_experts} experts")
    per = n_experts // world
    return rank * per, (rank + 1) * per


class CudaSteps:
    """The three computing steps on this rank's GPU (the C library).  The workspaces are kept
    from call to call (grown when a call needs more), so a steady stream of calls allocates nothing
    new; the last calls' device status words are read with dispatch_status / experts_status."""

    def __init__(self, path: int = PATH_AUTO):
        self.path = path
        self.ws_dispatch = None
        self.ws_experts = None

    @staticmethod
    def _grow(ws, need, device):
        if ws is None or ws.numel() < need or ws.device != device:
            ws = torch.empty(need, dtype=torch.uint8, device=device)
        return ws

    def dispatch(self, x, router_W, router_bias, world):
        need = jamba_moe_ep_dispatch_workspace_size(x.shape[0], x.shape[1])
        self.ws_dispatch = self._grow(self.ws_dispatch, need, x.device)
        return jamba_moe_ep_dispatch(x, router_W, router_bias, world, workspace=self.ws_dispatch)

    def experts(self, xr, expert, w, weights):
        Q1, S1, Q3, S3, Q2, S2 = weights
        need = jamba_moe_ep_experts_workspace_size(xr.shape[0], xr.shape[1], Q1.shape[1])
        self.ws_experts = self._grow(self.ws_experts, need, xr.device)
        return jamba_moe_ep_experts(xr, expert, w, Q1, S1, Q3, S3, Q2, S2, workspace=self.ws_experts,
                                    path=self.path)

    def dispatch_status(self) -> int:
        return 0 if self.ws_dispatch is None else jamba_moe_read_device_status(self.ws_dispatch)

    def experts_status(self) -> int:
        return 0 if self.ws_experts is None else jamba_moe_read_device_status(self.ws_experts)

    def combine(self, ret, pos):
        return jamba_moe_ep_combine(ret, pos)


def _all_to_all(send: torch.Tensor, send_counts, recv_counts, group):
    """Rows of `send` (first dim) to every rank: send_counts[g] rows to rank g, recv_counts[g]
    rows from rank g.  bf16 rows (an even number of elements) travel as pairs in 32-bit words."""
    bf16 = send.dtype == torch.bfloat16
    wire = send.contiguous().view(torch.int32) if bf16 else send.contiguous()
    recv = torch.empty((sum(recv_counts),) + tuple(wire.shape[1:]), dtype=wire.dtype, device=send.device)
    dist.all_to_all_single(recv, wire, output_split_sizes=list(recv_counts), input_split_sizes=list(send_counts),
                           group=group)
    return recv.view(torch.bfloat16) if bf16 else recv


def ep_forward(x: torch.Tensor, router_W: torch.Tensor, router_bias: Optional[torch.Tensor], weights,
               group=None, steps=None, stats: Optional[dict] = None):
    """The MoE layer on this rank's tokens x [T][d] (bf16), experts spread over the ranks of `group`.

    weights = (Q1, S1, Q3, S3, Q2, S2) of this rank's experts (expert_range), as produced by
    jamba_moe_quantize; router_W [16][d] and router_bias are replicated.  Returns
    (y bf16 [T][d], topk_ids int32 [T][2], topk_w fp32 [T][2]).  Collective: every rank of the
    group calls it once per layer call, in the same order.  If `stats` is given, it receives the
    rows sent to and received from every rank and the local expert index of every received row.
    """
    steps = steps or CudaSteps()
    world = dist.get_world_size(group)
    d = steps.dispatch(x, router_W, router_bias, world)
    send_counts = d["send_counts"]
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts.contiguous(), group=group)
    sc = [int(v) for v in send_counts.tolist()]  # host copies size the row exchange (one sync)
    rc = [int(v) for v in recv_counts.tolist()]
    n_send = sum(sc)
    xr = _all_to_all(d["send_x"][:n_send], sc, rc, group)
    er = _all_to_all(d["send_expert"][:n_send], sc, rc, group)
    wr = _all_to_all(d["send_w"][:n_send], sc, rc, group)
    if stats is not None:
        stats.update(send_counts=sc, recv_counts=rc, recv_expert=er)
    out = steps.experts(xr, er, wr, weights)
    ret = _all_to_all(out, rc, sc, group)
    y = steps.combine(ret, d["pos"])
    return y, d["topk_ids"], d["topk_w"]
