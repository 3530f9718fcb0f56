"""Expert parallelism on CPU ranks (gloo): the exchange logic of ep_forward, with the three
computing steps (CUDA kernels in the product) replaced by stand-ins built from the oracle and
following the same contract.  Each rank holds only its own experts' weights and its own batch;
its y must equal the whole layer's oracle output on its tokens, so a row sent to the wrong rank,
in the wrong order or combined into the wrong token fails."""
import dataclasses
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class OracleSteps:
    """dispatch / experts / combine with the contract of include/jmoe.h's jamba_moe_ep_* calls."""

    def __init__(self, oracle, per_rank):
        self.oracle = oracle
        self.per = per_rank

    def dispatch(self, x, router_W, router_bias, world):
        xb = x.view(torch.int16).numpy().view(np.uint16)
        ids, w = self.oracle.route(xb, router_W.numpy(), None if router_bias is None else router_bias.numpy())
        flat = ids.reshape(-1)
        order = np.argsort(flat, kind="stable")  # expert, then assignment (token) order
        pos = np.empty(flat.size, np.int32)
        pos[order] = np.arange(flat.size)
        counts = [int(((flat >= g * self.per) & (flat < (g + 1) * self.per)).sum()) for g in range(world)]
        return dict(send_x=torch.from_numpy(xb[order // 2].view(np.int16)).view(torch.bfloat16),
                    send_expert=torch.from_numpy((flat[order] % self.per).astype(np.int32)),
                    send_w=torch.from_numpy(w.reshape(-1)[order].astype(np.float64)),
                    send_counts=torch.tensor(counts, dtype=torch.int64),
                    pos=torch.from_numpy(pos.reshape(-1, 2)), topk_ids=torch.from_numpy(ids), topk_w=torch.from_numpy(w))

    def experts(self, xr, er, wr, weights):
        q1, s1, q3, s3, q2, s2 = weights
        xb = xr.view(torch.int16).numpy().view(np.uint16)
        e = er.numpy()
        out = np.zeros((xb.shape[0], xb.shape[1]), np.float64)
        for le in np.unique(e):
            rows = np.nonzero(e == le)[0]
            y = self.oracle.mlp_forward(xb[rows], q1[le], s1[le], q3[le], s3[le], q2[le], s2[le])["y"]
            out[rows] = wr.numpy()[rows, None] * y
        return torch.from_numpy(out)

    def combine(self, ret, pos):
        p = pos.numpy()
        return torch.from_numpy(ret.numpy()[p[:, 0]] + ret.numpy()[p[:, 1]])


def _worker(rank, world, port, T, out):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    import synth
    from helpers import workload
    from int8_expert_weight_b200.ep import ep_forward, expert_range

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = dataclasses.replace(workload("tiny"), T=T)  # router and expert weights: shared seed
        inp = dict(x=synth.gen_x(dataclasses.replace(wl, seed=100 + rank)),  # this rank's own tokens
                   wr=synth.gen_router(wl), bias=synth.gen_bias(wl))
        e0, e1 = expert_range(rank, world)
        qs = {}
        for which in ("w1", "w3", "w2"):  # only this rank's experts
            q, s = oracle.quantize(np.stack([synth.gen_expert(wl, which, e) for e in range(e0, e1)]))
            qs[which] = (q, s)
        weights = (*qs["w1"], *qs["w3"], *qs["w2"])
        x = torch.from_numpy(inp["x"].view(np.int16)).view(torch.bfloat16)
        bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"])
        y, ids, w = ep_forward(x, torch.from_numpy(inp["wr"]), bias, weights,
                               steps=OracleSteps(oracle, 16 // world))
        # the whole layer, all 16 experts, on one process
        full = {}
        for which in ("w1", "w3", "w2"):
            full[which] = oracle.quantize(synth.gen_experts(wl, which))
        ref = oracle.moe_forward(inp["x"], inp["wr"], inp["bias"], *full["w1"], *full["w3"], *full["w2"])
        err = float(np.max(np.abs(y.numpy() - ref["y"]) / (1e-30 + np.abs(ref["y"]).max())))
        out[rank] = (err, bool(np.array_equal(ids.numpy(), ref["ids"])))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T", [(2, 64), (4, 37), (2, 1)])
def test_ep_forward_gloo_ranks(world, T):
    port = free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, T, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        err, ids_same = out[r]
        assert ids_same, f"rank {r}: routing differs"
        assert err <= 1e-12, f"rank {r}: y differs from the whole layer by {err:.3e}"


def test_expert_range_partitions_the_experts():
    from int8_expert_weight_b200.ep import expert_range
    for world in (1, 2, 4, 8, 16):
        owned = [e for r in range(world) for e in range(*expert_range(r, world))]
        assert owned == list(range(16))
    with pytest.raises(ValueError):
        expert_range(0, 3)
