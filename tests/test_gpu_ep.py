"""Expert parallelism on one GPU: G ranks emulated in one process, each with its own tokens and
only its own experts' weights, the all-to-all exchanges done by copying between the ranks' buffers
(no kernel waits on another rank).  The dispatch, expert and combine kernels are the ones
ep_forward runs over NCCL; every rank's y is checked against the fp64 oracle of the whole layer."""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import int8_expert_weight_b200 as jm  # noqa: E402
from int8_expert_weight_b200.ep import expert_range  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402
from gpu_layer import bf16_to_dev, dev_to_bf16_bits  # noqa: E402
from helpers import assert_routing, assert_y_close, gap_inputs, workload  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from int8_expert_weight_b200 import build
    build.build()
    jm.load_library()


def emulate(wl, world, path):
    """Per rank: inputs, y, ids, w from the emulated expert-parallel layer."""
    ranks = []
    for r in range(world):
        inp = gap_inputs(dataclasses.replace(wl, seed=wl.seed + 1000 * (r + 1)), router_wl=wl)
        e0, e1 = expert_range(r, world)
        wts = []
        for which in ("w1", "w3", "w2"):
            q, s = jm.jamba_moe_quantize(bf16_to_dev(np.stack([synth.gen_expert(wl, which, e) for e in range(e0, e1)])))
            wts += [q, s]
        bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).cuda()
        d = jm.jamba_moe_ep_dispatch(bf16_to_dev(inp["x"]), torch.from_numpy(inp["wr"]).cuda(), bias, world)
        ranks.append(dict(inp=inp, weights=wts, d=d, counts=d["send_counts"].cpu().numpy().astype(np.int64)))
    # exchange: rank g receives, from every rank r in rank order, the rows r packed for g
    outs = []
    for g in range(world):
        parts = []
        for r in range(world):
            c = ranks[r]["counts"]
            lo, hi = int(c[:g].sum()), int(c[:g + 1].sum())
            parts.append((ranks[r]["d"]["send_x"][lo:hi], ranks[r]["d"]["send_expert"][lo:hi],
                          ranks[r]["d"]["send_w"][lo:hi]))
        xr = torch.cat([p[0] for p in parts]).contiguous()
        er = torch.cat([p[1] for p in parts]).contiguous()
        wr = torch.cat([p[2] for p in parts]).contiguous()
        Q1, S1, Q3, S3, Q2, S2 = ranks[g]["weights"]
        out = jm.jamba_moe_ep_experts(xr, er, wr, Q1, S1, Q3, S3, Q2, S2, path=path)
        sizes = [int(ranks[r]["counts"][g]) for r in range(world)]
        outs.append(torch.split(out, sizes))
    results = []
    for r in range(world):
        ret = torch.cat([outs[g][r] for g in range(world)]).contiguous()  # back in send order
        y = jm.jamba_moe_ep_combine(ret, ranks[r]["d"]["pos"])
        torch.cuda.synchronize()
        results.append((ranks[r]["inp"], dev_to_bf16_bits(y), ranks[r]["d"]["topk_ids"].cpu().numpy(),
                        ranks[r]["d"]["topk_w"].cpu().numpy()))
    return results


def full_layer_ref(wl, inp):
    qs = {w: oracle.quantize(synth.gen_experts(wl, w)) for w in ("w1", "w3", "w2")}
    return oracle.moe_forward(inp["x"], inp["wr"], inp["bias"], *qs["w1"], *qs["w3"], *qs["w2"])


@pytest.mark.parametrize("path", [pytest.param(jm.PATH_AUTO, id="auto"), pytest.param(jm.PATH_GEMV, id="gemv"),
                                  pytest.param(jm.PATH_GEMM, id="gemm")])
@pytest.mark.parametrize("world,T,d,F", [(1, 64, 256, 512), (2, 64, 256, 512), (4, 37, 384, 640),
                                         (2, 300, 256, 512), (8, 130, 128, 256)])
def test_ep_layer_matches_oracle(world, T, d, F, path):
    wl = dataclasses.replace(workload("tiny"), T=T, d=d, F=F)
    for r, (inp, y, ids, w) in enumerate(emulate(wl, world, path)):
        ref = full_layer_ref(wl, inp)
        _, _, z = oracle.route(inp["x"], inp["wr"], inp["bias"], want_logits=True)
        assert_routing(ids, w, ref["ids"], ref["w"], z)
        assert_y_close(y, ref["y"], f"rank {r} of {world}")


def test_ep_skewed_routing_two_ranks():
    """The skewed router (+2 on experts 3 and 11): one rank gets far more rows than the other."""
    wl = dataclasses.replace(workload("skewed"), T=200, d=256, F=512)
    for r, (inp, y, ids, w) in enumerate(emulate(wl, 2, jm.PATH_AUTO)):
        ref = full_layer_ref(wl, inp)
        assert np.array_equal(np.sort(ids, 1), np.sort(ref["ids"], 1))
        assert_y_close(y, ref["y"], f"rank {r}")
