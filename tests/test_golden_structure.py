"""The workloads and the library's supported shape match the structure the pages print."""
import os

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "jamba_moe_structure.txt")


def load_golden():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kv, _cite = line.split("|", 1)
        k, v = kv.split()
        out[k] = v
    return out


def test_workloads_follow_the_pages():
    g = load_golden()
    for wl in synth.WORKLOADS.values():
        assert wl.E == int(g["n_experts"])
        assert wl.K == int(g["top_k"])
    assert synth.WORKLOADS["large_decode"].d == int(g["hidden_large"])
    assert synth.WORKLOADS["large_prefill"].d == int(g["hidden_large"])
    assert g["weight_storage_bits"] == "8" and g["compute_dtype"] == "bf16"
