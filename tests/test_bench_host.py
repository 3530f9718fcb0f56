"""Host-side pieces of bench.py that the JSON line depends on: the algorithmic work per launch that
divides into the roofline, and the source key that decides whether a stored ncu traffic figure
still belongs to the kernel being timed (a stale figure is reported as null)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def test_algorithmic_work_of_the_decode_workload():
    wl = synth.WORKLOADS["v01_decode"]
    d, F, T = wl.d, wl.F, wl.T
    kind, b13 = bench.algorithmic("gemv13", wl, T, touched=16, rows_padded=2048)
    assert kind == "bytes"
    # every touched expert's W1 and W3 once (int8 codes + fp32 row scales), x rows in, h rows out
    assert b13 == 16 * (2 * F * d + 2 * F * 4) + 2 * T * d * 2 + 2 * T * F * 2
    kind, b2 = bench.algorithmic("gemv2", wl, T, touched=16, rows_padded=2048)
    assert kind == "bytes" and b2 == 16 * (d * F + d * 4) + 2 * T * F * 2 + 2 * T * d * 4 + 2 * T * 8
    # bf16 weights: twice the weight bytes, no scales
    _, b13w = bench.algorithmic("gemv13", wl, T, 16, 2048, wbytes=2)
    assert b13w == 16 * (2 * F * d * 2) + 2 * T * d * 2 + 2 * T * F * 2
    # fewer touched experts: fewer weight bytes
    assert bench.algorithmic("gemv13", wl, T, 5, 2048)[1] < b13


def test_algorithmic_flops_of_the_prefill_workload():
    wl = synth.WORKLOADS["v01_prefill"]
    kind, f13 = bench.algorithmic("gemm13", wl, wl.T, 16, 0)
    assert kind == "flops" and f13 == 2.0 * (2 * wl.T) * wl.d * (2 * wl.F)
    kind, f2 = bench.algorithmic("gemm2", wl, wl.T, 16, 0)
    assert kind == "flops" and f2 == 2.0 * (2 * wl.T) * wl.F * wl.d


def test_algorithmic_work_of_the_dense_mlp():
    wl = synth.MLP_WORKLOADS["mlp_v01_decode"]
    d, F, T = wl.d, wl.F, wl.T
    # one weight set, every token once; the down-projection writes y in bf16
    assert bench.algorithmic("gemv2", wl, T, 1, 128)[1] == d * F + d * 4 + T * F * 2 + T * d * 2
    assert bench.algorithmic("gemm13", synth.MLP_WORKLOADS["mlp_v01_prefill"], 8192, 1, 0)[1] == \
        2.0 * 8192 * d * 2 * F


def test_source_key_ignores_comments_only(tmp_path, monkeypatch):
    csrc = tmp_path / "int8_expert_weight_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "common.cuh").write_text("// header\nint a;\n")
    (csrc / "gemv.cu").write_text("/* notes */\nint f() { return 1; }  // one\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    k0 = bench.kernel_source_hash("gemv13")
    (csrc / "gemv.cu").write_text("/* other notes,\n   two lines */\nint f() { return 1; }  // uno\n")
    assert bench.kernel_source_hash("gemv13") == k0
    # a comment block removed with its lines, re-indented code: still the same key
    (csrc / "gemv.cu").write_text("\n\n\nint  f()\n{ return 1; }\n")
    assert bench.kernel_source_hash("gemv13") == k0
    (csrc / "gemv.cu").write_text("int f() { return 2; }\n")
    assert bench.kernel_source_hash("gemv13") != k0



def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON line with the
    keys of the bench contract, no host/device copies and a CPU-baseline record of itself."""
    import json
    import subprocess

    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1", "--workload", "tiny"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 1
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"] == "tiny"
    assert abs(d["value"] - d["config"]["T"] * 1e3 / d["ms_per_step"]) <= 1e-6 * d["value"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_parity_on_sample_measures():
    """parity_stats, which puts the sampled GPU-vs-oracle comparison into the bench line: the
    oracle's own output rounded to bf16 is within tolerance, a 10 % error is not, and a token whose
    expert pair differs is counted and left out of the y measures."""
    wl = synth.WORKLOADS["tiny"]
    setup = bench.oracle_setup(wl, wl.seed)
    toks = np.arange(0, wl.T, 5)
    ref = bench.oracle_forward(wl, setup, toks, 1)
    y_bits = synth.f32_to_bf16_bits(ref["y"].astype(np.float32))
    ok = bench.parity_stats(y_bits, ref["ids"], ref)
    assert ok["tokens"] == len(toks) and ok["id_mismatch_tokens"] == 0 and ok["within_tolerance"]
    assert 0 < ok["max_err_rel"] < 1e-2 and ok["mean_rel_err"] < 5e-3
    bad = bench.parity_stats(synth.f32_to_bf16_bits((ref["y"] * 1.1).astype(np.float32)), ref["ids"], ref)
    assert not bad["within_tolerance"]
    ids = ref["ids"].copy()
    ids[3] = (ids[3] + 1) % 16
    y_off = y_bits.copy()
    y_off[3] = synth.f32_to_bf16_bits(np.full(wl.d, 1e3, np.float32))  # that token's y is then unrelated
    mism = bench.parity_stats(y_off, ids, ref)
    assert mism["id_mismatch_tokens"] == 1 and mism["within_tolerance"]
    mlp = bench.parity_stats(y_bits, None, {"y": ref["y"]})
    assert "id_mismatch_tokens" not in mlp and mlp["within_tolerance"]
