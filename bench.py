"""Benchmark of the ExpertsInt8 MoE layer (tokens/s through jamba_moe_forward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one forward pass of the whole layer (router, permutation, expert GEMMs with in-kernel
int8 -> bf16 dequantization, weighted combine) over one batch of T synthetic tokens.  The int8
weights are quantized once, before timing (load time), by the library's quantize kernel, which is
timed on its own and reported under "quantize".  Under torchrun every rank runs its own batch with
replicated weights (weak scaling, no collective on the data path); the time is the max over ranks.

Prints one JSON line (rank 0).  --impl reference times the fp64 CPU oracle on bounded samples of the
same workload on the host cores (rank 0 only).
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "MoE-layer tokens/sec (int8 experts) at 1 B200; % of HBM / BF16 roofline"
METRIC_MLP = "dense-MLP tokens/sec (ExpertsInt8 weights) at 1 B200; % of HBM / BF16 roofline"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "skewed"  # the largest single-GPU configuration: T=65536, d=4096, ffn=14336


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.ALL_WORKLOADS),
                    help="MoE layer workloads, or mlp_* for the dense ExpertsInt8 MLP")
    ap.add_argument("--tokens", type=int, default=None,
                    help="run the workload's layer shape on this many tokens instead of its own T")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="auto", choices=["auto", "gemv", "gemm"])
    ap.add_argument("--weights", default="int8", choices=["int8", "bf16", "fp8"],
                    help="int8: ExpertsInt8 (the method); bf16: the unquantized comparator layer; "
                         "fp8: the FP8 (E4M3 weights and activations) comparator layer")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "ep"],
                    help="replicas: every rank runs the whole layer on its own batch (no collective); "
                         "ep: experts split over the ranks, rows exchanged by NCCL all-to-all")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ algorithmic work per launch
def algorithmic(kind, wl, T, touched, rows_padded, wbytes=1):
    """Bytes (HBM-bound kernels) or FLOPs (tensor-bound kernels) one launch must move / do.
    touched = experts with >= 1 token; rows_padded = permuted rows incl. per-expert padding;
    wbytes = bytes per weight (1: int8 codes, plus 4-byte scales per row; 2: bf16, no scales)."""
    d, F, TK = wl.d, wl.F, T * wl.K
    sc = 4 if wbytes == 1 else 0
    if wl.layer == "mlp":  # one weight matrix set, every token once (K = 1); y written in bf16 by gemv2/gemm2
        if kind == "gemv2":
            return "bytes", d * F * wbytes + d * sc + T * F * 2 + T * d * 2
        if kind == "permute":
            return "bytes", rows_padded * 4 + T * 4
    if kind == "gemv13":
        return "bytes", touched * (2 * F * d * wbytes + 2 * F * sc) + TK * d * 2 + TK * F * 2
    if kind == "gemv2":
        return "bytes", touched * (d * F * wbytes + d * sc) + TK * F * 2 + TK * d * 4 + TK * 4 * 2
    if kind == "gemm13":
        return "flops", 2.0 * TK * d * (2 * F)
    if kind == "gemm2":
        return "flops", 2.0 * TK * F * d
    if kind == "combine":
        return "bytes", TK * d * 4 + T * d * 2
    if kind == "router":
        return "bytes", T * d * 2 + wl.E * d * 4 + TK * 8
    if kind == "gather":
        return "bytes", rows_padded * d * 2 + TK * d * 2
    if kind == "permute":
        return "bytes", TK * 4 * 3
    if kind == "act_quant":  # FP8 layer, per launch on average: x (bf16 -> E4M3) and h (fp32 -> E4M3)
        return "bytes", (T * d * 3 + TK * F * 5) / 2
    if kind == "quantize":
        return "bytes", 3 * (2 * F * d + d * F) * wl.E
    return "bytes", 0


def kernel_source_hash(kind):
    files = {"gemv13": ["gemv.cu"], "gemv2": ["gemv.cu"], "gemm13": ["gemm_ts.cu", "tc.cuh"],
             "gemm2": ["gemm_ts.cu", "tc.cuh"],
             "quantize": ["quantize.cu"], "router": ["router.cu"], "combine": ["combine.cu"],
             "permute": ["permute.cu"], "gather": ["permute.cu"]}.get(kind, [])
    # the code only: comments are stripped and whitespace collapsed, so an edit of a comment keeps a
    # capture valid
    h = hashlib.sha256()
    for f in files + ["common.cuh"]:
        p = os.path.join(ROOT, "int8_expert_weight_b200", "csrc", f)
        if os.path.exists(p):
            src = re.sub(r"/\*.*?\*/", "", open(p).read(), flags=re.S)
            src = re.sub(r"//[^\n]*", "", src)
            h.update(" ".join(src.split()).encode())  # layout-insensitive: whitespace runs count as one
    return h.hexdigest()[:16]


def ncu_traffic(kind, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(f"{kind}@{workload}")
    if not rec or rec.get("source_sha256") != kernel_source_hash(kind):
        return None
    return rec.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks during the timed region
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"jmoe_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[4]), parts[5:]))
            except ValueError:
                continue
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[2] > 0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3][1:5]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(loaded)}


# ------------------------------------------------------------------ CPU oracle (baseline / reference arm)
def oracle_setup(wl, seed_x):
    """Host copies for the oracle: bf16 x, router, and the oracle's own quantization of the weights."""
    import oracle
    x = synth.gen_x(synth_replace(wl, seed=seed_x))
    wr = synth.gen_router(wl) if wl.layer == "moe" else None
    bias = synth.gen_bias(wl)
    qs = {}
    for which in ("w1", "w3", "w2"):
        rows, cols = synth.weight_shape(wl, which)
        q = np.empty((wl.E, rows, cols), np.int8)
        s = np.empty((wl.E, rows), np.float32)
        for e in range(wl.E):
            q[e], s[e] = oracle.quantize(synth.gen_expert(wl, which, e))
        qs[which] = (q, s)
    return x, wr, bias, qs


def synth_replace(wl, **kw):
    import dataclasses
    return dataclasses.replace(wl, **kw)


def oracle_forward(wl, setup, tokens, threads):
    """The oracle's layer (the MoE layer, or the dense MLP for mlp_* workloads) on the listed tokens."""
    import oracle
    x, wr, bias, qs = setup
    if wl.layer == "mlp":
        q1, s1 = qs["w1"]
        q3, s3 = qs["w3"]
        q2, s2 = qs["w2"]
        return oracle.mlp_forward(x, q1[0], s1[0], q3[0], s3[0], q2[0], s2[0], tokens=tokens, threads=threads)
    return oracle.moe_forward(x, wr, bias, *qs["w1"], *qs["w3"], *qs["w2"], tokens=tokens, threads=threads)


def oracle_rate(wl, setup, budget_s, max_tokens=None):
    """Tokens/s of the oracle forward on a bounded sample (tokens spread over the batch), with the
    sampled tokens and the oracle's result on them."""
    import oracle
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    oracle_forward(wl, setup, [0], 1)
    per_token_1t = time.perf_counter() - t0
    n = max(1, min(wl.T, int(budget_s * threads / max(per_token_1t, 1e-9))))
    if max_tokens:
        n = min(n, max_tokens)
    toks = np.linspace(0, wl.T - 1, n).round().astype(np.int64)
    t0 = time.perf_counter()
    ref = oracle_forward(wl, setup, toks, threads)
    dt = time.perf_counter() - t0
    used = min(threads, n)
    return n / dt, used, n, dt, toks, ref


def parity_stats(y_bits, ids, ref):
    """The layer's parity measures on sampled tokens: y_bits bf16 bits [n][d] and ids int32 [n][K]
    (None for the dense MLP) from the GPU, ref the oracle's result on the same tokens.  The bench
    batch is not filtered for near-tied router logits, so a token may legitimately take another
    pair of experts; such tokens are counted and left out of the y measures."""
    y = synth.bf16_bits_to_f32(np.asarray(y_bits, np.uint16)).astype(np.float64)
    r = np.asarray(ref["y"], np.float64)
    same = np.ones(len(r), bool)
    out = {"tokens": int(len(r))}
    if ids is not None and "ids" in ref:
        same = (np.sort(np.asarray(ids), 1) == np.sort(ref["ids"], 1)).all(1)
        out["id_mismatch_tokens"] = int((~same).sum())
    err = np.abs(y[same] - r[same])
    den = np.abs(r[same]).sum()
    out["max_err_rel"] = float((err / (1.0 + np.abs(r[same]))).max()) if err.size else 0.0
    out["mean_rel_err"] = float(err.sum() / den) if den > 0 else 0.0
    out["within_tolerance"] = bool(out["max_err_rel"] <= 2e-2 and out["mean_rel_err"] <= 5e-3)
    return out


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    wl = workload_of(args)
    setup = oracle_setup(wl, wl.seed)
    import oracle
    threads = oracle.default_threads()
    # calibrate one token on one thread, then size every step to fit a few minutes in total
    t0 = time.perf_counter()
    oracle_forward(wl, setup, [0], 1)
    per_tok = time.perf_counter() - t0
    step_budget = min(args.cpu_budget_s, 150.0 / max(1, args.steps + args.warmup))
    n = int(max(1, min(wl.T, step_budget * threads / per_tok)))
    toks = np.linspace(0, wl.T - 1, n).round().astype(np.int64)
    for _ in range(args.warmup):
        oracle_forward(wl, setup, toks, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_forward(wl, setup, toks, threads)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    sample = f"{n} of {wl.T} tokens per step (evenly spaced), full fp64 layer per token"
    out = {
        "metric": METRIC if wl.layer == "moe" else METRIC_MLP, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": run_config(wl, args, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(threads, n), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


def workload_of(args):
    """The named workload, with its token count replaced when --tokens is given."""
    wl = synth.ALL_WORKLOADS[args.workload]
    return synth_replace(wl, T=args.tokens) if args.tokens else wl


def run_config(wl, args, world):
    """The `config` object of both arms' JSON lines (the same keys and values for the same run)."""
    fp8, int8w = args.weights == "fp8", args.weights == "int8"
    par = (f"ep{world}" if getattr(args, "parallel", "replicas") == "ep" else
           f"replicas{world}" if world > 1 else "1gpu")
    return dict(workload_config(wl, args.path), parallelism=par,
                weights=("int8 codes + fp32 per-output-channel scales" if int8w else
                         "E4M3 codes + fp32 per-output-channel scales; E4M3 activations with "
                         "per-row scales (FP8 comparator)" if fp8 else "bf16 (unquantized comparator)"))


def workload_config(wl, path):
    return {"workload": wl.name, "layer": wl.layer, "T": wl.T, "d": wl.d, "ffn": wl.F, "experts": wl.E,
            "top_k": wl.K,
            "weights": "int8 codes + fp32 per-output-channel scales", "activations": "bf16",
            "path": path, "l2": l2_note(wl)}


def l2_note(wl):
    wbytes = 3 * wl.E * wl.d * wl.F
    if wbytes > 126e6:
        return "inputs larger than L2: int8 expert weights %.2f GB > 126 MB L2, no flush" % (wbytes / 1e9)
    return "inputs fit in L2 (%.1f MB): not a roofline workload" % (wbytes / 1e6)


# ------------------------------------------------------------------ multi-rank helpers
def rank_seed(wl, rank):
    """Each rank draws its own batch of tokens (weak scaling); weights use the workload seed."""
    return wl.seed + rank


def max_over_ranks(value, device):
    """The largest value over all ranks (one all-reduce); the value itself with one process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(world, T, steps, max_ms):
    """Whole-job throughput: every rank processed T tokens per step; time = slowest rank."""
    return world * T * steps / (max_ms / 1e3)


# ------------------------------------------------------------------ the CUDA arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    import int8_expert_weight_b200 as jm

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    ep = args.parallel == "ep"
    if world > 1 or ep:
        import datetime
        if world == 1:  # a one-rank group for the expert-parallel path on a single GPU
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(29500 + os.getpid() % 1000))
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    wl = workload_of(args)
    mlp = wl.layer == "mlp"
    if mlp and args.weights != "int8":
        raise SystemExit("the dense MLP workloads run with ExpertsInt8 weights only")
    if ep and (mlp or args.weights != "int8"):
        raise SystemExit("the expert-parallel path runs the MoE layer with ExpertsInt8 weights")
    if ep:
        from int8_expert_weight_b200.ep import CudaSteps, ep_forward, expert_range
        e_first, e_last = expert_range(rank, world)
    else:
        e_first, e_last = 0, wl.E
    T, d, F, E = wl.T, wl.d, wl.F, wl.E
    path = {"auto": jm.PATH_AUTO, "gemv": jm.PATH_GEMV, "gemm": jm.PATH_GEMM}[args.path]
    peaks = load_peaks()

    # ---- inputs: this rank's batch (own seed), replicated weights quantized by the library (load time)
    seed_x = rank_seed(wl, rank)
    x_bits = synth.gen_x(synth_replace(wl, seed=seed_x))
    to_dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev).view(torch.bfloat16)  # noqa
    x = to_dev(x_bits)
    wr = None if mlp else torch.from_numpy(synth.gen_router(wl)).to(dev)
    bias_np = synth.gen_bias(wl)
    bias = None if bias_np is None else torch.from_numpy(bias_np).to(dev)
    int8w = args.weights == "int8"
    fp8 = args.weights == "fp8"
    wbytes = 2 if args.weights == "bf16" else 1
    Q, S, Wb = {}, {}, {}
    q_ms = 0.0
    jm.jamba_moe_timing_start(3)  # the quantize launches (one per matrix), timed by the library's own events
    for which in ("w1", "w3", "w2"):
        rows, cols = synth.weight_shape(wl, which)
        Wb[which] = torch.empty((e_last - e_first, rows, cols), dtype=torch.bfloat16, device=dev)
        for e in range(e_first, e_last):  # drawn expert by expert on the host, to bound host memory
            Wb[which][e - e_first].copy_(to_dev(synth.gen_expert(wl, which, e)))
        if int8w:
            Q[which], S[which] = jm.jamba_moe_quantize(Wb[which])
            del Wb[which]
        elif fp8:
            Q[which], S[which] = jm.jamba_moe_quantize_fp8(Wb[which])
            del Wb[which]
    torch.cuda.synchronize()
    q_ms = jm.jamba_moe_timing_collect().get("quantize", (0.0, 0))[0]
    jm.jamba_moe_timing_start(0)
    q_bytes = algorithmic("quantize", wl, T, 0, 0)[1]
    ws_bytes = (jm.jamba_mlp_workspace_size(T, d, F) if mlp else
                jm.jamba_moe_workspace_size_fp8(T, d, F) if fp8 else jm.jamba_moe_workspace_size(T, d, F))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    ids = torch.empty((T, 2), dtype=torch.int32, device=dev)
    tw = torch.empty((T, 2), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    ep_stats = {}
    ep_steps = CudaSteps(path) if ep else None
    y_ep = [y]

    def forward(xin, y=y):
        if ep:
            y_ep[0], ids_ep, _ = ep_forward(xin, wr, bias, (Q["w1"], S["w1"], Q["w3"], S["w3"], Q["w2"], S["w2"]),
                                            steps=ep_steps, stats=ep_stats)
            ids.copy_(ids_ep)
        elif mlp:
            jm.jamba_mlp_forward(xin, Q["w1"][0], S["w1"][0], Q["w3"][0], S["w3"][0], Q["w2"][0], S["w2"][0], y=y,
                                 workspace=ws, path=path)
        elif int8w:
            jm.jamba_moe_forward(xin, wr, bias, Q["w1"], S["w1"], Q["w3"], S["w3"], Q["w2"], S["w2"], y=y,
                                 topk_ids=ids, topk_w=tw, workspace=ws, path=path)
        elif fp8:
            jm.jamba_moe_forward_fp8(xin, wr, bias, Q["w1"], S["w1"], Q["w3"], S["w3"], Q["w2"], S["w2"], y=y,
                                     topk_ids=ids, topk_w=tw, workspace=ws, path=path)
        else:
            jm.jamba_moe_forward_bf16w(xin, wr, bias, Wb["w1"], Wb["w3"], Wb["w2"], y=y, topk_ids=ids, topk_w=tw,
                                       workspace=ws, path=path)

    def step():
        forward(x)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    def read_status():
        if ep:  # the expert-parallel calls keep their own workspaces: the worse of the two
            return max(ep_steps.dispatch_status(), ep_steps.experts_status())
        return jm.jamba_moe_read_device_status(ws)

    # JMOE_OK = 0 after each pass (none read before any call has run)
    status = {"warmup": read_status() if args.warmup > 0 else None}

    # ---- timed region: K forward steps on resident inputs.  A CUDA event recorded between two
    # launches ends their programmatic overlap, so the per-kernel durations come from a second,
    # identical pass of K steps with the library's per-launch events on the launching stream.
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed_pass(per_kernel):
        if per_kernel:
            jm.jamba_moe_timing_start(args.steps * 16)
        barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        kern = None
        if per_kernel:
            kern = jm.jamba_moe_timing_collect()
            jm.jamba_moe_timing_start(0)
        return ev0.elapsed_time(ev1), kern

    with ClockSampler(local_rank) as clk:
        ms_plain, _ = timed_pass(False)
        ms_events, kernels = timed_pass(True)
    status["timed"] = read_status()
    T_work = T  # tokens whose assignments this rank's expert kernels process
    if ep:
        # this rank's kernels work on the rows it received, one assignment each
        counts = np.bincount(ep_stats["recv_expert"].cpu().numpy(), minlength=E)
        touched = int((counts > 0).sum())
        T_work = sum(ep_stats["recv_counts"]) / wl.K
    else:
        ids_np = np.zeros((T, 1), np.int32) if mlp else ids.cpu().numpy()
        touched = int(np.unique(ids_np).size)
        counts = np.bincount(ids_np.reshape(-1), minlength=E)
    rows_padded = int(sum((c + 127) // 128 * 128 for c in counts))
    ms = max_over_ranks(ms_plain, dev)
    ms_events = max_over_ranks(ms_events, dev)
    value = aggregate_tokens_per_s(world, T, args.steps, ms)

    # ---- end to end through the public call with host buffers: pinned x in, pinned y out.  Every
    # step copies its x from pinned host memory and its y back; the copies run on their own
    # streams (one per direction) with two device buffers, so step i+1's input copy and step i-1's
    # output copy overlap step i's layer, as a serving loop would.  The expert-parallel path keeps
    # the plain sequential loop (its outputs are allocated by the exchange).
    x_host = torch.empty((T, d), dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(x.cpu())
    y_host = torch.empty((T, d), dtype=torch.bfloat16, pin_memory=True)
    x_dev = [torch.empty_like(x) for _ in range(2)]
    y_dev = [y, torch.empty_like(y)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n):
        """n steps; ends with the compute stream waiting for the last output copy."""
        for i in range(n):
            b = i & 1
            if ep:
                x_dev[0].copy_(x_host, non_blocking=True)
                forward(x_dev[0])
                y_host.copy_(y_ep[0], non_blocking=True)
                continue
            if i == 0:
                s_in.wait_stream(stream)  # the first copy starts after the timing event
            elif i >= 2:
                s_in.wait_event(ev_done[b])  # step i-2's layer has read x_dev[b]
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # step i-2's output copy has left y_dev[b]
            forward(x_dev[b], y_dev[b])
            ev_done[b].record(stream)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                y_host.copy_(y_dev[b], non_blocking=True)
                ev_out[b].record(s_out)
        if not ep and n > 0:
            stream.wait_event(ev_out[(n - 1) & 1])

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    barrier()
    ev0.record(stream)
    e2e_steps(args.steps)
    ev1.record(stream)
    torch.cuda.synchronize()
    status["e2e"] = read_status()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    e2e_value = aggregate_tokens_per_s(world, T, args.steps, e2e_ms)

    # ---- roofline of the dominant kernel
    dom = max(kernels, key=lambda k: kernels[k][0])
    dom_ms, dom_n = kernels[dom]
    unit_kind, work = algorithmic(dom, wl, T_work, touched, rows_padded, wbytes)
    avg_s = dom_ms / dom_n / 1e3
    if unit_kind == "bytes":
        achieved, peak, unit, bound = work / avg_s / 1e9, peaks["hbm_gbs"], "GB/s", "hbm"
    else:
        # the burst bf16 peak (each kernel is timed alone by its own events); FP8 MMAs: the measured
        # bf16 peak times the nominal fp8 / bf16 ratio (4.5 / 2.25)
        achieved, peak, unit, bound = (work / avg_s / 1e12, peaks["bf16_tflops"] * (2.0 if fp8 else 1.0),
                                       "TFLOP/s", "tensor")
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": ncu_traffic(dom, wl.name) if args.weights == "int8" else None, "kernel": dom,
                "algorithmic_per_launch": work,
                "peak_source": peaks["source"] + (" burst" if bound == "tensor" else "") +
                               (" bf16 x 2 (nominal fp8/bf16 ratio)" if fp8 and bound == "tensor" else "")}
    if bound == "tensor":
        sus = peaks["bf16_tflops_sustained"] * (2.0 if fp8 else 1.0)
        roofline["peak_sustained"] = sus
        roofline["frac_of_sustained"] = achieved / sus
    clocks = clk.summary()
    if clocks.get("sm_mhz"):
        # the same rate per SM clock: comparable across runs that ran at different clocks
        roofline["achieved_per_sm_mhz"] = achieved / clocks["sm_mhz"]
    per_kernel = {}
    for k, (kms, n) in sorted(kernels.items(), key=lambda kv: -kv[1][0]):
        uk, wk = algorithmic(k, wl, T_work, touched, rows_padded, wbytes)
        a = wk / (kms / n / 1e3)
        per_kernel[k] = {"launches": n, "avg_us": kms / n * 1e3,
                         ("GB/s" if uk == "bytes" else "TFLOP/s"): a / (1e9 if uk == "bytes" else 1e12)}

    cpu = parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and int8w:
        setup = oracle_setup(wl, seed_x)
        rate, cores, n, dt, toks, ref = oracle_rate(wl, setup, args.cpu_budget_s)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{n} of {wl.T} tokens (evenly spaced) of the same batch, fp64, {dt:.1f} s"}
        try:  # the last forward's output on the oracle's sample: a record, never a reason to fail the run
            y_bits = (y_ep[0] if ep else y).view(torch.int16).cpu().numpy().view(np.uint16)[toks]
            parity = parity_stats(y_bits, None if mlp else ids.cpu().numpy()[toks], ref)
        except Exception as ex:  # noqa: BLE001
            parity = {"error": repr(ex)[:200]}

    if rank == 0:
        out = {
            "metric": METRIC_MLP if mlp else METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16", "data": "synthetic",
            "config": run_config(wl, args, world),
            "roofline": roofline, "cpu_baseline": cpu, "parity_on_sample": parity,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": T * d * 2,
                    "d2h_bytes_per_step": T * d * 2},
            "gpu_launches": int(sum(n for _, n in kernels.values())),
            "ms_per_step_with_kernel_events": ms_events / args.steps,
            "clocks": clocks, "kernels": per_kernel, "device_status": status,
            "routing": {"touched_experts": touched, "max_tokens_per_expert": int(counts.max())},
            "quantize": ({"ms": q_ms, "GB/s": q_bytes / (q_ms / 1e3) / 1e9,
                          "frac_of_hbm": q_bytes / (q_ms / 1e3) / 1e9 / peaks["hbm_gbs"]} if q_ms > 0 else None),
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()
    bad = {k: v for k, v in status.items() if v}
    if bad:  # a bounded wait ran out or a kernel skipped a bad index: the numbers above are void
        print(f"rank {rank}: device status {bad} ({jm.jamba_moe_status_string(max(bad.values()))})", file=sys.stderr)
        return 3
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
