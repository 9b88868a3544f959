#!/usr/bin/env python
"""Benchmark of the fine-grained MoE expert layer on B200.

One step = the whole path on one batch: routing (router logits, softmax, top-K,
permutation), forward (up-proj + SwiGLU, down-proj, aggregation) and backward
(dH + dS, dW2, dX~, dW1, router backward, dX aggregation), all through the
library's C ABI.  Default workload: the DeepSeek-V3-shaped layer, T=8192
tokens, d=7168, E=256, n=2048, top-8, Zipf(1.1) expert popularity -- the
largest of the workloads that fits one GPU; --config NAME runs another.
Synthetic seeded inputs (workloads package).  Multi-GPU: one process per GPU
(torchrun), each with its own batch (weak scaling); the weight gradients are
all-reduced over NCCL as the data-parallel exchange step.

Prints one JSON line on rank 0.  --impl reference times the fp64 CPU oracle on
a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd+bwd TFLOP/s (bf16) and % of B200 tensor peak; tokens/sec"
WORKLOADS = {
    "dsv3": ("DeepSeek-V3-shaped MoE layer fwd+bwd: T=8192, d=7168, E=256, n=2048, top-8, SwiGLU, "
             "Zipf(1.1) expert popularity (router bias -1.1 ln rank)"),
    "7b": ("fine-grained 7B-class MoE layer fwd+bwd: T=16384, d=1536, E=128, n=256, top-8, SwiGLU, "
           "skewed router (bias ~N(0,0.5))"),
    "qwen3": ("Qwen3-MoE-shaped layer fwd+bwd: T=32768, d=2048, E=128, n=768, top-8, SwiGLU, balanced router"),
    "olmoe": ("OLMoE-shaped layer fwd+bwd: T=32768, d=2048, E=64, n=1024, top-8, SwiGLU, balanced router"),
    "tiny": ("tiny MoE layer fwd+bwd: T=512, d=128, E=16, n=64, top-2, SwiGLU"),
}
# a timed region at least this long runs under the power cap: its roofline
# uses the sustained tensor peak; a shorter one uses the burst peak
SUSTAINED_WINDOW_S = 2.0


def workload_text(name, cfg):
    if name in WORKLOADS:
        return WORKLOADS[name]
    return (f"{name} MoE layer fwd+bwd: T={cfg.T}, d={cfg.d}, E={cfg.E}, n={cfg.n}, top-{cfg.K}, SwiGLU, "
            f"router bias {cfg.bias}, rounding mode {cfg.round_mode}")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="dsv3",
                    help="workload (default: the DeepSeek-V3-shaped layer, the largest that fits one GPU)")
    ap.add_argument("--cpu-sample-tokens", type=int, default=None,
                    help="tokens of the CPU oracle's sample (default: about 10 s of fp64 work)")
    ap.add_argument("--cpu-min-seconds", type=float, default=10.0,
                    help="repeat the oracle step on the sample until this much CPU time has run (at most 4 times)")
    ap.add_argument("--ref-sample-tokens", type=int, default=None,
                    help="tokens per reference-arm step (default: about 1 s of fp64 work)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--parallel", default="dp", choices=["dp", "ep"],
                    help="dp: every rank holds all experts and its own tokens, weight gradients all-reduced; "
                         "ep: rank r holds experts [rE/N, (r+1)E/N), routed rows exchanged by all-to-all")
    ap.add_argument("--mxfp8-forward", action="store_true",
                    help="forward GEMMs on MXFP8 operands (moe_forward_mxfp8); backward unchanged")
    ap.add_argument("--comm-sms", type=int, default=16,
                    help="N>1: SMs left to NCCL while the gradient all-reduces overlap the backward "
                         "(0: all-reduce after the step, no overlap)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- algorithmic work per kernel
def kernel_work(cfg, R):
    """Algorithmic FLOPs and HBM bytes of one launch of each kernel (R = routed
    pairs T*K; bf16 = 2 bytes).  Bytes assume every operand is read once."""
    T, d, E, n = cfg.T, cfg.d, cfg.E, cfg.n
    w = {
        "up_proj_gemm": (4 * R * d * n, 2 * T * d + 4 * E * d * n + 6 * R * n),
        "down_proj_gemm": (2 * R * d * n, 2 * R * n + 2 * E * d * n + 2 * R * d),
        "dh_gemm": (2 * R * d * n, 2 * T * d + 2 * E * d * n + 10 * R * n + 4 * R),
        "dw2_gemm": (2 * R * d * n, 2 * R * n + 2 * T * d + 2 * E * d * n),
        # dX~ with the router path dz * Wr^T added in its epilogue
        "dxt_gemm": (4 * R * d * n + 2 * R * d, 4 * R * n + 4 * E * d * n + 2 * R * d + 4 * E * d + 8 * R),
        "dw1_gemm": (4 * R * d * n, 2 * T * d + 4 * R * n + 4 * E * d * n),
        "aggregate_fwd": (2 * R * d, 2 * R * d + 2 * T * d + 8 * R),
        "aggregate_bwd": (R * d, 2 * R * d + 2 * T * d + 4 * R + 4 * T),
        "router_logits_gemm": (2 * T * d * E, 2 * T * d + 4 * d * E + 4 * T * E),
        "router_dwr_gemm": (2 * T * d * E, 2 * T * d + 4 * T * E + 4 * d * E),
        # MXFP8 forward: 1-byte codes plus one scale byte per 32
        "up_proj_gemm_mx": (4 * R * d * n, T * d * 33 // 32 + 2 * E * d * n * 33 // 32 + 4 * R * n + R * n * 33 // 32),
        "down_proj_gemm_mx": (2 * R * d * n, R * n * 33 // 32 + E * d * n * 33 // 32 + 2 * R * d),
        "mx_quant_x": (0, 2 * T * d + T * d * 33 // 32),
        # W1 and W2 read (bf16), codes and their scale tiles written
        "mx_quant_w": (0, 6 * E * d * n + 3 * E * d * n * 33 // 32),
    }
    return w


def source_digest():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fine_grained_mixture_top_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel, workload_key):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    if there is none for this kernel and workload or the sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        data = json.load(f)
    rec = data.get(f"{kernel}@{workload_key}") or data.get(kernel)  # one record per kernel and workload
    if not rec or rec.get("src_digest") != source_digest() or rec.get("workload") != workload_key:
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle (baseline / reference arm)
# fp64 bytes per expert the oracle holds: W1[e], W2[e] and their gradients
def _expert_f64_bytes(cfg):
    return 8 * 6 * cfg.d * cfg.n


def oracle_sample_plan(cfg, X, Wr, bias, tokens, budget_bytes=8 << 30):
    """The bounded sample the CPU oracle runs: the first `tokens` tokens, and
    the experts their pairs go to, most-loaded first, as many as fit
    `budget_bytes` of fp64 weights and weight gradients (all of them on the
    smaller layers).  Returns the expert ids."""
    import numpy as np
    from oracle import moe_oracle as orc
    rt = orc.route(X[:tokens].double().numpy(), Wr.double().numpy(),
                   None if bias is None else bias.double().numpy(), cfg.K)
    counts = np.bincount(rt["pair_expert"], minlength=cfg.E)
    cap = max(1, budget_bytes // _expert_f64_bytes(cfg))
    used = [int(e) for e in np.argsort(-counts, kind="stable") if counts[e] > 0]
    return sorted(used[:cap])


def oracle_sample_step(cfg, smp):
    """One step of the fp64 oracle (as it stands) on the sample `smp`: route
    the sample's tokens over all E experts, keep the pairs that go to the
    sample's experts (all pairs when every expert is in it), then forward and
    backward with the router path.  Returns (seconds, pairs, threads)."""
    import numpy as np
    from oracle import moe_oracle as orc
    X, dO, Wr, b, W1, W2, S = (smp[k] for k in ("X", "dO", "Wr", "bias", "W1", "W2", "experts"))
    t0 = time.perf_counter()
    rt = orc.route(X, Wr, b, cfg.K)
    if len(S) == cfg.E:
        sub, Wr_s = rt, Wr
    else:
        remap = -np.ones(cfg.E, np.int64)
        remap[S] = np.arange(len(S))
        keep = remap[rt["pair_expert"]] >= 0
        pair_tok = np.repeat(np.arange(X.shape[0]), np.diff(rt["tok_ptr"]))
        tok_ptr = np.concatenate([[0], np.cumsum(np.bincount(pair_tok[keep], minlength=X.shape[0]))])
        sub = {"z": rt["z"][:, S], "probs": rt["probs"][:, S], "topk_idx": rt["topk_idx"], "tok_ptr": tok_ptr,
               "pair_expert": remap[rt["pair_expert"][keep]], "pair_gate": rt["pair_gate"][keep]}
        Wr_s = Wr[:, S]
    fw = orc.forward(X, Wr_s, None, W1, W2, cfg.K, routing=sub)
    orc.backward(fw, dO, X, Wr_s, W1, W2)
    dt = time.perf_counter() - t0
    return dt, int(sub["tok_ptr"][-1]), blas_threads()


def oracle_sample(cfg, inp, tokens, experts):
    """Host fp64 copies of the sample's tensors (`inp` may live on any device;
    W1/W2 either full or already restricted to `experts`)."""
    def f64(t):
        return t.detach().to("cpu").double().numpy()
    full = inp["W1"].shape[0] == cfg.E
    idx = experts if full else list(range(len(experts)))
    import torch
    sel = torch.as_tensor(idx, device=inp["W1"].device)
    return {"X": f64(inp["X"][:tokens]), "dO": f64(inp["dO"][:tokens]), "Wr": f64(inp["Wr"]),
            "bias": None if inp["bias"] is None else f64(inp["bias"]),
            "W1": f64(inp["W1"].index_select(0, sel)), "W2": f64(inp["W2"].index_select(0, sel)),
            "experts": list(experts)}


def default_sample_tokens(cfg, seconds):
    """Tokens whose fp64 forward + backward (18 K d n flops each) take about
    `seconds` at 0.15 TFLOP/s, the oracle's rate on a 16-thread host; at
    least 16, a multiple of 16."""
    per_tok = 18.0 * cfg.K * cfg.d * cfg.n
    return int(max(16, min(cfg.T, seconds * 0.15e12 / per_tok)) // 16 * 16)


def sample_text(cfg, tokens, experts, pairs):
    if len(experts) == cfg.E:
        return f"first {tokens} of {cfg.T} tokens of the batch with all {cfg.E} experts ({pairs} routed pairs)"
    return (f"first {tokens} of {cfg.T} tokens of the batch, routed over all {cfg.E} experts; the {pairs} "
            f"pairs that go to the {len(experts)} experts most loaded by them (the fp64 weights of all "
            f"{cfg.E} would not fit the host), same per-pair work")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from workloads import CONFIGS, make_inputs
    cfg = CONFIGS[args.config]
    tokens = min(args.ref_sample_tokens or default_sample_tokens(cfg, 1.0), cfg.T)
    base = make_inputs(cfg, "cpu", experts=[])
    experts = oracle_sample_plan(cfg, base["X"], base["Wr"], base["bias"], tokens)
    inp = make_inputs(cfg, "cpu", experts=experts)
    smp = oracle_sample(cfg, inp, tokens, experts)
    pairs = 0
    for _ in range(args.warmup):
        oracle_sample_step(cfg, smp)
    times = []
    threads = 1
    for _ in range(args.steps):
        dt, pairs, threads = oracle_sample_step(cfg, smp)
        times.append(dt)
    tot = sum(times)
    flops = 6 * 3 * pairs * cfg.d * cfg.n
    value = flops * args.steps / tot / 1e12
    sample = sample_text(cfg, tokens, experts, pairs) + " per step, fp64 numpy oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_text(args.config, cfg), "T": cfg.T, "d": cfg.d, "E": cfg.E, "n": cfg.n,
                   "K": cfg.K, "parallelism": "single host process"},
        "tokens_per_s": pairs / cfg.K * args.steps / tot,
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


# ---------------------------------------------------------------- GPU arm
def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    from fine_grained_mixture_top_b200 import moe
    from workloads import CONFIGS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    overlap = world > 1 and args.comm_sms > 0
    if overlap:  # NCCL reads this when its communicator is created
        os.environ.setdefault("NCCL_MAX_CTAS", str(args.comm_sms))
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    cfg = CONFIGS[args.config]
    workload = workload_text(args.config, cfg)
    inp = make_inputs(cfg, dev, rank=rank)
    layer = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, round_mode=cfg.round_mode, router_grad=1,
                         seed=cfg.seed, device=dev)
    X, Wr, b, W1, W2, dO = (inp[k] for k in ("X", "Wr", "bias", "W1", "W2", "dO"))
    layer.mxfp8 = args.mxfp8_forward
    if args.mxfp8_forward:
        workload += "; forward GEMMs on MXFP8 operands (E4M3, E8M0 scale per 32 along K)"
    stream = torch.cuda.current_stream()
    ep = None
    if args.parallel == "ep":
        if args.mxfp8_forward:
            raise SystemExit("--parallel ep runs the bf16 forward")
        if world == 1:  # the all-to-alls still need a (one-rank) group
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(_free_port()))
            dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=180),
                                    device_id=dev)
        from fine_grained_mixture_top_b200.ep import CudaEngine, ExpertParallelMoE
        E_loc = cfg.E // world
        W1 = W1[rank * E_loc:(rank + 1) * E_loc].contiguous()
        W2 = W2[rank * E_loc:(rank + 1) * E_loc].contiguous()
        eng = CudaEngine(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, world, device=dev, seed=cfg.seed,
                         round_mode=cfg.round_mode)
        ep = ExpertParallelMoE(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, eng)
        layer = eng  # routing statistics below
        overlap = False
        workload += f"; expert parallel over {world} rank(s), {E_loc} experts each, all-to-all of routed rows"
    if overlap:
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        moe.moe_set_sm_budget(sms - args.comm_sms)
        reducer = moe.OverlappedGradReduce(layer)

    def step():
        if ep is not None:
            ep.forward(X, Wr, b, W1, W2)
            ep.backward(dO, X, Wr, W1, W2)
            return
        if overlap:
            reducer.step(X, Wr, b, W1, W2, dO)
            return
        layer.step(X, Wr, b, W1, W2, dO)
        if world > 1:
            for g in (layer.dW1, layer.dW2, layer.dWr):
                dist.all_reduce(g)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    code, where = moe.moe_get_status()
    if code != 0:
        raise RuntimeError(f"device status {moe.status_str(code)} at {where}")
    R = int(layer.routing["tok_ptr"][cfg.T].item())
    counts = layer.routing["counts"].cpu().tolist()

    # ---- breakdown pass (outside the timed region): every launch bracketed
    # by CUDA events on its stream, to find the dominant kernel and the launch
    # count of a step.  Bracketing every launch costs about 0.2 ms per step, so
    # the timed region below brackets only the dominant kernel.
    n_breakdown = 3
    moe.moe_profile_select(None)
    moe.moe_profile_enable(True)
    for _ in range(n_breakdown):
        step()
    torch.cuda.synchronize()
    moe.moe_profile_enable(False)
    recs_all = moe.moe_profile_records()
    launches_per_step = len(recs_all) // n_breakdown
    per = {}
    for name, t in recs_all:
        per.setdefault(name, []).append(t)
    # the dominant kernel among those whose algorithmic work is known (the
    # roofline needs it); every kernel still appears in the breakdown
    work0 = kernel_work(cfg, R)
    dom = max((k for k in per if k in work0), key=lambda k: sum(per[k]))

    # ---- device-timed region
    vis = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    smi_index = vis[local_rank].strip() if local_rank < len(vis) and vis[local_rank].strip().isdigit() else local_rank
    sampler = ClockSampler(smi_index)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.2)
    moe.moe_profile_select(dom)
    moe.moe_profile_enable(True)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    moe.moe_profile_enable(False)
    moe.moe_profile_select(None)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    ms_t = torch.tensor([ms], device=dev)
    if world > 1:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())
    recs_dom = moe.moe_profile_records()
    code, where = moe.moe_get_status()
    if code != 0:
        raise RuntimeError(f"device status {moe.status_str(code)} at {where}")

    flops_step = 18 * cfg.T * cfg.K * cfg.d * cfg.n
    ms_step = ms_max / args.steps
    value = flops_step * world / (ms_step * 1e-3) / 1e12

    # ---- per-kernel breakdown (breakdown pass) and the dominant kernel's
    # roofline (its launches inside the timed region)
    peaks, peak_src = load_peaks()
    work = kernel_work(cfg, R)
    step_bd = sum(t for _, t in recs_all) / n_breakdown
    breakdown = {}
    for name, ts in per.items():
        avg = sum(ts) / len(ts)
        entry = {"launches_per_step": len(ts) // n_breakdown, "avg_us": round(1e3 * avg, 2),
                 "share": round(sum(ts) / n_breakdown / max(step_bd, 1e-9), 4)}
        if name in work:
            fl, by = work[name]
            entry["tflops"] = round(fl / (avg * 1e-3) / 1e12, 1)
            entry["gbs"] = round(by / (avg * 1e-3) / 1e9, 1)
        breakdown[name] = entry
    # forward / backward split of the breakdown pass (routing counted apart)
    fwd_k = {"up_proj_gemm", "down_proj_gemm", "aggregate_fwd", "up_proj_gemm_mx", "down_proj_gemm_mx",
             "mx_quant_x", "mx_quant_w"}
    route_us = fwd_us = bwd_us = 0.0
    for name, ts in per.items():
        us = 1e3 * sum(ts) / n_breakdown
        if name.startswith(("router_split", "router_logits", "router_softmax", "permute_", "round_")):
            route_us += us
        elif name in fwd_k:
            fwd_us += us
        else:
            bwd_us += us
    fl_tok = cfg.T * cfg.K * cfg.d * cfg.n
    phases = {"route_us": round(route_us, 1), "fwd_us": round(fwd_us, 1), "bwd_us": round(bwd_us, 1),
              "fwd_tflops": round(6 * fl_tok / (fwd_us * 1e-6) / 1e12, 1),
              "bwd_tflops": round(12 * fl_tok / (bwd_us * 1e-6) / 1e12, 1),
              "note": "sums of the breakdown pass's kernel times; fwd = up-proj, down-proj, aggregation; "
                      "route = router logits/softmax/top-K, permutation and token rounding"}
    dom_times = [t for n, t in recs_dom if n == dom]
    avg_dom = sum(dom_times) / len(dom_times)
    fl, by = work.get(dom, (0, 0))
    intensity = fl / max(by, 1)
    # The tensor peak that applies: the burst figure for a timed region
    # shorter than SUSTAINED_WINDOW_S (the clocks have not settled under the
    # power cap yet), the sustained one for a longer region.
    window_s = ms_max * 1e-3
    sustained = window_s >= SUSTAINED_WINDOW_S
    tensor_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    ridge = tensor_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if intensity >= ridge:
        achieved = fl / (avg_dom * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tensor_peak, "unit": "TFLOP/s"}
        roof["frac"] = round(achieved / tensor_peak, 4)
        roof["frac_of_burst"] = round(achieved / peaks["bf16_tflops"], 4)
        roof["frac_of_sustained"] = round(achieved / peaks["bf16_tflops_sustained"], 4)
    else:
        achieved = by / (avg_dom * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        roof["frac"] = round(achieved / peaks["hbm_gbs"], 4)
    roof["kernel"] = dom
    roof["peak_source"] = (f"{peak_src} " + (("sustained bf16" if sustained else "burst bf16") +
                                             f" (timed region {window_s:.2f} s)"
                                             if roof["bound"] == "tensor" else "copy bandwidth"))
    roof["traffic"] = measured_traffic(dom, args.config)

    # ---- end-to-end through the public API with host buffers: every step
    # copies its X and dO from pinned host memory and its per-token outputs O
    # and dX back to pinned host memory (HostFedRunner overlaps those copies
    # with the kernels)
    e2e = None
    if not args.no_e2e:
        Xh = X.cpu().pin_memory()
        dOh = dO.cpu().pin_memory()
        Oh = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory()
        dXh = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory()
        if ep is None:
            runner = moe.HostFedRunner(layer)

            def e2e_step():
                runner.step(Xh, dOh, Oh, Wr, b, W1, W2, dXh=dXh)
                if world > 1:
                    for g in (layer.dW1, layer.dW2, layer.dWr):
                        dist.all_reduce(g)
        else:
            class _Copies:  # host copies in line with the expert-parallel step
                def finish(self):
                    pass
            runner = _Copies()

            def e2e_step():
                X.copy_(Xh, non_blocking=True)
                dO.copy_(dOh, non_blocking=True)
                Oh.copy_(ep.forward(X, Wr, b, W1, W2), non_blocking=True)
                dXh.copy_(ep.backward(dO, X, Wr, W1, W2)[0], non_blocking=True)

        for _ in range(3):
            e2e_step()
        runner.finish()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        runner.finish()
        e1.record(stream)
        torch.cuda.synchronize()
        ems = torch.tensor([e0.elapsed_time(e1)], device=dev)
        if world > 1:
            dist.all_reduce(ems, op=dist.ReduceOp.MAX)
        e_ms_step = float(ems.item()) / args.steps
        e2e = {"value": round(flops_step * world / (e_ms_step * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(Xh.numel() * 2 + dOh.numel() * 2),
               "d2h_bytes_per_step": int(Oh.numel() * 2 + dXh.numel() * 2), "ms_per_step": round(e_ms_step, 4),
               "api": "HostFedRunner.step (pinned host X, dO in; O, dX out)"}

    # ---- CPU baseline: the oracle on a bounded sample of the same batch
    # (the device's own input bytes), rank 0 at N=1 only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tokens = min(args.cpu_sample_tokens or default_sample_tokens(cfg, args.cpu_min_seconds), cfg.T)
        experts = oracle_sample_plan(cfg, X.cpu(), Wr.cpu(), None if b is None else b.cpu(), tokens)
        smp = oracle_sample(cfg, inp, tokens, experts)
        dt, reps, fl = 0.0, 0, 0
        while reps < 4 and (reps == 0 or dt < args.cpu_min_seconds):
            step_s, pairs, threads = oracle_sample_step(cfg, smp)
            dt += step_s
            fl += 18 * pairs * cfg.d * cfg.n
            reps += 1
        del smp
        cpu = {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s",
               "cores": threads, "kind": "oracle", "seconds": round(dt, 2),
               "sample": sample_text(cfg, tokens, experts, pairs) + f", {reps} x route+forward+backward of the "
                         "fp64 numpy oracle"}

    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16+mxfp8" if args.mxfp8_forward else "bf16", "data": "synthetic",
            "config": {"workload": workload, "T": cfg.T, "d": cfg.d, "E": cfg.E, "n": cfg.n, "K": cfg.K,
                       "router_bias": cfg.bias, "round_mode": cfg.round_mode,
                       "parallelism": (f"ep{world} (NCCL all-to-all of routed rows and dS, all-reduce of dWr)"
                                       if ep is not None else
                                       f"dp{world}" + ((" (NCCL all-reduce of dW2, dW1, dWr overlapping the backward, "
                                                        f"{args.comm_sms} SMs left to NCCL)") if overlap else
                                                       (" (NCCL all-reduce of dW1, dW2, dWr)" if world > 1 else ""))),
                       "l2": "inputs larger than L2 (%d MB of X, dO, W1, W2 per step)" % (
                           (4 * cfg.T * cfg.d + 6 * cfg.E * cfg.d * cfg.n) // 2**20)},
            "tokens_per_s": round(cfg.T * world / (ms_step * 1e-3), 1),
            "pct_of_tensor_peak": round(100 * value / world / tensor_peak, 2),
            "roofline": roof,
            "phases": phases,
            "kernels": breakdown,
            "kernels_note": (f"per-kernel CUDA events from {n_breakdown} steps with every launch bracketed, run "
                             "before the timed region; the timed region brackets only the dominant kernel"),
            "gpu_launches": launches_per_step * args.steps,
            "routed_pairs": R,
            "expert_load": {"min": min(counts), "max": max(counts), "mean": sum(counts) / len(counts)},
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
