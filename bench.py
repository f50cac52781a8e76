#!/usr/bin/env python
"""Throughput of one mHC layer, forward + backward, on B200.

A step is one pass of the whole hot path over one batch of synthetic tokens:
  mhc_pre -> mhc_post (with a supplied f_out standing in for F's output) ->
  mhc_backward_map -> mhc_backward_apply
``--forward fused`` times one layer of a deep stack in steady state instead:
  mhc_layer_input -> mhc_post_fused (x_next and the next layer's maps) ->
  mhc_backward_map -> mhc_backward_apply
(the layer's own maps then come from one mhc_pre before timing).  Both run at
T = 16384 tokens per GPU, n = 4 streams, C = 7168 channels, bf16
activations, Sinkhorn t_max = 20.  Under torchrun each rank runs its own
16384 tokens (data parallel over tokens, weak scaling) and the step ends with
the one exchange the backward has: an all-reduce of grad_phi / grad_b /
grad_alpha (2.75 MB).

Timing: W warm-up steps, then exactly K steps between a barrier +
synchronize on each side, CUDA events on the launching stream, max over
ranks.  Every input tensor (x, grad_x_next: 940 MB each) is larger than the
126 MB L2, so no flush is needed between steps.  CUDA events recorded
between the calls give each call's device time; the roofline line is taken
for the longest single-kernel call.

``--impl reference`` times the fp64 CPU oracle (the reference arm of this
library) on a bounded sample of the same workload instead.

Two more workloads print their own line (the default line is the layer's):
``--workload sinkhorn``: the standalone batched Sinkhorn-Knopp on 2^22
matrices for n = 4, 8, 16 (20 iterations) and the depth-product Amax gain
over L = 64 layers of 2^16 tokens; ``--workload depth``: a 24-layer stack
(T = 65536 tokens per GPU, n = 4, C = 7168, F_l(h) = s_l h) forward and
backward through ``DepthStack`` with block recompute.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mHC layer tokens/s (fwd+bwd, n=4, C=7168) and achieved HBM GB/s vs B200 peak"
T_TOK, N_STR, C_CH, T_MAX = 16384, 4, 7168, 20
SINKHORN_METRIC = ("batched Sinkhorn-Knopp matrices/s (2^22 matrices each for n=4,8,16, "
                   "20 iterations)")
DEPTH_METRIC = "mHC depth-stack tokens/s (24 layers fwd+bwd with recompute, n=4, C=7168)"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, the spec figure


def layer_metric(n: int) -> str:
    """The layer line's metric for n streams."""
    return METRIC if n == N_STR else METRIC.replace("n=4", f"n={n}")


def per_token_bytes(n=N_STR, C=C_CH, act=2):
    """Algorithmic bytes per token of each call (bf16 activations, fp32 maps)."""
    M = n * n + 2 * n
    nC = n * C
    coef = ((n * n + 2 * n + M + 1) + 3) // 4 * 4 * 4  # per-token record of the split backward
    return {
        "pre": nC * act + C * act + 4 * (2 * n + n * n),                  # x in; h_in, H out
        "post": nC * act + C * act + 4 * (n + n * n) + nC * act,           # x, f, H in; x_next out
        "layer_input": nC * act + C * act + 4 * n,                         # x, H_pre in; h_in out
        "post_fused": nC * act + C * act + 4 * (n + n * n) + nC * act + 4 * (2 * n + n * n),
        # x, G, g, f in; records out
        "bwd_map": 2 * nC * act + 2 * C * act + coef,
        # x, G, g, records in; grads out
        "bwd_apply": 2 * nC * act + C * act + coef + nC * act + C * act,
        # one pass: x, G, g, f in; grads out
        "bwd_min": 2 * nC * act + 2 * C * act + nC * act + C * act,
    }


def per_call_param_bytes(n=N_STR, C=C_CH):
    K, M = n * C, n * n + 2 * n
    phi = K * M * 4
    return {"pre": phi, "post": 0, "layer_input": 0, "post_fused": phi, "bwd_map": phi,
            "bwd_apply": 2 * phi}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha(files):
    h = hashlib.sha256()
    for f in files:
        path = os.path.join(ROOT, "manifold_constrained_hyper_token_b200", "csrc", f)
        with open(path, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# kernels behind each single-kernel call, for matching ncu traffic to sources
# (keys: the call at n = 4; "<call>_n8" at n = 8)
CALL_SOURCES = {
    "post": ["k_post.cu", "mhc_common.cuh"],
    "bwd_map": ["k_map_tc.cu", "tc_sm100.cuh", "mhc_common.cuh"],
    "bwd_apply": ["k_apply_tc.cu", "tc_sm100.cuh", "mhc_common.cuh"],
    "pre": ["k_map_tc.cu", "k_post.cu", "tc_sm100.cuh", "mhc_common.cuh"],
    "layer_input": ["k_post.cu", "mhc_common.cuh"],
    "post_fused": ["k_map_tc.cu", "tc_sm100.cuh", "mhc_common.cuh"],
    "post_n8": ["k_post.cu", "mhc_common.cuh"],
    "layer_input_n8": ["k_post.cu", "mhc_common.cuh"],
}


def traffic_key(call, n):
    return call if n == N_STR else "%s_n%d" % (call, n)


def ncu_traffic(key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of that kernel; else None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[key]
        if e.get("source_sha") != kernel_source_sha(CALL_SOURCES[key]):
            return None
        return float(e["bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for k, v in zip(names, r[5:9]):
                if v.strip().lower().startswith("active"):
                    reasons.add(k)
        sm.sort()
        med = sm[len(sm) // 2] if sm else None
        return {"sm_mhz": med, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def oracle_layer_pass(n: int = N_STR, seed: int = 0, pool: int = 0):
    """One timed pass of the fp64 oracle over the layer: pre + post + backward on
    the first S tokens of the seeded workload with n streams.  Returns
    run(S) -> seconds (the inputs are drawn before the clock starts).  With
    pool > 0 the tokens come from one pool of that many, drawn once."""
    import torch

    import oracle
    from manifold_constrained_hyper_token_b200 import synth

    params = synth.layer_params(n, C_CH, seed)
    alpha = float(params["alpha"][0])
    held = synth.activations(pool, n, C_CH, seed, torch.bfloat16, backward=True) if pool else None

    def run(S):
        if held is not None:
            d = {k: v[:S] for k, v in held.items()}
        else:
            d = synth.activations(S, n, C_CH, seed, torch.bfloat16, backward=True)
        t0 = time.perf_counter()
        o = oracle.pre(d["x"], params["phi"], params["b"], alpha, iters=T_MAX)
        oracle.post(d["x"], d["f_out"], o["H_post"], o["H_res"])
        oracle.backward(d["x"], params["phi"], params["b"], alpha, d["f_out"], d["grad_x_next"],
                        d["grad_h_in"], iters=T_MAX)
        return time.perf_counter() - t0

    return run


def oracle_sinkhorn_pass():
    """One timed pass of the fp64 oracle's batched Sinkhorn on the first S
    matrices of each n's seeded batch (n = 4, 8, 16; 20 iterations): run(S) ->
    seconds for 3 S matrices."""
    import oracle
    from manifold_constrained_hyper_token_b200 import synth

    def run(S):
        lg = [synth.sinkhorn_logits(S, n, seed=100 + n) for n in (4, 8, 16)]
        t0 = time.perf_counter()
        for x in lg:
            oracle.sinkhorn(x, T_MAX)
        return time.perf_counter() - t0

    return run


def oracle_depth_pass(L: int = 24):
    """One timed pass of the fp64 oracle through the L-layer stack (F_l(h) = s_l
    h) on the first S tokens of chunk 0: forward, then each layer's backward
    with grad_h_in = s_l grad_f_out, last layer first.  run(S) -> seconds."""
    import numpy as np
    import oracle
    from manifold_constrained_hyper_token_b200 import synth

    prms = [synth.layer_params(N_STR, C_CH, seed=l) for l in range(L)]
    gains = [synth.depth_gain(l) for l in range(L)]

    def run(S):
        d = synth.depth_stack_chunk(S, N_STR, C_CH, chunk=0)
        t0 = time.perf_counter()
        xs, fs = [d["x0"]], []
        for l in range(L):
            a = float(prms[l]["alpha"][0])
            r = oracle.pre(xs[l], prms[l]["phi"], prms[l]["b"], a, iters=T_MAX)
            fs.append(gains[l] * r["h_in"])
            xs.append(oracle.post(xs[l], fs[l], r["H_post"], r["H_res"]))
        G = d["G_last"]
        for l in reversed(range(L)):
            a = float(prms[l]["alpha"][0])
            zero = np.zeros((S, C_CH))
            gf = oracle.backward(xs[l], prms[l]["phi"], prms[l]["b"], a, fs[l], G, zero,
                                 iters=T_MAX)["grad_f_out"]
            G = oracle.backward(xs[l], prms[l]["phi"], prms[l]["b"], a, fs[l], G, gains[l] * gf,
                                iters=T_MAX)["grad_x"]
        return time.perf_counter() - t0

    return run


def _grow(run, seconds, start, cap):
    """Grow the sample size from `start` until one timed pass takes about
    `seconds` / 4 or more (or the cap is reached); returns (size, seconds)."""
    S = start
    dt = run(S)
    while dt < seconds / 4 and S < cap:
        S = min(cap, int(S * max(2.0, min(8.0, seconds / max(dt, 1e-3) / 2))))
        dt = run(S)
    return S, dt


def _both_thread_counts(run, seconds, start, cap, small):
    """The oracle with every host thread on a grown sample, then with one thread
    on a `small` sample of the same workload."""
    import oracle
    S, dt = _grow(run, seconds, start, cap)
    cores = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        dt1 = run(small)
    finally:
        oracle.set_num_threads(cores)
    return S, dt, cores, small, dt1


def cpu_reference(seconds: float, seed: int = 0):
    """The fp64 oracle, as it stands, on the first S tokens of the layer workload:
    pre + post + backward.  S is grown until one pass takes about `seconds`."""
    S, dt, cores, S1, dt1 = _both_thread_counts(oracle_layer_pass(N_STR, seed), seconds, 32,
                                                8192, 64)
    return {"value": S / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {S} tokens of the T={T_TOK}, n={N_STR}, C={C_CH} bf16 workload, "
                      f"pre+post+backward in fp64, {dt:.2f} s",
            "single_thread": {"value": S1 / dt1, "unit": "tokens/s", "cores": 1,
                              "sample": f"first {S1} tokens, {dt1:.2f} s"}}


def cpu_sinkhorn(seconds: float):
    """The fp64 oracle's batched Sinkhorn on the first S matrices of each n's batch
    (n = 4, 8, 16; the same seeded logits; 20 iterations): matrices/s."""
    S, dt, cores, S1, dt1 = _both_thread_counts(oracle_sinkhorn_pass(), seconds, 1024, 1 << 22,
                                                16384)
    return {"value": 3 * S / dt, "unit": "matrices/s", "cores": cores, "kind": "oracle",
            "sample": f"first {S} matrices of each of the n=4, 8, 16 batches, 20 iterations "
                      f"in fp64, {dt:.2f} s",
            "single_thread": {"value": 3 * S1 / dt1, "unit": "matrices/s", "cores": 1,
                              "sample": f"first {S1} matrices per n, {dt1:.2f} s"}}


def cpu_depth(seconds: float, L: int = 24):
    """The fp64 oracle through the L-layer stack on the first S tokens of chunk 0,
    forward and backward: tokens/s."""
    S, dt, cores, S1, dt1 = _both_thread_counts(oracle_depth_pass(L), seconds, 4, 4096, 8)
    return {"value": S / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {S} tokens of the stack input, {L} layers forward and backward "
                      f"(the per-layer backward run twice: grad_f_out, then grad_x) in fp64, "
                      f"{dt:.2f} s",
            "single_thread": {"value": S1 / dt1, "unit": "tokens/s", "cores": 1,
                              "sample": f"first {S1} tokens, {dt1:.2f} s"}}


def _reference_sample(run, start, cap, warmup, steps, budget_s):
    """Reference-arm sample size: one calibration pass of at least one unit per
    host thread (the oracle spreads tokens or matrices over its threads), then
    the S (at most `cap`) for which the warm-up and timed passes together take
    about budget_s.  Returns S, the seconds of the `steps` timed passes and the
    threads the oracle kept busy."""
    import oracle
    threads = oracle.num_threads()
    start = min(cap, max(start, threads))
    rate = start / run(start)
    S = int(max(start, min(cap, budget_s * rate / (warmup + steps))))
    for _ in range(warmup):
        run(S)
    return S, sum(run(S) for _ in range(steps)), min(S, threads)


def run_reference(args, rank, world):
    """Reference arm: the fp64 oracle on the host cores, for the workload the
    arguments name (the layer with --streams n, the batched Sinkhorn, or the
    depth stack), with that arm's metric and unit.  Each step runs the oracle
    on a bounded sample of S units of the workload; S comes from a short
    calibration so that the W + K steps take about --reference-seconds."""
    if rank != 0:
        return
    W, K, budget = args.warmup, args.steps, args.reference_seconds
    if args.workload == "sinkhorn":
        S, total, cores = _reference_sample(oracle_sinkhorn_pass(), 1024, 1 << 22, W, K,
                                            budget)
        metric, unit, units = SINKHORN_METRIC, "matrices/s", 3 * S
        sample = (f"first {S} matrices of each of the n=4, 8, 16 batches per step, 20 "
                  f"iterations in fp64")
        cfg = {"workload": f"standalone Sinkhorn-Knopp, oracle on the first {S} matrices per n "
                           f"of the 2^22-matrix batches (n in {{4, 8, 16}}, logits N(0, 2), "
                           f"{T_MAX} iterations) per step",
               "matrices_per_step": units, "B_sampled_from": 1 << 22, "t_max": T_MAX}
    elif args.workload == "depth":
        L = 24
        T = args.tokens if args.tokens != T_TOK else 65536
        S, total, cores = _reference_sample(oracle_depth_pass(L), 4, 4096, W, K, budget)
        metric, unit, units = DEPTH_METRIC, "tokens/s", S
        sample = (f"first {S} tokens of the stack input per step, {L} layers forward and "
                  f"backward in fp64")
        cfg = {"workload": f"depth stack, oracle on the first {S} tokens of the L={L}, "
                           f"T={T}, n={N_STR}, C={C_CH}, F_l(h)=s_l h workload per step",
               "tokens_per_step": S, "T_sampled_from": T, "L": L, "n": N_STR, "C": C_CH,
               "t_max": T_MAX}
    else:
        n = args.streams
        S, total, cores = _reference_sample(oracle_layer_pass(n, 0, pool=256), 32, 256, W, K,
                                            budget)
        metric, unit, units = layer_metric(n), "tokens/s", S
        sample = (f"{S} tokens per step of the T={args.tokens}, n={n}, C={C_CH} bf16 "
                  f"workload, pre+post+backward in fp64")
        cfg = {"workload": f"mHC layer fwd+bwd, oracle on a sample of S={S} tokens per step "
                           f"drawn from the T={args.tokens}, n={n}, C={C_CH}, t_max={T_MAX} "
                           f"bf16 workload",
               "tokens_per_step": S, "T_sampled_from": args.tokens, "n": n, "C": C_CH,
               "t_max": T_MAX}
    cfg["parallelism"] = "host cores (oracle)"
    val = K * units / total
    # a step here is the sample the oracle ran, and ms_per_step its measured time
    line = {"metric": metric, "value": val, "unit": unit, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": 1000.0 * total / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": cfg,
            "cpu_baseline": {"value": val, "unit": unit, "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample-seconds", type=float, default=12.0)
    ap.add_argument("--reference-seconds", type=float, default=120.0,
                    help="--impl reference: host seconds for the warm-up and timed steps together")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--tokens", type=int, default=T_TOK,
                    help="tokens per GPU (default 16384; smaller values for profiler captures)")
    ap.add_argument("--workload", default="layer", choices=["layer", "sinkhorn", "depth"],
                    help="layer: the fwd+bwd layer step (the default line); sinkhorn: batched "
                         "Sinkhorn-Knopp and depth gain; depth: the 24-layer stack")
    ap.add_argument("--streams", type=int, default=N_STR, choices=[4, 8, 16],
                    help="layer workload stream count n (default 4, the headline; 8 runs its "
                         "tensor-core mapping and apply; 16 its tensor-core projection with the "
                         "CUDA-core reductions, Sinkhorn and apply)")
    ap.add_argument("--forward", default="unfused", choices=["fused", "unfused"],
                    help="fused: layer input + post merge fused with the next layer's mapping; "
                         "unfused: mhc_pre + mhc_post")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    if args.workload == "sinkhorn":
        run_sinkhorn(args, dev, rank, world, local_rank)
    elif args.workload == "depth":
        run_depth(args, dev, rank, world, local_rank)
    else:
        run_layer(args, dev, rank, world, local_rank)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def step_stats(ms):
    """Median and spread of per-step device times (ms)."""
    v = sorted(ms)
    if not v:
        return None
    q = lambda f: v[min(len(v) - 1, int(round(f * (len(v) - 1))))]
    return {"median": q(0.5), "p10": q(0.1), "p90": q(0.9), "min": v[0], "max": v[-1],
            "n": len(v)}


def run_layer(args, dev, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import manifold_constrained_hyper_token_b200 as mhc
    from manifold_constrained_hyper_token_b200 import parallel, synth

    T, n, C = args.tokens, args.streams, C_CH
    K, M = n * C, n * n + 2 * n
    prm = synth.layer_params(n, C, seed=0)
    act = synth.activations(T, n, C, seed=rank, dtype=torch.bfloat16, backward=True)
    phi, b, alpha = (prm["phi"].to(dev), prm["b"].to(dev), prm["alpha"].to(dev))
    x, f_out = act["x"].to(dev), act["f_out"].to(dev)
    G, g = act["grad_x_next"].to(dev), act["grad_h_in"].to(dev)
    h_in = torch.empty(T, C, dtype=torch.bfloat16, device=dev)
    Hpre = torch.empty(T, n, dtype=torch.float32, device=dev)
    Hpost = torch.empty(T, n, dtype=torch.float32, device=dev)
    Hres = torch.empty(T, n, n, dtype=torch.float32, device=dev)
    x_next = torch.empty_like(x)
    gx = torch.empty_like(x)
    gf = torch.empty_like(f_out)
    pgrads, gphi, gb, ga = parallel.param_grad_buffer(n, C, dev)  # one all-reduce buffer
    ws = torch.empty(mhc.mhc_backward_workspace_size(n, T, C, torch.bfloat16), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()
    fused = args.forward == "fused"
    calls = (["layer_input", "post_fused"] if fused else ["pre", "post"]) + ["bwd_map", "bwd_apply"]
    # this library's kernels per call: pre = phi split + mapping + layer input;
    # bwd_map = phi split + mapping; post_fused = phi split + fused kernel;
    # bwd_apply = one kernel at n = 4; n = 8: grad_x with phi u, bias sums,
    # grad_phi and its finish (k_gxu8, k_bias8, k_gphi8, k_gphi8_fin);
    # n = 16: pre = phi split + projection + epilogue + layer input, bwd_map =
    # phi split + projection + reductions + epilogue
    launches_per_call = {"pre": 3, "post": 1, "layer_input": 1, "post_fused": 2, "bwd_map": 2,
                         "bwd_apply": 1 if n == N_STR else 4}
    if n == 8:  # the fused post is k_post, then the phi split and the mapping; the
        # backward mapping is the phi split, the tensor-core reductions, the mapping
        launches_per_call.update({"post_fused": 3, "bwd_map": 3})
    if n == 16:  # the apply: U rows, phi u, grad_x, grad_phi and its finish, bias sums
        launches_per_call.update({"pre": 4, "bwd_map": 4, "post_fused": 4, "bwd_apply": 6})
    # the layer's maps; in a stack the previous layer's post_fused computes them
    mhc.mhc_pre(x, phi, b, alpha, t_max=T_MAX, out=(h_in, Hpre, Hpost, Hres), stream=stream)
    nxt = (torch.empty_like(Hpre), torch.empty_like(Hpost), torch.empty_like(Hres))
    pre_ws = torch.empty(max(1, mhc.mhc_pre_workspace_size(n, T, C, torch.bfloat16)),
                         dtype=torch.uint8, device=dev)

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        if fused:
            mhc.mhc_layer_input(x, Hpre, out=h_in, stream=stream)
        else:
            mhc.mhc_pre(x, phi, b, alpha, t_max=T_MAX, out=(h_in, Hpre, Hpost, Hres),
                        workspace=pre_ws, stream=stream)
        if evs is not None:
            evs[1].record(stream)
        if fused:
            mhc.mhc_post_fused(x, f_out, Hpost, Hres, phi, b, alpha, t_max=T_MAX,
                               out=(x_next,) + nxt, workspace=pre_ws, stream=stream)
        else:
            mhc.mhc_post(x, f_out, Hpost, Hres, out=x_next, stream=stream)
        if evs is not None:
            evs[2].record(stream)
        mhc.mhc_backward_map(x, phi, b, alpha, f_out, G, g, ws, t_max=T_MAX, stream=stream)
        if evs is not None:
            evs[3].record(stream)
        mhc.mhc_backward_apply(x, phi, G, g, ws, t_max=T_MAX, out=(gx, gphi, gb, ga, gf),
                               stream=stream)
        if evs is not None:
            evs[4].record(stream)
        if world > 1:
            parallel.allreduce_param_grads(pgrads)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)  # let the sampler come up before the timed region
    t_start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    per_call = {c: 0.0 for c in calls}
    for s in range(args.steps):
        for i, c in enumerate(calls):
            per_call[c] += evs[s][i].elapsed_time(evs[s][i + 1])
    per_call = {c: v / args.steps for c, v in per_call.items()}
    per_step = [evs[s][0].elapsed_time(evs[s][len(calls)]) for s in range(args.steps)]
    elapsed_ms = parallel.max_over_ranks(elapsed_ms, dev)
    ms_per_step = elapsed_ms / args.steps
    tokens_per_s = T * world / (ms_per_step / 1000.0)

    # ---- roofline of the longest single-kernel call, and the whole step
    peak, peak_kind = load_peaks()
    tb = per_token_bytes(n, C)
    pb = per_call_param_bytes(n, C)
    call_bytes = {c: T * tb[c] + pb[c] for c in calls}
    # the roofline is read for a call whose time is one kernel's (the phi split
    # ahead of the n = 4 backward mapping is 5 us of its 0.5 ms and is counted
    # in; at n = 8 and 16 the backward mapping and the apply are several
    # kernels each and are not such calls)
    single = [c for c in calls
              if c in ("post", "layer_input") or (c in ("bwd_map", "bwd_apply") and n == N_STR)]
    dom = max(single, key=lambda c: per_call[c])
    achieved = call_bytes[dom] / (per_call[dom] / 1000.0) / 1e9
    traffic = ncu_traffic(traffic_key(dom, n))
    fwd_calls = calls[:2]
    step_alg_bytes = (T * (sum(tb[c] for c in fwd_calls) + tb["bwd_min"]) +
                      sum(pb[c] for c in fwd_calls) + pb["bwd_apply"])
    step_gbs = step_alg_bytes / (ms_per_step / 1000.0) / 1e9

    # ---- end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0:
        hx, hf = act["x"].pin_memory(), act["f_out"].pin_memory()
        hG, hg = act["grad_x_next"].pin_memory(), act["grad_h_in"].pin_memory()
        hout = torch.empty(K * M + M + 1, dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hx, hf, hG, hg))
        d2h = hout.numel() * hout.element_size()

        def e2e_step():
            x.copy_(hx, non_blocking=True)
            f_out.copy_(hf, non_blocking=True)
            G.copy_(hG, non_blocking=True)
            g.copy_(hg, non_blocking=True)
            step()
            hout.copy_(pgrads, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = parallel.max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dev)
        e2e = {"value": T * world / (e_ms / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "ms_per_step": e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and n == N_STR:
        cpu = cpu_reference(args.cpu_sample_seconds)

    if rank == 0:
        line = {
            "metric": layer_metric(n),
            "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"mHC layer fwd+bwd per GPU: T={T} tokens, n={n}, C={C}, "
                                   f"t_max={T_MAX}, bf16 activations, fp32 maps; " +
                                   ("one layer of a stack: layer input, post merge fused with "
                                    "the next layer's mapping, backward" if fused else
                                    "pre, post, backward (no cross-layer fusion)"),
                       "forward": args.forward,
                       "T_per_gpu": T, "n": n, "C": C, "t_max": T_MAX,
                       "parallelism": f"dp{world} over tokens",
                       "l2": f"inputs larger than L2 (x and grad_x_next are "
                             f"{T * n * C * 2 / 1e6:.0f} MB each); no flush"},
            "hbm": {"achieved_gbs": step_gbs, "peak_gbs": peak, "frac": step_gbs / peak,
                    "peak_kind": peak_kind, "frac_vs_nominal": step_gbs / NOMINAL_HBM_GBS,
                    "alg_bytes_per_step": step_alg_bytes},
            "per_call_ms": per_call,
            "step_ms": step_stats(per_step),
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                         "frac_vs_nominal": achieved / NOMINAL_HBM_GBS,
                         "alg_bytes_per_launch": call_bytes[dom], "peak_kind": peak_kind},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * sum(launches_per_call[c] for c in calls),
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def _timed(fn, steps, warmup, stream):
    """Device times (ms) of `steps` calls of fn after `warmup` untimed ones."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for e0, e1 in evs:
        e0.record(stream)
        fn()
        e1.record(stream)
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in evs]


def sinkhorn_ops(n, iters):
    """fp32 operations of one n x n Sinkhorn-Knopp estimate as the kernel runs it: the
    row maxima, shift and exp (3 n^2), then per normalisation n^2 adds, n reciprocals
    and n^2 multiplies."""
    return 3 * n * n + 2 * iters * (2 * n * n + n)


def run_sinkhorn(args, dev, rank, world, local_rank):
    """Batched Sinkhorn-Knopp on 2^22 matrices (n = 4, 8, 16; logits N(0, 2); 20
    iterations) and the depth-product Amax gain over L = 64 layers of 2^16 tokens.
    Each rank runs its own batch (weak scaling)."""
    import torch

    import manifold_constrained_hyper_token_b200 as mhc
    from manifold_constrained_hyper_token_b200 import parallel, synth

    B, iters, Tdep, Ldep = 1 << 22, T_MAX, 1 << 16, 64
    stream = torch.cuda.current_stream()
    peak, peak_kind = load_peaks()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(local_rank)
    sampler.start()
    per_n = {}
    total_ms, total_mat = 0.0, 0
    for n in (4, 8, 16):
        lg = synth.sinkhorn_logits(B, n, seed=100 + n + rank).to(dev)
        out = torch.empty_like(lg)
        ms = _timed(lambda: mhc.mhc_sinkhorn_knopp(lg, iters, out=out, stream=stream),
                    args.steps, args.warmup, stream)
        t = parallel.max_over_ranks(sum(ms) / len(ms), dev)
        byts = B * 8 * n * n
        ops = B * sinkhorn_ops(n, iters)
        per_n[str(n)] = {"ms": t, "matrices_per_s": B * world / (t / 1e3),
                         "hbm_gbs": byts / (t / 1e3) / 1e9,
                         "hbm_frac": byts / (t / 1e3) / 1e9 / peak,
                         "gops": ops / (t / 1e3) / 1e9, "step_ms": step_stats(ms)}
        total_ms += t
        total_mat += B
        del lg, out
    # depth product over 64 layers of 20-iteration Sinkhorn outputs (n = 4)
    H = mhc.mhc_sinkhorn_knopp(synth.sinkhorn_logits(Tdep * Ldep, 4, seed=300 + rank).to(dev),
                               iters).view(Tdep, Ldep, 4, 4)
    gf = torch.empty(Tdep, device=dev)
    gb = torch.empty(Tdep, device=dev)
    ms = _timed(lambda: mhc.mhc_depth_amax(H, out=(gf, gb), stream=stream), args.steps,
                args.warmup, stream)
    td = parallel.max_over_ranks(sum(ms) / len(ms), dev)
    dbytes = Tdep * Ldep * 16 * 4 + 2 * Tdep * 4
    clocks = sampler.stop()
    sm_mhz = clocks.get("sm_mhz") or 1965.0
    # fp32 add / multiply issue rate: 128 lanes per SM per clock
    alu_peak_gops = props.multi_processor_count * 128 * sm_mhz * 1e6 / 1e9
    for v in per_n.values():
        v["alu_frac"] = v["gops"] / alu_peak_gops
    dom = max(per_n, key=lambda k: per_n[k]["ms"])
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_sinkhorn(args.cpu_sample_seconds)
    if rank == 0:
        d = per_n[dom]
        bound = "hbm" if d["hbm_frac"] >= d["alu_frac"] else "alu"
        line = {
            "metric": SINKHORN_METRIC,
            "value": total_mat * world / (total_ms / 1e3), "unit": "matrices/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "standalone Sinkhorn-Knopp: 2^22 matrices per n in {4, 8, 16}, "
                                   "logits N(0, 2), 20 iterations; depth gain over L=64 layers "
                                   "x 2^16 tokens (n=4)",
                       "l2": "inputs larger than L2 (n=4: 268 MB of logits); no flush"},
            "per_n": per_n,
            "depth_amax": {"ms": td, "tokens_per_s": Tdep * world / (td / 1e3),
                           "hbm_gbs": dbytes / (td / 1e3) / 1e9,
                           "hbm_frac": dbytes / (td / 1e3) / 1e9 / peak},
            "roofline": {"bound": bound, "kernel": f"k_sinkhorn n={dom}",
                         "achieved": d["hbm_gbs"] if bound == "hbm" else d["gops"],
                         "peak": peak if bound == "hbm" else alu_peak_gops,
                         "unit": "GB/s" if bound == "hbm" else "Gop/s",
                         "frac": d["hbm_frac"] if bound == "hbm" else d["alu_frac"],
                         "traffic": None, "peak_kind": peak_kind if bound == "hbm" else
                         "148 SMs x 128 fp32 lanes x median SM clock"},
            "cpu_baseline": cpu,
            "gpu_launches": 4 * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def run_depth(args, dev, rank, world, local_rank):
    """24 mHC layers, T tokens per GPU (default 65536), n = 4, C = 7168, bf16,
    F_l(h) = s_l h, forward and backward through DepthStack (block recompute,
    backward in training order)."""
    import torch

    from manifold_constrained_hyper_token_b200 import parallel, synth
    from manifold_constrained_hyper_token_b200.depth import DepthStack

    L, n, C = 24, N_STR, C_CH
    T = args.tokens if args.tokens != T_TOK else 65536
    layers = [{k: v.to(dev) for k, v in synth.layer_params(n, C, seed=l).items()}
              for l in range(L)]
    gains = [synth.depth_gain(l) for l in range(L)]
    F = lambda l, h: h * gains[l]
    Fb = lambda l, h, f, gfo: gfo * gains[l]
    stack = DepthStack(layers, F, Fb, n)
    d = synth.depth_stack_chunk(T, n, C, chunk=rank)
    x0, GL = d["x0"].to(dev), d["G_last"].to(dev)
    del d
    stream = torch.cuda.current_stream()

    def step():
        stack.forward(x0)
        stack.backward(GL)

    sampler = ClockSampler(local_rank)
    sampler.start()
    ms = _timed(step, args.steps, args.warmup, stream)
    clocks = sampler.stop()
    t = parallel.max_over_ranks(sum(ms) / len(ms), dev)
    peak, peak_kind = load_peaks()
    tb = per_token_bytes(n, C)
    alg = L * T * (tb["pre"] + tb["post"] + tb["bwd_min"])
    # this library's launches per step: forward pre (phi split, mapping, layer
    # input) + post per layer; backward: each recompute's pre (+ post when the
    # next layer's input is rebuilt), then post_backward + pre_backward (phi
    # split, split mapping, apply) per layer
    rec = [st for st in stack.bwd_steps if st[0] == "recompute"]
    launches = 4 * L + sum(3 + (1 if st[2] else 0) for st in rec) + 4 * L
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_depth(args.cpu_sample_seconds)
    gbs = alg / (t / 1e3) / 1e9
    if rank == 0:
        line = {
            "metric": DEPTH_METRIC,
            "value": T * world / (t / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"depth stack: L={L} layers, T={T} tokens per GPU, n={n}, "
                                   f"C={C}, bf16, F_l(h)=s_l h, recompute block "
                                   f"{stack.block}, backward in training order",
                       "l2": "inputs larger than L2; no flush"},
            "step_ms": step_stats(ms),
            "hbm": {"alg_bytes_per_step": alg, "achieved_gbs": alg / (t / 1e3) / 1e9,
                    "peak_gbs": peak, "frac": alg / (t / 1e3) / 1e9 / peak,
                    "peak_kind": peak_kind,
                    "note": "24 x 415,920 B/token (one forward and a one-pass backward per "
                            "layer); the recompute forward and F are extra"},
            "roofline": {"bound": "hbm", "kernel": "whole step (24 layers, every kernel)",
                         "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": None, "peak_kind": peak_kind},
            "cpu_baseline": cpu,
            "gpu_launches": launches * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
