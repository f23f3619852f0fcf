"""Benchmark: chunkwise GLA forward + backward on B200 (one process per GPU).

One step = gla_fwd + gla_bwd over one batch of the 1.3B-layer workload
(B=2, H=4, T=4096, d_k=256, d_v=512, bf16, vector gates with z ~ N(-1,1)),
inputs resident in HBM.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 launch with torchrun; every rank runs its own replica of the workload
(weak scaling, no collective on the data path), and the line also reports the
same sequence split across the ranks (sequence_parallel.ranks).  --seqpar makes
that split the headline (strong scaling: each rank runs its piece of one
sequence, with one NCCL all-gather of the pieces' state summaries per direction).
--impl reference times the float64 CPU oracle (the only reference
implementation) on a bounded sample.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GLA fwd+bwd tokens/s and TFLOP/s vs T; % of B200 bf16 tensor peak / HBM BW"
WORKLOAD = dict(B=2, H=4, T=4096, K=256, V=512, C=64, z_mean=-1.0, gate="vector")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def counted_flops(B, H, T, K, V, C):
    """Contraction FLOPs per step (fwd 4KV + C(K+V), bwd 10KV + C(3K+2V) per token-head)."""
    th = B * H * T
    return th * (4 * K * V + C * (K + V)) + th * (10 * K * V + C * (3 * K + 2 * V))


def algorithmic_bytes(B, H, T, K, V, gate="vector"):
    """Inputs + outputs of fwd and bwd (bf16 q,k,v,o,do,dq,dk,dv; fp32 gates; no states)."""
    th = B * H * T
    g = 4 * K if gate == "vector" else (4 if gate == "scalar" else 0)
    fwd = th * (2 * K + 2 * K + 2 * V + g + 2 * V)
    bwd = th * (2 * K + 2 * K + 2 * V + g + 2 * V + 2 * K + 2 * K + 2 * V + g)
    return fwd + bwd


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) measured by ncu on
# the full-size workload, with the sha256 of the kernel sources it was measured on.  It is
# reported only while the sources are unchanged (a changed kernel has unknown traffic).
NCU_TRAFFIC = {"src_sha256": "cdee8da559628cfc47ae53331168aec32159d565ba6b25d6d0ad903d9718a49c",
               "per_launch_bytes": {"tc_walk": 116625216, "tc_bwd": 461712256, "tc_prep": 71790848, "segment_starts": 12621184}}


def kernel_src_sha256():
    """sha256 over the sources of the step's kernels (the tc_* files and seqpar.cu)."""
    d = os.path.join(ROOT, "chunkwise_linear_rnn_fwd_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(x for x in os.listdir(d) if x.startswith("tc_") or x == "seqpar.cu"):
        h.update(f.encode())
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(kernel):
    if NCU_TRAFFIC["src_sha256"] != kernel_src_sha256():
        return None
    return NCU_TRAFFIC["per_launch_bytes"].get(kernel)


def bench_config(w, world):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": f"gla fwd+bwd, B={w['B']} H={w['H']} T={w['T']} d_k={w['K']} d_v={w['V']} C={w['C']}, "
                        f"bf16, {w['gate']} gates z~N({w['z_mean']:g},1), fp32 state",
            "global_batch": w["B"] * world, "seq_len": w["T"], "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (~268 MB touched per step)"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        busy = [x for x in sm if x > 0.5 * (smax or 1)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def reduce_max_ms(ms_local: float, world: int, device=None) -> float:
    """Max of a per-rank duration over all ranks (the slowest rank defines the step)."""
    if world <= 1:
        return ms_local
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms_local], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(tokens_per_rank_step: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank_step * world * steps / (ms_max / 1e3)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ----------------------------------------------------------------------------------- oracle
def oracle_sample_rate(w, T_sample=1024, seed=0, min_seconds=0.0):
    """Time the float64 oracle (fwd + BPTT bwd) on all heads of the workload for the
    first T_sample tokens, repeated until at least min_seconds have passed; returns
    (tokens/s, seconds, threads, description)."""
    import torch

    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs
    from oracle import oracle

    x = make_inputs(w["B"], w["H"], T_sample, w["K"], w["V"], dtype=torch.bfloat16, gate=w["gate"], seed=seed,
                    z_mean=w["z_mean"])
    f = lambda a: None if a is None else a.double().numpy()
    q, k, v, la, do = f(x.q), f(x.k), f(x.v), f(x.log_alpha), f(x.do)
    oracle.build()
    reps, dt = 0, 0.0
    while reps == 0 or dt < min_seconds:
        t0 = time.perf_counter()
        oracle.fwd(q, k, v, la, gate=w["gate"])
        oracle.bwd(q, k, v, la, do, gate=w["gate"])
        dt += time.perf_counter() - t0
        reps += 1
    threads = min(oracle.threads(), w["B"] * w["H"])
    desc = (f"fwd+bwd of all {w['B'] * w['H']} heads over the first {T_sample} of {w['T']} tokens "
            f"(d_k={w['K']}, d_v={w['V']}), float64, OpenMP over heads, {reps} repetition(s)")
    return reps * w["B"] * T_sample / dt, dt, threads, desc


def host_cpu():
    """The host the oracle ran on: cores available to this process and the CPU model.
    `cores` in cpu_baseline is the number of threads the oracle actually used (its
    OpenMP loop runs over the B*H heads, so it cannot use more threads than heads)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        avail = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        avail = os.cpu_count()
    return {"host_cores_available": avail, "cpu_model": model}


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_sample_rate(w, T_sample=args.ref_tokens)
    rates, secs = [], 0.0
    threads, desc = 1, ""
    for _ in range(args.steps):
        r, dt, threads, desc = oracle_sample_rate(w, T_sample=args.ref_tokens)
        rates.append(r)
        secs += dt
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc,
                         **host_cpu()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------ ours
def walk_segments(w, sms):
    """Segment count the library picks for the walks (one wave of one CTA per SM over
    the heads' 128-column d_v tiles)."""
    B, H, T, K, V, C = w["B"], w["H"], w["T"], w["K"], w["V"], w["C"]
    N = -(-T // C)
    nvt = -(-V // 128)
    P = max(1, sms // (B * H * nvt))
    P = min(P, N)
    L = -(-N // P)
    return -(-N // L)


def kernel_io_bytes(name, w, sms=148):
    """Bytes the launches of `name` in one fwd+bwd step must move at minimum (their own
    inputs + outputs, each once), divided by the number of those launches."""
    B, H, T, K, V, C = w["B"], w["H"], w["T"], w["K"], w["V"], w["C"]
    BH, N = B * H, -(-T // C)
    Tp = N * C
    if name == "tc_walk":
        P = walk_segments(w, sms)
        f = (P - 1) / P                       # share of chunks a pre-pass covers
        kx = BH * Tp * K * 2                  # qg or kg
        vy = BH * T * V * 2                   # V or dO
        seg = BH * (P - 1) * K * V * 4        # segment contributions (written, then read)
        states = BH * N * K * V * 2           # bf16 chunk states h_n or dh_n
        pt = BH * N * C * C * 2
        pre = f * (kx + vy) + seg
        # forward: pre-pass + output walk that also stores h_n (saved states);
        # backward: reverse pre-pass + adjoint walk storing dh_n
        fwd_out = 2 * kx + vy + pt + seg + vy + BH * K * V * 4 + states
        # reverse walk: qg, dO (the adjoint) and kg, P^T (dv) in; dh_n and dv out
        dh_walk = 2 * kx + vy + pt + seg + states + vy
        launches = 2 * (2 if P > 1 else 1)
        total = 2 * (pre if P > 1 else 0) + fwd_out + dh_walk
        return total / launches
    g = 4 * K if w["gate"] == "vector" else (4 if w["gate"] == "scalar" else 0)
    if name == "tc_prep":
        return BH * T * (2 * K + 2 * K + g) + BH * Tp * 2 * (2 * K) + BH * N * (4 * K + 2 * C * C)
    if name == "tc_bwd":
        return (BH * N * K * V * 2 * 2 + BH * T * (2 * V * 2 + 2 * K * 2 + g) + BH * Tp * 2 * K
                + BH * N * 2 * C * C + BH * T * (2 * K * 2 + 2 * V + g))
    return None


# Which of the step's algorithmic tensors (inputs and outputs of the forward and the
# backward, each counted once per pass as in algorithmic_bytes) each kernel moves
# between HBM and the chip: a kernel's algorithmic share of the step.
KERNEL_ALG_TENSORS = {
    "tc_prep": ("q", "k", "la"),                          # the forward's reads of q, k, log alpha
    "tc_walk": ("v", "o", "h_final", "do", "dv"),         # forward: v in, o, h_final out; reverse: dO in, dv out
    "tc_bwd": ("q", "k", "la", "v", "dq", "dk", "dla"),   # the backward's reads of q, k, log alpha, v and its outputs
}


def kernel_alg_bytes(name, w):
    """Algorithmic bytes per step that kernel `name` is responsible for (its share of
    algorithmic_bytes: the tensors of KERNEL_ALG_TENSORS, no workspace)."""
    B, H, T, K, V = w["B"], w["H"], w["T"], w["K"], w["V"]
    th = B * H * T
    g = 4 * K if w["gate"] == "vector" else (4 if w["gate"] == "scalar" else 0)
    size = {"q": th * 2 * K, "k": th * 2 * K, "v": th * 2 * V, "la": th * g, "o": th * 2 * V, "do": th * 2 * V,
            "dq": th * 2 * K, "dk": th * 2 * K, "dv": th * 2 * V, "dla": th * g, "h_final": B * H * K * V * 4}
    names = KERNEL_ALG_TENSORS.get(name)
    return None if names is None else sum(size[n] for n in names)


DECODE_WORKLOAD = dict(B=128, H=4, K=256, V=512)


def measure_decode(args, dev, stream, peaks, peak_src, seed=0):
    """The recurrent decode step (one token per head, state updated in place) on a batch
    whose fp32 state (256 MB) exceeds L2: device time per step and the HBM roofline of
    its algorithmic bytes (state read + write, q, k, v, log alpha read, o written)."""
    import torch

    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs

    w = DECODE_WORKLOAD
    B, H, K, V = w["B"], w["H"], w["K"], w["V"]
    x = make_inputs(B, H, 1, K, V, dtype=torch.bfloat16, gate="vector", seed=seed, with_h0=True)
    q, k, v = (t[:, :, 0].contiguous().to(dev) for t in (x.q, x.k, x.v))
    la = x.log_alpha[:, :, 0].contiguous().to(dev)
    S = x.h0.to(dev).contiguous()
    o = torch.empty(B, H, V, dtype=torch.bfloat16, device=dev)
    for _ in range(max(3, args.warmup)):
        pkg.gla_decode_step(q, k, v, la, S, o=o, stream=stream)
    torch.cuda.synchronize()
    n = max(10, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        pkg.gla_decode_step(q, k, v, la, S, o=o, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    nbytes = B * H * (2 * K * V * 4 + 2 * K * 2 + V * 2 + K * 4 + V * 2)
    gbs = nbytes / (ms / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    return {"workload": f"decode step, B={B} H={H} d_k={K} d_v={V}, bf16 q/k/v/o, fp32 state, vector gates",
            "ms_per_step": ms, "tokens_per_s": B / (ms / 1e3), "bytes_per_step": nbytes,  # one token per sequence
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "peak_source": peak_src}}


def measure_epilogue(args, w, dev, stream, peaks, peak_src, seed=0):
    """The layer epilogue (LayerNorm of each head's output times the Swish output gate)
    on the bench workload's output shape: device time of the forward and of the
    backward (with dw, db) and their HBM rooflines on algorithmic bytes."""
    import torch

    import chunkwise_linear_rnn_fwd_b200 as pkg

    B, H, T, V = w["B"], w["H"], w["T"], w["V"]
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    o, r, dy = (torch.randn(B, H, T, V, device=dev, generator=g).to(torch.bfloat16) for _ in range(3))
    wt = torch.ones(V, device=dev)
    bs = torch.zeros(V, device=dev)
    y = torch.empty_like(o)
    ws = pkg.alloc_workspace(pkg.epilogue_workspace_size(B, H, T, V, torch.bfloat16), dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # twice the L2
    res = {}
    for name, fn in (("fwd", lambda: pkg.gla_epilogue_fwd(o, r, wt, bs, y=y, workspace=ws, stream=stream)),
                     ("bwd", lambda: pkg.gla_epilogue_bwd(o, r, dy, wt, bs, workspace=ws, stream=stream))):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        # device time of every launch (library events on the launch stream), L2 flushed
        # before each call so that no input is served from the previous iteration's L2
        n = max(10, args.steps)
        pkg.timing_enable(True)
        pkg.timing_collect()
        for _ in range(n):
            flush.fill_(1)  # on torch's current stream, which is the launch stream
            fn()
        torch.cuda.synchronize()
        launches = pkg.timing_collect()
        pkg.timing_enable(False)
        per_kernel = {}
        for kname, kms in launches:
            per_kernel[kname] = per_kernel.get(kname, 0.0) + kms / n
        ms = sum(per_kernel.values())
        elems = B * H * T * V
        nbytes = elems * 2 * (3 if name == "fwd" else 5) + 4 * 4 * V
        gbs = nbytes / (ms / 1e3) / 1e9
        res[name] = {"ms": ms, "kernels_ms": per_kernel, "bytes": nbytes, "achieved_gbs": gbs,
                     "frac_of_hbm": gbs / float(peaks["hbm_gbs"]), "l2": "flushed before every call"}
    res["workload"] = f"layer epilogue, B={B} H={H} T={T} d_v={V}, bf16 (fwd: o, r -> y; bwd: o, r, dy -> do, dr, dw, db)"
    res["peak_source"] = peak_src
    res["fused_forward"] = measure_fused_epilogue(args, w, dev, stream, r, wt, bs, res["fwd"]["ms"], seed=seed)
    return res


def measure_fused_epilogue(args, w, dev, stream, r, wt, bs, separate_ms, seed=0):
    """The forward with the epilogue fused into its output store (gla_fwd_epilogue)
    against the plain forward (gla_fwd) on the bench workload: the fused store's
    extra device time beside the separate pass's."""
    import torch

    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs

    B, H, T, K, V, C = w["B"], w["H"], w["T"], w["K"], w["V"], w["C"]
    x = make_inputs(B, H, T, K, V, dtype=torch.bfloat16, gate=w["gate"], seed=seed, z_mean=w["z_mean"])
    q, k, v, la = (t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha))
    o, y = torch.empty_like(v), torch.empty_like(v)
    ws = pkg.alloc_workspace(pkg.workspace_size(B, H, T, K, V, torch.bfloat16, w["gate"], C, False), dev)
    n = max(10, args.steps)
    plain = lambda: pkg.gla_fwd(q, k, v, la, None, chunk=C, o=o, want_final=False, workspace=ws, stream=stream)
    fused = lambda: pkg.gla_fwd_epilogue(q, k, v, la, r, wt, bs, chunk=C, o=o, y=y, want_final=False, workspace=ws,
                                         stream=stream)
    res = {"plain_fwd_ms": _time_steps(plain, stream, n, max(3, args.warmup)),
           "fused_fwd_ms": _time_steps(fused, stream, n, max(3, args.warmup))}
    pkg.timing_enable(True)
    pkg.timing_collect()
    for _ in range(n):
        fused()
    torch.cuda.synchronize()
    per = {}
    for kname, kms in pkg.timing_collect():
        per[kname] = per.get(kname, 0.0) + kms / n
    pkg.timing_enable(False)
    res["fused_kernels_ms"] = per
    res["extra_ms"] = res["fused_fwd_ms"] - res["plain_fwd_ms"]
    res["separate_pass_ms"] = separate_ms
    res["workload"] = (f"gla_fwd vs gla_fwd_epilogue, B={B} H={H} T={T} d_k={K} d_v={V}, bf16, "
                       f"{w['gate']} gates; o and y both written")
    return res


def measure_seqpar(args, w, dev, stream, seed=0, pieces=8):
    """Sequence parallelism's cost per rank when the bench workload is one piece of a
    sequence split over `pieces` ranks: a piece's whole training step (summaries,
    folds over the gathered summaries of the other pieces -- the worst-placed rank
    folds pieces - 1 -- and the reruns, one workspace, seqpar.LibraryOps) against the
    plain step on the same inputs, both timed with events around `steps` steps.  The
    all-gather itself needs several GPUs and is reported in bytes."""
    import torch

    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200 import seqpar
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs

    B, H, T, K, V = w["B"], w["H"], w["T"], w["K"], w["V"]
    x = make_inputs(B, H, T, K, V, dtype=torch.bfloat16, gate=w["gate"], seed=seed, z_mean=w["z_mean"])
    q, k, v, la, do = (t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha, x.do))
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    gammas = torch.rand(pieces, B, H, K, device=dev, generator=g)
    deltas = torch.randn(pieces, B, H, K, V, device=dev, generator=g)
    ops = seqpar.LibraryOps(w["C"], stream)
    ws = pkg.alloc_workspace(pkg.workspace_size(B, H, T, K, V, torch.bfloat16, w["gate"], w["C"], True,
                                                flags=pkg.FLAG_SAVE_STATES), dev)

    def sp_step():
        ops.fwd_state(q, k, v, la, None)
        h_in = ops.state_scan(gammas, deltas, pieces - 1, False)
        ops.fwd(q, k, v, la, h_in)
        ops.bwd_state(q, k, la, do, None)
        dh_out = ops.state_scan(gammas, deltas, 0, True)
        ops.bwd(q, k, v, la, do, h_in, dh_out)

    def plain_step():
        pkg.gla_fwd(q, k, v, la, None, chunk=w["C"], workspace=ws, stream=stream, save_states=True)
        pkg.gla_bwd(q, k, v, la, do, None, None, chunk=w["C"], workspace=ws, stream=stream, reuse_prep=True,
                    saved_states=True)

    res = {}
    for name, fn in (("plain_step", plain_step), ("sp_step", sp_step)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        n = max(5, min(args.steps, 20))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        res[name + "_ms"] = e0.elapsed_time(e1) / n
    pkg.timing_enable(True)
    pkg.timing_collect()
    sp_step()
    torch.cuda.synchronize()
    per = {}
    for kname, kms in pkg.timing_collect():
        per[kname] = per.get(kname, 0.0) + kms
    pkg.timing_enable(False)
    return {"workload": f"one piece of {pieces}: B={B} H={H} T={T} d_k={K} d_v={V} bf16, {w['gate']} gates",
            **res, "overhead": res["sp_step_ms"] / res["plain_step_ms"] - 1.0,
            "sp_step_kernels_ms": per,
            "allgather_bytes_per_rank_per_direction": (B * H * K * V + B * H * K) * 4}


# --------------------------------------------------------- sequence parallelism across ranks
def seqpar_bounds(T, world, chunk=64):
    """Token range [cuts[r], cuts[r+1]) of rank r's piece of a T-token sequence:
    consecutive pieces of whole chunks, as equal as the chunk count allows; the last
    piece takes the ragged tail.  Every piece holds at least one chunk."""
    n = -(-T // chunk)
    if n < world:
        raise ValueError(f"{T} tokens make {n} chunks of {chunk}: fewer than {world} pieces")
    cuts = [min(T, (n * r // world) * chunk) for r in range(world)] + [T]
    return cuts


def seqpar_step(ops, piece, h0=None, dh_final=None, group=None):
    """One training step of this rank's piece through seqpar's protocol: the forward
    (one all-gather of the pieces' summaries) then the backward (one more).  piece =
    (q, k, v, log_alpha, do) of this rank; h0 / dh_final are read on the first / the
    last rank only.  Returns (o, dq, dk, dv, dlog_alpha, h_out, dh_in)."""
    from chunkwise_linear_rnn_fwd_b200 import seqpar
    q, k, v, la, do = piece
    o, h_out, h_in = seqpar.sp_gla_fwd(q, k, v, la, h0, group=group, ops=ops)
    dq, dk, dv, dla, dh_in = seqpar.sp_gla_bwd(q, k, v, la, do, h_in, dh_final, group=group, ops=ops)
    return o, dq, dk, dv, dla, h_out, dh_in


def gather_pieces(t, cuts, group=None):
    """The whole sequence's [B, H, T, ...] tensor, on every rank, from each rank's piece
    t (token dimension 2): one all-gather of the pieces zero-padded to the longest."""
    import torch
    import torch.distributed as dist
    world = len(cuts) - 1
    if world == 1:
        return t
    lens = [cuts[r + 1] - cuts[r] for r in range(world)]
    pad = t.new_zeros(*t.shape[:2], max(lens), *t.shape[3:])
    pad[:, :, :t.shape[2]] = t
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:, :, :n] for p, n in zip(parts, lens)], dim=2)


def tensor_rel_err(a, b):
    """max |a - b| / max |b| over the whole tensor (0 for two empty or zero tensors)."""
    a, b = a.float(), b.float()
    den = b.abs().max().item() if b.numel() else 0.0
    num = (a - b).abs().max().item() if b.numel() else 0.0
    return num / den if den > 0 else num


def measure_seqpar_ranks(args, w, dev, stream, rank, world):
    """The workload's one sequence split across the job's ranks (strong scaling): rank r
    runs seqpar_step on its piece through seqpar.LibraryOps, with one NCCL all-gather
    of the pieces' summaries per direction; every rank draws the same whole-sequence
    inputs.  Returns the step's device time (max over ranks, events on the launch
    stream), the all-gather's own time and bytes, the per-kernel durations of one
    rank, the end-to-end time with this rank's piece in pinned host memory, and the
    gathered pieces compared on rank 0 with the single-GPU gla_fwd / gla_bwd of the
    whole sequence (the same library; its parity with the oracle is in tests/)."""
    import torch
    import torch.distributed as dist

    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200 import seqpar
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs

    B, H, T, K, V, C = w["B"], w["H"], w["T"], w["K"], w["V"], w["C"]
    cuts = seqpar_bounds(T, world, C)
    lo, hi = cuts[rank], cuts[rank + 1]
    x = make_inputs(B, H, T, K, V, dtype=torch.bfloat16, gate=w["gate"], seed=0, z_mean=w["z_mean"])
    whole = [None if t is None else t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha, x.do)]
    piece = [None if t is None else t[:, :, lo:hi].contiguous() for t in whole]
    ops = seqpar.LibraryOps(C, stream)
    group = None

    def step():
        return seqpar_step(ops, piece, group=group)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    n = max(5, args.steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = reduce_max_ms(e0.elapsed_time(e1), world, dev) / n

    # the exchange alone: one all-gather of (gamma, delta) as the protocol packs them
    gam = torch.rand(B, H, K, device=dev)
    dlt = torch.randn(B, H, K, V, device=dev)
    ag_ms = 0.0
    if world > 1:
        for _ in range(3):
            seqpar.gather_summaries(gam, dlt, group)
        torch.cuda.synchronize()
        dist.barrier()
        e0.record(stream)
        for _ in range(n):
            seqpar.gather_summaries(gam, dlt, group)
        e1.record(stream)
        torch.cuda.synchronize()
        ag_ms = reduce_max_ms(e0.elapsed_time(e1), world, dev) / n

    # this rank's kernels, one event pair per launch (a second pass of the same steps)
    pkg.timing_enable(True)
    pkg.timing_collect()
    for _ in range(n):
        step()
    torch.cuda.synchronize()
    launches = pkg.timing_collect()
    pkg.timing_enable(False)
    per_kernel = {}
    for name, t in launches:
        d = per_kernel.setdefault(name, [0, 0.0])
        d[0] += 1
        d[1] += t / n

    # end to end: this rank's piece from pinned host memory, its gradients and output back
    outs = step()
    host_in = [None if t is None else t.cpu().pin_memory() for t in piece]
    host_out = [None if t is None else torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs[:5]]
    h2d = sum(t.numel() * t.element_size() for t in host_in if t is not None)
    d2h = sum(t.numel() * t.element_size() for t in host_out if t is not None)

    def e2e_step():
        for dst, src in zip(piece, host_in):
            if dst is not None:
                dst.copy_(src, non_blocking=True)
        res = step()
        for dst, src in zip(host_out, res[:5]):
            if dst is not None:
                dst.copy_(src, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(n):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max_ms(e0.elapsed_time(e1), world, dev) / n

    # the gathered pieces against the whole sequence on one GPU (rank 0 compares;
    # every rank takes part in the gathers)
    outs = step()
    gathered = [None if t is None else gather_pieces(t, cuts, group) for t in outs[:5]]
    h_final = outs[5].contiguous()
    if world > 1:
        dist.broadcast(h_final, src=world - 1, group=group)
    check = None
    if rank == 0:
        q, k, v, la, do = whole
        o, hT = pkg.gla_fwd(q, k, v, la, None, chunk=C, stream=stream)
        dq, dk, dv, dla, _ = pkg.gla_bwd(q, k, v, la, do, None, None, chunk=C, stream=stream, want_dh0=False)
        torch.cuda.synchronize()
        names = ("o", "dq", "dk", "dv", "dlog_alpha")
        check = {nm: tensor_rel_err(g, r) for nm, g, r in zip(names, gathered, (o, dq, dk, dv, dla))
                 if g is not None}
        check["h_final"] = tensor_rel_err(h_final, hT)
        check["measure"] = "max |pieces - whole| / max |whole| per tensor (tensor scale)"
    if world > 1:
        dist.barrier()
    return {
        "ms_per_step": ms, "tokens_per_step": B * T, "pieces": cuts, "piece_tokens": hi - lo,
        "allgather_ms": ag_ms, "allgathers_per_step": 2 if world > 1 else 0,
        "allgather_bytes_per_rank_per_direction": (B * H * K + B * H * K * V) * 4 if world > 1 else 0,
        "kernels_ms_per_step": {k2: v2[1] for k2, v2 in per_kernel.items()},
        "gpu_launches_per_step": sum(v2[0] for v2 in per_kernel.values()) / n,
        "e2e_ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
        "vs_whole_sequence": check,
    }


def measure_general_gate(args, w, dev, stream, seed=0):
    """The general gate alpha_t^T beta_t (CUDA-core path, fp32 arithmetic) on the
    bench workload with log beta drawn like log alpha: forward + backward step time
    from events around `steps` steps (inputs larger than L2)."""
    import torch

    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs

    B, H, T, K, V = w["B"], w["H"], w["T"], w["K"], w["V"]
    x = make_inputs(B, H, T, K, V, dtype=torch.bfloat16, gate=w["gate"], seed=seed, z_mean=w["z_mean"],
                    with_log_beta=True)
    q, k, v, la, lb, do = (t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha, x.log_beta, x.do))
    wsf = pkg.alloc_workspace(pkg.general_workspace_size(B, H, T, K, V, torch.bfloat16, w["gate"], w["C"]), dev)
    wsb = pkg.alloc_workspace(pkg.general_workspace_size(B, H, T, K, V, torch.bfloat16, w["gate"], w["C"], True),
                              dev)

    def step():
        pkg.gla_fwd_general(q, k, v, la, lb, chunk=w["C"], workspace=wsf, stream=stream)
        pkg.gla_bwd_general(q, k, v, la, lb, do, chunk=w["C"], workspace=wsb, stream=stream)

    step()
    torch.cuda.synchronize()
    n = 3
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    # bound "alu": fp32 FMA on CUDA cores; peak from the unit counts and the clock
    # (148 SMs x 128 fp32 lanes x 2 FLOP x SM clock), the contraction FLOPs counted as
    # for the alpha-only step (the beta factors add only elementwise work)
    flops = B * H * T * (4 * K * V + w["C"] * (K + V) + 10 * K * V + w["C"] * (3 * K + 2 * V))
    peak = 148 * 128 * 2 * FALLBACK_PEAKS["sm_max_mhz"] * 1e6 / 1e12
    achieved = flops / (ms / 1e3) / 1e12
    return {"workload": f"general gate, B={B} H={H} T={T} d_k={K} d_v={V} bf16 in/out, {w['gate']} alpha + vector beta",
            "path": "CUDA cores, fp32 arithmetic, materialised chunk states", "ms_per_step": ms,
            "tokens_per_s": B * T / (ms / 1e3),
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz"}}


def _time_steps(fn, stream, steps, warmup=3):
    """Mean device time of fn() over `steps` calls (CUDA events on the launch stream)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def measure_variants(args, w, dev, stream, seed=0):
    """The forward/backward variants of the workload, each a whole fwd+bwd step:
    saved_states  the forward stores its bf16 chunk states, the backward reads them;
    recompute     the backward recomputes the chunk states with a forward walk of its own;
    materialized  the MATERIALIZED forward (every chunk state in fp32, then all chunk
                  outputs in parallel), the backward reading the saved bf16 states.
    All reuse the forward's prep outputs in the backward."""
    import torch

    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs

    B, H, T, K, V, C = w["B"], w["H"], w["T"], w["K"], w["V"], w["C"]
    x = make_inputs(B, H, T, K, V, dtype=torch.bfloat16, gate=w["gate"], seed=seed, z_mean=w["z_mean"])
    q, k, v, la, do = (t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha, x.do))
    o = torch.empty(B, H, T, V, dtype=torch.bfloat16, device=dev)
    dq, dk, dv, dla = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(la)
    out = {}
    n = max(5, min(args.steps, 20))
    for name, save, variant in (("saved_states", True, "auto"), ("recompute", False, "auto"),
                                ("materialized", True, "materialized")):
        flags = pkg.FLAG_REUSE_PREP | (pkg.FLAG_SAVE_STATES if save else 0)
        ws = pkg.alloc_workspace(pkg.workspace_size(B, H, T, K, V, torch.bfloat16, w["gate"], C, True, flags=flags,
                                                    variant=variant), dev)

        def fwd():
            pkg.gla_fwd(q, k, v, la, None, chunk=C, o=o, want_final=False, workspace=ws, stream=stream,
                        save_states=save, variant=variant)

        def step():
            fwd()
            pkg.gla_bwd(q, k, v, la, do, None, None, chunk=C, dq=dq, dk=dk, dv=dv, dlog_alpha=dla, want_dh0=False,
                        workspace=ws, stream=stream, reuse_prep=True, saved_states=save, variant=variant)

        out[name] = {"step_ms": _time_steps(step, stream, n), "fwd_ms": _time_steps(fwd, stream, n)}
        del ws
    out["workload"] = (f"B={B} H={H} T={T} d_k={K} d_v={V} C={C} bf16, {w['gate']} gates; fwd+bwd and fwd alone, "
                       "device time per call")
    return out


SWEEP_T = [dict(name=f"config 5: fwd+bwd, B*T=32768 H=4 d_k=256 d_v=512, T={T}", B=32768 // T, H=4, T=T, K=256,
                V=512, gate=g, z_mean=0.0, bwd=True)
           for T in (1024, 2048, 4096, 8192, 16384) for g in ("vector", "scalar", "none")]


def time_workload(c, args, dev, stream, peaks, C=64):
    """Device time of one workload configuration `c` (dict with B, H, T, K, V, gate,
    z_mean, bwd): the forward (and backward) as bench.py's step launches them, inputs
    drawn on the device with the workload's distributions (timing only; parity is in
    tests/)."""
    import torch

    import chunkwise_linear_rnn_fwd_b200 as pkg

    B, H, T, K, V = c["B"], c["H"], c["T"], c["K"], c["V"]
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    q = torch.randn(B, H, T, K, device=dev, generator=g).to(torch.bfloat16)
    k = (torch.randn(B, H, T, K, device=dev, generator=g) / K ** 0.5).to(torch.bfloat16)
    v = torch.randn(B, H, T, V, device=dev, generator=g).to(torch.bfloat16)
    do = torch.randn(B, H, T, V, device=dev, generator=g).to(torch.bfloat16)
    shape = {"vector": (B, H, T, K), "scalar": (B, H, T)}.get(c["gate"])
    la = None if shape is None else torch.nn.functional.logsigmoid(
        torch.randn(*shape, device=dev, generator=g) + c["z_mean"]) / 16
    o = torch.empty_like(v)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dla = None if la is None else torch.empty_like(la)
    flags = pkg.FLAG_REUSE_PREP | pkg.FLAG_SAVE_STATES if c["bwd"] else 0
    ws = pkg.alloc_workspace(pkg.workspace_size(B, H, T, K, V, torch.bfloat16, c["gate"], C, c["bwd"],
                                                flags=flags), dev)

    def step():
        pkg.gla_fwd(q, k, v, la, None, chunk=C, gate=c["gate"], o=o, want_final=False, workspace=ws,
                    stream=stream, save_states=c["bwd"])
        if c["bwd"]:
            pkg.gla_bwd(q, k, v, la, do, None, None, chunk=C, gate=c["gate"], dq=dq, dk=dk, dv=dv,
                        dlog_alpha=dla, want_dh0=False, workspace=ws, stream=stream, reuse_prep=True,
                        saved_states=True)

    ms = _time_steps(step, stream, args.steps, max(3, args.warmup))
    th = B * H * T
    flops = th * (4 * K * V + C * (K + V)) + (th * (10 * K * V + C * (3 * K + 2 * V)) if c["bwd"] else 0)
    abytes = algorithmic_bytes(B, H, T, K, V, c["gate"]) if c["bwd"] else th * (4 * K + 4 * V) + (
        th * 4 * K if c["gate"] == "vector" else (th * 4 if c["gate"] == "scalar" else 0))
    peak_t = float(peaks.get("bf16_tflops", 1590)) * 1e12
    peak_b = float(peaks["hbm_gbs"]) * 1e9
    return {"workload": c["name"], "gate": c["gate"], "ms_per_step": ms, "tokens_per_s": B * T / (ms / 1e3),
            "tflops": flops / (ms / 1e3) / 1e12, "frac_of_tensor_peak": flops / (ms / 1e3) / peak_t,
            "frac_of_roofline": max(flops / peak_t, abytes / peak_b) / (ms / 1e3)}


def measure_e2e(args, x, step_on, dev_in, dev_out, stream, world, dev):
    """The step end to end through the public API with the inputs in pinned host
    memory and the results read back to it, every step: a copy-in stream, the compute
    stream and a copy-out stream with two sets of device buffers, so that step j's
    computation overlaps the copy-in of step j + 1 and the copy-out of step j - 1
    (each on its own copy engine).  Timed with events from the first copy-in to the
    last copy-out (max over ranks).  Also the same steps with the copies and the
    computation in one stream (serial_ms_per_step), for comparison."""
    import torch
    import torch.distributed as dist

    pin = lambda t: t.cpu().pin_memory()
    h_in = [pin(t) for t in (x.q, x.k, x.v, x.log_alpha, x.do)]
    h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dev_out]
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    ins = [list(dev_in), [torch.empty_like(t) for t in dev_in]]
    outs = [list(dev_out), [torch.empty_like(t) for t in dev_out]]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    in_ready, done, out_copied = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for b in range(2):  # every buffer starts free
        done[b].record(stream)
        out_copied[b].record(stream)

    def run(n):
        for j in range(n):
            b = j & 1
            s_in.wait_event(done[b])  # step j - 2 has read these inputs
            with torch.cuda.stream(s_in):
                for dst, src in zip(ins[b], h_in):
                    dst.copy_(src, non_blocking=True)
            in_ready[b].record(s_in)
            stream.wait_event(in_ready[b])
            stream.wait_event(out_copied[b])  # step j - 2's results have left these outputs
            step_on(ins[b], outs[b], stream)
            done[b].record(stream)
            s_out.wait_event(done[b])
            with torch.cuda.stream(s_out):
                for dst, src in zip(h_out, outs[b]):
                    dst.copy_(src, non_blocking=True)
            out_copied[b].record(s_out)

    run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    n = max(2, args.steps // 2)
    f0, f1 = ev(), ev()
    f0.record(s_in)
    run(n)
    f1.record(s_out)
    torch.cuda.synchronize()
    ms_total = reduce_max_ms(f0.elapsed_time(f1), world, dev)

    # the serial form: copy-in, step, copy-out on the compute stream
    def serial():
        for dst, src in zip(ins[0], h_in):
            dst.copy_(src, non_blocking=True)
        step_on(ins[0], outs[0], stream)
        for dst, src in zip(h_out, outs[0]):
            dst.copy_(src, non_blocking=True)

    serial()
    torch.cuda.synchronize()
    g0, g1 = ev(), ev()
    g0.record(stream)
    for _ in range(n):
        serial()
    g1.record(stream)
    torch.cuda.synchronize()
    serial_ms = reduce_max_ms(g0.elapsed_time(g1), world, dev) / n
    return {"steps": n, "ms_total": ms_total, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "serial_ms_per_step": serial_ms,
            "pipeline": "copy-in, compute and copy-out streams, two device buffer sets: step j overlaps the "
                        "copy-in of step j+1 and the copy-out of step j-1"}


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import chunkwise_linear_rnn_fwd_b200 as pkg
    from chunkwise_linear_rnn_fwd_b200.synth import make_inputs

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pkg.load()

    B, H, T, K, V, C = w["B"], w["H"], w["T"], w["K"], w["V"], w["C"]
    x = make_inputs(B, H, T, K, V, dtype=torch.bfloat16, gate=w["gate"], seed=rank, z_mean=w["z_mean"])
    q, k, v, la, do = (t.to(dev) for t in (x.q, x.k, x.v, x.log_alpha, x.do))
    o = torch.empty(B, H, T, V, dtype=torch.bfloat16, device=dev)
    hT = torch.empty(B, H, K, V, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dla = torch.empty_like(la)
    # one workspace for both calls: the forward stores its bf16 chunk states there
    # (GLA_FLAG_SAVE_STATES) and the backward reads them and the forward's per-chunk
    # prep outputs (GLA_FLAG_REUSE_PREP) instead of recomputing them
    flags = pkg.FLAG_REUSE_PREP | pkg.FLAG_SAVE_STATES
    ws = pkg.alloc_workspace(pkg.workspace_size(B, H, T, K, V, torch.bfloat16, w["gate"], C, True, flags=flags), dev)
    stream = torch.cuda.current_stream()

    def step_on(ins, outs, st):
        """One training step of the workload: gla_fwd then gla_bwd on `st`, inputs
        (q, k, v, log_alpha, do) and outputs (o, dq, dk, dv, dlog_alpha) as given."""
        qq, kk, vv, ll, dd = ins
        oo, dqq, dkk, dvv, dll = outs
        pkg.gla_fwd(qq, kk, vv, ll, None, chunk=C, o=oo, h_final=hT, workspace=ws, stream=st, save_states=True)
        pkg.gla_bwd(qq, kk, vv, ll, dd, None, None, chunk=C, dq=dqq, dk=dkk, dv=dvv, dlog_alpha=dll, want_dh0=False,
                    workspace=ws, stream=st, reuse_prep=True, saved_states=True)

    def step():
        step_on((q, k, v, la, do), (o, dq, dk, dv, dla), stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- timed region: K steps bracketed by device events on the launch stream ----------
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_local = e0.elapsed_time(e1)
    clocks = sampler.stop()

    # ---- per-kernel durations: the same K steps again with a CUDA-event pair around
    # every launch (on the launch stream).  The pairs keep a kernel from starting while
    # its predecessor drains, so this pass gives each kernel's duration, not the step time.
    pkg.timing_enable(True)
    pkg.timing_collect()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    launches = pkg.timing_collect()
    pkg.timing_enable(False)
    ms = reduce_max_ms(ms_local, world, dev)
    ms_per_step = ms / args.steps
    value = aggregate_value(B * T, world, args.steps, ms)

    # ---- end to end through the public API with host buffers ----------------------------
    e2e = measure_e2e(args, x, step_on, (q, k, v, la, do), (o, dq, dk, dv, dla), stream, world, dev)
    e2e_value = aggregate_value(B * T, world, e2e["steps"], e2e["ms_total"])

    # ---- roofline of the dominant kernel --------------------------------------------------
    peaks, peak_src = load_peaks()
    per_kernel = {}
    for name, t in launches:
        d = per_kernel.setdefault(name, [0, 0.0])
        d[0] += 1
        d[1] += t
    dom = max(per_kernel.items(), key=lambda kv: kv[1][1])[0] if per_kernel else None
    roofline = None
    if dom is not None:
        n_l, tot = per_kernel[dom]
        avg_ms = tot / n_l
        launches_per_step = n_l / args.steps
        alg = kernel_alg_bytes(dom, w)
        io = kernel_io_bytes(dom, w, torch.cuda.get_device_properties(dev).multi_processor_count)
        if alg is not None:
            # achieved = the kernel's algorithmic bytes per launch / its mean launch time
            alg_launch = alg / launches_per_step
            achieved = alg_launch / (avg_ms / 1e3) / 1e9
            peak = float(peaks["hbm_gbs"])
            roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak, "traffic": measured_traffic(dom), "peak_source": peak_src,
                        "bytes_per_launch": alg_launch, "bytes_source": "algorithmic share (no workspace)",
                        "launches_per_step": launches_per_step, "avg_launch_ms": avg_ms}
            if io is not None:
                # the same kernel's own input + output bytes, workspace included
                roofline["bytes_per_launch_incl_workspace"] = io
                roofline["frac_incl_workspace"] = io / (avg_ms / 1e3) / 1e9 / peak
    flops = counted_flops(B, H, T, K, V, C)
    abytes = algorithmic_bytes(B, H, T, K, V, w["gate"])
    t_tensor = flops / (float(peaks.get("bf16_tflops", 1590)) * 1e12)
    t_hbm = abytes / (float(peaks["hbm_gbs"]) * 1e9)
    step_s = ms_per_step / 1e3
    step_roofline = {
        "bound": "hbm" if t_hbm >= t_tensor else "tensor", "tflops": flops / step_s / 1e12,
        "frac_of_tensor_peak": (flops / step_s) / (float(peaks.get("bf16_tflops", 1590)) * 1e12),
        "gbs_algorithmic": abytes / step_s / 1e9, "frac_of_roofline": max(t_hbm, t_tensor) / step_s,
        "flops_per_step": flops, "algorithmic_bytes_per_step": abytes, "peak_source": peak_src,
    }

    decode = epilogue = seqpar = variants = general = sweep_T = None
    if not args.step_only:
        decode = measure_decode(args, dev, stream, peaks, peak_src, seed=rank)
        epilogue = measure_epilogue(args, w, dev, stream, peaks, peak_src, seed=rank)
        seqpar = measure_seqpar(args, w, dev, stream, seed=rank)
        if world > 1:
            # the same job, one sequence split across its ranks (all ranks take part)
            seqpar["ranks"] = measure_seqpar_ranks(args, w, dev, stream, rank, world)
        variants = measure_variants(args, w, dev, stream, seed=rank)
        sweep_args = argparse.Namespace(steps=5, warmup=2)
        sweep_T = [time_workload(c, sweep_args, dev, stream, peaks) for c in SWEEP_T]
        general = measure_general_gate(args, w, dev, stream, seed=rank)
        general["vs_alpha_only_step"] = general["ms_per_step"] / ms_per_step

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.step_only:
        r, dt, threads, desc = oracle_sample_rate(w, T_sample=w["T"], min_seconds=args.cpu_seconds)
        cpu = {"value": r, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc, "seconds": dt,
               **host_cpu()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(w, world),
            "tflops": step_roofline["tflops"], "step_roofline": step_roofline, "roofline": roofline,
            "kernels": {k2: {"launches": v2[0], "ms_total": v2[1], "share": v2[1] / max(1e-9, sum(x[1] for x in per_kernel.values()))}
                        for k2, v2 in sorted(per_kernel.items(), key=lambda kv: -kv[1][1])},
            "gpu_launches": len(launches),
            "kernel_timing": "separate pass of the same K steps with a CUDA-event pair around each launch",
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                    "d2h_bytes_per_step": e2e["d2h_bytes_per_step"], "ms_per_step": e2e["ms_total"] / e2e["steps"],
                    "pipeline": e2e["pipeline"], "serial_ms_per_step": e2e["serial_ms_per_step"]},
            "clocks": clocks, "cpu_baseline": cpu, "decode_step": decode, "layer_epilogue": epilogue,
            "sequence_parallel": seqpar, "general_gate": general, "variants": variants,
            "sweep_vs_T": None if sweep_T is None else {
                "workloads": sweep_T, "steps": 5, "peak_source": peak_src,
                "l2": "inputs larger than L2 (B*T = 32768 tokens, >= 1 GB per step)"},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_seqpar(args, w):
    """--seqpar: one JSON line for the workload's sequence split across the job's ranks
    (strong scaling; value = the sequence's tokens per second of the slowest rank)."""
    import torch
    import torch.distributed as dist

    import chunkwise_linear_rnn_fwd_b200 as pkg

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pkg.load()
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    r = measure_seqpar_ranks(args, w, dev, stream, rank, world)
    clocks = sampler.stop()
    peaks, peak_src = load_peaks()
    ms = r["ms_per_step"]
    B, H, T, K, V, C = w["B"], w["H"], w["T"], w["K"], w["V"], w["C"]
    kms = r["kernels_ms_per_step"]
    roofline = None
    if kms:
        dom = max(kms, key=kms.get)
        wp = dict(w, T=r["piece_tokens"])
        alg = kernel_alg_bytes(dom, wp)
        if alg is not None:
            achieved = alg / (kms[dom] / 1e3) / 1e9
            peak = float(peaks["hbm_gbs"])
            roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak, "traffic": None, "peak_source": peak_src,
                        "bytes_source": "algorithmic share of rank 0's piece (no workspace)",
                        "ms_per_step": kms[dom]}
    flops = counted_flops(B, H, T, K, V, C)
    if rank == 0:
        line = {
            "metric": METRIC, "value": B * T / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": max(5, args.steps), "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(bench_config(w, 1), parallelism=f"sequence x{world}",
                           pieces=r["pieces"]),
            "tflops": flops / (ms / 1e3) / 1e12, "roofline": roofline,
            "gpu_launches": int(round(r["gpu_launches_per_step"] * max(5, args.steps))),
            "e2e": {"value": B * T / (r["e2e_ms_per_step"] / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": r["h2d_bytes_per_step"] * world,
                    "d2h_bytes_per_step": r["d2h_bytes_per_step"] * world},
            "clocks": clocks, "cpu_baseline": None, "sequence_parallel_ranks": r,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


SWEEP = ([dict(name="config 2: fwd, B=8 H=4 T=2048 d_k=128 d_v=256", B=8, H=4, T=2048, K=128, V=256, gate=g,
               z_mean=0.0, bwd=False) for g in ("vector", "none")]
         + [dict(name="config 3: fwd+bwd, B=8 H=4 T=2048 d_k=128 d_v=256", B=8, H=4, T=2048, K=128, V=256,
                 gate="vector", z_mean=0.0, bwd=True)]
         + [dict(name="config 4: fwd+bwd, B=2 H=4 T=4096 d_k=256 d_v=512", B=2, H=4, T=4096, K=256, V=512,
                 gate="vector", z_mean=-1.0, bwd=True)]
         + SWEEP_T)


def run_sweep(args):
    """Device time of every workload configuration (one JSON line, --sweep)."""
    import torch

    import chunkwise_linear_rnn_fwd_b200 as pkg

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    pkg.load()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()
    out = [time_workload(c, args, dev, stream, peaks) for c in SWEEP]
    print(json.dumps({"metric": METRIC, "sweep": out, "peak_source": peak_src}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--ref-tokens", type=int, default=1024, help="tokens per head in the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="minimum oracle time of the CPU baseline")
    ap.add_argument("--batch", type=int, default=None, help="override B (smaller profiling captures)")
    ap.add_argument("--heads", type=int, default=None, help="override H")
    ap.add_argument("--seqlen", type=int, default=None, help="override T")
    ap.add_argument("--sweep", action="store_true", help="time every workload configuration (one JSON line)")
    ap.add_argument("--seqpar", action="store_true",
                    help="split the workload's sequence across the job's ranks (sequence parallelism, one NCCL "
                         "all-gather per direction; strong scaling) instead of running a replica per rank")
    ap.add_argument("--step-only", action="store_true",
                    help="time the fwd+bwd step alone (no decode, epilogue, sequence-parallel, variant, sweep, "
                         "general-gate or CPU measurements): the command line of the profiler captures")
    ap.add_argument("--fused-epilogue-once", action="store_true",
                    help="run gla_fwd_epilogue (the forward with the layer epilogue fused into its output store) "
                         "three times on the workload and exit (a small case for profiler captures; prints no "
                         "bench line)")
    ap.add_argument("--epilogue-once", action="store_true",
                    help="run the layer epilogue forward and backward twice on the workload's output shape and "
                         "exit (a small case for profiler captures; prints no bench line)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = dict(WORKLOAD)
    for key, val in (("B", args.batch), ("H", args.heads), ("T", args.seqlen)):
        if val is not None:
            w[key] = val
    if args.impl == "reference":
        return run_reference(args, w)
    if args.sweep:
        return run_sweep(args)
    if args.epilogue_once:
        return run_epilogue_once(w)
    if args.fused_epilogue_once:
        return run_fused_epilogue_once(w)
    if args.seqpar:
        return run_seqpar(args, w)
    return run_ours(args, w)


def run_fused_epilogue_once(w):
    """Three calls of gla_fwd_epilogue on the workload (inputs drawn on the device),
    then the device status word.  Launch order per call: prep, pre-pass walk, start
    fold, fused output walk."""
    import torch

    import chunkwise_linear_rnn_fwd_b200 as pkg

    dev = torch.device("cuda", 0)
    B, H, T, K, V, C = w["B"], w["H"], w["T"], w["K"], w["V"], w["C"]
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    q = torch.randn(B, H, T, K, device=dev, generator=g).to(torch.bfloat16)
    k = (torch.randn(B, H, T, K, device=dev, generator=g) / K ** 0.5).to(torch.bfloat16)
    v, r = (torch.randn(B, H, T, V, device=dev, generator=g).to(torch.bfloat16) for _ in range(2))
    la = torch.nn.functional.logsigmoid(torch.randn(B, H, T, K, device=dev, generator=g) + w["z_mean"]) / 16
    ws = pkg.alloc_workspace(pkg.workspace_size(B, H, T, K, V, torch.bfloat16, w["gate"], C, False), dev)
    for _ in range(3):
        pkg.gla_fwd_epilogue(q, k, v, la, r, workspace=ws, chunk=C)
    torch.cuda.synchronize()
    st = pkg.poll_status(ws)
    print(json.dumps({"fused_epilogue_once": {"B": B, "H": H, "T": T, "d_k": K, "d_v": V, "status": st}}))
    return 0 if st == 0 else 1


def run_epilogue_once(w):
    """Two forward + backward calls of the layer epilogue on [B,H,T,d_v] bf16 inputs,
    then the device status word.  Launch order: fwd, bwd, reduce, fwd, bwd, reduce."""
    import torch

    import chunkwise_linear_rnn_fwd_b200 as pkg

    dev = torch.device("cuda", 0)
    B, H, T, V = w["B"], w["H"], w["T"], w["V"]
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    o, r, dy = (torch.randn(B, H, T, V, device=dev, generator=g).to(torch.bfloat16) for _ in range(3))
    wt, bs = torch.ones(V, device=dev), torch.zeros(V, device=dev)
    ws = pkg.alloc_workspace(pkg.epilogue_workspace_size(B, H, T, V, torch.bfloat16), dev)
    for _ in range(2):
        pkg.gla_epilogue_fwd(o, r, wt, bs, workspace=ws)
        pkg.gla_epilogue_bwd(o, r, dy, wt, bs, workspace=ws)
    torch.cuda.synchronize()
    st = pkg.poll_status(ws)
    print(json.dumps({"epilogue_once": {"B": B, "H": H, "T": T, "d_v": V, "status": st}}))
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
