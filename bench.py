"""Benchmark of the Swimba layer forward on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl swimba|reference] [--workload NAME]

A step is one swimba_layer_fwd (router -> dispatch -> expert projections with the fused mix ->
chunked scan) over one batch of synthetic inputs already resident in HBM.  Default workload: the base
layer B4 T2048 D768 H24 P64 N128 E8 k2 Q256 (bf16 weights and activations, fp32 state).  With N > 1
(torchrun) every rank runs its own batch (weak scaling, no data-path collective; the process group only
carries the barrier and the max-over-ranks of the timings).

On one GPU the default run adds two nested measurements to the same JSON line, timed the same way:
"decode" (swimba_step on 256 sequences, D2048 H64 N128 P64 E16 k2, state from a 512-token prefill; bound
by HBM), "esweep" (the base layer at E in {8, 16, 32, 64}: layer and scan-stage times, which the
method's cost statement says are flat in E, plus the separated-trajectory scan that runs k trajectories) and
"out_proj" (the output projection y W_out^T on the base layer's y, bound by the tensor cores), "mixed_A"
(the base layer with the expert-mixed transition A~ = sum_j pi_j A_exp[K_j]), "groups" (the base layer
with B and C shared by G in {H, H/4, 1} groups of heads: layer and scan times), "scan_bwd" (the scan
gradients at the base sizes, bound by fp32 CUDA-core arithmetic) and "layer_bwd" (the whole layer's gradients
at the base workload, tensor-core expert products plus CUDA-core scan gradients).

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events on the launching stream,
with a write of 2x the L2 size between steps (outside the events) so every step reads its inputs from
HBM.  A second pass of K steps with the library's own per-stage events on gives the stage breakdown and
the dominant kernel's duration for the roofline (the headline pass records no stage events).
`--impl reference` times the fp64 CPU oracle (the reference for this layer) on a bounded sample.
"""
import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from parameter_space_moe_b200 import configs, inputs  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------------ work model

def scan_chunk_of(w):
    """Chunk length the scan actually solves in: the tensor-core scan (bf16, N = 128, P in {64, 128})
    always uses 128-token sub-chunks; the CUDA-core scan uses the workload's chunk."""
    if w.dtype == "bf16" and w.dstate == 128 and w.headdim in (64, 128):
        return 128
    return w.chunk


def ssd_flops(w, T=None):
    """Algorithmic FLOPs of the chunked solve at the chunk length the kernel runs (causal half of the
    intra-chunk products counted)."""
    T = T or w.seqlen
    Q, k, N, P = scan_chunk_of(w), w.top_k, w.dstate, w.headdim
    total = 0
    for c in range(math.ceil(T / Q)):
        L = min(Q, T - c * Q)
        tri = L * (L + 1) / 2
        total += 2 * tri * k * N + 2 * tri * k * P + 2 * N * P * k * L + 2 * L * N * P
    return total * w.batch * w.nheads


def work(w):
    """Per-step algorithmic FLOPs and bytes of each stage and of the layer."""
    M, D, E, H, k = w.M, w.d_model, w.n_experts, w.nheads, w.top_k
    ab = 2 if w.dtype == "bf16" else 4          # activation / weight bytes
    sb = 2 if w.dtype == "bf16" else 4          # stream bytes (fp16 or fp32)
    used_experts = E if M * k >= 4 * E else min(E, M * k)
    gemm_flops = 2.0 * M * k * D * w.W_e
    streams = M * k * (2 * w.G * w.dstate + H * w.headdim) * sb
    states = w.batch * H * w.dstate * w.headdim * 4
    layer_bytes = (M * D * ab + used_experts * w.W_e * D * ab + (E + H) * D * ab + M * H * w.headdim * ab + states)
    return {
        "router": {"flops": 2.0 * M * D * (E + H), "bytes": M * D * ab + (E + H) * D * ab + M * (2 * k + H) * 4},
        "expert_proj_mix": {"flops": gemm_flops, "bytes": M * k * D * ab + used_experts * w.W_e * D * ab + streams},
        "ssd_scan": {"flops": ssd_flops(w), "bytes": streams + M * H * 4 + M * H * w.headdim * ab + states},
        "layer": {"flops": 2.0 * M * D * (E + H) + gemm_flops + ssd_flops(w), "bytes": layer_bytes},
    }


def decode_work(w):
    """Per-step algorithmic FLOPs and bytes of the recurrent decode step (one token per sequence)."""
    B, D, E, H, k, N, P = w.batch, w.d_model, w.n_experts, w.nheads, w.top_k, w.dstate, w.headdim
    used = min(E, B * k)
    weights = used * w.W_e * D * 2
    streams = B * k * (2 * w.G * N + H * P) * 2
    state = 2 * B * H * N * P * 4
    return {
        "router": {"flops": 2.0 * B * D * (E + H), "bytes": B * D * 2 + (E + H) * D * 2},
        "expert_proj_mix": {"flops": 2.0 * B * k * D * w.W_e, "bytes": weights + streams + B * k * D * 2},
        "state_update": {"flops": 2.0 * B * H * N * P * (k + 1), "bytes": state + streams + B * H * P * 2},
        "layer": {"flops": 2.0 * B * k * D * w.W_e + 2.0 * B * D * (E + H),
                  "bytes": weights + state + B * D * 2 + B * H * P * 2},
    }


# ------------------------------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock, power and throttle reasons through NVML every ~10 ms while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                util = self.nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, util))
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        loaded = [m for m, u in self.samples if u > 0] or [m for m, _ in self.samples]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------ reference arm

def cpu_oracle_sample(w, inp, budget_s=20.0, min_tokens=256):
    """Time the fp64 oracle on the first batch rows of the workload that fit ~budget_s of CPU work."""
    from oracle import swimba_oracle as O
    f = inputs.to_f64
    wt = [f(inp[k]) for k in ("W_r", "W_dt", "b_dt", "A", "W_exp")]
    T = w.seqlen if w.seqlen <= min_tokens else min_tokens
    t0 = time.perf_counter()
    O.layer_fwd(f(inp["X"][:1, :T]), *wt, w.nheads, w.headdim, w.dstate, w.G, w.top_k)
    probe = time.perf_counter() - t0
    per_token = probe / T
    rows = max(1, min(w.batch, int(budget_s / (per_token * w.seqlen))))
    if per_token * w.seqlen > budget_s:
        rows, T = 1, max(T, int(budget_s / per_token))
    else:
        T = w.seqlen
    X = f(inp["X"][:rows, :T])
    t0 = time.perf_counter()
    O.layer_fwd(X, *wt, w.nheads, w.headdim, w.dstate, w.G, w.top_k)
    dt = time.perf_counter() - t0
    return rows * T / dt, f"{rows} batch row(s) x {T} tokens of {w.name} ({rows * T} tokens), fp64 oracle"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, w):
    rank, _, _ = rank_env()
    if rank != 0:  # under torchrun only rank 0 times the oracle; the others exit without work
        return
    inp = inputs.make_inputs(w)
    from oracle import swimba_oracle as O
    f = inputs.to_f64
    wt = [f(inp[k]) for k in ("W_r", "W_dt", "b_dt", "A", "W_exp")]
    T = min(w.seqlen, 256)
    X = f(inp["X"][:1, :T])
    for _ in range(args.warmup):
        O.layer_fwd(X, *wt, w.nheads, w.headdim, w.dstate, w.G, w.top_k)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.layer_fwd(X, *wt, w.nheads, w.headdim, w.dstate, w.G, w.top_k)
        times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = args.steps * T / tot
    sample = f"each step: 1 batch row x {T} tokens of {w.name}, fp64 oracle"
    cores = blas_threads()
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ------------------------------------------------------------------------------------------ GPU arm

METRIC = "Swimba layer fwd tokens/s (E=8,k=2,T=2048); % of tensor/HBM roofline"


def config_of(w):
    return {"workload": w.name, "batch": w.batch, "seq_len": w.seqlen, "d_model": w.d_model, "nheads": w.nheads,
            "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.G, "n_experts": w.n_experts, "top_k": w.top_k,
            "chunk": w.chunk, "l2": "flushed between steps (2x L2 write outside the timed events)"}


class LayerSession:
    """Forward-pass workloads: one step = swimba_layer_fwd over B x T tokens."""

    def __init__(self, w, dev, inp, swimba, mixed_A=False):
        self.w, self.sw = w, swimba
        self.d = swimba.dims_of(w)
        self.W = swimba.WeightSet(*(inp[k].to(dev) for k in ("W_r", "W_dt", "b_dt", "A", "W_exp")),
                                  A_exp=inp["A_exp"].to(dev) if mixed_A else None)
        self.X = inp["X"].to(dev).reshape(w.M, w.d_model)
        odt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.y = torch.empty(w.M, w.nheads * w.headdim, dtype=odt, device=dev)
        self.fin = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, device=dev)
        self.ws = torch.empty(swimba.workspace_size(self.d), dtype=torch.uint8, device=dev)
        self.Xh = inp["X"].reshape(w.M, w.d_model).pin_memory()
        self.yh = torch.empty(self.y.shape, dtype=odt).pin_memory()
        self.tokens = w.M
        self.metric = METRIC
        self.work = work(w)

    def step(self):
        self.sw.layer_fwd(self.d, self.X, self.W, None, self.y, self.fin, None, None, self.ws)

    def e2e_step(self):
        """Host X in, host y out through swimba_layer_fwd_host: 4 time segments of every sequence chained
        through the final state, each segment's copies overlapping another segment's compute."""
        self.sw.layer_fwd_host(self.d, self.Xh, self.W, None, self.yh, self.fin, self.X, self.y, self.ws, chunks=4)

    def extras(self, stream, steps):
        """Separated-trajectory variant ("k scans") on this layer's streams, timed alone."""
        w, sw = self.w, self.sw
        sdt = torch.float16 if w.dtype == "bf16" else torch.float32
        dev = self.X.device
        idx = torch.empty(w.M, w.top_k, dtype=torch.int32, device=dev)
        wts = torch.empty(w.M, w.top_k, device=dev)
        dt = torch.empty(w.M, w.nheads, device=dev)
        sw.router_topk(self.d, self.X, self.W, idx, wts, dt)
        Z = torch.empty(w.M, w.top_k, w.W_e, device=dev)
        sw.expert_proj(self.d, self.X, self.W, idx, Z, self.ws)
        B = torch.empty(w.M, w.top_k, w.G, w.dstate, dtype=sdt, device=dev)
        Xs = torch.empty(w.M, w.top_k, w.nheads, w.headdim, dtype=sdt, device=dev)
        C = torch.empty_like(B)
        sw.mix(self.d, Z, wts, sw.MIX_UNSCALED_B, B, Xs, C)
        del Z
        A = self.W.tensors[3]
        ys = torch.empty_like(self.y)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(3):
            sw.separated_scan(self.d, B, Xs, C, dt, A, None, ys, None, self.ws)
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(steps):
            e0.record(stream)
            sw.separated_scan(self.d, B, Xs, C, dt, A, None, ys, None, self.ws)
            e1.record(stream)
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        return {"separated_scan_ms": tot / steps, "separated_trajectories": w.top_k, "mixed_trajectories": 1}


class DecodeSession:
    """Recurrent decode: one step = swimba_step, one new token for each of `batch` sequences, on a state
    built by a prefill of `prefill` tokens through swimba_layer_fwd."""

    def __init__(self, w, dev, inp, swimba):
        self.w, self.sw = w, swimba
        self.W = swimba.WeightSet(*(inp[k].to(dev) for k in ("W_r", "W_dt", "b_dt", "A", "W_exp")))
        dp = swimba.dims_of(w, seqlen=w.prefill)
        Mp = w.batch * w.prefill
        self.state = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, device=dev)
        wsp = torch.empty(swimba.workspace_size(dp), dtype=torch.uint8, device=dev)
        yp = torch.empty(Mp, w.nheads * w.headdim, dtype=torch.bfloat16, device=dev)
        swimba.layer_fwd(dp, inp["X"].to(dev).reshape(Mp, w.d_model), self.W, None, yp, self.state, None, None, wsp)
        torch.cuda.synchronize()
        del wsp, yp
        torch.cuda.empty_cache()  # the prefill's workspace goes back to the driver: the step needs far less
        self.d = swimba.dims_of(w, seqlen=1)
        self.X = inp["X_step"].to(dev)
        self.y = torch.empty(w.batch, w.nheads * w.headdim, dtype=torch.bfloat16, device=dev)
        self.ws = torch.empty(swimba.workspace_size(self.d), dtype=torch.uint8, device=dev)
        self.Xh = inp["X_step"].pin_memory()
        self.yh = torch.empty(self.y.shape, dtype=self.y.dtype).pin_memory()
        self.tokens = w.batch
        self.metric = "Swimba decode step tokens/s (256 seqs, H64 N128 P64 E16 k2); % of HBM roofline"
        self.work = decode_work(w)

    def step(self):
        self.sw.step(self.d, self.X, self.W, self.state, self.y, None, self.ws)

    def e2e_step(self):
        """Host X in, host y out: copy, swimba_step, copy back (one step is too small to split)."""
        self.X.copy_(self.Xh, non_blocking=True)
        self.step()
        self.yh.copy_(self.y, non_blocking=True)

    def extras(self, stream, steps):
        return {}


def rank_env():
    """(rank, world size, local rank) from the torchrun environment (1 process when absent)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_workload(w, rank):
    """Weak scaling: every rank runs the same shapes on its own batch (its own input seed)."""
    return w.with_(seed=w.seed + 1000 * rank)


def max_over_ranks(values, dist, device):
    """Element-wise maximum of a list of floats over all ranks (the job's time is its slowest rank's)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(tokens_per_rank, world, steps, total_ms):
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank * world * steps / (total_ms / 1e3)


def measure(sess, args, flush, stream, dist, local, swimba, e2e=True):
    """Warm-up, then K device-timed steps (L2 flushed between steps, outside the events), a second pass of K
    steps with the library's stage events on (so the headline carries no profiling events), and K end-to-end
    steps through the host-memory entry point.  Times are this rank's totals in milliseconds."""
    for _ in range(args.warmup):
        sess.step()
    torch.cuda.synchronize()
    assert swimba.check_device_status() == 0
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = swimba.launch_count()
    with sampler:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            sess.step()
            ends[i].record(stream)
        torch.cuda.synchronize()
    launches = swimba.launch_count() - n0
    if dist:
        dist.barrier()
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    assert swimba.check_device_status() == 0

    stage_ms = {}
    swimba.profile_enable(True)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        sess.step()
        for name, ms in swimba.profile_read():
            stage_ms[name] = stage_ms.get(name, 0.0) + ms
    torch.cuda.synchronize()
    swimba.profile_enable(False)

    e2e_ms = None
    if e2e:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(2):
            sess.e2e_step()
        torch.cuda.synchronize()
        e2e_ms = 0.0
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            e0.record(stream)
            sess.e2e_step()
            e1.record(stream)
            e1.synchronize()
            e2e_ms += e0.elapsed_time(e1)
    assert swimba.check_device_status() == 0
    return {"total_ms": total_ms, "stage_ms": stage_ms, "launches": launches, "clocks": sampler.summary(),
            "e2e_ms": e2e_ms}


def esweep_measure(args, dev, flush, stream, swimba):
    """The base layer at E in {8, 16, 32, 64}: per-step layer and stage times (the scan's work does not
    depend on E), plus the separated-trajectory scan ("k scans") at E = 8 on the same streams."""
    out = {"E": [], "layer_ms": [], "scan_ms": [], "expert_proj_ms": [], "scan_roofline_frac": []}
    peaks, _ = load_peaks()
    for E in configs.ESWEEP_E:
        w = configs.esweep(E)
        sess = LayerSession(w, dev, inputs.make_inputs(w), swimba)
        m = measure(sess, args, flush, stream, None, dev.index or 0, swimba, e2e=False)
        K = args.steps
        scan_s = m["stage_ms"].get("ssd_scan", 0.0) / K / 1e3
        out["E"].append(E)
        out["layer_ms"].append(m["total_ms"] / K)
        out["scan_ms"].append(scan_s * 1e3)
        out["expert_proj_ms"].append(m["stage_ms"].get("expert_proj_mix", 0.0) / K)
        out["scan_roofline_frac"].append(sess.work["ssd_scan"]["bytes"] / scan_s / 1e9 / peaks["hbm_gbs"])
        if E == configs.ESWEEP_E[0]:
            sep = sess.extras(stream, args.steps)
            out["separated_scan_ms"] = sep["separated_scan_ms"]
            out["trajectories"] = {"mixed": sep["mixed_trajectories"], "separated": sep["separated_trajectories"]}
        del sess
        torch.cuda.empty_cache()
    out["scan_ms_spread"] = max(out["scan_ms"]) / min(out["scan_ms"]) - 1.0
    return out


def scan_bwd_flops(w):
    """FLOPs the scan-gradient kernels execute (2 per FMA), 64-token sub-chunks of L tokens, T2 = L (L + 1) / 2
    causal pairs: per sub-chunk and head k [3 L N P + T2 (3 N + 2 P)] + 2 L N P FMAs (end states, the carried-
    state terms, the score tiles, and the Xs, Bpi and C~ contractions)."""
    N, P, k = w.dstate, w.headdim, w.top_k
    total = 0
    for t0 in range(0, w.seqlen, 64):
        L = min(64, w.seqlen - t0)
        T2 = L * (L + 1) // 2
        total += k * (3 * L * N * P + T2 * (3 * N + 2 * P)) + 2 * L * N * P
    return 2.0 * total * w.batch * w.nheads


def scan_bwd_tensor_flops(w):
    """The part of scan_bwd_flops the tensor cores run for fp16 streams with N = 128 and P in {64, 128}: the
    sub-chunk end states (k L N P FMAs) and adjoint sources (L N P), algorithmic counts (the hi/lo split's
    second MMA not counted); 0 where the CUDA-core kernels run them."""
    if w.dtype != "bf16" or w.dstate != 128 or w.headdim not in (64, 128):
        return 0.0
    return 2.0 * (w.top_k + 1) * w.seqlen * w.dstate * w.headdim * w.batch * w.nheads


def scan_bwd_measure(args, dev, flush, stream, swimba):
    """The scan gradients (swimba_ssd_scan_bwd) at the base layer's sizes on seeded streams, timed alone.  The
    end states and adjoint sources run on the tensor cores, the rest on CUDA cores: the floor is the sum of
    their FLOPs at the bf16 burst peak and at the fp32 ALU peak (148 SMs x 128 lanes x 2 FLOP x the maximum SM
    clock); achieved counts all of the work against the ALU peak as well, for comparison with the CUDA-core
    kernels alone."""
    w = configs.BASE
    g = torch.Generator().manual_seed(131)
    M, k, H, P, N = w.M, w.top_k, w.nheads, w.headdim, w.dstate
    Bpi = (0.5 * torch.randn(M, k, H, N, generator=g)).half().to(dev)
    Xs = torch.randn(M, k, H, P, generator=g).half().to(dev)
    Cpi = (0.5 * torch.randn(M, k, H, N, generator=g)).half().to(dev)
    dt = (1e-3 + 0.099 * torch.rand(M, H, generator=g)).to(dev)
    A = inputs.make_inputs(w, with_x=False)["A"].to(dev)
    dy = torch.randn(M, H, P, generator=g).to(dev)
    outs = [torch.empty(M, k, H, N, device=dev), torch.empty(M, k, H, P, device=dev), torch.empty(M, H, N, device=dev),
            torch.empty(M, H, device=dev), torch.empty(H, device=dev)]
    d = swimba.dims_of(w)
    ws = torch.empty(swimba.workspace_size(d), dtype=torch.uint8, device=dev)
    call = lambda: swimba.ssd_scan_bwd(d, Bpi, Xs, Cpi, dt, A, None, dy, *outs, None, ws)
    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tot = 0.0
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e0.record(stream)
        call()
        e1.record(stream)
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    if swimba.check_device_status() != 0:
        raise RuntimeError("swimba_ssd_scan_bwd raised a device status")
    secs = tot / args.steps / 1e3
    flops = scan_bwd_flops(w)
    mhz = 1965.0
    try:
        import pynvml
        pynvml.nvmlInit()
        mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(pynvml.nvmlDeviceGetHandleByIndex(dev.index or 0),
                                                     pynvml.NVML_CLOCK_SM))
    except Exception:
        pass
    peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
    tflops = scan_bwd_tensor_flops(w)
    peaks, psrc = load_peaks()
    floor = tflops / (peaks["bf16_tflops"] * 1e12) + (flops - tflops) / (peak * 1e12)
    return {"ms": secs * 1e3, "flops": flops, "tensor_flops": tflops,
            "roofline": {"bound": "alu", "achieved": flops / secs / 1e12, "peak": peak, "unit": "TFLOP/s",
                         "frac": flops / secs / 1e12 / peak,
                         "peak_source": f"148 SMs x 128 fp32 lanes x 2 FLOP x {mhz:.0f} MHz (max SM clock)"},
            "floor": {"bound": "tensor+alu", "floor_ms": floor * 1e3, "frac": floor / secs,
                      "tensor_peak_tflops": peaks["bf16_tflops"], "peak_source": f"bf16 burst ({psrc})"}}


def layer_bwd_measure(args, sess, inp, flush, stream, swimba):
    """The layer gradients (swimba_layer_bwd) at the base workload with a seeded dy, timed alone: one call
    recomputes the forward's router, dispatch and projections, runs the scan gradients (end states and adjoint
    sources on the tensor cores, the rest on CUDA cores), the mix and router gradients, the two expert products
    dz W_e and dz^T X (tensor cores, on a bf16 hi/lo split of dz) and the router and dt weight gradients.  The
    roofline is the sum of two floors: the tensor-core FLOPs (forward recompute GEMM and router, the scan's
    end states and adjoint sources, the two expert products; algorithmic counts, the split's second MMA not
    counted) at the bf16 burst peak plus the CUDA-core FLOPs (the rest of the scan gradients, the router and
    dt products) at the fp32 ALU peak.  The expert products also get their own roofline from their stage time (pack of dz included)."""
    w = sess.w
    dev = sess.X.device
    g = torch.Generator().manual_seed(151)
    dy = torch.randn(w.M, w.nheads, w.headdim, generator=g).to(dev)
    outs = [torch.empty(w.M, w.d_model, device=dev), torch.empty(w.n_experts, w.d_model, device=dev),
            torch.empty(w.nheads, w.d_model, device=dev), torch.empty(w.nheads, device=dev),
            torch.empty(w.nheads, device=dev), torch.empty(w.n_experts, w.W_e, w.d_model, device=dev)]
    ws = torch.empty(swimba.layer_bwd_workspace_size(sess.d), dtype=torch.uint8, device=dev)
    call = lambda: swimba.layer_bwd(sess.d, sess.X, sess.W, None, dy, *outs, None, ws)
    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tot = 0.0
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e0.record(stream)
        call()
        e1.record(stream)
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    stages = {}
    swimba.profile_enable(True)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        call()
        for name, ms in swimba.profile_read():
            stages[name] = stages.get(name, 0.0) + ms / args.steps
    swimba.profile_enable(False)
    if swimba.check_device_status() != 0:
        raise RuntimeError("swimba_layer_bwd raised a device status")
    secs = tot / args.steps / 1e3
    peaks, psrc = load_peaks()
    gemm = 2.0 * w.M * w.top_k * w.W_e * w.d_model          # one expert product over all (token, slot) rows
    small = 2.0 * w.M * (w.n_experts + w.nheads) * w.d_model  # one router + dt product over all tokens
    st = scan_bwd_tensor_flops(w)                            # scan end states and adjoint sources
    t_flops = 3 * gemm + small + st                          # recompute GEMM and router, dz W_e, dz^T X
    a_flops = scan_bwd_flops(w) - st + 2 * small             # rest of the scan gradients, dg^T X / du^T X, dX terms
    tpk = peaks["bf16_tflops"]
    apk = 148 * 128 * 2 * 1965e6 / 1e12
    floor = t_flops / (tpk * 1e12) + a_flops / (apk * 1e12)
    eg = stages.get("expert_grad", 0.0) / 1e3
    res = {"ms": secs * 1e3, "stages_ms": stages, "tensor_flops": t_flops, "alu_flops": a_flops,
           "roofline": {"bound": "tensor+alu", "floor_ms": floor * 1e3, "frac": floor / secs,
                        "tensor_peak_tflops": tpk, "alu_peak_tflops": apk,
                        "peak_source": f"bf16 burst ({psrc}); fp32 ALU = 148 SMs x 128 lanes x 2 FLOP x 1965 MHz"}}
    if eg > 0:
        res["expert_grad"] = {"ms": eg * 1e3, "flops": 2 * gemm, "achieved": 2 * gemm / eg / 1e12, "peak": tpk,
                              "unit": "TFLOP/s", "frac": 2 * gemm / eg / 1e12 / tpk, "peak_source": psrc}
    return res


def out_proj_measure(args, sess, inp, flush, stream, swimba):
    """The output projection out = y W_out^T (swimba_out_proj) on the layer's own y, timed alone: K launches
    between L2 flushes, against the burst bf16 peak (a kernel timed alone)."""
    w = sess.w
    W_out = inp["W_out"].to(sess.X.device)
    out = torch.empty(w.M, w.d_model, dtype=sess.y.dtype, device=sess.X.device)
    for _ in range(max(args.warmup, 3)):
        swimba.out_proj(sess.d, sess.y, W_out, out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tot = 0.0
    for _ in range(args.steps):
        flush.fill_(1)
        e0.record(stream)
        swimba.out_proj(sess.d, sess.y, W_out, out)
        e1.record(stream)
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    if swimba.check_device_status() != 0:
        raise RuntimeError("swimba_out_proj raised a device status")
    peaks, src = load_peaks()
    HP = w.nheads * w.headdim
    flops = 2.0 * w.M * w.d_model * HP
    nbytes = (w.M * HP + w.d_model * HP + w.M * w.d_model) * out.element_size()
    secs = tot / args.steps / 1e3
    return {"ms": secs * 1e3, "shape": f"[{w.M} x {HP}] x [{HP} x {w.d_model}]", "flops": flops, "bytes": nbytes,
            "roofline": {"bound": "tensor", "achieved": flops / secs / 1e12, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": flops / secs / 1e12 / peaks["bf16_tflops"],
                         "peak_source": f"bf16 dense, burst, {src}"}}


def groups_measure(args, dev, flush, stream, swimba, base_out):
    """The base layer with B and C shared by groups of heads, G in {H, H/4, 1}: per-step layer and scan
    times (the heads of a group read the same B and C rows, which L2 then serves)."""
    w0 = configs.BASE
    res = {"G": [w0.G], "layer_ms": [base_out["ms_per_step"]],
           "scan_ms": [base_out["stages_ms_per_step"].get("ssd_scan")]}
    for w in (configs.BASE_G6, configs.BASE_G1):
        G = w.G
        torch.cuda.empty_cache()
        sess = LayerSession(w, dev, inputs.make_inputs(w), swimba)
        m = measure(sess, args, flush, stream, None, dev.index or 0, swimba, e2e=False)
        res["G"].append(G)
        res["layer_ms"].append(m["total_ms"] / args.steps)
        res["scan_ms"].append(m["stage_ms"].get("ssd_scan", 0.0) / args.steps)
        del sess
    return res


def run_measure(args):
    """One nested measurement alone (layer gradients, scan gradients or output projection) on the base workload,
    one GPU: the same timing as inside the default line, printed as its own JSON object."""
    from parameter_space_moe_b200 import swimba
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    swimba.lib()
    w = configs.BASE
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    if args.measure == "scan_bwd":
        res = scan_bwd_measure(args, dev, flush, stream, swimba)
    else:
        inp = inputs.make_inputs(w)
        sess = LayerSession(w, dev, inp, swimba)
        fn = layer_bwd_measure if args.measure == "layer_bwd" else out_proj_measure
        res = fn(args, sess, inp, flush, stream, swimba)
    print(json.dumps({"measure": args.measure, "workload": w.name, "steps": args.steps, "warmup": args.warmup,
                      **res}))


def run_gpu(args, w):
    from parameter_space_moe_b200 import swimba
    rank, world, local = rank_env()
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    swimba.lib()
    wr = rank_workload(w, rank)
    inp = inputs.make_inputs(wr)
    sess = (DecodeSession if w.prefill else LayerSession)(w, dev, inp, swimba)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    m = measure(sess, args, flush, stream, dist, local, swimba)
    extras = sess.extras(stream, args.steps) if args.separated else {}

    t = max_over_ranks([m["total_ms"], m["e2e_ms"]] + [m["stage_ms"].get(n, 0.0) for n in sorted(m["stage_ms"])],
                       dist, dev)
    m["total_ms"], m["e2e_ms"] = t[0], t[1]
    m["stage_ms"] = {n: t[2 + i] for i, n in enumerate(sorted(m["stage_ms"]))}
    out = summarize(args, w, sess, world, m, inp, extras)
    # one GPU, default workload: the decode step and the expert-count sweep in the same line
    if world == 1 and w.name == configs.BASE.name and not args.no_extras:
        out["out_proj"] = out_proj_measure(args, sess, inp, flush, stream, swimba)
        out["layer_bwd"] = layer_bwd_measure(args, sess, inp, flush, stream, swimba)
        del sess
        torch.cuda.empty_cache()
        msess = LayerSession(w, dev, inp, swimba, mixed_A=True)
        mm = measure(msess, args, flush, stream, None, local, swimba, e2e=False)
        out["mixed_A"] = {"layer_ms": mm["total_ms"] / args.steps,
                          "stages_ms_per_step": {n: v / args.steps for n, v in mm["stage_ms"].items()}}
        del msess
        out["groups"] = groups_measure(args, dev, flush, stream, swimba, out)
        torch.cuda.empty_cache()
        out["scan_bwd"] = scan_bwd_measure(args, dev, flush, stream, swimba)
        torch.cuda.empty_cache()
        dw = configs.DECODE
        dsess = DecodeSession(dw, dev, inputs.make_inputs(dw), swimba)
        dm = measure(dsess, args, flush, stream, None, local, swimba)
        d = summarize(args, dw, dsess, 1, dm, None, {})
        out["decode"] = {k: d[k] for k in ("metric", "value", "unit", "ms_per_step", "config", "roofline",
                                           "layer_roofline", "stages_ms_per_step", "e2e", "gpu_launches", "clocks")}
        del dsess
        torch.cuda.empty_cache()
        out["esweep"] = esweep_measure(args, dev, flush, stream, swimba)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline and not w.prefill:
            v, sample = cpu_oracle_sample(w, inp)
            out["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                   "sample": sample}
        print(json.dumps(out))
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum, bytes per launch) of a stage's kernel from one
# ncu capture of the current kernel build; a stage/workload not listed reports null.  An entry is removed
# whenever its kernel changes.
PROFILED_TRAFFIC = {
    ("base_B4_T2048_D768_H24_E8_k2", "expert_proj_mix"): 120178688 + 205011456,     # proj_tc_pair_kernel
    ("decode_B256_D2048_H64_E16_k2", "expert_proj_mix"): 1347068672 + 21526528,     # proj_tc_kernel
}


def tensor_peak(peaks, clocks):
    """The bf16 GEMM peak that applies: the sustained figure when the timed region ran under the power
    cap (sw_power_cap seen, or the median SM clock well below its maximum), else the burst figure."""
    capped = "sw_power_cap" in clocks.get("reasons", []) or (
        clocks.get("sm_mhz") and clocks.get("sm_max_mhz") and clocks["sm_mhz"] < 0.95 * clocks["sm_max_mhz"])
    if capped:
        return peaks["bf16_tflops_sustained"], "sustained"
    return peaks["bf16_tflops"], "burst"


def stage_roofline(model, secs, peaks, tpeak):
    """Bound (tensor or hbm), achieved, peak and unit of one stage from its work model and duration."""
    t_tensor = model["flops"] / (tpeak * 1e12)
    t_hbm = model["bytes"] / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        return "tensor", model["flops"] / secs / 1e12, tpeak, "TFLOP/s", model["flops"]
    return "hbm", model["bytes"] / secs / 1e9, peaks["hbm_gbs"], "GB/s", model["bytes"]


def summarize(args, w, sess, world, m, inp, extras):
    """The JSON object of one measured workload (the headline fields of the bench contract)."""
    peaks, src = load_peaks()
    wk = sess.work
    K = args.steps
    total_ms, e2e_ms, stage_ms, clocks = m["total_ms"], m["e2e_ms"], m["stage_ms"], m["clocks"] or {}
    tokens = sess.tokens * world * K
    value = job_throughput(sess.tokens, world, K, total_ms)
    # dominant kernel stage (among those with a work model) and its roofline
    dom = max((n for n in stage_ms if n in wk), key=stage_ms.get)
    avg_s = stage_ms[dom] / K / 1e3
    tpeak, tkind = tensor_peak(peaks, clocks)
    bound, achieved, peak, unit, alg = stage_roofline(wk[dom], avg_s, peaks, tpeak)
    peak_note = (f"bf16 dense, {tkind}, {src}" if bound == "tensor" else f"HBM copy, {src}")
    roof_s = max(wk["layer"]["flops"] / (tpeak * 1e12), wk["layer"]["bytes"] / (peaks["hbm_gbs"] * 1e9))
    h2d = sess.Xh.numel() * sess.Xh.element_size()
    d2h = sess.yh.numel() * sess.yh.element_size()
    out = {
        "metric": sess.metric, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic", "config": config_of(w),
        "roofline": {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "traffic": PROFILED_TRAFFIC.get((w.name, dom)),
                     "peak_source": peak_note, "algorithmic": alg},
        "layer_roofline": {"time_us": roof_s * 1e6, "frac": roof_s / (total_ms / K / 1e3),
                           "flops": wk["layer"]["flops"], "bytes": wk["layer"]["bytes"]},
        "stages_ms_per_step": {n: v / K for n, v in stage_ms.items()},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": m["launches"],
        "clocks": m["clocks"],
    }
    out.update(extras)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="swimba", choices=["swimba", "reference"])
    ap.add_argument("--workload", default=configs.BASE.name, choices=sorted(configs.ALL))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--separated", action="store_true",
                    help="also time the separated-trajectory scan (k scans) on the layer's streams")
    ap.add_argument("--no-extras", action="store_true",
                    help="default workload on one GPU: skip the nested decode and expert-count sweep measurements")
    ap.add_argument("--measure", choices=["layer_bwd", "scan_bwd", "out_proj"],
                    help="one GPU, base workload: run only this nested measurement and print its JSON")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = configs.ALL[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    elif args.measure:
        run_measure(args)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
