#!/usr/bin/env python
"""Benchmark of the LongCat-Flash MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N ...

One step = one pass of the whole hot path over one batch: router logits + softmax/top-K
+ histogram (moe_route_packed, with the router weight packed once at set-up), permutation
(moe_permute), grouped SwiGLU FFN on the tensor cores (moe_grouped_ffn; the deterministic
combine by default: the down GEMM stores y per permuted row), the combine (moe_combine:
each token's slots summed in slot order plus the zero-expert term) and the PID bias update
(moe_pid_bias_update, written to a second bias buffer so every step routes the same
batch). --combine fused times the fused epilogue (fp32 atomics into the token's
accumulator) and the finalize instead. Workload: the full-shape prefill layer (hidden
6144, 512 SwiGLU FFN experts of intermediate 2048 + 256 zero-computation experts, K = 12,
8192 tokens, bf16, synthetic seeded inputs). The default run also times the same layer in
the decode regime (128 tokens, against the HBM roofline), the skewed-routing workload
(16384 tokens, drawn Zipf-skewed logits, with its 50-step PID trajectory) and the
768-wide proxy layer (4096 tokens).

Multi-GPU: every rank runs its own replica of the layer on its own batch (no exchange in
the forward pass: weak scaling); the time is the max over ranks.

--impl reference times the CPU oracle (float64 numpy) on a bounded sample of the same
workload on the host cores; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import gc
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_layer_29_b200 import abi  # noqa: E402
from mixture_experts_layer_29_b200 import workloads as wl  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200; % of bf16 TC peak (prefill) / HBM BW (decode)"
UNIT = "tokens/s"
PID_GAINS = (0.01, 0.001, 0.0, 8 / 12)
# faster integral action for the skewed workload's closed loop (reported beside the
# default gains; the pages do not print theirs)
PID_GAINS_FAST = (0.01, 0.05, 0.0, 8 / 12)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "mixture_experts_layer_29_b200", "csrc")


# ------------------------------------------------------------------------------ helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(files) -> str:
    """Hash of the named csrc/ files (the traffic figures hold only for the code they were
    taken on)."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_entry(key: str):
    """The committed ncu DRAM figures for `key` (see profiles/traffic.json), or None when
    any of the sources they were taken on changed since."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(key)
    if not e or e.get("source_sha") != source_hash(e.get("sources", [])):
        return None
    return e


class ClockSampler:
    """SM clock and clock-event (throttle) reasons during the timed region, read only: NVML
    every 5 ms from a thread, the GPU found by the CUDA device's UUID; nvidia-smi every 50 ms
    where NVML is not importable."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvmlClocksEventReason*)
    BITS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
            ("hw_thermal_slowdown", 0x40))

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []          # (sm MHz, max sm MHz, set of reasons)
        self.proc = None
        self.nv = None
        self.stop = threading.Event()
        self.t = None
        self.source = None

    def _nvml(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            u = str(torch.cuda.get_device_properties(self.gpu).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)
        except Exception:  # noqa: BLE001
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        return pynvml, h

    def __enter__(self):
        try:
            self.nv, self.h = self._nvml()
            self.max_sm = float(self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.source = "nvml"
            self.t = threading.Thread(target=self._poll_nvml, daemon=True)
            self.t.start()
            return self
        except Exception:  # noqa: BLE001
            self.nv = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
            self.t = threading.Thread(target=self._read_smi, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _poll_nvml(self):
        nv, h = self.nv, self.h
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                bits = int(get_reasons(h))
                self.samples.append((sm, self.max_sm, {n for n, b in self.BITS if bits & b}))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def _read_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            r = [c.strip() for c in line.split(",")]
            if len(r) > 8 and r[1].replace(".", "").isdigit() and r[2].replace(".", "").isdigit():
                self.samples.append((float(r[1]), float(r[2]),
                                     {n for n, v in zip(names, r[5:9]) if v.lower() == "active"}))

    def __exit__(self, *a):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=5)
        if self.nv is not None:
            try:
                self.nv.nvmlShutdown()
            except Exception:  # noqa: BLE001
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clocks not sampled"]}
        sm = [x[0] for x in self.samples]
        reasons = set().union(*(x[2] for x in self.samples))
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": sorted(reasons), "samples": len(self.samples), "source": self.source}


def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def oracle_sample(cfg, w, x_dev, tokens, logits_dev=None, cache=None):
    """Time the oracle on `tokens` of the workload: logits (float64), routing, and the
    SwiGLU experts of those tokens. Weights of the experts they hit are copied to the
    host and converted to float64 first (outside the timed region; `cache`, a dict, keeps
    them across calls). Where the workload's logits are an input (`logits_dev`, the
    skewed workload), the oracle takes those rows instead of computing them.
    Returns (seconds, tokens)."""
    import oracle.moe_oracle as orc
    x = x_dev[tokens].float().cpu().numpy()
    wr = w.w_router.cpu().numpy()
    bias = w.bias.cpu().numpy()
    given = None if logits_dev is None else logits_dev[tokens].cpu().numpy()
    # routing decides which experts' weights to stage; staging is not timed
    L_probe = given if given is not None else orc.router_logits(x, wr).astype(np.float32)
    r = orc.route(L_probe, bias, cfg.n_ffn, cfg.K)
    experts = sorted({int(e) for e in r.topk_idx.ravel() if e < cfg.n_ffn})
    # the oracle computes in float64: hand it float64 weights, so that the timed region
    # holds its arithmetic, not the conversion of every touched expert's 75 MB of weights
    cache = {} if cache is None else cache
    for e in experts:
        if e not in cache:
            cache[e] = (w.w_gate_up[e].float().cpu().numpy().astype(np.float64),
                        w.w_down[e].float().cpu().numpy().astype(np.float64))
    wgu = {e: cache[e][0] for e in experts}
    wd = {e: cache[e][1] for e in experts}
    t0 = time.perf_counter()
    L = given if given is not None else orc.router_logits(x, wr).astype(np.float32)
    orc.moe_layer_forward(x, L, bias, wgu, wd, cfg.n_ffn, cfg.K, cfg.ffn_out_scale)
    return time.perf_counter() - t0, len(tokens)


def cpu_baseline_sample(cfg, w, x, logits_in, first: int, target_s: float, max_slices: int = 5):
    """The oracle on a bounded token sample sized for about `target_s` seconds of oracle
    time. The tokens are a fixed-seed random permutation of the batch, taken in slices:
    `first` tokens, then each further slice sized from the previous slice's rate to fill
    the time left. A slice's cost per token falls as the slice grows (an expert's weights
    serve more rows per matrix product), so one linear extrapolation undershoots. The
    float64 weights of the experts a slice hits are staged once, outside the timed region.
    Stops at 90% of the target, at the end of the batch or after `max_slices` slices.
    Returns (seconds, tokens)."""
    order = np.random.default_rng(0).permutation(cfg.T).tolist()
    secs, n = 0.0, 0
    size = min(first, cfg.T)
    cache = {}
    for _ in range(max_slices):
        s1, n1 = oracle_sample(cfg, w, x, sorted(order[n:n + size]), logits_in, cache)
        secs, n = secs + s1, n + n1
        left = target_s - secs
        if n >= cfg.T or left <= 0.1 * target_s:
            break
        size = min(cfg.T - n, max(1, int(n1 * left / max(s1, 1e-9))))
    return secs, n


# ------------------------------------------------------------------------------ our arm

class Stepper:
    """The layer's ABI steps on one stream, with CUDA events around each call."""

    def __init__(self, cfg, w, x, logits_in, combine, device):
        self.cfg, self.w, self.x, self.logits_in = cfg, w, x, logits_in
        self.shape = abi.shape_of(cfg, combine)
        self.b = abi.StepBuffers.allocate(self.shape, device)
        # the router weight in the tensor cores' three-part bf16 form, packed once like any
        # weight layout (model-load time), not per step
        self.w_packed = None
        if self.shape.dtype == abi.MOE_BF16 and logits_in is None:
            self.w_packed = torch.empty(cfg.E, 3 * cfg.H, dtype=torch.bfloat16, device=device)
            abi.router_pack(self.shape, w.w_router, self.w_packed)
        self.bias_next = w.bias.clone()
        self.pid = abi.Pid(*PID_GAINS)
        self.state = torch.empty(3 * cfg.n_ffn, dtype=torch.float32, device=device)
        self.stats = torch.zeros(8, dtype=torch.float32, device=device)
        abi.pid_init(self.shape, w.bias, self.state)

    def step(self, ev=None):
        s, b, w = self.shape, self.b, self.w

        def mark(i):
            if ev is not None:
                ev[i].record()
        mark(0)
        if self.w_packed is not None:
            abi.route_packed(s, self.x, self.w_packed, w.bias, b.logits, b.topk_idx,
                             b.topk_gate, b.counts, b.nffn_hist, b.zgate, b.ws)
        else:
            abi.route(s, self.x, w.w_router, self.logits_in, w.bias,
                      None if self.logits_in is not None else b.logits, b.topk_idx,
                      b.topk_gate, b.counts, b.nffn_hist, b.zgate, b.ws)
        mark(1)
        xp = b.x_perm
        abi.permute(s, b.topk_idx, b.topk_gate, b.zgate, self.x, b.offsets, b.perm_token,
                    b.row_of, b.row_gate, xp, b.out_acc, b.ws)
        mark(2)
        abi.grouped_ffn(s, self.x, xp, b.offsets, w.w_gate_up, w.w_down, b.perm_token,
                        b.row_gate, b.h, b.y_perm, b.out_acc, b.ws)
        mark(3)
        abi.combine(s, self.x, b.y_perm, b.out_acc, b.topk_gate, b.row_of, b.zgate, b.out)
        mark(4)
        abi.pid_bias_update(self.pid, s, b.counts, b.nffn_hist, self.bias_next, self.state,
                            self.stats)
        mark(5)


PHASES = ["route", "permute", "grouped_ffn", "combine", "pid"]


def graph_step_ms(st: Stepper, n: int) -> float:
    """One step captured into a CUDA graph (the calls neither allocate nor synchronise),
    then `n` replays between CUDA events: the step without the host's launch work."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        st.step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st.step()
    for _ in range(3):
        g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(n):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / n


def timed_loop(st: Stepper, steps: int, warmup: int, dist_on: bool, phases: bool = True):
    """Time `steps` steps (after `warmup`) between CUDA events on the launching stream.
    phases=True also records an event between the layer's calls for the per-call
    breakdown; the step time itself is taken without them (phases=False), because an
    event between two kernels makes the second wait for the first to finish instead of
    starting as a programmatic dependent launch."""
    for _ in range(warmup):
        st.step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)] \
        if phases else None
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    n0 = abi.launch_count()
    start.record()
    for k in range(steps):
        st.step(evs[k] if phases else None)
    end.record()
    torch.cuda.synchronize()
    launches = abi.launch_count() - n0
    if dist_on:
        torch.distributed.barrier()
    total = start.elapsed_time(end)
    per = {p: [evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(steps)]
           for i, p in enumerate(PHASES)} if phases else None
    return total, per, launches


def scmoe_overlap(st: Stepper, device, seed: int, iters: int, warmup: int) -> dict:
    """The layer's dense SwiGLU FFN (intermediate 12288) beside its MoE step, on one GPU.

    The shortcut-connected MoE (LongCat-Flash Technical Report digest, Key claims, report
    §2.2) runs a layer's dense FFN while its MoE is under way; across GPUs that hides the
    dispatch / combine all-to-all, and here the closest analogue is two streams: the MoE
    step on the launching stream, the dense FFN (the grouped-FFN kernels with one group) on
    a second one. Times the MoE step alone, the dense FFN alone, both on one stream, and
    both on two streams, each the mean over `iters` after `warmup`."""
    cfg = st.cfg
    wgu, wd = wl.draw_dense_ffn(cfg, device, seed=seed)
    dense = abi.DenseFFN(cfg.T, wgu, wd)
    xd = torch.zeros(cfg.T + 128, cfg.H, dtype=torch.bfloat16, device=device)
    xd[: cfg.T].copy_(st.x)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream(device=device)

    def timed(fn) -> float:
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        for _ in range(iters):
            fn()
        e1.record(main)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / iters

    def concurrent():
        fork = torch.cuda.Event()
        fork.record(main)
        side.wait_event(fork)
        with torch.cuda.stream(side):
            dense.forward(xd)
        st.step()
        join = torch.cuda.Event()
        join.record(side)
        main.wait_event(join)

    t_moe = timed(st.step)
    t_dense = timed(lambda: dense.forward(xd))
    t_serial = timed(lambda: (st.step(), dense.forward(xd)))
    t_conc = timed(concurrent)
    flops = 6.0 * cfg.T * cfg.H * wl.DENSE_FFN_INTER
    saved = t_serial - t_conc
    out = {"tokens": cfg.T, "dense_inter": wl.DENSE_FFN_INTER,
           "moe_ms": round(t_moe, 4), "dense_ffn_ms": round(t_dense, 4),
           "dense_ffn_tflops": round(flops / (t_dense / 1e3) / 1e12, 1),
           "one_stream_ms": round(t_serial, 4), "two_streams_ms": round(t_conc, 4),
           "saved_ms": round(saved, 4),
           "saved_of_shorter": round(saved / min(t_moe, t_dense), 4)}
    del dense, wgu, wd, xd
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def time_backward(st: Stepper, device, seed: int, iters: int, warmup: int) -> dict:
    """moe_backward on the batch of the last timed step (deterministic-mode forward), for a
    random bf16 output gradient; mean CUDA-event time per call.

    Training mode: the forward's moe_grouped_ffn keeps G | U (gu_out) and the backward
    takes them. Also timed: the backward that recomputes G | U itself, and the forward's
    grouped FFN with and without keeping G | U. Algorithmic work of the backward's expert
    GEMMs: dh (2 R H I), the rows' dx (4 R H I) and the two weight gradients (2 + 4 R H I),
    12 R H I in all (16 R H I with the recompute); the router's GEMMs are 4 T E H."""
    cfg, b = st.cfg, st.b
    g = torch.Generator(device=device).manual_seed(seed + 77)
    dout = (torch.randn(cfg.T, cfg.H, device=device, generator=g) * 0.5).to(torch.bfloat16)
    dx = torch.empty(cfg.T, cfg.H, dtype=torch.float32, device=device)
    d_router = torch.empty(cfg.E, cfg.H, dtype=torch.float32, device=device)
    d_gu = torch.empty(cfg.n_ffn, 2 * cfg.I, cfg.H, dtype=torch.float32, device=device)
    d_d = torch.empty(cfg.n_ffn, cfg.H, cfg.I, dtype=torch.float32, device=device)
    ws = torch.zeros(abi.backward_workspace_size(b.shape), dtype=torch.uint8, device=device)
    gu = torch.empty(cfg.T * cfg.K + 128, 2 * cfg.I, dtype=torch.bfloat16, device=device)
    w = st.w

    def ffn(keep):
        abi.grouped_ffn(b.shape, st.x, b.x_perm, b.offsets, w.w_gate_up, w.w_down, b.perm_token,
                        b.row_gate, b.h, b.y_perm, b.out_acc, b.ws, gu_out=gu if keep else None)

    def bwd(saved):
        abi.backward(b.shape, dout, st.x, w.w_router, w.w_gate_up, w.w_down, b.logits,
                     b.topk_idx, b.topk_gate, b.offsets, b.row_of, b.x_perm, b.h, b.y_perm,
                     dx, d_router, d_gu, d_d, ws, gu=gu if saved else None)

    def timed(fn, n):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    ffn_plain = timed(lambda: ffn(False), iters)
    ffn_keep = timed(lambda: ffn(True), iters)      # leaves G | U of this batch in gu
    ms = timed(lambda: bwd(True), iters)
    ms_re = timed(lambda: bwd(False), iters)
    assert abi.read_device_status(ws) == 0
    rows = int(b.counts[: cfg.n_ffn].sum().item())
    flop = 12.0 * rows * cfg.H * cfg.I
    out = {"workload": st.cfg.name, "tokens": cfg.T, "ms_per_call": round(ms, 4),
           "expert_gemm_flop": flop, "ffn_rows": rows,
           "expert_gemm_tflops_over_call": round(flop / (ms / 1e3) / 1e12, 1),
           "ms_per_call_recompute_gu": round(ms_re, 4),
           "forward_grouped_ffn_ms": round(ffn_plain, 4),
           "forward_grouped_ffn_keep_gu_ms": round(ffn_keep, 4),
           "router_flop": 4.0 * cfg.T * cfg.E * cfg.H,
           "note": "whole moe_backward call given the forward's G | U (gu_out); "
                   "the recompute variant runs the gate/up GEMM again"}
    del dout, dx, d_router, d_gu, d_d, ws, gu
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def pid_trajectory(cfg, w, device, seed: int, gains=PID_GAINS) -> dict:
    """The skewed workload's closed loop, untimed: for each of cfg.pid_steps steps, route
    that step's drawn logits with the current bias (moe_route) and update the FFN experts'
    biases from the histogram (moe_pid_bias_update), starting from the workload's bias.
    Reports, after every step, the FFN activation ratio (mean FFN picks per token / K),
    the spread of FFN picks per token and the FFN experts' max / mean load."""
    shape = abi.shape_of(cfg)
    b = abi.StepBuffers.allocate(abi.shape_of(cfg.with_(H=128, I=128)), device)
    ws = torch.zeros(abi.scratch_size(shape), dtype=torch.uint8, device=device)
    bias = w.bias.clone()
    state = torch.empty(3 * cfg.n_ffn, dtype=torch.float32, device=device)
    stats = torch.zeros(8, dtype=torch.float32, device=device)
    abi.pid_init(shape, bias, state)
    pid = abi.Pid(*gains)
    ratio, spread, imbalance = [], [], []
    for k in range(cfg.pid_steps):
        logits = wl.draw_skewed_logits(cfg, device, seed=seed, step=k)
        abi.route(shape, None, None, logits, bias, None, b.topk_idx, b.topk_gate, b.counts,
                  b.nffn_hist, b.zgate, ws)
        abi.pid_bias_update(pid, shape, b.counts, b.nffn_hist, bias, state, stats)
        st = stats.cpu()
        ratio.append(round(float(st[0]), 4))
        spread.append(round(float(st[2]), 3))
        imbalance.append(round(float(st[3]), 2))
    assert abi.read_device_status(ws) == 0
    return {"steps": cfg.pid_steps, "target_ratio": round(gains[3], 4),
            "gains": {"kp": gains[0], "ki": gains[1], "kd": gains[2]},
            "ffn_ratio": ratio, "ffn_picks_std": spread, "ffn_max_over_mean_load": imbalance}


def ffn_roofline(workload: str, rows: int, cfg, ffn_ms: float, timed_ms: float) -> dict:
    """The grouped FFN (gate/up + down tcgen05 GEMMs) against the bf16 tensor-core peak.
    Algorithmic work: 6 H I FLOP per FFN row (gate, up and down projections). The timed
    region lasts well under a second, so the burst peak applies; the sustained one (a
    seconds-long loop under the power cap) is printed beside it."""
    pk, pk_kind = peaks()
    flop = rows * 6.0 * cfg.H * cfg.I
    achieved = flop / (ffn_ms / 1e3) / 1e12
    burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sustained = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    te = traffic_entry(f"{workload}:grouped_ffn")
    return {"bound": "tensor", "kernel": "grouped_ffn (gate/up + down tcgen05 GEMMs)",
            "achieved": round(achieved, 1), "peak": burst, "unit": "TFLOP/s",
            "frac": round(achieved / burst, 4),
            "traffic": te["dram_bytes_per_call"] if te else None,
            "peak_kind": f"bf16 burst, {pk_kind} (timed region {timed_ms / 1e3:.2f} s)",
            "frac_of_sustained": round(achieved / sustained, 4), "sustained_peak": sustained,
            "algorithmic_flop_per_call": flop, "ffn_rows": rows,
            "kernel_ms": round(ffn_ms, 4)}


def max_over_ranks(v: float, dist_on: bool) -> float:
    """The largest of the ranks' values (the job's time is the slowest replica's)."""
    if not dist_on:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_seed(cfg, rank: int) -> int:
    """Each replica routes its own batch: the token seed moves with the rank (the weights
    are the same on every rank)."""
    return cfg.seed + rank


def job_throughput(tokens_per_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_step * steps * world / (max_ms / 1e3)


def workload(args):
    cfg = wl.CONFIGS[args.workload]
    kw = {}
    if args.tokens is not None:
        kw["T"] = args.tokens
    if args.ffn_experts is not None:
        kw["n_ffn"] = args.ffn_experts
    if args.zero_experts is not None:
        kw["n_zero"] = args.zero_experts
    return cfg.with_(**kw) if kw else cfg


def time_workload(name: str, args, device, rank: int, dist_on: bool, world: int) -> dict:
    """Another workload of the layer, timed like the main one in the same run: its own
    weights, batch (and drawn logits), the same step, the per-call breakdown and the
    grouped FFN's roofline; for the skewed workload also its closed PID loop, with the
    default gains and with PID_GAINS_FAST."""
    cfg = wl.CONFIGS[name]
    seed = replica_seed(cfg, rank)
    w = wl.draw_weights(cfg, device, seed=cfg.seed)
    x = wl.draw_tokens(cfg, device, seed=seed)
    logits_in = wl.draw_skewed_logits(cfg, device, seed=seed) if cfg.skewed else None
    st = Stepper(cfg, w, x, logits_in, args.combine, device)
    # short steps get more of them, so that the timed region is not a few microseconds
    steps = max(args.steps, 200) if cfg.T * cfg.H < 8192 * 6144 // 4 else args.steps
    ms, _, launches = timed_loop(st, steps, max(args.warmup, 3), dist_on, phases=False)
    _, per, _ = timed_loop(st, min(steps, 30), 0, dist_on, phases=True)
    ms = max_over_ranks(ms, dist_on)
    counts = st.b.counts.cpu().numpy()
    rows = int(counts[: cfg.n_ffn].sum())
    out = {"workload": name, "tokens": cfg.T, "hidden": cfg.H, "expert_intermediate": cfg.I,
           "ffn_experts": cfg.n_ffn, "zero_experts": cfg.n_zero, "top_k": cfg.K,
           "value": round(job_throughput(cfg.T, steps, world, ms), 1), "unit": UNIT,
           "ms_per_step": round(ms / steps, 4), "steps": steps,
           "gpu_launches": int(launches) * world,
           "breakdown_ms": {p: round(float(np.mean(v)), 4) for p, v in per.items()},
           "roofline": ffn_roofline(name, rows, cfg, float(np.mean(per["grouped_ffn"])), ms),
           "routing": {"ffn_rows": rows, "ffn_experts_hit": int((counts[: cfg.n_ffn] > 0).sum()),
                       "max_rows_per_expert": int(counts[: cfg.n_ffn].max())}}
    if cfg.H * cfg.I * cfg.n_ffn * 6 < 126e6:
        out["l2"] = "the experts' weights fit in the 126 MB L2; no flush between steps"
    if cfg.pid_steps > 0 and rank == 0:
        out["pid_trajectory"] = pid_trajectory(cfg, w, device, seed)
        out["pid_trajectory_fast"] = pid_trajectory(cfg, w, device, seed, PID_GAINS_FAST)
    del st, w, x, logits_in
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def workload_config(args, cfg) -> dict:
    """The `config` keys both arms report: the workload and the layer's sizes."""
    name = args.workload if cfg == wl.CONFIGS[args.workload] else \
        f"{args.workload} (overridden: T={cfg.T}, n_ffn={cfg.n_ffn}, n_zero={cfg.n_zero})"
    return {"workload": name, "tokens": cfg.T, "hidden": cfg.H, "expert_intermediate": cfg.I,
            "ffn_experts": cfg.n_ffn, "zero_experts": cfg.n_zero, "top_k": cfg.K}


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    cfg = workload(args)
    seed = replica_seed(cfg, rank)
    w = wl.draw_weights(cfg, device, seed=cfg.seed)
    x = wl.draw_tokens(cfg, device, seed=seed)
    logits_in = wl.draw_skewed_logits(cfg, device, seed=seed) if cfg.skewed else None
    st = Stepper(cfg, w, x, logits_in, args.combine, device)

    with ClockSampler(local) as clk:
        total_ms, _, launches = timed_loop(st, args.steps, args.warmup, dist_on, phases=False)
        _, per, _ = timed_loop(st, min(args.steps, 30), 0, dist_on, phases=True)
    total_ms = max_over_ranks(total_ms, dist_on)
    ms_step = total_ms / args.steps
    value = job_throughput(cfg.T, args.steps, world, total_ms)

    counts = st.b.counts.cpu().numpy()
    rows = int(counts[: cfg.n_ffn].sum())
    ffn_ms = float(np.mean(per["grouped_ffn"]))
    roofline = ffn_roofline(args.workload, rows, cfg, ffn_ms, total_ms)

    # ---- decode regime: same layer (same weights), 128 tokens ---------------------------
    decode = None
    dst = None
    if args.workload == "prefill_bf16" and not args.no_decode:
        dcfg = cfg.with_(T=wl.CONFIGS["decode_bf16"].T)
        dx = wl.draw_tokens(dcfg, device, seed=seed)
        dst = Stepper(dcfg, w, dx, None, args.combine, device)
        dsteps = max(args.steps, 20)
        dms, _, _ = timed_loop(dst, dsteps, max(args.warmup, 3), dist_on, phases=False)
        _, dper, _ = timed_loop(dst, min(dsteps, 30), 0, dist_on, phases=True)
        dms = max_over_ranks(dms, dist_on)
        dc = dst.b.counts.cpu().numpy()
        touched = int((dc[: dcfg.n_ffn] > 0).sum())
        dbytes = (touched * 3.0 * dcfg.H * dcfg.I * 2 + dcfg.E * dcfg.H * 4
                  + 2 * dcfg.T * dcfg.H * 2)
        dstep = dms / dsteps
        dte = traffic_entry("decode_bf16:step")
        dtraffic = dte["dram_bytes_per_step"] if dte else None
        dach = dbytes / (dstep / 1e3) / 1e9
        pk, pk_kind = peaks()
        hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        dgraph = graph_step_ms(dst, dsteps) if not dist_on else None
        decode = {"workload": "decode_bf16", "value": round(dcfg.T * dsteps * world / (dms / 1e3), 1),
                  "unit": UNIT, "ms_per_step": round(dstep, 4),
                  "graph_ms_per_step": round(dgraph, 4) if dgraph else None,
                  "breakdown_ms": {p: round(float(np.mean(v)), 4) for p, v in dper.items()},
                  "roofline": {"bound": "hbm", "scope": "whole layer step",
                               "achieved": round(dach, 1), "peak": hbm, "unit": "GB/s",
                               "frac": round(dach / hbm, 4), "frac_of_8TBs": round(dach / 8000, 4),
                               "traffic": dtraffic, "algorithmic_bytes_per_step": dbytes,
                               "touched_experts": touched, "peak_kind": pk_kind}}

    # ---- end to end through the public API from pinned host memory ----------------------
    # moe_host_pipeline_*: every step copies its x (and given logits) in from page-locked
    # host memory and its output back, each copy overlapped with a neighbouring step's
    # kernels; the serial figure (moe_forward between two copies on one stream) is context.
    e2e = None
    if not args.no_e2e:
        layer = abi.MoELayer(abi.shape_of(cfg, args.combine), w.w_router, w.bias.clone(),
                             w.w_gate_up, w.w_down)
        xh = x.cpu().pin_memory()
        lh = logits_in.cpu().pin_memory() if logits_in is not None else None
        ohs = [torch.empty(cfg.T, cfg.H, dtype=x.dtype).pin_memory() for _ in range(2)]
        pipe = abi.HostPipeline(layer, with_logits=lh is not None)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def e2e_loop(n, serial):
            if dist_on:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            s0.record()
            for i in range(n):
                if serial:
                    layer.forward_host(xh, ohs[i % 2], logits_in)
                else:
                    pipe.submit(xh, ohs[i % 2], lh)
            if not serial:
                pipe.join()
            s1.record()
            torch.cuda.synchronize()
            return max_over_ranks(s0.elapsed_time(s1), dist_on)

        e2e_loop(max(args.warmup, 3), False)
        ems = e2e_loop(args.steps, False)
        nser = min(args.steps, 20)
        e2e_loop(2, True)
        sms = e2e_loop(nser, True)
        pipe.close()
        bi = xh.numel() * xh.element_size() + (lh.numel() * 4 if lh is not None else 0)
        e2e = {"value": round(cfg.T * args.steps * world / (ems / 1e3), 1), "unit": UNIT,
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": ohs[0].numel() * ohs[0].element_size(),
               "ms_per_step": round(ems / args.steps, 4),
               "serial_ms_per_step": round(sms / nser, 4),
               "note": "moe_host_pipeline_submit per step: page-locked x in and the output "
                       "back, each step's copies overlapped with its neighbours' kernels; "
                       "serial_ms_per_step: copy in, moe_forward, copy out on one stream"}
        del layer

    bwd = None
    if not args.no_backward and not dist_on and cfg.dtype == wl.BF16 and \
            args.combine == "deterministic" and not cfg.skewed:
        bwd = time_backward(st, device, seed, 5, 2)

    overlap = None
    if not args.no_overlap and not dist_on and cfg.dtype == wl.BF16:
        overlap = {"prefill": scmoe_overlap(st, device, seed, 20, 3)}
        if decode is not None:
            overlap["decode"] = scmoe_overlap(dst, device, seed, 50, 5)

    pid_traj = None
    if cfg.pid_steps > 0 and rank == 0:
        pid_traj = pid_trajectory(cfg, w, device, seed)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, n = cpu_baseline_sample(cfg, w, x, logits_in, args.cpu_tokens, args.cpu_seconds)
        cpu = {"value": round(n / secs, 3), "unit": UNIT, "cores": oracle_threads(),
               "kind": "oracle",
               "sample": f"{n} of the {cfg.T} tokens, drawn with a fixed seed (logits, routing "
                         f"and SwiGLU experts in float64 numpy), {secs:.1f} s of oracle time"}

    # ---- the other workloads of the layer, after the main one's weights are freed ---------
    others = None
    if args.workload == "prefill_bf16" and not args.no_others:
        del st, dst, w, x, logits_in
        gc.collect()
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        others = {"skew_pid": time_workload("skew_pid_bf16", args, device, rank, dist_on, world),
                  "proxy": time_workload("proxy_bf16", args, device, rank, dist_on, world)}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded normal inputs and random-init weights of the layer's shape)",
        "config": {**workload_config(args, cfg), "combine": args.combine,
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "no flush: each step streams the touched experts' weights "
                         f"({roofline['ffn_rows']} FFN rows) and writes x_perm, both far above "
                         "the 126 MB L2"},
        "breakdown_ms": {p: round(float(np.mean(v)), 4) for p, v in per.items()},
        "roofline": roofline,
        "decode": decode,
        "scmoe_overlap": overlap,
        "backward": bwd,
        "pid_trajectory": pid_traj,
        "workloads": others,
        "e2e": e2e,
        "gpu_launches": int(launches) * world,
        "cpu_baseline": cpu,
        "clocks": clk.summary(),
        "routing": {"ffn_rows": rows, "ffn_experts_hit": int((counts[: cfg.n_ffn] > 0).sum()),
                    "max_rows_per_expert": int(counts[: cfg.n_ffn].max())},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


# ------------------------------------------------------------------------------ reference arm

def run_reference(args):
    """The oracle, timed on the host cores on a bounded sample of the same workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = workload(args)
    device = "cuda" if torch.cuda.is_available() else "cpu"
    if device == "cpu" and cfg.H * cfg.I * cfg.n_ffn > 2**31:
        print(json.dumps({"impl": "reference", "unavailable":
                          "no GPU to draw the full-shape weights of the workload on"}))
        return 0
    w = wl.draw_weights(cfg, device)
    x = wl.draw_tokens(cfg, device)
    logits_in = wl.draw_skewed_logits(cfg, device) if cfg.skewed else None
    rng = np.random.default_rng(1)
    times, n_tok = [], 0
    cache = {}      # float64 weights of the experts seen so far, staged once per run
    for k in range(args.warmup + args.steps):
        toks = sorted(rng.choice(cfg.T, size=args.ref_tokens, replace=False).tolist())
        secs, n = oracle_sample(cfg, w, x, toks, logits_in, cache)
        if k >= args.warmup:
            times.append(secs)
            n_tok += n
    total = sum(times)
    value = n_tok / total
    cores = oracle_threads()
    sample = (f"{args.ref_tokens} random tokens per step of the {cfg.T}-token batch: float64 "
              f"logits, routing and SwiGLU experts (each expert's weights staged in float64 "
              f"once per run, outside the timed region)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args, cfg),
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_bf16", choices=sorted(wl.CONFIGS))
    ap.add_argument("--combine", default="deterministic", choices=["fused", "deterministic"])
    ap.add_argument("--cpu-tokens", type=int, default=400,
                    help="first slice of the oracle's token sample")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="oracle time the CPU baseline's sample is sized for")
    ap.add_argument("--ref-tokens", type=int, default=256,
                    help="tokens of the batch the reference arm's oracle runs per step")
    ap.add_argument("--tokens", type=int, default=None, help="override the workload's T")
    ap.add_argument("--ffn-experts", type=int, default=None, help="override n_ffn (profiling)")
    ap.add_argument("--zero-experts", type=int, default=None, help="override n_zero (profiling)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip timing moe_backward")
    ap.add_argument("--no-overlap", action="store_true",
                    help="skip the dense-FFN-beside-MoE (two streams) measurement")
    ap.add_argument("--no-others", action="store_true",
                    help="skip the skewed-routing + PID and proxy workloads of the default run")
    return ap


def main(argv=None):
    args = parser().parse_args(argv)
    if args.impl == "ours":
        args.warmup = max(args.warmup, 3)     # timing rule: at least 3 untimed steps
    return run_reference(args) if args.impl == "reference" else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
