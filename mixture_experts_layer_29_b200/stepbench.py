"""Time one step of the layer in isolation (for profiling single kernels).

    python -m mixture_experts_layer_29_b200.stepbench --workload prefill_bf16 --step route
    python -m mixture_experts_layer_29_b200.stepbench --step ffn --ffn-experts 32 --zero-experts 16

Steps: route (moe_route: router logits + top-K), permute (moe_permute), ffn
(moe_grouped_ffn), combine (moe_combine), pid (moe_pid_bias_update), layer (all of them),
backward (moe_backward after one deterministic-mode forward; fp32 weight gradients of
every expert are allocated, so keep n_ffn modest at full width).
Only what the chosen step needs is drawn: the route and permute steps never allocate the
FFN weights, so they run at the full-shape T and E in well under a GB of device memory.
Prints one JSON line with the mean CUDA-event time per call.
"""
from __future__ import annotations

import argparse
import json
import sys

import torch

from . import abi
from . import workloads as wl

STEPS = ("route", "permute", "ffn", "combine", "pid", "layer", "backward")


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--workload", default="prefill_bf16", choices=sorted(wl.CONFIGS))
    ap.add_argument("--step", default="route", choices=STEPS)
    ap.add_argument("--combine", default="deterministic", choices=["fused", "deterministic"])
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--ffn-experts", type=int, default=None)
    ap.add_argument("--zero-experts", type=int, default=None)
    ap.add_argument("--gather", action="store_true",
                    help="no permuted copy of x: the gate/up GEMM gathers the token rows")
    ap.add_argument("--tune", action="append", default=[], metavar="KNOB=VALUE",
                    help="moe_set_tuning switch by its abi.TUNE_* name without the prefix, "
                         "e.g. --tune GATE_UP_BAND=8 (repeatable)")
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args(argv)

    for kv in a.tune:
        k, v = kv.split("=")
        abi.set_tuning(getattr(abi, "TUNE_" + k.upper()), int(v))
    cfg = wl.CONFIGS[a.workload]
    kw = {k: v for k, v in (("T", a.tokens), ("n_ffn", a.ffn_experts),
                            ("n_zero", a.zero_experts)) if v is not None}
    cfg = cfg.with_(**kw) if kw else cfg
    dev = torch.device("cuda", 0)
    need_ffn = a.step in ("ffn", "combine", "layer", "backward")
    if a.step == "backward":
        a.combine = "deterministic"
    w = wl.draw_weights(cfg, dev, ffn=need_ffn)
    x = wl.draw_tokens(cfg, dev)
    logits_in = wl.draw_skewed_logits(cfg, dev) if cfg.skewed else None
    shape = abi.shape_of(cfg, a.combine)
    b = abi.StepBuffers.allocate(shape, dev)
    pid = abi.Pid(0.01, 0.001, 0.0, 8 / 12)
    state = torch.empty(3 * cfg.n_ffn, dtype=torch.float32, device=dev)
    bias_next = w.bias.clone()
    abi.pid_init(shape, w.bias, state)

    def route():
        abi.route(shape, x, w.w_router, logits_in, w.bias,
                  None if logits_in is not None else b.logits, b.topk_idx, b.topk_gate,
                  b.counts, b.nffn_hist, b.zgate, b.ws)

    xp = None if a.gather else b.x_perm

    def permute():
        abi.permute(shape, b.topk_idx, b.topk_gate, b.zgate, x, b.offsets, b.perm_token,
                    b.row_of, b.row_gate, xp, b.out_acc, b.ws)

    def ffn():
        abi.grouped_ffn(shape, x, xp, b.offsets, w.w_gate_up, w.w_down, b.perm_token,
                        b.row_gate, b.h, b.y_perm, b.out_acc, b.ws)

    def combine():
        abi.combine(shape, x, b.y_perm, b.out_acc, b.topk_gate, b.row_of, b.zgate, b.out)

    def pid_step():
        abi.pid_bias_update(pid, shape, b.counts, b.nffn_hist, bias_next, state)

    bwd = {}
    if a.step == "backward":
        g = torch.Generator(device=dev).manual_seed(9)
        bwd["dout"] = (torch.randn(cfg.T, cfg.H, device=dev, generator=g) * 0.5).to(torch.bfloat16)
        bwd["dx"] = torch.empty(cfg.T, cfg.H, device=dev)
        bwd["dr"] = torch.empty(cfg.E, cfg.H, device=dev)
        bwd["dgu"] = torch.empty(cfg.n_ffn, 2 * cfg.I, cfg.H, device=dev)
        bwd["dd"] = torch.empty(cfg.n_ffn, cfg.H, cfg.I, device=dev)
        bwd["ws"] = torch.zeros(abi.backward_workspace_size(shape), dtype=torch.uint8, device=dev)

    def backward():
        abi.backward(shape, bwd["dout"], x, w.w_router, w.w_gate_up, w.w_down, b.logits,
                     b.topk_idx, b.topk_gate, b.offsets, b.row_of, b.x_perm, b.h, b.y_perm,
                     bwd["dx"], bwd["dr"], bwd["dgu"], bwd["dd"], bwd["ws"])

    steps = {"route": route, "permute": permute, "ffn": ffn, "combine": combine,
             "pid": pid_step, "layer": lambda: (route(), permute(), ffn(), combine()),
             "backward": backward}
    # inputs of the timed step come from the steps before it
    order = ["route", "permute", "ffn", "combine", "backward"]
    if a.step in order[1:]:
        for s in order[: order.index(a.step)]:
            steps[s]()
    if a.step == "pid":
        route()
    fn = steps[a.step]
    for _ in range(a.warmup):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    n0 = abi.launch_count()
    e0.record()
    for _ in range(a.iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.iters
    print(json.dumps({"workload": a.workload, "T": cfg.T, "n_ffn": cfg.n_ffn,
                      "n_zero": cfg.n_zero, "step": a.step, "ms_per_call": round(ms, 5),
                      "kernels_per_call": (abi.launch_count() - n0) / a.iters,
                      "device_status": abi.read_device_status(b.ws)}))
    return 0


if __name__ == "__main__":
    sys.exit(main())
