"""Programmatic dependent launch changes when kernels start, never what they compute.

The same seeded layer steps run in two child processes, one with the library's kernels
launched with the programmatic stream-serialisation attribute (the default) and one with
moe_set_tuning(MOE_TUNE_PDL, 0) (plain stream order); in the deterministic combine mode every output is a
fixed function of the inputs, so the two runs must agree bit for bit. Each child runs
several steps back to back, with a PID bias update between them, so every kernel of the
chain has a predecessor still in flight when it is launched. The step calls leave host
gaps between the calls, so each child also runs moe_forward (the whole chain from one C
call, no gaps) on several fresh batches in a row, fp32 and bf16, and two layers stacked
with the first layer's output as the second layer's x: a kernel that read a predecessor's
output through a non-coherent load before the data was final would differ there."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
from mixture_experts_layer_29_b200 import abi, workloads as wl
abi.set_tuning(abi.TUNE_PDL, int(sys.argv[3]))
assert abi.get_tuning(abi.TUNE_PDL) == int(sys.argv[3])
out = {}
for name, T in (("proxy_bf16", 4096), ("proxy_bf16", 200), ("decode_bf16", 128), ("tiny_fp32", 64)):
    cfg = wl.CONFIGS[name].with_(T=T)
    w = wl.draw_weights(cfg, "cuda", seed=3)
    x = wl.draw_tokens(cfg, "cuda", seed=3)
    shape = abi.shape_of(cfg, "deterministic")
    b = abi.StepBuffers.allocate(shape, "cuda")
    state = torch.empty(3 * cfg.n_ffn, dtype=torch.float32, device="cuda")
    abi.pid_init(shape, w.bias, state)
    pid = abi.Pid(0.01, 0.001, 0.0, 8 / 12)
    for step in range(3):
        abi.run_steps(b, x, w.w_router, None, w.bias, w.w_gate_up, w.w_down)
        abi.pid_bias_update(pid, shape, b.counts, b.nffn_hist, w.bias, state)
    torch.cuda.synchronize()
    assert abi.read_device_status(b.ws) == 0
    for k, t in (("out", b.out), ("idx", b.topk_idx), ("gate", b.topk_gate),
                 ("counts", b.counts), ("hist", b.nffn_hist), ("logits", b.logits),
                 ("bias", w.bias)):
        out[f"{name}_{T}_{k}"] = t.detach().cpu().clone()
for name, T in (("tiny_fp32", 64), ("proxy_bf16", 512)):
    cfg = wl.CONFIGS[name].with_(T=T)
    w = wl.draw_weights(cfg, "cuda", seed=4)
    xs = [wl.draw_tokens(cfg, "cuda", seed=30 + i) for i in range(6)]
    layer = abi.MoELayer(abi.shape_of(cfg, "deterministic"), w.w_router, w.bias, w.w_gate_up,
                         w.w_down)
    torch.cuda.synchronize()
    got = [layer.forward(x)[0].clone() for x in xs]
    torch.cuda.synchronize()
    for i, o in enumerate(got):
        out[f"forward_{name}_{T}_{i}"] = o[:T].cpu()
    # two layers stacked: layer 2 reads layer 1's output buffer as its x, so the first
    # kernels of the second call depend on the last kernel of the first
    w2 = wl.draw_weights(cfg, "cuda", seed=5)
    layer2 = abi.MoELayer(abi.shape_of(cfg, "deterministic"), w2.w_router, w2.bias,
                          w2.w_gate_up, w2.w_down)
    torch.cuda.synchronize()
    stacked = []
    for x in xs:
        o1 = layer.forward(x)[0]
        stacked.append(layer2.forward(o1[:T])[0].clone())
    torch.cuda.synchronize()
    for i, o in enumerate(stacked):
        out[f"stacked_{name}_{T}_{i}"] = o[:T].cpu()
torch.save(out, sys.argv[2])
"""


def _run(tmp_path, pdl: str):
    path = os.path.join(tmp_path, f"pdl{pdl}.pt")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, path, pdl], capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return torch.load(path)


def test_pdl_on_and_off_agree_bit_for_bit(cuda_device, tmp_path):
    on = _run(str(tmp_path), "1")
    off = _run(str(tmp_path), "0")
    assert on.keys() == off.keys()
    for k in on:
        assert torch.equal(on[k], off[k]), k
