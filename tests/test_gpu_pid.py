"""The histogram + PID bias update on the GPU against the oracle over 50 steps of the
skewed-routing workload (hidden 6144, 512 + 256 experts, K = 12, T = 16384): biases
bit-exact after every step given the same counts; routing bit-exact on sampled steps."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle.moe_oracle as orc
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GAINS = dict(kp=0.01, ki=0.001, kd=0.0, target_ratio=8 / 12)


@pytest.mark.parametrize("kd", [0.0, 0.005])
def test_pid_fifty_steps_bit_exact(cuda_device, kd):
    cfg = wl.CONFIGS["skew_pid_bf16"]
    w = wl.draw_weights(cfg, "cuda", ffn=False)
    shape = abi.shape_of(cfg)
    b = abi.StepBuffers.allocate(abi.shape_of(cfg.with_(H=128, I=128)), "cuda")  # routing bufs
    pid = abi.Pid(GAINS["kp"], GAINS["ki"], kd, GAINS["target_ratio"])
    state = torch.empty(3 * cfg.n_ffn, dtype=torch.float32, device="cuda")
    stats = torch.zeros(8, dtype=torch.float32, device="cuda")
    ws = torch.zeros(abi.scratch_size(shape), dtype=torch.uint8, device="cuda")
    abi.pid_init(shape, w.bias, state)
    o_bias = gh.host(w.bias).copy()
    o_state = orc.pid_init(o_bias, cfg.n_ffn)
    ratios = []
    for step in range(cfg.pid_steps):
        logits = wl.draw_skewed_logits(cfg, "cuda", step=step)
        abi.route(shape, None, None, logits, w.bias, None, b.topk_idx, b.topk_gate, b.counts,
                  b.nffn_hist, b.zgate, ws)
        counts_before = b.counts.clone()
        abi.pid_bias_update(pid, shape, b.counts, b.nffn_hist, w.bias, state, stats)
        torch.cuda.synchronize()
        counts = gh.host(counts_before)
        hist = gh.host(b.nffn_hist)
        if step % 10 == 0 or step == cfg.pid_steps - 1:
            r = orc.route(gh.host(logits), o_bias, cfg.n_ffn, cfg.K)
            gh.compare_topk(gh.host(b.topk_idx), gh.host(b.topk_gate), r)
        o_bias_new, o_state = orc.pid_update(counts, cfg.T, cfg.K, cfg.n_ffn, o_bias, o_state,
                                             pid.kp, pid.ki, pid.kd, pid.target_ratio)
        got = gh.host(w.bias)
        assert got.tobytes() == o_bias_new.tobytes(), f"step {step}"
        assert got[cfg.n_ffn:].tobytes() == o_bias[cfg.n_ffn:].tobytes()
        st = gh.host(state)
        assert st[cfg.n_ffn:2 * cfg.n_ffn].tobytes() == o_state.integral.tobytes()
        assert st[2 * cfg.n_ffn:].tobytes() == o_state.prev_err.tobytes()
        o_stats = orc.pid_stats(counts, hist, cfg.T, cfg.K, cfg.n_ffn, o_state.prev_err)
        np.testing.assert_allclose(gh.host(stats), o_stats, rtol=1e-6, atol=1e-7)
        o_bias = o_bias_new
        ratios.append(float(o_stats[0]))
    print("\nFFN activation ratio per step:", " ".join(f"{r:.3f}" for r in ratios))
