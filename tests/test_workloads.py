"""The seeded input generators: deterministic, right shapes and distributions."""
import math

import torch

from mixture_experts_layer_29_b200 import workloads as wl


def test_configs_have_the_pages_shapes():
    c = wl.CONFIGS["prefill_bf16"]
    assert (c.n_ffn, c.n_zero, c.K, c.H, c.I) == (512, 256, 12, 6144, 2048)
    assert wl.CONFIGS["decode_bf16"].T == 128 and wl.CONFIGS["skew_pid_bf16"].T == 16384
    assert wl.CONFIGS["proxy_bf16"].H * 8 == c.H            # 768-wide proxy, m = 8
    assert math.isclose(c.w_std, 0.02 / math.sqrt(8))


def test_draws_are_seeded_and_shaped():
    c = wl.CONFIGS["tiny_fp32"]
    a, b = wl.draw_weights(c), wl.draw_weights(c)
    assert torch.equal(a.w_gate_up, b.w_gate_up) and torch.equal(a.w_down, b.w_down)
    assert a.w_gate_up.shape == (16, 256, 256) and a.w_down.shape == (16, 256, 128)
    assert a.w_router.shape == (24, 256) and a.bias.shape == (24,)
    assert torch.equal(a.bias, torch.zeros(24))
    x1, x2 = wl.draw_tokens(c), wl.draw_tokens(c, seed=1)
    assert x1.shape == (64, 256) and not torch.equal(x1, x2)
    assert abs(float(a.w_gate_up.std()) - 0.02) < 1e-3


def test_proxy_bias_range_and_dtype():
    c = wl.CONFIGS["proxy_bf16"].with_(T=64, n_ffn=4)
    w = wl.draw_weights(c)
    assert w.w_gate_up.dtype == torch.bfloat16 and w.w_router.dtype == torch.float32
    assert float(w.bias.min()) >= -0.1 and float(w.bias.max()) <= 0.1


def test_skewed_logits_structure():
    c = wl.CONFIGS["skew_pid_bf16"].with_(T=2048)
    L0 = wl.draw_skewed_logits(c, step=0)
    L1 = wl.draw_skewed_logits(c, step=1)
    assert L0.shape == (2048, 768) and not torch.equal(L0, L1)
    zipf, _ = wl.skew_offsets(c)
    assert abs(float(zipf.mean())) < 1e-5
    # the per-expert offset survives averaging over tokens on FFN experts
    col = L0[:, :512].mean(0)
    assert float(torch.corrcoef(torch.stack([col, zipf[:512]]))[0, 1]) > 0.95
