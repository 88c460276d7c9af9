"""Seeded synthetic workloads for the LongCat-Flash MoE layer.

This module only draws random inputs with the shapes and value distributions of the
layer's workloads. It holds none of the layer's arithmetic (no logits, softmax,
selection, permutation, FFN or bias update): the CUDA path and the CPU oracle both take
their inputs from here and nothing else is shared between them.

Shapes follow the LongCat-Flash Technical Report digest, "Key claims" (report §2.1 and
§2.4 Model Configurations): 512 FFN experts plus 256 zero-computation experts, K = 12,
hidden 6144, per-expert FFN intermediate 2048; and the 768-wide proxy with width factor
m = 8 (report §3.1.1, Table 1).

Expert order in every tensor: FFN experts are indices [0, n_ffn), zero-computation
experts are [n_ffn, n_ffn + n_zero).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

BF16 = "bf16"
FP32 = "fp32"


@dataclass(frozen=True)
class MoEConfig:
    """One workload: layer shape, dtypes and the distributions its inputs are drawn from."""

    name: str
    T: int                 # tokens in the batch
    H: int                 # hidden width
    I: int                 # per-expert FFN intermediate width
    n_ffn: int             # SwiGLU FFN experts
    n_zero: int            # zero-computation (identity) experts
    K: int                 # experts chosen per token
    dtype: str             # "bf16" or "fp32": x, FFN weights, x_perm, h, y and out
    w_std: float           # std of the FFN weights and of the router weight
    bias_lo: float         # per-expert bias ~ U(bias_lo, bias_hi)
    bias_hi: float
    seed: int = 0
    ffn_out_scale: float = 1.0
    # skewed-routing workload: logits are drawn directly (see draw_skewed_logits)
    skewed: bool = False
    zipf_s: float = 1.1
    zero_offset_range: float = 4.0
    pid_steps: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def E(self) -> int:
        return self.n_ffn + self.n_zero

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


_FULL_STD = 0.02 / math.sqrt(8.0)   # N(0, 0.02) on the 768 proxy, divided by sqrt(m), m = 8

CONFIGS: dict[str, MoEConfig] = {
    # tiny fp32 layer the oracle finishes in well under a second
    "tiny_fp32": MoEConfig("tiny_fp32", T=64, H=256, I=128, n_ffn=16, n_zero=8, K=4,
                           dtype=FP32, w_std=0.02, bias_lo=0.0, bias_hi=0.0),
    # 768-wide proxy layer
    "proxy_bf16": MoEConfig("proxy_bf16", T=4096, H=768, I=256, n_ffn=64, n_zero=32, K=6,
                            dtype=BF16, w_std=0.02, bias_lo=-0.1, bias_hi=0.1),
    # full-shape prefill layer
    "prefill_bf16": MoEConfig("prefill_bf16", T=8192, H=6144, I=2048, n_ffn=512, n_zero=256,
                              K=12, dtype=BF16, w_std=_FULL_STD, bias_lo=-0.05, bias_hi=0.05),
    # the same layer in the decode regime
    "decode_bf16": MoEConfig("decode_bf16", T=128, H=6144, I=2048, n_ffn=512, n_zero=256,
                             K=12, dtype=BF16, w_std=_FULL_STD, bias_lo=-0.05, bias_hi=0.05),
    # skewed routing + 50 PID steps; the bias starts at zero
    "skew_pid_bf16": MoEConfig("skew_pid_bf16", T=16384, H=6144, I=2048, n_ffn=512,
                               n_zero=256, K=12, dtype=BF16, w_std=_FULL_STD, bias_lo=0.0,
                               bias_hi=0.0, skewed=True, pid_steps=50),
}


def torch_dtype(cfg: MoEConfig) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == BF16 else torch.float32


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


@dataclass
class LayerWeights:
    """Layer parameters.

    w_router  [E, H]       float32
    bias      [E]          float32 (FFN experts first, then zero experts)
    w_gate_up [n_ffn, 2I, H] rows [0, I) are the gate projection, rows [I, 2I) the up projection
    w_down    [n_ffn, H, I]
    """

    w_router: torch.Tensor
    bias: torch.Tensor
    w_gate_up: torch.Tensor
    w_down: torch.Tensor


def draw_weights(cfg: MoEConfig, device="cpu", seed: int | None = None,
                 ffn: bool = True) -> LayerWeights:
    """Draw the layer's parameters: every weight ~ N(0, w_std^2), bias ~ U(bias_lo, bias_hi).

    ffn=False skips the FFN weights (w_gate_up and w_down are None); the router weight and
    the bias are the same values either way (they are drawn first)."""
    seed = cfg.seed if seed is None else seed
    g = _gen(device, seed * 7919 + 1)
    dt = torch_dtype(cfg)
    w_router = torch.empty(cfg.E, cfg.H, dtype=torch.float32, device=device)
    w_router.normal_(0.0, cfg.w_std, generator=g)
    bias = torch.empty(cfg.E, dtype=torch.float32, device=device)
    if cfg.bias_hi > cfg.bias_lo:
        bias.uniform_(cfg.bias_lo, cfg.bias_hi, generator=g)
    else:
        bias.fill_(cfg.bias_lo)
    if not ffn:
        return LayerWeights(w_router, bias, None, None)
    w_gate_up = torch.empty(cfg.n_ffn, 2 * cfg.I, cfg.H, dtype=dt, device=device)
    w_down = torch.empty(cfg.n_ffn, cfg.H, cfg.I, dtype=dt, device=device)
    # one expert at a time keeps the generator's temporaries small on the full shape
    for e in range(cfg.n_ffn):
        w_gate_up[e].normal_(0.0, cfg.w_std, generator=g)
    for e in range(cfg.n_ffn):
        w_down[e].normal_(0.0, cfg.w_std, generator=g)
    return LayerWeights(w_router, bias, w_gate_up, w_down)


# The dense FFN that sits beside the MoE in a LongCat-Flash layer (report §2.4 Model
# Configurations: dense-FFN intermediate 12288; the shortcut-connected MoE of report §2.2
# runs it while the MoE's dispatch and combine are under way).
DENSE_FFN_INTER = 12288


def draw_dense_ffn(cfg: MoEConfig, device="cpu", seed: int | None = None,
                   inter: int = DENSE_FFN_INTER):
    """A dense SwiGLU FFN of the layer's width: (w_gate_up [1, 2*inter, H], w_down
    [1, H, inter]) ~ N(0, w_std^2), laid out as one expert of the grouped-FFN weights."""
    seed = cfg.seed if seed is None else seed
    g = _gen(device, seed * 7919 + 5)
    dt = torch_dtype(cfg)
    w_gate_up = torch.empty(1, 2 * inter, cfg.H, dtype=dt, device=device)
    w_down = torch.empty(1, cfg.H, inter, dtype=dt, device=device)
    w_gate_up.normal_(0.0, cfg.w_std, generator=g)
    w_down.normal_(0.0, cfg.w_std, generator=g)
    return w_gate_up, w_down


def draw_tokens(cfg: MoEConfig, device="cpu", seed: int | None = None) -> torch.Tensor:
    """Draw the token activations x [T, H] ~ N(0, 1) in the layer's dtype."""
    seed = cfg.seed if seed is None else seed
    g = _gen(device, seed * 7919 + 2)
    x = torch.empty(cfg.T, cfg.H, dtype=torch_dtype(cfg), device=device)
    x.normal_(0.0, 1.0, generator=g)
    return x


def skew_offsets(cfg: MoEConfig, device="cpu", seed: int | None = None):
    """Per-expert Zipf offsets and per-token zero-expert offsets of the skewed workload.

    zipf[e] = -s * ln(rank[e]) (then centred), rank a seeded random permutation of 1..E;
    zero_off[t] ~ U(-r, r), added to every zero-computation expert's logit of token t.
    """
    seed = cfg.seed if seed is None else seed
    g = _gen("cpu", seed * 7919 + 3)
    rank = torch.randperm(cfg.E, generator=g).to(torch.float64) + 1.0
    zipf = -cfg.zipf_s * torch.log(rank)
    zipf = (zipf - zipf.mean()).to(torch.float32)
    zero_off = torch.empty(cfg.T, dtype=torch.float32)
    zero_off.uniform_(-cfg.zero_offset_range, cfg.zero_offset_range, generator=g)
    return zipf.to(device), zero_off.to(device)


def draw_skewed_logits(cfg: MoEConfig, device="cpu", seed: int | None = None,
                       step: int = 0) -> torch.Tensor:
    """Router logits of the skewed workload, drawn directly as an input.

    base ~ N(0, sigma^2) with sigma = sqrt(H) * w_std (the spread x . w_r would have for
    x ~ N(0, 1) and w_r ~ N(0, w_std^2)), plus the Zipf per-expert offsets (fixed over
    steps) and, on zero-computation experts, the per-token offset (fresh every step).
    """
    seed = cfg.seed if seed is None else seed
    zipf, _ = skew_offsets(cfg, "cpu", seed)
    g = _gen("cpu", seed * 7919 + 1000 + step)
    zero_off = torch.empty(cfg.T, dtype=torch.float32)
    zero_off.uniform_(-cfg.zero_offset_range, cfg.zero_offset_range, generator=g)
    sigma = math.sqrt(cfg.H) * cfg.w_std
    gd = _gen(device, seed * 7919 + 2000 + step)
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=device)
    logits.normal_(0.0, sigma, generator=gd)
    logits += zipf.to(device)[None, :]
    logits[:, cfg.n_ffn:] += zero_off.to(device)[:, None]
    return logits


def draw_forced_logits(T: int, n_ffn: int, n_zero: int, zero_only_tokens, device="cpu",
                       seed: int = 0) -> torch.Tensor:
    """Logits for edge cases: tokens listed in zero_only_tokens get +50 on every zero
    expert, so that with K <= n_zero they pick zero-computation experts only."""
    g = _gen("cpu", seed * 7919 + 4)
    E = n_ffn + n_zero
    logits = torch.empty(T, E, dtype=torch.float32)
    logits.normal_(0.0, 1.0, generator=g)
    for t in zero_only_tokens:
        logits[t, n_ffn:] += 50.0
    return logits.to(device)
