"""GPU parity of the load-balance loss (moe_lb_loss) against the CPU oracle.

The loss and the mean probabilities are computed from the GPU's own logits and counts
on both sides: loss within 1e-6 relative, every P_i within 1e-6 relative (+1e-12
absolute). Sums run in double on the device in a fixed order, so the call is
bit-reproducible."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle.moe_oracle as orc
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

pytestmark = pytest.mark.gpu

RTOL = 1e-6


def _lb(shape, logits, counts, ws):
    E = shape.n_ffn + shape.n_zero
    P = torch.empty(E, dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    abi.lb_loss(shape, logits, counts, P, loss, ws)
    torch.cuda.synchronize()
    return float(loss.item()), P.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name,T", [("tiny_fp32", 64), ("proxy_bf16", 4096), ("proxy_bf16", 1000),
                                    ("decode_bf16", 128), ("skew_pid_bf16", 16384)])
def test_lb_loss_matches_oracle(cuda_device, name, T):
    cfg = wl.CONFIGS[name].with_(T=T)
    case = gh.Case(cfg, ffn=False)
    b = case.buffers()
    case.route(b)
    L = case.logits_in if case.logits_in is not None else b.logits
    loss, P = _lb(b.shape, L, b.counts, b.ws)
    ref, refP = orc.lb_loss(gh.host(L), gh.host(b.counts), cfg.n_ffn, cfg.K)
    assert abs(loss - ref) <= RTOL * abs(ref), (loss, ref)
    np.testing.assert_allclose(P, refP, rtol=RTOL, atol=1e-12)
    # bit-reproducible
    loss2, P2 = _lb(b.shape, L, b.counts, b.ws)
    assert loss2 == loss and np.array_equal(P2, P)


def test_lb_loss_balanced_batch_is_one(cuda_device):
    """Equal logits and K T / E picks on every expert give f_i = 1 and P_i = 1/E: loss 1."""
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=96 * 4)          # E = 96, K = 6: 24 picks each
    shape = abi.shape_of(cfg)
    ws = torch.zeros(abi.scratch_size(shape), dtype=torch.uint8, device="cuda")
    L = torch.full((cfg.T, cfg.E), 0.375, dtype=torch.float32, device="cuda")
    counts = torch.full((cfg.E,), cfg.K * cfg.T // cfg.E, dtype=torch.int32, device="cuda")
    loss, P = _lb(shape, L, counts, ws)
    assert abs(loss - 1.0) < 1e-6
    np.testing.assert_allclose(P, 1.0 / cfg.E, rtol=1e-6)


def test_lb_loss_empty_batch_is_zero(cuda_device):
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=0)
    shape = abi.shape_of(cfg)
    ws = torch.zeros(abi.scratch_size(shape), dtype=torch.uint8, device="cuda")
    counts = torch.zeros(cfg.E, dtype=torch.int32, device="cuda")
    P = torch.full((cfg.E,), 7.0, device="cuda")
    loss = torch.full((1,), 7.0, device="cuda")
    abi.lb_loss(shape, None, counts, P, loss, ws)
    torch.cuda.synchronize()
    assert float(loss.item()) == 0.0 and bool((P == 0).all())
