"""The dense SwiGLU FFN beside the MoE (shortcut-connected MoE, on one GPU).

abi.DenseFFN runs a dense FFN on the grouped-FFN kernels with one group of all tokens;
its rows are compared with the oracle's SwiGLU expert (float64), max per-row relative
error <= 2e-2. Running it on a second stream concurrently with the MoE layer's steps must
give bit-identical results to running the two one after the other."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle.moe_oracle as orc
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _dense(cfg, inter, seed=2):
    wgu, wd = wl.draw_dense_ffn(cfg, "cuda", seed=seed, inter=inter)
    x = wl.draw_tokens(cfg, "cuda", seed=seed)
    xd = torch.zeros(cfg.T + 128, cfg.H, dtype=torch.bfloat16, device="cuda")
    xd[: cfg.T].copy_(x)
    return abi.DenseFFN(cfg.T, wgu, wd), xd, wgu, wd


@pytest.mark.parametrize("name,T,inter,nrows", [("proxy_bf16", 300, 1536, 300),
                                                 ("prefill_bf16", 300, 12288, 6),
                                                 ("prefill_bf16", 1100, 12288, 6)])
def test_dense_ffn_matches_oracle(cuda_device, name, T, inter, nrows):
    """T = 300 runs the one-CTA kernel, T = 1100 the CTA-pair kernel (ragged last tile)."""
    cfg = wl.CONFIGS[name].with_(T=T)
    dense, xd, wgu, wd = _dense(cfg, inter)
    y = dense.forward(xd)
    torch.cuda.synchronize()
    rows = np.unique(np.r_[np.linspace(0, T - 1, nrows).astype(int), T - 1])
    ref = orc.swiglu_expert(gh.host(xd[rows]), gh.host(wgu[0]), gh.host(wd[0]))
    err = gh.row_rel_err(gh.host(y[rows]), ref)
    assert err <= gh.TOL["bf16"], err
    assert abi.read_device_status(dense.ws) == 0


def test_dense_ffn_beside_moe_on_two_streams_is_bit_identical(cuda_device):
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=2048)
    case = gh.Case(cfg, seed=3)
    b = case.buffers("deterministic")
    dense, xd, _, _ = _dense(cfg, 1536)

    def moe():
        return abi.run_steps(b, case.x, case.w.w_router, None, case.w.bias, case.w.w_gate_up,
                             case.w.w_down)
    out1 = moe().clone()
    y1 = dense.forward(xd).clone()
    b.out.zero_()
    dense.y.zero_()
    main, side = torch.cuda.current_stream(), torch.cuda.Stream()
    fork = torch.cuda.Event()
    fork.record(main)
    side.wait_event(fork)
    with torch.cuda.stream(side):
        dense.forward(xd)
    moe()
    join = torch.cuda.Event()
    join.record(side)
    main.wait_event(join)
    torch.cuda.synchronize()
    assert torch.equal(b.out, out1)
    assert torch.equal(dense.y[: cfg.T], y1)
