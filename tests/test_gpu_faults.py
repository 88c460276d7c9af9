"""Device-side checks report through the status word instead of trapping: a corrupted
expert index handed to moe_permute sets MOE_ERR_DEVICE_CHECK, and a tensor-core GEMM
whose wait runs out sets MOE_ERR_TIMEOUT; the context stays usable and the next call runs
clean. (The bad input is made on the host; the stalled wait is a pipeline stage that the
GEMM's producer, told so by the host, never loads, so nothing is in flight on it.)"""
import time

import numpy as np
import pytest
import torch

import gpu_harness as gh
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bad", ["too_large", "negative", "repeated"])
def test_corrupted_expert_index_sets_status(cuda_device, bad):
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=100)
    case = gh.Case(cfg)
    b = case.buffers()
    case.route(b)
    torch.cuda.synchronize()
    assert abi.read_device_status(b.ws) == 0
    idx = b.topk_idx.clone()
    if bad == "too_large":
        idx[3, 1] = cfg.E + 7
    elif bad == "negative":
        idx[50, 0] = -2
    else:
        idx[9, 2] = idx[9, 0]
    abi.permute(b.shape, idx, b.topk_gate, b.zgate, case.x, b.offsets, b.perm_token, b.row_of,
                b.row_gate, b.x_perm, b.out_acc, b.ws)
    assert abi.read_device_status(b.ws) == -6
    assert abi.read_device_status(b.ws) == 0            # reading clears it
    # the context is intact: a clean call works and reports nothing
    abi.permute(b.shape, b.topk_idx, b.topk_gate, b.zgate, case.x, b.offsets, b.perm_token,
                b.row_of, b.row_gate, b.x_perm, b.out_acc, b.ws)
    torch.cuda.synchronize()
    gh.check_permutation(case, b, zero_init=True)
    assert abi.read_device_status(b.ws) == 0


def test_bad_arguments_raise_before_launch(cuda_device):
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=64)
    case = gh.Case(cfg)
    b = case.buffers()
    before = abi.launch_count()
    with pytest.raises(abi.MoEError) as e:
        abi.route(b.shape, case.x, case.w.w_router, None, case.w.bias, b.logits, b.topk_idx,
                  b.topk_gate, b.counts, b.nffn_hist, b.zgate, b.ws[:100])
    assert e.value.code == -5
    odd = torch.empty(1000, dtype=torch.uint8, device="cuda")[4:]
    with pytest.raises(abi.MoEError) as e:
        abi.route(b.shape, case.x, case.w.w_router, None, odd, b.logits, b.topk_idx,
                  b.topk_gate, b.counts, b.nffn_hist, b.zgate, b.ws)
    assert e.value.code == -3
    assert abi.launch_count() == before


@pytest.mark.parametrize("T", [4096, 512])     # CTA-pair GEMM / one-CTA GEMM
def test_gemm_wait_that_runs_out_reports_timeout(cuda_device, T):
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=T)
    case = gh.Case(cfg, seed=11)
    b = case.buffers("deterministic")
    w = case.w

    def ffn():
        abi.grouped_ffn(b.shape, case.x, b.x_perm, b.offsets, w.w_gate_up, w.w_down,
                        b.perm_token, b.row_gate, b.h, b.y_perm, None, b.ws)
        abi.combine(b.shape, case.x, b.y_perm, None, b.topk_gate, b.row_of, b.zgate, b.out)

    abi.run_steps(b, case.x, w.w_router, None, w.bias, w.w_gate_up, w.w_down)
    torch.cuda.synchronize()
    assert abi.read_device_status(b.ws) == 0
    want = b.out.clone()
    # the next gate/up GEMM leaves the first k-block of its first tile unloaded: the MMA
    # thread's wait on that stage runs out after its 2 s limit, every role of the CTA (of
    # the CTA pair) winds down, and the call reports MOE_ERR_TIMEOUT
    abi.set_tuning(abi.TUNE_TEST_STALL, 1)
    try:
        t0 = time.perf_counter()
        ffn()
        torch.cuda.synchronize()
        waited = time.perf_counter() - t0
    finally:
        armed = abi.get_tuning(abi.TUNE_TEST_STALL)
        abi.set_tuning(abi.TUNE_TEST_STALL, 0)
    assert armed == 0                                  # one shot: consumed by that launch
    assert abi.read_device_status(b.ws) == -7
    assert 1.5 < waited < 60, waited
    # the context is intact: the same call again gives the clean run's bits
    ffn()
    torch.cuda.synchronize()
    assert abi.read_device_status(b.ws) == 0
    assert torch.equal(b.out, want)
    L = case.gpu_logits(b)
    toks = np.arange(cfg.T)
    o_out = gh.oracle_layer(case, L, toks)[0]
    assert gh.row_rel_err(gh.host(b.out), o_out) <= gh.TOL[cfg.dtype]
