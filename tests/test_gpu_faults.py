"""Device-side checks report through the status word instead of trapping: a corrupted
expert index handed to moe_permute sets MOE_ERR_DEVICE_CHECK, the context stays usable
and the next call runs clean. (The bad input is made on the host.)"""
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
