"""End-to-end runs from host memory: MoELayer.forward_host and the overlapped
moe_host_pipeline_* calls.

Each batch's output, copied back into page-locked host memory, must be bit-identical to
the same layer's moe_forward on the same tokens already on the device (deterministic
combine), whatever the neighbouring batches are. One batch of the proxy layer is also
checked against the oracle, so the pipeline cannot agree with the device path on a wrong
answer."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle.moe_oracle as orc
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _layer(cfg, seed=5):
    w = wl.draw_weights(cfg, "cuda", seed=seed)
    return abi.MoELayer(abi.shape_of(cfg, "deterministic"), w.w_router, w.bias, w.w_gate_up,
                        w.w_down), w


def _device_out(layer, x, logits=None):
    out = layer.forward(x, logits)[0]
    torch.cuda.synchronize()
    return out[: x.shape[0]].clone()


def test_forward_host_matches_device_forward(cuda_device):
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=1000)
    layer, _ = _layer(cfg)
    x = wl.draw_tokens(cfg, "cuda", seed=11)
    want = _device_out(layer, x)
    xh = x.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    layer.forward_host(xh, oh)
    torch.cuda.synchronize()
    assert torch.equal(oh, want.cpu())


@pytest.mark.parametrize("name,T", [("proxy_bf16", 300), ("proxy_bf16", 2048), ("tiny_fp32", 64)])
def test_pipeline_batches_match_device_forward(cuda_device, name, T):
    """Five batches through two slots: every slot is reused, and each batch's input copy
    overlaps the previous batch's kernels (bf16 on both GEMM kernels, and an fp32 layer)."""
    cfg = wl.CONFIGS[name].with_(T=T)
    layer, _ = _layer(cfg)
    xs = [wl.draw_tokens(cfg, "cuda", seed=20 + i) for i in range(5)]
    want = [_device_out(layer, x) for x in xs]
    xh = [x.cpu().pin_memory() for x in xs]
    oh = [torch.full_like(x, 7.0).pin_memory() for x in xh]
    pipe = abi.HostPipeline(layer)
    for a, o in zip(xh, oh):
        pipe.submit(a, o)
    pipe.join()
    torch.cuda.synchronize()
    for i, (o, w) in enumerate(zip(oh, want)):
        assert torch.equal(o, w.cpu()), i
    assert abi.read_device_status(layer.ws) == 0
    # a second sequence on the same pipeline (the copy streams fork again)
    for a, o in zip(xh[:2], oh[:2]):
        o.fill_(7.0)
        pipe.submit(a, o)
    pipe.join()
    torch.cuda.synchronize()
    assert torch.equal(oh[0], want[0].cpu()) and torch.equal(oh[1], want[1].cpu())
    pipe.close()


def test_pipeline_with_given_logits(cuda_device):
    """Logits passed from host memory take the place of the router, as logits_in does."""
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=512)
    layer, _ = _layer(cfg)
    xs = [wl.draw_tokens(cfg, "cuda", seed=40 + i) for i in range(3)]
    g = torch.Generator(device="cuda").manual_seed(3)
    ls = [torch.randn(cfg.T, cfg.E, device="cuda", generator=g) for _ in range(3)]
    want = [_device_out(layer, x, lg) for x, lg in zip(xs, ls)]
    pipe = abi.HostPipeline(layer, with_logits=True)
    oh = []
    for x, lg in zip(xs, ls):
        o = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()
        pipe.submit(x.cpu().pin_memory(), o, lg.cpu().pin_memory())
        oh.append(o)
    pipe.join()
    torch.cuda.synchronize()
    for o, w in zip(oh, want):
        assert torch.equal(o, w.cpu())
    pipe.close()


@pytest.mark.parametrize("n_zero", [32, 0])
def test_pipeline_output_matches_oracle(cuda_device, n_zero):
    """Given logits from host memory, the oracle routes exactly as the GPU does (away from
    near ties) and the output is within the bf16 bar on every row. Without zero experts
    the output is the FFN part alone, which the zero experts' g * x would otherwise
    dominate below bf16's resolution."""
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=256, n_zero=n_zero)
    layer, w = _layer(cfg)
    x = wl.draw_tokens(cfg, "cuda", seed=9)
    g = torch.Generator(device="cuda").manual_seed(4)
    L = torch.randn(cfg.T, cfg.E, device="cuda", generator=g) * 2.0
    oh = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory()
    pipe = abi.HostPipeline(layer, with_logits=True)
    pipe.submit(x.cpu().pin_memory(), oh, L.cpu().pin_memory())
    pipe.join()
    torch.cuda.synchronize()
    pipe.close()
    out, _, _, _, r = orc.moe_layer_forward(gh.host(x), gh.host(L), gh.host(w.bias),
                                            gh.host(w.w_gate_up), gh.host(w.w_down),
                                            cfg.n_ffn, cfg.K, cfg.ffn_out_scale)
    # bit-exact selection away from near ties (both sides decide in fp32)
    clear = r.gap >= gh.NEAR_TIE
    assert clear.mean() > 0.95
    idx = gh.host(layer.topk_idx)
    assert np.array_equal(idx[clear], r.topk_idx[clear])
    assert gh.row_rel_err(gh.host(oh)[clear], out[clear]) <= gh.TOL["bf16"]
