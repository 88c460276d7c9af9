"""The layer captured into a CUDA graph and replayed.

The library neither allocates nor synchronises inside a call, so a stream that runs the
four step calls (or moe_forward) can be captured once and replayed. Every replay must give
the bits of an eager run on the same inputs, and a replay after the inputs change in place
must follow the new inputs (the graph reads the buffers, it does not bake values in)."""
import pytest
import torch

import gpu_harness as gh
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _capture(fn, mode):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()                                   # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode=mode):
        fn()
    return g


@pytest.mark.parametrize("mode", ["global", "thread_local"])
@pytest.mark.parametrize("name,T", [("proxy_bf16", 128), ("proxy_bf16", 2048), ("tiny_fp32", 64)])
def test_step_calls_replay_bit_identical(cuda_device, name, T, mode):
    """T = 128: the small-batch kernels (split-K router sum, one-CTA permutation index);
    T = 2048: the CTA-pair GEMMs; the fp32 layer: the CUDA-core router and FFN."""
    cfg = wl.CONFIGS[name].with_(T=T)
    case = gh.Case(cfg, seed=12)
    b = case.buffers("deterministic")
    x = case.x.clone()

    def step():
        abi.run_steps(b, x, case.w.w_router, None, case.w.bias, case.w.w_gate_up, case.w.w_down)

    step()
    torch.cuda.synchronize()
    want = b.out.clone()
    want_idx = b.topk_idx.clone()
    g = _capture(step, mode)
    for _ in range(3):
        b.out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(b.out, want)
        assert torch.equal(b.topk_idx, want_idx)
    # new tokens in the same buffer: the replay follows them
    x.copy_(wl.draw_tokens(cfg, "cuda", seed=99))
    g.replay()
    torch.cuda.synchronize()
    got = b.out.clone()
    step()
    torch.cuda.synchronize()
    assert torch.equal(got, b.out)
    assert not torch.equal(got, want)
    assert abi.read_device_status(b.ws) == 0


def test_moe_forward_replay_bit_identical(cuda_device):
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=512)
    w = wl.draw_weights(cfg, "cuda", seed=13)
    layer = abi.MoELayer(abi.shape_of(cfg, "deterministic"), w.w_router, w.bias, w.w_gate_up,
                         w.w_down)
    x = wl.draw_tokens(cfg, "cuda", seed=14)
    out = layer.forward(x)[0]
    torch.cuda.synchronize()
    want = out.clone()
    g = _capture(lambda: layer.forward(x), "global")
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, want)
