"""moe_permute_static_scratch against moe_permute, on the GPU, through the C ABI.

The static-scratch call is for callers that cannot hand the library a device workspace:
code whose stream is being captured into a CUDA graph in a mode where cudaMalloc is an
error, plugins of a framework that owns all device memory, and latency-bound paths that
cannot afford an allocation. It must give exactly what moe_permute gives with its
workspace (the permutation is bit-exact), on consecutive calls that share its scratch
array: the second call here has a different token count and inputs, so anything the first
call left behind would show.

This file is collected last so that a stop at the first failure has run every other test.
"""
import ctypes

import pytest
import torch

import gpu_harness as gh
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _outputs(b, T, K, R, copy):
    got = [b.offsets.clone(), b.perm_token[:R].clone(), b.row_of[: T * K].clone(),
           b.row_gate[:R].clone(), b.out_acc[:T].clone()]
    return got + [b.x_perm[:R].clone()] if copy else got


def _compare_one(cfg, seed, copy=True):
    """moe_permute with its workspace, then the static-scratch call on wiped outputs; every
    output bit for bit. copy=False passes x_perm = NULL to both (indices only, for the
    gathered-rows FFN): nothing is written to x_perm then."""
    case = gh.Case(cfg, seed=seed, ffn=False)
    b = case.buffers("fused")
    case.route(b)
    xp = b.x_perm if copy else None
    abi.permute(b.shape, b.topk_idx, b.topk_gate, b.zgate, case.x, b.offsets, b.perm_token,
                b.row_of, b.row_gate, xp, b.out_acc, b.ws)
    torch.cuda.synchronize()
    assert abi.read_device_status(b.ws) == 0
    R = int(b.offsets[-1])
    want = _outputs(b, cfg.T, cfg.K, R, copy)
    # wipe the outputs, then the static-scratch call
    for t in (b.offsets, b.perm_token, b.row_of, b.row_gate, b.x_perm, b.out_acc):
        t.zero_()
    abi.permute_static_scratch(b.shape, b.topk_idx, b.topk_gate, b.zgate, case.x, b.offsets,
                               b.perm_token, b.row_of, b.row_gate, xp, b.out_acc)
    torch.cuda.synchronize()
    got = _outputs(b, cfg.T, cfg.K, R, copy)
    for w_, g_ in zip(want, got):
        assert torch.equal(w_, g_)
    if not copy:
        assert not b.x_perm.any()
    return R


def test_static_scratch_matches_workspace_call_on_two_calls_in_a_row(cuda_device):
    base = wl.CONFIGS["proxy_bf16"]
    r1 = _compare_one(base, seed=0)                 # 4096 tokens: the three-kernel path
    r2 = _compare_one(base.with_(T=777), seed=1)    # fewer tokens, other inputs
    assert r1 > 0 and r2 > 0


def test_static_scratch_small_batches_and_indices_only(cuda_device):
    """T <= 512 takes the one-CTA index kernel plus the row copy; x_perm = NULL writes the
    indices only. Each call follows the previous one's leftovers in the shared array."""
    base = wl.CONFIGS["proxy_bf16"]
    assert _compare_one(base.with_(T=128), seed=2) > 0
    assert _compare_one(base.with_(T=512), seed=3, copy=False) > 0
    assert _compare_one(base.with_(T=4096), seed=4, copy=False) > 0
    assert _compare_one(base.with_(T=33), seed=5) > 0


def test_static_scratch_rejects_shapes_beyond_its_size(cuda_device):
    cfg = wl.CONFIGS["prefill_bf16"]
    big = abi.shape_of(cfg, T=32737)                # needs just over the 4 MiB
    p = ctypes.c_void_p(1 << 20)                    # never dereferenced: rejected on the host
    before = abi.launch_count()
    rc = abi.lib().moe_permute_static_scratch(ctypes.byref(big), *([p] * 10), None)
    assert rc == -5
    assert abi.launch_count() == before
    # an empty batch is accepted and launches nothing
    assert abi.lib().moe_permute_static_scratch(ctypes.byref(abi.shape_of(cfg, T=0)),
                                                *([p] * 10), None) == 0
