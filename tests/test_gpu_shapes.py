"""The layer on shapes the named workloads do not reach, against the oracle.

The named workloads have hidden sizes that are multiples of 256, E a multiple of 8 and
K >= 4. These bf16 layers put the other edges under test:
  * H % 256 == 128 (a half-valid last N tile of the down GEMM and of the router);
  * I an odd multiple of 128 (gate/up N tiles of 128 gate + 128 up rows);
  * H = 128 (two k-blocks);
  * E not a multiple of 8 or 32, K = 1, no zero experts;
  * T on both sides of the CTA-pair threshold (1024), ragged against every tile.
Each runs the four step calls in both combine modes and checks routing bit for bit (away
from near ties), every permuted row's y (deterministic mode) and the whole output within
the bf16 bar, on every token. One shape also runs the backward."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
import oracle.moe_oracle as orc
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

pytestmark = pytest.mark.gpu

SHAPES = {
    #            T,    H,   I,  N,  Z, K
    "h384":    (777, 384, 128, 8, 4, 3),
    "h640_pair": (1100, 640, 384, 12, 0, 2),
    "e27":     (513, 896, 256, 20, 7, 5),
    "k1_i640": (2048, 384, 640, 6, 2, 1),
    "h128":    (64, 128, 128, 3, 1, 2),
}


def _cfg(name):
    T, H, I, N, Z, K = SHAPES[name]
    return wl.CONFIGS["proxy_bf16"].with_(name=f"shape_{name}", T=T, H=H, I=I, n_ffn=N,
                                          n_zero=Z, K=K)


@pytest.mark.parametrize("name", sorted(SHAPES))
@pytest.mark.parametrize("combine", ["deterministic", "fused"])
def test_odd_shape_layer_matches_oracle(cuda_device, name, combine):
    cfg = _cfg(name)
    case = gh.Case(cfg, seed=21)
    b = case.buffers(combine)
    out = abi.run_steps(b, case.x, case.w.w_router, None, case.w.bias, case.w.w_gate_up,
                        case.w.w_down)
    torch.cuda.synchronize()
    assert abi.read_device_status(b.ws) == 0
    gh.check_routing(case, b)
    gh.check_permutation(case, b, zero_init=False)
    L = case.gpu_logits(b)
    toks = list(range(cfg.T))
    o_out, _, _, y_rows, _, _ = gh.oracle_layer(case, L, toks)
    # tokens whose selection is a near tie may route differently on the two sides
    r = orc.route(L, gh.host(case.w.bias), cfg.n_ffn, cfg.K)
    same = np.all(np.sort(gh.host(b.topk_idx), 1) == np.sort(r.topk_idx, 1), axis=1)
    err = gh.row_rel_err(gh.host(out)[: cfg.T][same], o_out[same])
    assert err <= gh.TOL["bf16"], err
    if combine == "deterministic":
        row_of = gh.host(b.row_of).reshape(cfg.T, cfg.K)
        yp = gh.host(b.y_perm)
        keys = [key for key in sorted(y_rows) if same[key[0]]]
        if keys:
            got = np.stack([yp[row_of[t, k]] for (t, k) in keys])
            want = np.stack([y_rows[key] for key in keys])
            assert gh.row_rel_err(got, want) <= gh.TOL["bf16"]


def test_odd_shape_backward_matches_oracle(cuda_device):
    """H = 384 (half-valid last N tiles in every backward GEMM), I = 384, E = 16."""
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=600, H=384, I=384, n_ffn=12, n_zero=4, K=3)
    case = gh.Case(cfg, seed=22)
    b = case.buffers("deterministic")
    abi.run_steps(b, case.x, case.w.w_router, None, case.w.bias, case.w.w_gate_up, case.w.w_down)
    g = torch.Generator(device="cuda").manual_seed(5)
    dout = (torch.randn(cfg.T, cfg.H, device="cuda", generator=g) * 0.5).to(torch.bfloat16)
    dx = torch.empty(cfg.T, cfg.H, dtype=torch.float32, device="cuda")
    d_router = torch.empty(cfg.E, cfg.H, dtype=torch.float32, device="cuda")
    d_gu = torch.zeros(cfg.n_ffn, 2 * cfg.I, cfg.H, dtype=torch.float32, device="cuda")
    d_d = torch.zeros(cfg.n_ffn, cfg.H, cfg.I, dtype=torch.float32, device="cuda")
    ws = torch.zeros(abi.backward_workspace_size(b.shape), dtype=torch.uint8, device="cuda")
    abi.backward(b.shape, dout, case.x, case.w.w_router, case.w.w_gate_up, case.w.w_down,
                 b.logits, b.topk_idx, b.topk_gate, b.offsets, b.row_of, b.x_perm, b.h,
                 b.y_perm, dx, d_router, d_gu, d_d, ws)
    torch.cuda.synchronize()
    assert abi.read_device_status(ws) == 0
    ref = orc.moe_layer_backward(gh.host(case.x), gh.host(case.w.w_router), gh.host(case.w.bias),
                                 gh.host(case.w.w_gate_up), gh.host(case.w.w_down), cfg.n_ffn,
                                 cfg.K, gh.host(dout), cfg.ffn_out_scale,
                                 topk_idx=gh.host(b.topk_idx))
    assert gh.row_rel_err(gh.host(dx), ref.dx) <= gh.TOL["bf16"]
    assert gh.row_rel_err(gh.host(d_router), ref.d_router) <= gh.TOL["bf16"]
    counts = gh.host(b.counts)[: cfg.n_ffn]
    for e in np.nonzero(counts > 0)[0]:
        for got, want in ((gh.host(d_gu[e]), ref.d_gate_up[e]), (gh.host(d_d[e]), ref.d_down[e])):
            assert np.abs(got - want).max() / max(np.abs(want).max(), 1e-30) <= gh.TOL["bf16"]


FP32_SHAPES = {
    #            T,   H,   I,  N, Z, K
    "f_odd":   (50, 112, 36, 5, 3, 2),
    "f_prime": (301, 272, 129, 9, 0, 4),
    "f_k1":    (97, 64, 1, 2, 5, 1),
    "f_t700":  (700, 144, 40, 6, 2, 3),
}


@pytest.mark.parametrize("name", sorted(FP32_SHAPES))
@pytest.mark.parametrize("combine", ["deterministic", "fused"])
def test_odd_fp32_shape_layer_matches_oracle(cuda_device, name, combine):
    """fp32 layers (the CUDA-core FFN) take any I >= 1 and H % 16 == 0: I = 1, 36, 129 and
    H = 112, 272 (not multiples of 32), against the oracle within 1e-5. T = 700 takes the
    large-batch permutation (H = 144: 36 16-byte vectors per row, so the copy's second
    vector round covers four lanes only)."""
    T, H, I, N, Z, K = FP32_SHAPES[name]
    cfg = wl.CONFIGS["tiny_fp32"].with_(name=f"shape_{name}", T=T, H=H, I=I, n_ffn=N,
                                        n_zero=Z, K=K)
    case = gh.Case(cfg, seed=23)
    b = case.buffers(combine)
    out = abi.run_steps(b, case.x, case.w.w_router, None, case.w.bias, case.w.w_gate_up,
                        case.w.w_down)
    torch.cuda.synchronize()
    assert abi.read_device_status(b.ws) == 0
    gh.check_routing(case, b)
    gh.check_permutation(case, b, zero_init=False)
    L = case.gpu_logits(b)
    o_out, _, _, _, _, _ = gh.oracle_layer(case, L, list(range(cfg.T)))
    r = orc.route(L, gh.host(case.w.bias), cfg.n_ffn, cfg.K)
    same = np.all(np.sort(gh.host(b.topk_idx), 1) == np.sort(r.topk_idx, 1), axis=1)
    err = gh.row_rel_err(gh.host(out)[: cfg.T][same], o_out[same])
    assert err <= gh.TOL["fp32"], err


@pytest.mark.parametrize("bands", [(3, 5, 1, 1, 1, 1, 0, 0), (8, 1, 0, 0, 1, 0, 0, 8),
                                   (64, 64, 1, 0, 1, 1, 0, 3), (1, 8, 0, 1, 1, 0, 0, 64),
                                   (1, 1, 0, 0, 1, 1, 0, 1), (1, 1, 0, 1, 0, 0, 0, 0),
                                   (1, 1, 0, 1, 1, 1, 1, 8)])
def test_tile_order_changes_no_bits(cuda_device, bands):
    """The CTA-pair GEMMs visit an expert's M tiles in bands (MOE_TUNE_GATE_UP_BAND /
    MOE_TUNE_DOWN_BAND) and spread the tiles of single-tile experts among the others
    (MOE_TUNE_PAIR_INTERLEAVE), load only the A rows of the group (MOE_TUNE_PAIR_A_TRIM;
    the MMA rows past the group see stale shared memory and are dropped), and may load
    single-tile experts' weights evict-first (MOE_TUNE_PAIR_STREAM_HINT). Every output
    tile is still one cluster's, summed over K in the same order from the same rows, so
    any setting gives the same bits as the default one; with the largest expert holding
    thousands of rows (a dozen M tiles) and several experts of one tile, the settings here
    cut it into full and partial bands, with and without the spread, the trim and L2
    prefetches ahead of the loads (MOE_TUNE_PAIR_PREFETCH). Swapped
    tiles of at most 128 rows (MOE_TUNE_PAIR_SWAP_AB) against M = 128 tiles, and such rows
    on the one-CTA kernel (MOE_TUNE_PAIR_TAILS), are other MMA shapes, so other fp32
    summation orders: those agree within rounding."""
    cfg = wl.CONFIGS["proxy_bf16"].with_(T=3001)
    case = gh.Case(cfg, seed=21)
    b = case.buffers("deterministic")
    args = (b, case.x, case.w.w_router, None, case.w.bias, case.w.w_gate_up, case.w.w_down)
    abi.run_steps(*args)
    torch.cuda.synchronize()
    R = int(b.offsets[-1].item())
    counts = b.counts[: cfg.n_ffn]
    assert int(counts.max().item()) > 6 * 256
    assert int(((counts > 0) & (counts <= 256)).sum().item()) >= 3     # single-tile experts
    want = [b.h[:R].clone(), b.y_perm[:R].clone(), b.out.clone()]
    try:
        abi.set_tuning(abi.TUNE_GATE_UP_BAND, bands[0])
        abi.set_tuning(abi.TUNE_DOWN_BAND, bands[1])
        abi.set_tuning(abi.TUNE_PAIR_INTERLEAVE, bands[2])
        abi.set_tuning(abi.TUNE_PAIR_A_TRIM, bands[3])
        abi.set_tuning(abi.TUNE_PAIR_SWAP_AB, bands[4])
        abi.set_tuning(abi.TUNE_PAIR_STREAM_HINT, bands[5])
        abi.set_tuning(abi.TUNE_PAIR_TAILS, bands[6])
        abi.set_tuning(abi.TUNE_PAIR_PREFETCH, bands[7])
        for t in (b.h, b.y_perm, b.out):
            t.zero_()
        abi.run_steps(*args)
        torch.cuda.synchronize()
    finally:
        abi.set_tuning(abi.TUNE_GATE_UP_BAND, 0)
        abi.set_tuning(abi.TUNE_DOWN_BAND, 0)
        abi.set_tuning(abi.TUNE_PAIR_INTERLEAVE, 0)
        abi.set_tuning(abi.TUNE_PAIR_A_TRIM, 1)
        abi.set_tuning(abi.TUNE_PAIR_SWAP_AB, 1)
        abi.set_tuning(abi.TUNE_PAIR_STREAM_HINT, 1)
        abi.set_tuning(abi.TUNE_PAIR_TAILS, 0)
        abi.set_tuning(abi.TUNE_PAIR_PREFETCH, 0)
    assert abi.read_device_status(b.ws) == 0
    same = [torch.equal(w_, g_) for w_, g_ in zip(want, [b.h[:R], b.y_perm[:R], b.out])]
    if bands[4] and not bands[6]:
        assert all(same)
    else:
        # M = 128 tiles instead of swapped ones: other MMA shapes, so other fp32 summation
        # orders in the tensor cores; both must stay within rounding of each other
        for w_, g_ in zip(want, [b.h[:R], b.y_perm[:R], b.out]):
            assert gh.row_rel_err(gh.host(g_), gh.host(w_)) < 1e-2
