"""Full-shape layers (hidden 6144, 512 FFN + 256 zero experts, K = 12, intermediate 2048)
on the GPU against the oracle: routing and permutation on every token, bit-exact; the
expert outputs and the layer output on a sample of tokens the oracle evaluates one by
one; in the launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _sample(cfg, n):
    rng = np.random.default_rng(123)
    toks = set(rng.choice(cfg.T, size=min(n, cfg.T), replace=False).tolist())
    toks |= {0, cfg.T - 1}
    return sorted(toks)


@pytest.fixture(scope="module", params=["prefill_bf16", "decode_bf16", "skew_pid_bf16"])
def full_case(request, cuda_device):
    case = gh.Case(wl.CONFIGS[request.param])
    yield case
    del case
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def test_full_shape_layer(full_case):
    case = full_case
    cfg = case.cfg
    report = {}
    results = {}
    for combine in ("fused", "deterministic"):
        b = case.buffers(combine)
        out = abi.run_steps(b, case.x, case.w.w_router, case.logits_in, case.w.bias,
                            case.w.w_gate_up, case.w.w_down)
        torch.cuda.synchronize()
        assert abi.read_device_status(b.ws) == 0
        gh.check_routing(case, b, report)
        gh.check_permutation(case, b, zero_init=False)
        if case.logits_in is None:
            gh.check_logits(case, b, rows=_sample(cfg, 64))
        results[combine] = b
    toks = _sample(cfg, 12 if cfg.T > 1000 else 24)
    L = case.gpu_logits(results["fused"])
    o_out, o_ffn, o_zg, y_rows, rr, experts = gh.oracle_layer(case, L, toks)
    tol = gh.TOL[cfg.dtype]
    for combine, b in results.items():
        err = gh.row_rel_err(gh.host(b.out)[toks], o_out)
        assert err <= tol, (combine, err)
    bd = results["deterministic"]
    row_of = gh.host(bd.row_of).reshape(cfg.T, cfg.K)
    keys = sorted(y_rows)
    got = np.stack([gh.host(bd.y_perm[int(row_of[t, k])]) for (t, k) in keys])
    want = np.stack([y_rows[k] for k in keys])
    err_y = gh.row_rel_err(got, want)
    assert err_y <= tol, err_y
    print(f"\n{cfg.name}: {report}, sampled tokens {len(toks)}, experts {len(experts)}, "
          f"y err {err_y:.2e}")


def test_full_shape_ffn_part_alone(full_case):
    """Fused epilogue into a zeroed accumulator: the FFN part of sampled tokens."""
    case = full_case
    cfg = case.cfg
    b = case.buffers("fused")
    case.route(b)
    abi.permute(b.shape, b.topk_idx, b.topk_gate, b.zgate, case.x, b.offsets, b.perm_token,
                b.row_of, b.row_gate, None, None, b.ws)
    b.out_acc.zero_()
    abi.grouped_ffn(b.shape, case.x, None, b.offsets, case.w.w_gate_up, case.w.w_down,
                    b.perm_token, b.row_gate, b.h, None, b.out_acc, b.ws)
    torch.cuda.synchronize()
    toks = _sample(cfg, 8)
    L = case.gpu_logits(b)
    _, o_ffn, _, _, _, _ = gh.oracle_layer(case, L, toks)
    has = np.abs(o_ffn).max(axis=1) > 0
    got = gh.host(b.out_acc)[toks]
    assert gh.row_rel_err(got[has], o_ffn[has]) <= gh.TOL[cfg.dtype]
    assert (got[~has] == 0).all()
