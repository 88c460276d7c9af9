"""Full-shape layers (hidden 6144, 512 FFN + 256 zero experts, K = 12, intermediate 2048)
on the GPU against the oracle, in the launch configuration the benchmark times (the
permuted copy of x, CTA-pair GEMMs for T >= 1024, one-CTA GEMMs at T = 128), on every
token:
  * routing and the permutation, bit-exact (near ties reported);
  * the router logits of every token (computed workloads);
  * every permuted row's expert output y (deterministic mode);
  * the layer output in both combine modes;
  * the FFN part alone (the fused epilogue into a zeroed accumulator), from the permuted
    copy and from rows gathered out of x, so that the zero-expert term, 10 to 100 times
    larger, cannot hide an FFN error.
The oracle runs over the batch 2048 tokens at a time, which keeps host memory bounded."""
import numpy as np
import pytest
import torch

import gpu_harness as gh
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CHUNK = 2048


@pytest.fixture(scope="module", params=["prefill_bf16", "decode_bf16", "skew_pid_bf16"])
def full_case(request, cuda_device):
    torch.cuda.empty_cache()
    case = gh.Case(wl.CONFIGS[request.param])
    yield case
    del case
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _ffn_alone(case, b, gathered: bool):
    """moe_grouped_ffn with the fused epilogue into a zeroed fp32 accumulator: the FFN part
    s * sum_k g_k y_k of every token, nothing else."""
    cfg = case.cfg
    acc = torch.zeros(cfg.T, cfg.H, dtype=torch.float32, device="cuda")
    abi.grouped_ffn(b.shape, case.x, None if gathered else b.x_perm, b.offsets,
                    case.w.w_gate_up, case.w.w_down, b.perm_token, b.row_gate, b.h, None, acc,
                    b.ws)
    return acc


def test_full_shape_layer_every_token(full_case, parity_report):
    case = full_case
    cfg = case.cfg
    report = {}
    results = {}
    for combine in ("fused", "deterministic"):
        b = case.buffers(combine)
        abi.run_steps(b, case.x, case.w.w_router, case.logits_in, case.w.bias,
                      case.w.w_gate_up, case.w.w_down)
        torch.cuda.synchronize()
        assert abi.read_device_status(b.ws) == 0
        gh.check_routing(case, b, report)
        gh.check_permutation(case, b, zero_init=False)
        results[combine] = b
    errs = {}
    if case.logits_in is None:
        errs["logits"] = gh.check_logits(case, results["fused"])        # every row
    bf, bd = results["fused"], results["deterministic"]
    ffn = {"ffn_copied": _ffn_alone(case, bf, False), "ffn_gathered": _ffn_alone(case, bf, True)}
    torch.cuda.synchronize()
    assert abi.read_device_status(bf.ws) == 0
    L = case.gpu_logits(bf)
    row_of = gh.host(bd.row_of).reshape(cfg.T, cfg.K)
    for k in ("out_fused", "out_deterministic", "y", "ffn_copied", "ffn_gathered"):
        errs[k] = 0.0
    n_rows = 0
    for t0 in range(0, cfg.T, CHUNK):
        t1 = min(cfg.T, t0 + CHUNK)
        toks = list(range(t0, t1))
        o_out, o_ffn, _, y_rows, _, _ = gh.oracle_layer(case, L, toks)
        for combine, b in results.items():
            e = gh.row_rel_err(gh.host(b.out[t0:t1]), o_out)
            errs[f"out_{combine}"] = max(errs[f"out_{combine}"], e)
        keys = list(y_rows)
        if keys:
            rows = torch.as_tensor([int(row_of[t, k]) for (t, k) in keys], device="cuda")
            got = gh.host(bd.y_perm[rows])
            want = np.stack([y_rows[key] for key in keys])
            errs["y"] = max(errs["y"], gh.row_rel_err(got, want))
            n_rows += len(keys)
        has = np.abs(o_ffn).max(axis=1) > 0
        for name, acc in ffn.items():
            got = gh.host(acc[t0:t1])
            errs[name] = max(errs[name], gh.row_rel_err(got[has], o_ffn[has]))
            assert (got[~has] == 0).all(), name            # no FFN pick: nothing added
    R = int(bd.offsets[-1].item())
    assert n_rows == R                                     # every permuted row was compared
    tol = gh.TOL[cfg.dtype]
    parity_report(
        f"{cfg.name}: T={cfg.T}, every token and all {R} FFN rows; max rel err "
        + ", ".join(f"{k} {v:.2e}" for k, v in errs.items() if k != "logits")
        + (f", logits {errs['logits']:.2e}" if "logits" in errs else "")
        + f" (bar {tol:g}); near ties {report['near_ties']}, set mismatches "
        f"{report['near_tie_set_mismatch']}, order near-ties {report['order_near_ties']}; "
        f"{report['ffn_hit']} FFN experts hit, max rows {report['max_rows']}")
    for k, v in errs.items():
        assert v <= (gh.LOGIT_RTOL if k == "logits" else tol), (k, v, errs)
