"""Shared helpers of the GPU parity tests: draw a workload on the GPU, run the layer
through the C ABI, bring results to the host and compare them with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle.moe_oracle as orc
from mixture_experts_layer_29_b200 import abi
from mixture_experts_layer_29_b200 import workloads as wl

NEAR_TIE = 1e-6          # tokens whose K-th / (K+1)-th score gap is below this are reported
GATE_RTOL = 1e-6
LOGIT_RTOL = 1e-5
TOL = {"bf16": 2e-2, "fp32": 1e-5}


def row_rel_err(a, b) -> float:
    """max over rows of max_j |a - b| / max_j |b| (rows with b == 0 compare absolutely)."""
    a = np.asarray(a, np.float64).reshape(len(a), -1)
    b = np.asarray(b, np.float64).reshape(len(b), -1)
    num = np.abs(a - b).max(axis=1)
    den = np.abs(b).max(axis=1)
    den = np.where(den > 0, den, 1.0)
    return float((num / den).max()) if len(a) else 0.0


def host(t) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


class Case:
    """Inputs of one workload on the GPU."""

    def __init__(self, cfg: wl.MoEConfig, device="cuda", ffn=True, logits=None, seed=None,
                 step=0):
        self.cfg = cfg
        self.w = wl.draw_weights(cfg, device, seed=seed, ffn=ffn)
        self.x = wl.draw_tokens(cfg, device, seed=seed)
        if logits is not None:
            self.logits_in = logits
        elif cfg.skewed:
            self.logits_in = wl.draw_skewed_logits(cfg, device, seed=seed, step=step)
        else:
            self.logits_in = None

    def shape(self, combine="fused") -> abi.Shape:
        return abi.shape_of(self.cfg, combine)

    def buffers(self, combine="fused") -> abi.StepBuffers:
        return abi.StepBuffers.allocate(self.shape(combine), self.x.device)

    def route(self, b: abi.StepBuffers):
        abi.route(b.shape, self.x, self.w.w_router, self.logits_in, self.w.bias,
                  None if self.logits_in is not None else b.logits, b.topk_idx, b.topk_gate,
                  b.counts, b.nffn_hist, b.zgate, b.ws)

    def gpu_logits(self, b: abi.StepBuffers) -> np.ndarray:
        return host(self.logits_in if self.logits_in is not None else b.logits)


def compare_topk(idx, gate, r, report: dict | None = None):
    """GPU top-K against the oracle's route result r.

    The chosen expert *sets* are bit-exact on every token whose K-th / (K+1)-th score gap
    is >= NEAR_TIE. Inside the K picks, the order (score descending) must match except
    between neighbours whose oracle scores differ by less than NEAR_TIE: the two sides
    compute p with different rounding, so such an order is a tie too. Gates compared per
    expert within GATE_RTOL. Returns the tokens whose sets differ (all near ties)."""
    T, K = idx.shape
    near = r.gap < NEAR_TIE
    clear = ~near
    set_gpu, set_orc = np.sort(idx, 1), np.sort(r.topk_idx, 1)
    np.testing.assert_array_equal(set_gpu[clear], set_orc[clear])
    set_mism = np.nonzero((set_gpu != set_orc).any(axis=1))[0]
    assert set(set_mism.tolist()) <= set(np.nonzero(near)[0].tolist())
    same_set = ~(set_gpu != set_orc).any(axis=1)
    order_ties = 0
    for t in np.nonzero(same_set & (idx != r.topk_idx).any(axis=1))[0]:
        sc = r.scores[t, idx[t]].astype(np.float64)       # oracle scores in the GPU's order
        assert (sc[:-1] >= sc[1:] - NEAR_TIE).all(), (t, idx[t], r.topk_idx[t])
        order_ties += 1
    # gates per expert on tokens with the same set
    og = np.take_along_axis(r.topk_gate, np.argsort(r.topk_idx, 1), 1)
    gg = np.take_along_axis(gate, np.argsort(idx, 1), 1)
    g_err = np.abs(gg[same_set] - og[same_set]) / np.maximum(np.abs(og[same_set]), 1e-30)
    assert g_err.max(initial=0) <= GATE_RTOL, g_err.max()
    if report is not None:
        report.update(near_ties=int(near.sum()), near_tie_set_mismatch=int(len(set_mism)),
                      order_near_ties=int(order_ties))
    return set_mism


def check_routing(case: Case, b: abi.StepBuffers, report: dict | None = None):
    """Routing of the GPU against the oracle given the GPU's own fp32 logits (see
    compare_topk); counts and histograms exact (and consistent with the GPU's own
    indices)."""
    cfg = case.cfg
    L = case.gpu_logits(b)
    r = orc.route(L, host(case.w.bias), cfg.n_ffn, cfg.K)
    idx, gate = host(b.topk_idx), host(b.topk_gate)
    rep = {} if report is None else report
    mism = compare_topk(idx, gate, r, rep)
    counts, hist = host(b.counts), host(b.nffn_hist)
    np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=cfg.E))
    per_tok = (idx < cfg.n_ffn).sum(1)
    np.testing.assert_array_equal(hist, np.bincount(per_tok, minlength=cfg.K + 1))
    if len(mism) == 0:
        np.testing.assert_array_equal(counts, r.counts)
        np.testing.assert_array_equal(hist, r.nffn_hist)
    same = ~(np.sort(idx, 1) != np.sort(r.topk_idx, 1)).any(axis=1)
    zg = host(b.zgate)
    np.testing.assert_allclose(zg[same], r.zgate[same], rtol=1e-6, atol=1e-12)
    rep.update(ffn_hit=int((counts[:cfg.n_ffn] > 0).sum()), max_rows=int(counts[:cfg.n_ffn].max()),
               R=int(counts[:cfg.n_ffn].sum()))
    return r


def check_logits(case: Case, b: abi.StepBuffers, rows=None):
    L = host(b.logits)
    rows = np.arange(case.cfg.T) if rows is None else np.asarray(rows)
    ref = orc.router_logits(host(case.x)[rows], host(case.w.w_router))
    err = row_rel_err(L[rows], ref)
    assert err <= LOGIT_RTOL, err
    return err


def check_permutation(case: Case, b: abi.StepBuffers, zero_init: bool, copied: bool = True):
    """copied: moe_permute wrote the permuted copy x_perm (else only the indices)."""
    cfg = case.cfg
    idx = host(b.topk_idx)
    pm = orc.permute(idx, cfg.n_ffn)
    R = int(pm.offsets[-1])
    np.testing.assert_array_equal(host(b.offsets), pm.offsets)
    np.testing.assert_array_equal(host(b.perm_token)[:R], pm.perm_token)
    np.testing.assert_array_equal(host(b.row_of).reshape(cfg.T, cfg.K), pm.row_of)
    # rows hold the token's activations bit for bit, and the pick's gate
    if copied:
        perm = torch.as_tensor(pm.perm_token, device=b.x_perm.device, dtype=torch.long)
        assert torch.equal(b.x_perm[:R], case.x[perm])
    gate = host(b.topk_gate)
    ro = pm.row_of
    sel = ro >= 0
    np.testing.assert_array_equal(host(b.row_gate)[ro[sel]], gate[sel])
    if zero_init:
        zg = host(b.zgate).astype(np.float32)
        want = zg[:, None] * host(case.x).astype(np.float32)     # one fp32 product
        np.testing.assert_array_equal(host(b.out_acc)[: cfg.T], want)
    return pm


class LazyExperts:
    """A device weight tensor [n_ffn, ...] that hands the oracle one expert at a time on
    the host, so that only the experts it touches are copied."""

    def __init__(self, w):
        self.w = w

    def __getitem__(self, e):
        return host(self.w[e])


def oracle_layer(case: Case, L: np.ndarray, tokens):
    """Oracle output for the given tokens (float64) from the GPU's logits; weights of the
    experts those tokens hit are brought to the host one expert at a time."""
    cfg = case.cfg
    r = orc.route(L, host(case.w.bias), cfg.n_ffn, cfg.K)
    experts = sorted({int(e) for t in tokens for e in r.topk_idx[t] if e < cfg.n_ffn})
    x = host(case.x)
    out, ffn, zg, y_rows, rr = orc.moe_layer_forward(
        x, L, host(case.w.bias), LazyExperts(case.w.w_gate_up), LazyExperts(case.w.w_down),
        cfg.n_ffn, cfg.K, cfg.ffn_out_scale, tokens=tokens)
    return out, ffn, zg, y_rows, rr, experts
