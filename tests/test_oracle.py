"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed form, brute
force on tiny inputs, an invariant the pages state, or an independent library routine
(torch / scipy in float64). The mutation tests at the end plant plausible mistakes in
the oracle and check that a pin catches each one.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle.moe_oracle as orc
from mixture_experts_layer_29_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng


# ----------------------------------------------------------------------------- logits

def test_logits_one_hot_selects_router_column():
    w = rng(1).standard_normal((5, 7))
    x = np.zeros((3, 7))
    x[0, 2] = 1.0
    x[1, 6] = 1.0
    x[2, 0] = -2.0
    L = orc.router_logits(x, w)
    assert L.shape == (3, 5)
    np.testing.assert_array_equal(L[0], w[:, 2])
    np.testing.assert_array_equal(L[1], w[:, 6])
    np.testing.assert_array_equal(L[2], -2.0 * w[:, 0])


def test_logits_match_torch_float64():
    x = rng(2).standard_normal((9, 33))
    w = rng(3).standard_normal((13, 33))
    ref = F.linear(torch.tensor(x), torch.tensor(w)).numpy()
    np.testing.assert_allclose(orc.router_logits(x, w), ref, rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------------------------- softmax

def test_softmax_two_experts_is_sigmoid_of_difference():
    L = rng(4).standard_normal((50, 2)) * 3
    p = orc.softmax_probs(L)
    ref = 1.0 / (1.0 + np.exp(L[:, 1] - L[:, 0]))
    np.testing.assert_allclose(p[:, 0], ref, rtol=2e-7)
    assert p.dtype == np.float32


def test_softmax_sums_to_one_and_matches_scipy():
    L = rng(5).standard_normal((64, 768)).astype(np.float32) * 0.55
    p = orc.softmax_probs(L)
    ref = scipy.special.softmax(L.astype(np.float64), axis=1)
    np.testing.assert_allclose(p, ref, rtol=1.5e-7, atol=0)
    np.testing.assert_allclose(p.astype(np.float64).sum(1), 1.0, atol=1e-5)
    # shift invariance of the exact softmax survives the float32 rounding
    np.testing.assert_array_equal(orc.softmax_probs(L.astype(np.float64) + 3.0), p)


# ----------------------------------------------------------------------------- selection

@pytest.mark.parametrize("E,K", [(6, 1), (6, 3), (8, 2), (8, 4), (10, 3)])
def test_topk_equals_brute_force_best_subset(E, K):
    r = rng(E * 10 + K)
    p = r.dirichlet(np.ones(E), size=200).astype(np.float32)
    b = r.uniform(-0.1, 0.1, E).astype(np.float32)
    s = orc.biased_scores(p, b)
    idx = orc.select_topk(s, K)
    for t in range(200):
        best = max(itertools.combinations(range(E), K),
                   key=lambda c: sum(float(s[t, e]) for e in c))
        assert set(idx[t]) == set(best)
        vals = [float(s[t, e]) for e in idx[t]]
        assert vals == sorted(vals, reverse=True)


def test_topk_ties_go_to_lower_index():
    s = np.array([[0.5, 0.7, 0.7, 0.1, 0.7, 0.0]], dtype=np.float32)
    assert list(orc.select_topk(s, 3)[0]) == [1, 2, 4]
    assert list(orc.select_topk(s, 4)[0]) == [1, 2, 4, 0]
    # -0 and +0 are the same score: index order decides
    p = np.array([[0.0, 0.25, 0.0]], dtype=np.float32)
    b = np.array([-0.0, -0.25, 0.0], dtype=np.float32)
    s = orc.biased_scores(p, b)
    assert list(orc.select_topk(s, 3)[0]) == [0, 1, 2]


def test_near_tie_gap_by_hand():
    s = np.array([[0.5, 0.3, 0.3, 0.125], [0.25, 0.75, 0.0, 0.5]], dtype=np.float32)
    np.testing.assert_array_equal(orc.near_tie_gap(s, 1), [0.5 - np.float32(0.3), 0.25])
    np.testing.assert_array_equal(orc.near_tie_gap(s, 2), [0.0, 0.25])
    np.testing.assert_array_equal(orc.near_tie_gap(s, 3), [np.float32(0.3) - 0.125, 0.25])
    assert np.isinf(orc.near_tie_gap(s, 4)).all()


def test_bias_moves_selection_not_gates():
    r = rng(7)
    L = r.standard_normal((300, 24)).astype(np.float32)
    b = r.uniform(-0.05, 0.05, 24).astype(np.float32)
    r0 = orc.route(L, np.zeros(24, np.float32), n_ffn=16, K=4)
    r1 = orc.route(L, b, n_ffn=16, K=4)
    assert not np.array_equal(r0.topk_idx, r1.topk_idx)          # selection moved
    for rr in (r0, r1):                                         # gate = unbiased p
        np.testing.assert_array_equal(rr.topk_gate, np.take_along_axis(rr.probs, rr.topk_idx, 1))
    np.testing.assert_array_equal(r0.probs, r1.probs)
    for t in range(300):                                        # same expert, same gate
        g0 = dict(zip(r0.topk_idx[t], r0.topk_gate[t]))
        g1 = dict(zip(r1.topk_idx[t], r1.topk_gate[t]))
        for e in set(g0) & set(g1):
            assert g0[e] == g1[e]


def test_constant_bias_shift_keeps_selection_off_near_ties():
    r = rng(8)
    L = r.standard_normal((400, 96)).astype(np.float32)
    b = r.uniform(-0.1, 0.1, 96).astype(np.float32)
    a = orc.route(L, b, 64, 6)
    c = orc.route(L, (b + np.float32(0.25)).astype(np.float32), 64, 6)
    clear = a.gap > 1e-6
    assert clear.mean() > 0.95
    np.testing.assert_array_equal(np.sort(a.topk_idx[clear], 1), np.sort(c.topk_idx[clear], 1))


def test_route_histograms():
    r = rng(9)
    L = r.standard_normal((257, 24)).astype(np.float32)
    res = orc.route(L, np.zeros(24, np.float32), 16, 4)
    assert res.counts.sum() == 257 * 4
    assert res.nffn_hist.sum() == 257
    per_tok = (res.topk_idx < 16).sum(1)
    assert (np.bincount(per_tok, minlength=5) == res.nffn_hist).all()
    for t in range(257):
        assert len(set(res.topk_idx[t])) == 4                  # K distinct experts
        z = sum(float(g) for e, g in zip(res.topk_idx[t], res.topk_gate[t]) if e >= 16)
        assert math.isclose(res.zgate[t], z, rel_tol=0, abs_tol=1e-15)
    assert (res.zgate < 1.0).all()                             # gates are not renormalised


# ----------------------------------------------------------------------------- permutation

def test_permutation_is_an_expert_grouped_bijection():
    r = rng(10)
    L = r.standard_normal((333, 40)).astype(np.float32)
    res = orc.route(L, r.uniform(-0.02, 0.02, 40).astype(np.float32), 30, 5)
    pm = orc.permute(res.topk_idx, 30)
    R = int((res.topk_idx < 30).sum())
    assert pm.offsets[-1] == R == len(pm.perm_token)
    np.testing.assert_array_equal(np.diff(pm.offsets), res.counts[:30])
    seen = np.zeros(R, bool)
    for t in range(333):
        for k in range(5):
            e, row = res.topk_idx[t, k], pm.row_of[t, k]
            if e >= 30:
                assert row == -1
                continue
            assert pm.offsets[e] <= row < pm.offsets[e + 1]
            assert pm.perm_token[row] == t
            assert not seen[row]
            seen[row] = True
    assert seen.all()
    for e in range(30):                                        # ascending tokens per group
        grp = pm.perm_token[pm.offsets[e]:pm.offsets[e + 1]]
        assert (np.diff(grp) > 0).all()


# ----------------------------------------------------------------------------- FFN / layer

def _torch_swiglu(x, wgu, wd):
    I = wgu.shape[0] // 2
    xt = torch.tensor(x, dtype=torch.float64)
    g = F.linear(xt, torch.tensor(wgu[:I], dtype=torch.float64))
    u = F.linear(xt, torch.tensor(wgu[I:], dtype=torch.float64))
    return F.linear(F.silu(g) * u, torch.tensor(wd, dtype=torch.float64)).numpy()


def test_single_ffn_expert_is_dense_swiglu_mlp():
    # one FFN expert, no zero experts, K = 1: p = 1 and the layer is a dense SwiGLU MLP
    r = rng(11)
    T, H, I = 7, 24, 10                     # non-square so a transposed weight shows
    x = r.standard_normal((T, H))
    wgu = r.standard_normal((1, 2 * I, H)) * 0.3
    wd = r.standard_normal((1, H, I)) * 0.3
    logits = r.standard_normal((T, 1)).astype(np.float32)
    out, ffn, zg, _, res = orc.moe_layer_forward(x, logits, np.zeros(1, np.float32), wgu, wd, 1, 1)
    assert (res.topk_gate == 1.0).all() and (zg == 0).all()
    np.testing.assert_allclose(out, _torch_swiglu(x, wgu[0], wd[0]), rtol=1e-12, atol=1e-12)


def test_textbook_topk_softmax_moe_without_zero_experts():
    # Z = 0 and b = 0: the layer is the plain top-K softmax MoE without renormalisation
    r = rng(12)
    T, H, I, N, K = 20, 16, 8, 6, 2
    x = r.standard_normal((T, H))
    wgu = r.standard_normal((N, 2 * I, H)) * 0.3
    wd = r.standard_normal((N, H, I)) * 0.3
    logits = (r.standard_normal((T, N)) * 2).astype(np.float32)
    out, _, zg, _, _ = orc.moe_layer_forward(x, logits, np.zeros(N, np.float32), wgu, wd, N, K,
                                             ffn_out_scale=1.0)
    # torch's softmax, rounded to float32 like the gates the layer carries
    p = torch.softmax(torch.tensor(logits, dtype=torch.float64), dim=1).float().double()
    top = torch.topk(p, K, dim=1)
    ref = np.zeros((T, H))
    for t in range(T):
        for g, e in zip(top.values[t].tolist(), top.indices[t].tolist()):
            ref[t] += g * _torch_swiglu(x[t:t + 1], wgu[e], wd[e])[0]
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    assert (zg == 0).all()


def test_zero_only_token_outputs_gate_sum_times_x_exactly():
    r = rng(13)
    T, H, I, N, Z, K = 12, 32, 8, 8, 6, 3
    x = r.standard_normal((T, H))
    wgu = r.standard_normal((N, 2 * I, H))
    wd = r.standard_normal((N, H, I))
    logits = wl.draw_forced_logits(T, N, Z, zero_only_tokens=[0, 3, 4, 11]).numpy()
    out, ffn, zg, _, res = orc.moe_layer_forward(x, logits, np.zeros(N + Z, np.float32), wgu, wd, N, K)
    p_ref = scipy.special.softmax(logits.astype(np.float64), axis=1)
    for t in [0, 3, 4, 11]:
        assert (res.topk_idx[t] >= N).all()
        assert (ffn[t] == 0).all()
        np.testing.assert_array_equal(out[t], zg[t] * x[t])       # identity experts
        # sum of the gates = mass of the K largest zero-expert probabilities (< 1: K < Z)
        want = np.sort(p_ref[t, N:])[::-1][:K].sum()
        assert math.isclose(zg[t], want, rel_tol=1e-6) and zg[t] < 1 - 1e-3


def test_output_is_linear_in_ffn_scale():
    r = rng(14)
    T, H, I, N, Z, K = 30, 16, 8, 5, 3, 3
    x = r.standard_normal((T, H))
    wgu = r.standard_normal((N, 2 * I, H)) * 0.5
    wd = r.standard_normal((N, H, I)) * 0.5
    L = r.standard_normal((T, N + Z)).astype(np.float32)
    b = np.zeros(N + Z, np.float32)
    o1, f1, zg, _, _ = orc.moe_layer_forward(x, L, b, wgu, wd, N, K, ffn_out_scale=1.0)
    o3, f3, _, _, _ = orc.moe_layer_forward(x, L, b, wgu, wd, N, K, ffn_out_scale=3.0)
    np.testing.assert_allclose(f3, 3.0 * f1, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(o3 - zg[:, None] * x, 3.0 * (o1 - zg[:, None] * x), rtol=1e-9,
                               atol=1e-12)


def test_sampled_tokens_equal_full_evaluation():
    r = rng(15)
    T, H, I, N, Z, K = 40, 16, 8, 6, 4, 3
    x = r.standard_normal((T, H))
    wgu = r.standard_normal((N, 2 * I, H))
    wd = r.standard_normal((N, H, I))
    L = r.standard_normal((T, N + Z)).astype(np.float32)
    b = r.uniform(-0.05, 0.05, N + Z).astype(np.float32)
    full, *_ = orc.moe_layer_forward(x, L, b, wgu, wd, N, K)
    part, *_ = orc.moe_layer_forward(x, L, b, wgu, wd, N, K, tokens=[3, 17, 39])
    # BLAS may block a different row count differently: equal up to float64 rounding
    np.testing.assert_allclose(part, full[[3, 17, 39]], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- PID

def _dyadic_counts(N, T, r):
    # counts chosen so that every float32 step below is exact
    return r.integers(0, T + 1, N)


def test_pid_integral_only_is_aux_loss_free_update():
    # kp = kd = 0: b_n = b0 + ki * sum_{j<=n} e_j; checked in exact rational arithmetic
    r = rng(16)
    N, Z, T, K = 8, 4, 64, 4
    ki, tr = 0.0625, 0.5
    bias = (r.integers(-64, 64, N + Z) / 1024.0).astype(np.float32)
    st = orc.pid_init(bias, N)
    b = bias
    acc = [Fraction(0)] * N
    tau = Fraction(tr) * K / N
    for _ in range(6):
        c = _dyadic_counts(N, T, r)
        b, st = orc.pid_update(np.concatenate([c, np.zeros(Z, int)]), T, K, N, b, st,
                               0.0, ki, 0.0, tr)
        for i in range(N):
            acc[i] += tau - Fraction(int(c[i]), T)
            assert Fraction(float(b[i])) == Fraction(float(bias[i])) + Fraction(ki) * acc[i]
        np.testing.assert_array_equal(b[N:], bias[N:])


def test_pid_constant_error_closed_form():
    # the same counts every step: e constant, I_n = n e, D_1 = e, D_n = 0 afterwards
    N, Z, T, K = 4, 2, 32, 4
    kp, ki, kd, tr = 0.5, 0.125, 0.25, 0.75
    counts = np.array([8, 0, 32, 16, 5, 7])
    bias = np.array([0.25, -0.5, 0.125, 0.0, 0.03125, -0.0625], np.float32)
    st = orc.pid_init(bias, N)
    b = bias
    tau = Fraction(3, 4) * 4 / 4
    e = [tau - Fraction(int(c), T) for c in counts[:N]]
    for n in range(1, 5):
        b, st = orc.pid_update(counts, T, K, N, b, st, kp, ki, kd, tr)
        for i in range(N):
            want = (Fraction(float(bias[i])) + Fraction(kp) * e[i] + Fraction(ki) * n * e[i]
                    + (Fraction(kd) * e[i] if n == 1 else 0))
            assert Fraction(float(b[i])) == want
        np.testing.assert_array_equal(b[N:], bias[N:])


def test_pid_leaves_zero_experts_bit_identical_and_moves_toward_target():
    r = rng(17)
    N, Z, T, K = 64, 32, 4096, 6
    bias = r.uniform(-0.1, 0.1, N + Z).astype(np.float32)
    bias[N + 3] = -0.0
    st = orc.pid_init(bias, N)
    counts = r.integers(0, 800, N + Z)
    b, st2 = orc.pid_update(counts, T, K, N, bias, st, 0.01, 0.001, 0.0, 8 / 12)
    assert b[N:].tobytes() == bias[N:].tobytes()
    tau = np.float32(np.float32(8 / 12) * np.float32(K)) / np.float32(N)
    over = counts[:N] / T > tau
    assert (b[:N][over] < bias[:N][over]).all()               # overloaded experts lose bias
    assert (b[:N][~over] >= bias[:N][~over]).all()


def test_pid_stats_from_histogram_match_per_token_values():
    r = rng(18)
    T, E, N, K = 500, 24, 16, 4
    L = r.standard_normal((T, E)).astype(np.float32)
    res = orc.route(L, r.uniform(-0.1, 0.1, E).astype(np.float32), N, K)
    st = orc.pid_stats(res.counts, res.nffn_hist, T, K, N)
    per_tok = (res.topk_idx < N).sum(1).astype(np.float64)
    assert math.isclose(st[1], per_tok.mean(), rel_tol=1e-12)
    assert math.isclose(st[2], per_tok.std(), rel_tol=1e-9)
    assert math.isclose(st[0], per_tok.mean() / K, rel_tol=1e-12)
    cf = res.counts[:N]
    assert math.isclose(st[3], cf.max() / cf.mean(), rel_tol=1e-12)
    assert st[4] == (cf > 0).sum()
    assert math.isclose(st[5], 1 - per_tok.sum() / (T * K), rel_tol=1e-12)


# ----------------------------------------------------------------------------- load-balance loss

@pytest.mark.parametrize("N,Z,K,T", [(4, 2, 3, 4), (16, 8, 4, 6), (8, 0, 2, 4), (6, 6, 4, 3)])
def test_lb_loss_balanced_batch_is_one(N, Z, K, T):
    """Uniform probabilities (p = 1/E) and counts K T / E on every expert: f_i = 1, so each
    FFN expert adds 1/E and the zero group adds Z/E; the loss is exactly 1."""
    E = N + Z
    assert (K * T) % E == 0
    loss, P = orc.lb_loss(np.zeros((T, E)), np.full(E, K * T // E), N, K)
    assert abs(loss - 1.0) < 1e-12
    np.testing.assert_allclose(P, 1.0 / E, rtol=1e-12)


def test_lb_loss_worked_example_by_hand():
    """Two tokens, two FFN and two zero experts, K = 2.
    Token 0 logits (ln 4, ln 2, 0, 0): exp = (4, 2, 1, 1) / 8 -> p = (1/2, 1/4, 1/8, 1/8).
    Token 1 logits (0, 0, ln 2, ln 4): p = (1/8, 1/8, 1/4, 1/2).
    P = mean over the tokens = (5/16, 3/16, 3/16, 5/16); f_i = 4 c_i / (2 * 2) = c_i.
    counts (2, 0, 1, 1): 2 * 5/16 + 0 + mean(1, 1) * (3/16 + 5/16) = 18/16.
    counts (0, 2, 2, 0): 0 + 2 * 3/16 + mean(2, 0) * 8/16 = 14/16."""
    L = np.array([[math.log(4), math.log(2), 0, 0], [0, 0, math.log(2), math.log(4)]])
    loss, P = orc.lb_loss(L, [2, 0, 1, 1], 2, 2)
    assert abs(loss - 18 / 16) < 1e-12
    np.testing.assert_allclose(P, [5 / 16, 3 / 16, 3 / 16, 5 / 16], rtol=1e-12)
    loss2, _ = orc.lb_loss(L, [0, 2, 2, 0], 2, 2)
    assert abs(loss2 - 14 / 16) < 1e-12


def test_lb_loss_zero_experts_form_one_virtual_group():
    """Moving picks between zero experts leaves the loss unchanged (one group); moving them
    between FFN experts does not. With a single zero expert every group is a singleton
    and the loss is DeepSeek's plain balance loss sum_i f_i P_i."""
    g = rng(5)
    T, N, Z, K = 50, 6, 4, 3
    L = g.standard_normal((T, N + Z)) * 2
    c = np.array([20, 10, 5, 5, 10, 0, 40, 20, 30, 10])
    base, _ = orc.lb_loss(L, c, N, K)
    c_zero_moved = c.copy(); c_zero_moved[6:] = [0, 50, 50, 0]
    assert abs(orc.lb_loss(L, c_zero_moved, N, K)[0] - base) < 1e-12
    c_ffn_moved = c.copy(); c_ffn_moved[:6] = [0, 0, 0, 0, 0, 50]
    assert abs(orc.lb_loss(L, c_ffn_moved, N, K)[0] - base) > 1e-3
    # Z = 1: singletons only
    L1 = L[:, : N + 1]
    c1 = c[: N + 1]
    p = scipy.special.softmax(L1, axis=1)
    plain = ((N + 1) * c1 / (K * T) * p.mean(axis=0)).sum()
    assert abs(orc.lb_loss(L1, c1, N, K)[0] - plain) < 1e-12


def test_lb_loss_collapsed_routing_reaches_E():
    """Every token sends its only pick (K = 1) to expert 0 with p_0 -> 1: f_0 = E, P_0 = 1,
    every other term 0, so the loss is E (its maximum)."""
    T, N, Z = 16, 5, 3
    L = np.zeros((T, N + Z)); L[:, 0] = 60.0
    c = np.zeros(N + Z, int); c[0] = T
    loss, P = orc.lb_loss(L, c, N, 1)
    assert abs(loss - (N + Z)) < 1e-9
    assert abs(P[0] - 1) < 1e-12


# ----------------------------------------------------------------------------- backward

def _bwd_case(seed=7, T=6, H=8, I=4, N=3, Z=2, K=3):
    g = rng(seed)
    x = g.standard_normal((T, H))
    wr = g.standard_normal((N + Z, H)) * 0.6
    bias = (g.uniform(-0.05, 0.05, N + Z)).astype(np.float32)
    wgu = g.standard_normal((N, 2 * I, H)) * 0.5
    wd = g.standard_normal((N, H, I)) * 0.5
    dout = g.standard_normal((T, H))
    return x, wr, bias, wgu, wd, dout, N, K


def _objective(x, wr, bias, wgu, wd, dout, N, K, s, idx):
    out, *_rest, r = orc.moe_layer_forward(x, x @ wr.T, bias, wgu, wd, N, K, s)
    assert (np.sort(r.topk_idx, 1) == np.sort(idx, 1)).all()     # selection unchanged
    return float((dout * out).sum())


def test_backward_matches_central_differences():
    """Directional derivatives of <dout, out> along random directions of each input, by
    central differences of the (pinned) forward, against the backward's gradients. The
    step keeps every token's selection (checked); the forward's float32 gates limit the
    agreement to ~1e-4 relative."""
    x, wr, bias, wgu, wd, dout, N, K = _bwd_case()
    s = 1.3
    b = orc.moe_layer_backward(x, wr, bias, wgu, wd, N, K, dout, s)
    g = rng(11)
    eps = 1e-3
    for name in ("x", "wr", "wgu", "wd"):
        args = dict(x=x, wr=wr, wgu=wgu, wd=wd)
        v = g.standard_normal(args[name].shape)
        grad = {"x": b.dx, "wr": b.d_router, "wgu": b.d_gate_up, "wd": b.d_down}[name]
        plus = dict(args); plus[name] = args[name] + eps * v
        minus = dict(args); minus[name] = args[name] - eps * v
        fd = (_objective(plus["x"], plus["wr"], bias, plus["wgu"], plus["wd"], dout, N, K, s, b.topk_idx)
              - _objective(minus["x"], minus["wr"], bias, minus["wgu"], minus["wd"], dout, N, K, s,
                           b.topk_idx)) / (2 * eps)
        an = float((grad * v).sum())
        assert abs(fd - an) <= 2e-3 * abs(an) + 1e-6, (name, fd, an)


def test_backward_matches_torch_autograd():
    """The same layer written with torch float64 ops, the selection fixed, differentiated
    by autograd: every gradient and the logit gradient agree to 1e-10."""
    x, wr, bias, wgu, wd, dout, N, K = _bwd_case(seed=3, T=9, Z=3, K=3)
    s = 0.7
    b = orc.moe_layer_backward(x, wr, bias, wgu, wd, N, K, dout, s)
    tx = torch.tensor(x, requires_grad=True)
    twr = torch.tensor(wr, requires_grad=True)
    twgu = torch.tensor(wgu, requires_grad=True)
    twd = torch.tensor(wd, requires_grad=True)
    I = wgu.shape[1] // 2
    logits = tx @ twr.T
    logits.retain_grad()
    p = torch.softmax(logits, dim=1)
    out = torch.zeros_like(tx)
    rows = []
    for t in range(x.shape[0]):
        acc = torch.zeros(x.shape[1], dtype=torch.float64)
        for k in range(K):
            e = int(b.topk_idx[t, k])
            if e < N:
                hh = F.silu(F.linear(tx[t], twgu[e, :I])) * F.linear(tx[t], twgu[e, I:])
                acc = acc + s * p[t, e] * F.linear(hh, twd[e])
            else:
                acc = acc + p[t, e] * tx[t]
        rows.append(acc)
    out = torch.stack(rows)
    (out * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(b.dx, tx.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(b.d_router, twr.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(b.d_gate_up, twgu.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(b.d_down, twd.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(b.d_logits, logits.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_restricted_to_tokens_and_experts_equals_the_full_one():
    """The backward restricted to some tokens (dx, gate and logit gradients) and some
    experts (weight gradients), as the full-size GPU check uses it, gives the same values
    as the full (pinned above) backward on those rows and experts, zero rows elsewhere
    and no router gradient."""
    x, wr, bias, wgu, wd, dout, N, K = _bwd_case(seed=5, T=12, N=4, Z=2, K=3)
    s = 0.9
    full = orc.moe_layer_backward(x, wr, bias, wgu, wd, N, K, dout, s)
    toks = [1, 4, 5, 11]
    hit = sorted({int(e) for e in full.topk_idx.ravel() if e < N})
    experts = hit[:2] + [e for e in range(N) if e not in hit][:1]
    part = orc.moe_layer_backward(x, wr, bias, wgu, wd, N, K, dout, s,
                                  topk_idx=full.topk_idx, tokens=toks, experts=experts)
    rest = np.setdiff1d(np.arange(x.shape[0]), toks)
    for a, b in ((part.dx, full.dx), (part.d_gate, full.d_gate), (part.d_logits, full.d_logits)):
        np.testing.assert_allclose(a[toks], b[toks], rtol=1e-12, atol=1e-14)
        assert (a[rest] == 0).all()
    assert part.d_router is None
    for e in experts:
        if e in hit:
            np.testing.assert_allclose(part.d_gate_up[e], full.d_gate_up[e], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(part.d_down[e], full.d_down[e], rtol=1e-12, atol=1e-14)
        else:
            assert e not in part.d_gate_up and e not in part.d_down
            assert (full.d_gate_up[e] == 0).all()
    assert set(part.d_gate_up) == set(experts) & set(hit)


# ----------------------------------------------------------------------------- pages' numbers

def test_activated_parameter_identity_from_the_pages():
    """12 FFN picks x 3 H x I matrices x 28 layers = max - min activated parameters.

    The pages print 18.6B-31.3B activated with K = 12 over 512 FFN + 256 zero experts,
    hidden 6144, expert intermediate 2048, 28 layers. Three H x I matrices per expert
    (a SwiGLU expert) make the span exactly the 12 FFN picks; two (a plain MLP) would not.
    """
    with open(os.path.join(GOLDEN, "longcat_flash_facts.json")) as f:
        facts = json.load(f)
    per_pick = 3 * facts["hidden"] * facts["expert_intermediate"] * facts["layers"]
    span = facts["activated_max_billion"] - facts["activated_min_billion"]
    assert abs(facts["top_k"] * per_pick / 1e9 - span) < 0.05 + 1e-9
    two_mat = 2 * facts["hidden"] * facts["expert_intermediate"] * facts["layers"]
    assert abs(facts["top_k"] * two_mat / 1e9 - span) > 3.0
    # the average activation corresponds to ~8 of 12 picks on FFN experts (PID target)
    mean_ffn = (facts["activated_avg_billion"] - facts["activated_min_billion"]) / (per_pick / 1e9)
    assert abs(mean_ffn - 8.0) < 0.1


# ----------------------------------------------------------------------------- mutation tests

def test_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible mistakes in the oracle (on the CPU) and check a pin fails."""
    # 1. gates renormalised over the K picks -> the zero-only identity pin breaks
    orig_route = orc.route

    def renorm_route(logits, bias32, n_ffn, K):
        r = orig_route(logits, bias32, n_ffn, K)
        g = r.topk_gate / r.topk_gate.sum(1, keepdims=True)
        r.topk_gate = g.astype(np.float32)
        r.zgate = np.where(r.topk_idx >= n_ffn, g, 0).sum(1)
        return r
    monkeypatch.setattr(orc, "route", renorm_route)
    with pytest.raises(AssertionError):
        test_zero_only_token_outputs_gate_sum_times_x_exactly()
    monkeypatch.setattr(orc, "route", orig_route)

    # 2. bias added to the gate as well -> the bias/gate pin breaks
    orig_take = np.take_along_axis

    def biased_route(logits, bias32, n_ffn, K):
        r = orig_route(logits, bias32, n_ffn, K)
        r.topk_gate = orig_take(r.scores, r.topk_idx, 1)
        return r
    monkeypatch.setattr(orc, "route", biased_route)
    with pytest.raises(AssertionError):
        test_bias_moves_selection_not_gates()
    monkeypatch.setattr(orc, "route", orig_route)

    # 3. gate and up projections swapped -> the dense SwiGLU pin breaks
    orig_sw = orc.swiglu_expert

    def swapped(x, wgu, wd):
        I = np.asarray(wgu).shape[0] // 2
        return orig_sw(x, np.concatenate([np.asarray(wgu)[I:], np.asarray(wgu)[:I]]), wd)
    monkeypatch.setattr(orc, "swiglu_expert", swapped)
    with pytest.raises(AssertionError):
        test_single_ffn_expert_is_dense_swiglu_mlp()
    monkeypatch.setattr(orc, "swiglu_expert", orig_sw)

    # 4. tie broken toward the higher index -> the tie pin breaks
    orig_sel = orc.select_topk
    monkeypatch.setattr(orc, "select_topk",
                        lambda s, K: (s.shape[1] - 1 - np.argsort(-s[:, ::-1], 1, kind="stable"))[:, :K])
    with pytest.raises(AssertionError):
        test_topk_ties_go_to_lower_index()
    monkeypatch.setattr(orc, "select_topk", orig_sel)

    # 5. derivative sign flipped in the PID -> the closed-form pin breaks
    orig_pid = orc.pid_update

    def bad_pid(c, T, K, N, b, st, kp, ki, kd, tr):
        return orig_pid(c, T, K, N, b, st, kp, ki, -kd, tr)
    monkeypatch.setattr(orc, "pid_update", bad_pid)
    with pytest.raises(AssertionError):
        test_pid_constant_error_closed_form()
    monkeypatch.setattr(orc, "pid_update", orig_pid)

    # 6. load-balance loss: the zero group's f summed instead of averaged -> the
    #    balanced-batch pin breaks; P averaged over experts instead of tokens -> the
    #    worked example breaks
    orig_lb = orc.lb_loss

    def lb_sum(logits, counts, n_ffn, K):
        loss, P = orig_lb(logits, counts, n_ffn, K)
        E = np.asarray(logits).shape[1]
        f = E * np.asarray(counts, float) / (K * np.asarray(logits).shape[0])
        return loss + (f[n_ffn:].sum() - f[n_ffn:].mean()) * P[n_ffn:].sum(), P
    monkeypatch.setattr(orc, "lb_loss", lb_sum)
    with pytest.raises(AssertionError):
        test_lb_loss_balanced_batch_is_one(4, 2, 3, 4)
    monkeypatch.setattr(orc, "lb_loss", orig_lb)

    def lb_axis(logits, counts, n_ffn, K):
        Lg = np.asarray(logits, float)
        p = np.exp(Lg - Lg.max(1, keepdims=True)); p /= p.sum(1, keepdims=True)
        P = np.resize(p.mean(axis=1), Lg.shape[1])          # wrong axis
        E = Lg.shape[1]
        f = E * np.asarray(counts, float) / (K * Lg.shape[0])
        return float((f[:n_ffn] * P[:n_ffn]).sum() + f[n_ffn:].mean() * P[n_ffn:].sum()), P
    monkeypatch.setattr(orc, "lb_loss", lb_axis)
    with pytest.raises(AssertionError):
        test_lb_loss_worked_example_by_hand()
    monkeypatch.setattr(orc, "lb_loss", orig_lb)

    # 7. backward: a gate/up gradient off by 0.1% -> the autograd pin; the down-projection
    #    gradient with its columns reversed -> the central-differences pin
    orig_bwd = orc.moe_layer_backward

    def bwd_scaled(x, wr, bias, wgu, wd, N, K, dout, s=1.0, topk_idx=None):
        r = orig_bwd(x, wr, bias, wgu, wd, N, K, dout, s, topk_idx)
        r.d_gate_up = r.d_gate_up * 0.999
        return r
    monkeypatch.setattr(orc, "moe_layer_backward", bwd_scaled)
    with pytest.raises(AssertionError):
        test_backward_matches_torch_autograd()
    monkeypatch.setattr(orc, "moe_layer_backward", orig_bwd)

    def bwd_wrong_down(x, wr, bias, wgu, wd, N, K, dout, s=1.0, topk_idx=None):
        r = orig_bwd(x, wr, bias, wgu, wd, N, K, dout, s, topk_idx)
        r.d_down = np.ascontiguousarray(np.flip(r.d_down, axis=2))
        return r
    monkeypatch.setattr(orc, "moe_layer_backward", bwd_wrong_down)
    with pytest.raises(AssertionError):
        test_backward_matches_central_differences()
    monkeypatch.setattr(orc, "moe_layer_backward", orig_bwd)
    monkeypatch.setattr(orc, "pid_update", orig_pid)
