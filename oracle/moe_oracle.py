"""Plain CPU oracle of the LongCat-Flash MoE layer forward and of its PID bias update.

TEST INFRASTRUCTURE. Only the tests, the package smoke check and the benchmark's CPU
baseline leg may import this module. The product path (the CUDA library and its Python
binding) never imports, calls or links anything here, and this module imports nothing
from the product path.

It is written to be read against the pages, not to be fast: float64 numpy for every
floating-point step (numpy's matmul, exp and sort serve as library primitives), except
where the method takes a decision that both sides must take in the same precision:

  * the softmax probabilities are rounded to float32 and the biased scores p + b are
    formed by one float32 addition, so that expert selection is decided in float32;
  * the PID bias update is float32 arithmetic in a fixed order without fused
    multiply-add, so that the device must reproduce it bit for bit.

Sources (page title, then the section or claim on that page):
  [pool]   "LongCat-Flash Technical Report" digest, Key claims, report §2.1 / §2.4: the pool
           holds 512 FFN experts and 256 zero-computation experts; the router chooses K = 12
           per token from the combined pool; a zero-computation expert is an identity map
           and costs nothing.
  [bias]   same page, Key claims, report §2.1.1 and Fig. 3(b)-(c): an expert bias updated
           by a PID controller over token-routing frequency, refining the aux-loss-free
           bias of DeepSeek-V3 (the bias moves selection; gates stay the softmax values).
  [excl]   same page, Key claims, report §2.1.1 / §2.1.2: zero-computation experts are
           excluded from the bias update.
  [target] same page, Method: a PID controller on each FFN expert's running bias keeps
           the average number of activated FFN experts near a target.
  [shape]  same page, Key claims, report §2.4: hidden 6144, per-expert FFN intermediate 2048.
  [scale]  same page, Key claims, report §2.3.2 Eq. 8: a variance-compensation factor on
           the fine-grained experts' outputs (ffn_out_scale here; its value is not printed).
  [zero]   "LongCat-Flash" blog, Key Innovations: zero-computation experts bypass
           computation for simple tokens.
  [lbloss] "LongCat-Flash Technical Report" digest, Key claims, report §2.1.1 / §2.1.2
           Eqs. 3-5: the zero-computation experts' share is held by a device-level
           load-balance loss, DeepSeek-V3's balance loss extended so that all
           zero-computation experts form one virtual group (the equations are not
           printed).

Readings where the pages are silent (the report's equations are not printed):
  softmax over all E experts; bias added to the float32 probability (not the logit);
  ties broken toward the lower expert index; gates not renormalised over the K picks;
  FFN experts are indices [0, n_ffn); SwiGLU experts W_down (silu(W_gate x) * W_up x);
  PID in position form with per-expert frequency target target_ratio * K / n_ffn;
  load-balance loss as in lb_loss below (DeepSeek's f_i P_i form, device-level grouping
  with one FFN expert per group and one group of every zero-computation expert);
  backward with the expert selection held fixed (it is piecewise constant in the inputs)
  and no gradient to the bias (it only moves the selection and is set by the PID).

Parity pins: every function here is pinned in tests/test_oracle.py against closed forms,
brute force, invariants or independent library routines; none is "parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "router_logits", "softmax_probs", "biased_scores", "select_topk", "near_tie_gap",
    "route", "permute", "swiglu_expert", "moe_layer_forward", "PidState", "pid_init",
    "pid_update", "pid_stats", "lb_loss", "moe_layer_backward", "BackwardResult",
    "RouteResult", "PermuteResult",
]


# ---------------------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------------------

def router_logits(x, w_router) -> np.ndarray:
    """Router logits L[t, e] = sum_h x[t, h] * w_router[e, h], in float64.

    [pool]: the router scores every expert of the combined pool for every token.
    """
    x64 = np.asarray(x, dtype=np.float64)
    w64 = np.asarray(w_router, dtype=np.float64)
    return x64 @ w64.T


def softmax_probs(logits) -> np.ndarray:
    """p[t, e] = exp(L[t, e] - max_j L[t, j]) / sum_j exp(L[t, j] - max_j L[t, j]).

    Computed in float64 over all E experts (FFN and zero alike: [pool] says K is chosen
    from the combined pool) and rounded once to float32, the precision in which the
    selection is decided.
    """
    L = np.asarray(logits, dtype=np.float64)
    m = L.max(axis=1, keepdims=True)
    ex = np.exp(L - m)
    return (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)


def biased_scores(p32: np.ndarray, bias32: np.ndarray) -> np.ndarray:
    """Selection scores sigma[t, e] = p[t, e] + b[e], one float32 addition.

    [bias]: the bias only steers selection. A zero result is stored as +0 so that the
    ordering of equal scores is decided by the expert index alone.
    """
    p32 = np.asarray(p32, dtype=np.float32)
    b32 = np.asarray(bias32, dtype=np.float32)
    s = (p32 + b32[None, :]).astype(np.float32)
    s[s == 0] = np.float32(0.0)
    return s


def select_topk(scores32: np.ndarray, K: int) -> np.ndarray:
    """The K experts with the largest score, listed by (score descending, index ascending).

    A stable sort of the negated scores keeps equal scores in index order, which is the
    lower-index tie-break.
    """
    order = np.argsort(-np.asarray(scores32, dtype=np.float32), axis=1, kind="stable")
    return order[:, :K].astype(np.int32)


def near_tie_gap(scores32: np.ndarray, K: int) -> np.ndarray:
    """Gap between the K-th and (K+1)-th largest score of each token (float64 of the
    float32 scores); +inf when K equals the number of experts."""
    s = np.asarray(scores32, dtype=np.float32)
    if K >= s.shape[1]:
        return np.full(s.shape[0], np.inf)
    srt = -np.sort(-s, axis=1)
    return srt[:, K - 1].astype(np.float64) - srt[:, K].astype(np.float64)


@dataclass
class RouteResult:
    probs: np.ndarray       # [T, E] float32
    scores: np.ndarray      # [T, E] float32
    topk_idx: np.ndarray    # [T, K] int32
    topk_gate: np.ndarray   # [T, K] float32 (unbiased, not renormalised)
    counts: np.ndarray      # [E] int64, tokens per expert
    nffn_hist: np.ndarray   # [K + 1] int64, tokens with n FFN picks
    zgate: np.ndarray       # [T] float64, sum of the zero-expert gates of each token
    gap: np.ndarray         # [T] float64, K-th minus (K+1)-th score


def route(logits, bias32, n_ffn: int, K: int) -> RouteResult:
    """Softmax, bias-adjusted top-K, gates and the per-batch expert histogram.

    [pool] K picks from the combined pool; [bias] the bias moves selection while the gate
    is the unbiased probability of the chosen expert; gates are not renormalised, so a
    token routed only to zero experts keeps the mass sum(g) < 1 ([zero]).
    """
    p = softmax_probs(logits)
    s = biased_scores(p, bias32)
    T, E = p.shape
    idx = select_topk(s, K)
    gate = np.take_along_axis(p, idx, axis=1).astype(np.float32)
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.int64)
    n_ffn_picks = (idx < n_ffn).sum(axis=1)
    nffn_hist = np.bincount(n_ffn_picks, minlength=K + 1).astype(np.int64)
    zgate = np.where(idx >= n_ffn, gate.astype(np.float64), 0.0).sum(axis=1)
    return RouteResult(p, s, idx, gate, counts, nffn_hist, zgate, near_tie_gap(s, K))


# ---------------------------------------------------------------------------------------
# Permutation into expert-contiguous groups
# ---------------------------------------------------------------------------------------

@dataclass
class PermuteResult:
    offsets: np.ndarray     # [n_ffn + 1] int64, exclusive scan of the FFN-expert counts
    perm_token: np.ndarray  # [R] int64, token of each permuted row
    row_of: np.ndarray      # [T, K] int64, permuted row of each pick, -1 for zero experts


def permute(topk_idx, n_ffn: int) -> PermuteResult:
    """Group the (token, FFN expert) picks by expert: group e holds, in ascending token
    order, the tokens that picked e, and the groups follow each other in expert order.
    Zero-expert picks get no row (they need no GEMM: [pool], [zero])."""
    idx = np.asarray(topk_idx)
    T, K = idx.shape
    row_of = np.full((T, K), -1, dtype=np.int64)
    perm = []
    offsets = np.zeros(n_ffn + 1, dtype=np.int64)
    for e in range(n_ffn):
        toks, slots = np.nonzero(idx == e)      # row-major: ascending token order
        base = len(perm)
        for j, (t, k) in enumerate(zip(toks, slots)):
            row_of[t, k] = base + j
            perm.append(int(t))
        offsets[e + 1] = len(perm)
    return PermuteResult(offsets, np.asarray(perm, dtype=np.int64), row_of)


# ---------------------------------------------------------------------------------------
# Experts and the combine
# ---------------------------------------------------------------------------------------

def swiglu_expert(x_rows, w_gate_up_e, w_down_e) -> np.ndarray:
    """One FFN expert on rows of x: y = W_down (silu(W_gate x) * (W_up x)), float64.

    w_gate_up_e is [2I, H] with the gate projection in rows [0, I) and the up projection
    in rows [I, 2I); w_down_e is [H, I]; silu(a) = a / (1 + exp(-a)). [shape] gives the
    intermediate width; the three H x I matrices per expert agree with the activated
    parameter range of [pool] (see the activation identity pin).
    """
    x64 = np.atleast_2d(np.asarray(x_rows, dtype=np.float64))
    wgu = np.asarray(w_gate_up_e, dtype=np.float64)
    wd = np.asarray(w_down_e, dtype=np.float64)
    I = wgu.shape[0] // 2
    G = x64 @ wgu[:I].T
    U = x64 @ wgu[I:].T
    with np.errstate(over="ignore"):
        h = G / (1.0 + np.exp(-G)) * U
    return h @ wd.T


def moe_layer_forward(x, logits, bias32, w_gate_up, w_down, n_ffn: int, K: int,
                      ffn_out_scale: float = 1.0, tokens=None):
    """The layer output out[t] = sum over FFN picks k of s * g_k * y_{e_k}(x_t)
    + (sum over zero-expert picks k of g_k) * x_t, in float64.

    [pool]/[zero]: a zero-computation expert adds g * x and runs no GEMM; [scale]: s is
    the factor on the FFN experts' outputs. No capacity limit and no token dropping.

    tokens: optional list of token indices to evaluate (sampled parity at full size).
    Returns (out [n, H], ffn_part [n, H], zgate [n], y_rows) where y_rows maps
    (token, slot) -> that expert's output row y (float64), and the route result.
    """
    x_all = np.asarray(x)
    r = route(logits, bias32, n_ffn, K)
    toks = np.arange(x_all.shape[0]) if tokens is None else np.asarray(tokens)
    H = x_all.shape[1]
    out = np.zeros((len(toks), H))
    ffn = np.zeros((len(toks), H))
    y_rows = {}
    # group the requested tokens by expert so each expert's weights are read once
    by_expert: dict[int, list] = {}
    for i, t in enumerate(toks):
        for k in range(K):
            e = int(r.topk_idx[t, k])
            if e < n_ffn:
                by_expert.setdefault(e, []).append((i, int(t), k))
    for e, items in sorted(by_expert.items()):
        xs = np.stack([np.asarray(x_all[t], dtype=np.float64) for (_, t, _) in items])
        ys = swiglu_expert(xs, w_gate_up[e], w_down[e])
        for (i, t, k), y in zip(items, ys):
            y_rows[(t, k)] = y
    for i, t in enumerate(toks):
        xt = np.asarray(x_all[t], dtype=np.float64)
        for k in range(K):
            if r.topk_idx[t, k] < n_ffn:
                ffn[i] += ffn_out_scale * float(r.topk_gate[t, k]) * y_rows[(int(t), k)]
        out[i] = ffn[i] + r.zgate[t] * xt
    return out, ffn, r.zgate[toks], y_rows, r


# ---------------------------------------------------------------------------------------
# PID bias update of the FFN experts
# ---------------------------------------------------------------------------------------

@dataclass
class PidState:
    b0: np.ndarray        # [n_ffn] float32, the bias the controller started from
    integral: np.ndarray  # [n_ffn] float32, running sum of the errors
    prev_err: np.ndarray  # [n_ffn] float32, last step's error


def pid_init(bias32, n_ffn: int) -> PidState:
    b = np.asarray(bias32, dtype=np.float32)
    return PidState(b[:n_ffn].copy(), np.zeros(n_ffn, np.float32), np.zeros(n_ffn, np.float32))


def pid_update(counts, T: int, K: int, n_ffn: int, bias32, state: PidState,
               kp: float, ki: float, kd: float, target_ratio: float):
    """One PID step on the FFN experts' biases ([bias], [target], [excl]).

    Each step, in float32 and in this order:
      f_i   = counts_i / T                      routing frequency of FFN expert i
      tau   = (target_ratio * K) / n_ffn        per-expert share of the FFN-pick target
      e_i   = tau - f_i
      I_i  += e_i
      D_i   = e_i - prev_i
      b_i   = ((b0_i + kp * e_i) + ki * I_i) + kd * D_i
      prev_i = e_i
    Zero-computation experts' biases are returned unchanged ([excl]). With kp = kd = 0
    this is the integral-only (aux-loss-free style) update b_i += ki * e_i.
    Returns (new bias [E] float32, new PidState).
    """
    f32 = np.float32
    c = np.asarray(counts)[:n_ffn].astype(np.float32)
    f = c / f32(T)
    tau = (f32(target_ratio) * f32(K)) / f32(n_ffn)
    err = (tau - f).astype(np.float32)
    integ = (state.integral + err).astype(np.float32)
    deriv = (err - state.prev_err).astype(np.float32)
    b = (state.b0 + f32(kp) * err).astype(np.float32)
    b = (b + f32(ki) * integ).astype(np.float32)
    b = (b + f32(kd) * deriv).astype(np.float32)
    new_bias = np.asarray(bias32, dtype=np.float32).copy()
    new_bias[:n_ffn] = b
    return new_bias, PidState(state.b0.copy(), integ, err)


def pid_stats(counts, nffn_hist, T: int, K: int, n_ffn: int, err=None) -> np.ndarray:
    """Statistics of one step, in float64:
      [0] FFN activation ratio = mean FFN picks per token / K
      [1] mean FFN picks per token        [2] their standard deviation over tokens
      [3] max / mean tokens per FFN expert [4] number of FFN experts hit
      [5] share of all picks that went to zero experts
      [6] mean |e_i|                       [7] max |e_i|   (0 when err is None)
    Fig. 3(b)-(c) of the report tracks the first three ([bias])."""
    h = np.asarray(nffn_hist, dtype=np.float64)
    n = np.arange(len(h), dtype=np.float64)
    mean = (h * n).sum() / T
    var = max(0.0, (h * n * n).sum() / T - mean * mean)
    c = np.asarray(counts, dtype=np.float64)
    cf = c[:n_ffn]
    mean_load = cf.sum() / n_ffn
    out = np.zeros(8)
    out[0] = mean / K
    out[1] = mean
    out[2] = math.sqrt(var)
    out[3] = cf.max() / mean_load if mean_load > 0 else 0.0
    out[4] = float((cf > 0).sum())
    out[5] = c[n_ffn:].sum() / (T * K)
    if err is not None:
        a = np.abs(np.asarray(err, dtype=np.float64))
        out[6] = a.mean()
        out[7] = a.max()
    return out


# ---------------------------------------------------------------------------------------
# Device-level load-balance loss (forward value)
# ---------------------------------------------------------------------------------------

def lb_loss(logits, counts, n_ffn: int, K: int):
    """Load-balance loss of one batch of T tokens over E = n_ffn + n_zero experts, and
    the mean router probability of every expert.

    [lbloss] names the loss without printing it; this follows DeepSeek's balance loss:
      f_i = E * c_i / (K * T)      c_i = tokens that picked expert i (counts)
      P_i = (1/T) sum_t p[t, i]     p = softmax over all E experts, float64
    and its device-level form, in which experts are grouped and a group g contributes
    (mean of f_i over g) * (sum of P_i over g). The groups are one per FFN expert and
    one virtual group holding every zero-computation expert:
      L = sum_{i < n_ffn} f_i P_i + mean_{i >= n_ffn}(f_i) * sum_{i >= n_ffn} P_i.
    A perfectly balanced batch (c_i = K T / E, p = 1/E) gives L = 1. The weight of the
    loss in the training objective is left to the caller. Returns (L, P) in float64.
    """
    L = np.asarray(logits, dtype=np.float64)
    c = np.asarray(counts, dtype=np.float64)
    T, E = L.shape
    m = L.max(axis=1, keepdims=True)
    ex = np.exp(L - m)
    p = ex / ex.sum(axis=1, keepdims=True)
    P = p.sum(axis=0) / T
    f = E * c / (K * T)
    loss = float((f[:n_ffn] * P[:n_ffn]).sum())
    if E > n_ffn:
        loss += float(f[n_ffn:].mean() * P[n_ffn:].sum())
    return loss, P


# ---------------------------------------------------------------------------------------
# Backward of the layer
# ---------------------------------------------------------------------------------------

@dataclass
class BackwardResult:
    dx: np.ndarray          # [T, H]
    d_router: np.ndarray    # [E, H]
    d_gate_up: np.ndarray   # [N, 2I, H]
    d_down: np.ndarray      # [N, H, I]
    d_logits: np.ndarray    # [T, E]
    d_gate: np.ndarray      # [T, K]: gradient of each pick's gate
    topk_idx: np.ndarray    # the selection the gradient was taken at


def moe_layer_backward(x, w_router, bias32, w_gate_up, w_down, n_ffn: int, K: int, dout,
                       ffn_out_scale: float = 1.0, topk_idx=None, tokens=None,
                       experts=None) -> BackwardResult:
    """Gradients of the layer output with respect to x, W_r, W_gu and W_d, given the
    gradient dout of the output, in float64.

    The forward is the one of moe_layer_forward with L = x W_r^T: out[t] = sum over FFN
    picks of s g_k y_{e_k}(x_t) + sum over zero picks of g_k x_t, g_k = p[t, e_k],
    p = softmax(L[t]) ([pool], [zero], [scale]). The selection is held fixed (it is
    piecewise constant in the inputs); the bias only moves the selection ([bias]) and gets
    no gradient. topk_idx: the selection to differentiate at (default: route() of the
    float64 logits). Per pick (t, k) of FFN expert e, with G = W_g x, U = W_u x,
    sig = 1 / (1 + exp(-G)), h = G sig U, y = W_d h:
      d_gate[t, k] = s <dout_t, y>,      dy = s g_k dout_t
      d_down[e]   += dy h^T,             dh = W_d^T dy
      dG = dh U sig (1 + G (1 - sig)),   dU = dh G sig
      d_gate_up[e] += [dG; dU] x_t^T,   dx_t += W_g^T dG + W_u^T dU
    per zero pick: d_gate[t, k] = <dout_t, x_t>, dx_t += g_k dout_t; then
      dp[t, e] = sum of d_gate over the picks of e,   dL = p * (dp - <p, dp>)
      d_router = dL^T x,   dx += dL W_r.

    tokens / experts (full-size checks, where every gradient at once does not fit in host
    memory): the same quantities for a part only. With tokens given, dx, d_gate and
    d_logits hold those tokens' rows (every other row is zero) and d_router is None: a
    token's dx, gate and logit gradients need only its own picks' rows. With experts given,
    d_gate_up and d_down are dicts holding those experts' gradients only: an expert's
    weight gradients need all of its rows, whatever `tokens` says.
    """
    x64 = np.asarray(x, dtype=np.float64)
    wr = np.asarray(w_router, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    T, H = x64.shape
    E = wr.shape[0]
    L = x64 @ wr.T
    if topk_idx is None:
        topk_idx = route(L, bias32, n_ffn, K).topk_idx
    idx = np.asarray(topk_idx)
    m = L.max(axis=1, keepdims=True)
    ex = np.exp(L - m)
    p = ex / ex.sum(axis=1, keepdims=True)
    s = float(ffn_out_scale)
    want = np.ones(T, dtype=bool)
    if tokens is not None:
        want = np.zeros(T, dtype=bool)
        want[np.asarray(tokens, dtype=np.int64)] = True
    dx = np.zeros((T, H))
    d_gate = np.zeros((T, K))
    N = n_ffn
    I = np.asarray(w_gate_up[0]).shape[0] // 2
    if experts is None:
        full = set(range(N))
        d_gu = np.zeros((N, 2 * I, H))
        d_d = np.zeros((N, H, I))
    else:
        full = {int(e) for e in experts}
        d_gu, d_d = {}, {}
    hit = {int(v) for v in idx[want].ravel() if v < n_ffn}
    for e in sorted(hit | {e for e in full if (idx == e).any()}):
        tk = np.argwhere(idx == e)                       # (t, k) of every pick of e
        if e not in full:
            tk = tk[want[tk[:, 0]]]                      # only the wanted tokens' rows
        ts, ks = tk[:, 0], tk[:, 1]
        wgu = np.asarray(w_gate_up[e], dtype=np.float64)
        wd = np.asarray(w_down[e], dtype=np.float64)
        X = x64[ts]
        G = X @ wgu[:I].T
        U = X @ wgu[I:].T
        with np.errstate(over="ignore"):
            sig = 1.0 / (1.0 + np.exp(-G))
        h = G * sig * U
        y = h @ wd.T
        g = p[ts, e]
        dy = s * g[:, None] * dout[ts]
        d_gate[ts, ks] = s * (dout[ts] * y).sum(axis=1)
        dh = dy @ wd
        dG = dh * U * sig * (1.0 + G * (1.0 - sig))
        dU = dh * G * sig
        if e in full:
            d_d[e] = dy.T @ h
            gu_e = np.empty((2 * I, H))
            gu_e[:I] = dG.T @ X
            gu_e[I:] = dU.T @ X
            d_gu[e] = gu_e
        dx[ts] += dG @ wgu[:I] + dU @ wgu[I:]            # a token picks e at most once
    zt, zk = np.nonzero((idx >= n_ffn) & want[:, None])
    d_gate[zt, zk] = (dout[zt] * x64[zt]).sum(axis=1)
    for t, k in zip(zt, zk):
        dx[t] += p[t, idx[t, k]] * dout[t]
    d_gate[~want] = 0.0
    dp = np.zeros((T, E))
    np.add.at(dp, (np.repeat(np.arange(T), K), idx.ravel()), d_gate.ravel())
    dL = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    dL[~want] = 0.0
    d_router = dL.T @ x64 if tokens is None else None
    dx += dL @ wr
    dx[~want] = 0.0
    return BackwardResult(dx, d_router, d_gu, d_d, dL, d_gate, idx)
