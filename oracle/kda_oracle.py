"""Float64 CPU oracle for the Kimi Delta Attention (KDA) layer.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` may import this module.  The product
path (the CUDA library and its Python binding) never imports it, and this
module imports nothing from the product package.

What it computes, and where each step comes from
------------------------------------------------
The pages describe the KDA layer only by its ingredients; the exact forms below
are the plainest reading consistent with all of them.

* llama.cpp PR #27754 "model: add GLM-5-Next", KDA commit description:
  - q|k|v are convolved together by ONE depthwise causal conv (the conv state
    is a single contiguous block), then SiLU is applied after the conv;
  - q and k are L2-normalised with the literal eps 1e-6 in the
    ``max(sqrt(sum), eps)`` form;
  - the decay gate is a bounded sigmoid (``gate_lower_bound`` is a required
    key), dt_bias is added per channel, A is per head and broadcast;
  - the decay acts on the KEY axis of the state (the value-axis spelling was
    the bug that commit fixed);
  - the output goes through a gated RMSNorm with a plain weight;
  - f, g and beta are read from the pre-conv hidden states, i.e. they enter
    as separate inputs here.
* glm53-flash-mlx README, quantization recipe: A_log and dt_bias are fp32.
* glm53-flash-mlx README, the published config: rms_norm_eps = 1e-5.

Readings taken where the pages are silent:

* log a_t = lb * sigmoid(exp(A_log[h]) * (f_t + dt_bias[h])), lb = -5 (bounded
  branch); with no lower bound, log a_t = -exp(A_log[h]) * softplus(f_t + dt_bias[h]);
* S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T, o_t = S_t^T q_t
  (state S is d_k x d_v, key axis = rows); b_t = sigmoid(beta_logit_t);
* conv: causal, left padded by the conv state (zeros when absent); tap K-1
  multiplies the current token; no bias; channel layout per head q(d)|k(d)|v(d);
* y = o / sqrt(mean(o^2) + 1e-5) * w * sigmoid(g), w of shape [d_v].

Everything here is float64 NumPy with explicit Python loops over tokens: slow
and meant to be read against the pages, not fast.
"""
from __future__ import annotations

import numpy as np

GATE_LOWER_BOUND = -5.0
L2_EPS = 1e-6
NORM_EPS = 1e-5


# ---------------------------------------------------------------------------
# elementwise pieces
# ---------------------------------------------------------------------------
def sigmoid(x):
    """Logistic function 1 / (1 + e^-x), evaluated without overflow."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def silu(x):
    """SiLU x * sigmoid(x), applied after the conv (PR #27754, KDA commit)."""
    x = np.asarray(x, dtype=np.float64)
    return x * sigmoid(x)


def l2_normalize(x, eps=L2_EPS):
    """x / max(||x||_2, eps) over the last axis.

    PR #27754, KDA commit: the q/k L2 eps is a literal 1e-6 and the norm is the
    ``max(sqrt(sum), eps)`` form, not ``sqrt(sum + eps)``.
    """
    x = np.asarray(x, dtype=np.float64)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, eps)


def softplus(x):
    """log(1 + e^x), evaluated without overflow."""
    return np.logaddexp(0.0, np.asarray(x, dtype=np.float64))


def log_decay(f, A_log, dt_bias, lb=GATE_LOWER_BOUND):
    """Per-key-channel log decay.

    Bounded-sigmoid branch (``lb`` given):
        log a = lb * sigmoid(exp(A_log[h]) * (f + dt_bias[h, :])), in [lb, 0].
    Softplus branch (``lb`` is None):
        log a = -exp(A_log[h]) * softplus(f + dt_bias[h, :]), in (-inf, 0].

    PR #27754, KDA commit: the bounded-sigmoid gate is selected by the
    ``gate_lower_bound`` key; dt_bias is added per channel before the reshape and
    the per-head A is broadcast over the channels.  PR #27754, "Metadata and
    tensor loading" commit: when that key is absent the softplus branch is
    selected, a different function rather than a missing clamp.  Its form here
    (the negative per-head rate exp(A_log) times softplus of the biased gate) is
    the plainest reading: the pages name the branch but do not write it out.
    f: [..., H, d]; A_log: [H]; dt_bias: [H, d].
    """
    f = np.asarray(f, dtype=np.float64)
    A = np.exp(np.asarray(A_log, dtype=np.float64))[:, None]
    z = f + np.asarray(dt_bias, dtype=np.float64)
    if lb is None:
        return -A * softplus(z)
    return lb * sigmoid(A * z)


def apply_key_decay(S, a):
    """Diag(a) S for a state S[..., d_k, d_v]: the decay scales the KEY axis.

    PR #27754, KDA commit: ne0 (the key axis) is the decay axis.
    """
    return a[..., :, None] * S


# ---------------------------------------------------------------------------
# prep: conv + SiLU + L2 norm + gate + beta
# ---------------------------------------------------------------------------
def causal_depthwise_conv(x, w, hist=None):
    """Depthwise causal conv over channels.

    x: [T, C] pre-conv inputs, w: [C, K], hist: [K-1, C] (oldest first) or None
    for zeros.  out[t, c] = sum_j w[c, j] * xp[t + j, c] where xp = [hist; x],
    so tap K-1 multiplies the current token.  Returns (out [T, C],
    new_hist [K-1, C] = the last K-1 rows of xp).
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    T, C = x.shape
    K = w.shape[1]
    if hist is None:
        hist = np.zeros((K - 1, C))
    xp = np.concatenate([np.asarray(hist, dtype=np.float64), x], axis=0)
    out = np.zeros((T, C))
    for j in range(K):
        out += w[:, j][None, :] * xp[j:j + T]
    return out, xp[T:].copy()


def prep(x, f, beta_logit, conv_w, A_log, dt_bias, conv_hist=None,
         lb=GATE_LOWER_BOUND, l2_eps=L2_EPS):
    """Prep for ONE sequence.

    x: [T, H, 3d] pre-conv q|k|v; f: [T, H, d]; beta_logit: [T, H];
    conv_w: [H, 3d, K]; A_log: [H]; dt_bias: [H, d];
    conv_hist: [K-1, H, 3d] or None (zeros); lb: the gate's lower bound, or
    None for the softplus branch (see ``log_decay``).
    Returns dict q, k, v [T, H, d], loga [T, H, d], beta [T, H],
    conv_hist [K-1, H, 3d] (new), window [K-1+T, H, 3d] (hist then x).
    """
    x = np.asarray(x, dtype=np.float64)
    T, H, C3 = x.shape
    d = C3 // 3
    K = conv_w.shape[-1]
    hist = None if conv_hist is None else np.asarray(conv_hist, np.float64).reshape(K - 1, H * C3)
    xt, new_hist = causal_depthwise_conv(x.reshape(T, H * C3),
                                         np.asarray(conv_w).reshape(H * C3, K), hist)
    xs = silu(xt).reshape(T, H, C3)
    q = l2_normalize(xs[..., :d], l2_eps)
    k = l2_normalize(xs[..., d:2 * d], l2_eps)
    v = xs[..., 2 * d:]
    loga = log_decay(f, A_log, dt_bias, lb)
    beta = sigmoid(beta_logit)
    hist_full = np.zeros((K - 1, H * C3)) if hist is None else hist
    window = np.concatenate([hist_full, x.reshape(T, H * C3)], axis=0).reshape(K - 1 + T, H, C3)
    return dict(q=q, k=k, v=v, loga=loga, beta=beta,
                conv_hist=new_hist.reshape(K - 1, H, C3), window=window)


# ---------------------------------------------------------------------------
# the recurrence (the definition)
# ---------------------------------------------------------------------------
def recurrence(q, k, v, loga, beta, S0=None, q_scale=1.0, return_states=False):
    """Token-by-token delta rule with per-key-channel decay.

    Per token t, for every leading unit (e.g. head) independently:
        S <- Diag(a_t) S                       (decay on the key axis)
        u  = b_t (v_t - S^T k_t)               (delta-rule correction)
        S <- S + k_t u^T                       (rank-1 write)
        o_t = q_scale * S^T q_t                (read after the write)
    which equals S_t = (I - b k k^T) Diag(a_t) S_{t-1} + b k v^T.  The order
    decay -> update -> read is the ordering PR #27754's KDA commit settles.

    q, k: [T, ..., d_k]; v: [T, ..., d_v]; loga: [T, ..., d_k]; beta: [T, ...];
    S0: [..., d_k, d_v] or None (zeros).  Returns (o [T, ..., d_v], S_T) or,
    with return_states, (o, S_T, states [T, ..., d_k, d_v]) where states[t] is
    the state after token t.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    loga = np.asarray(loga, np.float64)
    beta = np.asarray(beta, np.float64)
    T = q.shape[0]
    dk, dv = k.shape[-1], v.shape[-1]
    lead = k.shape[1:-1]
    S = np.zeros(lead + (dk, dv)) if S0 is None else np.array(S0, dtype=np.float64, copy=True)
    o = np.zeros((T,) + lead + (dv,))
    states = np.zeros((T,) + lead + (dk, dv)) if return_states else None
    for t in range(T):
        S = apply_key_decay(S, np.exp(loga[t]))
        r = np.einsum('...kv,...k->...v', S, k[t])
        u = beta[t][..., None] * (v[t] - r)
        S = S + k[t][..., :, None] * u[..., None, :]
        o[t] = q_scale * np.einsum('...kv,...k->...v', S, q[t])
        if return_states:
            states[t] = S
    if return_states:
        return o, S, states
    return o, S


def gated_rmsnorm(o, g, w, eps=NORM_EPS):
    """y = o / sqrt(mean(o^2) + eps) * w * sigmoid(g) over the last (d_v) axis.

    PR #27754, KDA commit: the output goes through an RMSNorm gated by sigmoid(g), with a
    plain per-channel weight;
    glm53-flash-mlx README: rms_norm_eps = 1e-5.
    """
    o = np.asarray(o, np.float64)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return o / np.sqrt(ms + eps) * np.asarray(w, np.float64) * sigmoid(g)


# ---------------------------------------------------------------------------
# whole layer, varlen
# ---------------------------------------------------------------------------
def layer(x, f, beta_logit, g, conv_w, A_log, dt_bias, norm_w, cu_seqlens,
          S0=None, conv_hist=None, lb=GATE_LOWER_BOUND, l2_eps=L2_EPS,
          norm_eps=NORM_EPS, q_scale=1.0, heads=None):
    """KDA layer over packed sequences.

    x: [Ttot, H, 3d]; f, g: [Ttot, H, d]; beta_logit: [Ttot, H];
    cu_seqlens: [N+1]; S0: [N, H, d, d] or None; conv_hist: [N, K-1, H, 3d]
    or None; lb as in ``prep`` (None selects the softplus decay branch).
    ``heads`` restricts the computation to a subset of heads (every
    head is independent); the returned arrays then hold only those heads.
    Returns dict y [Ttot, Hs, d], o, state [N, Hs, d, d], conv_hist
    [N, K-1, Hs, 3d], and the prep outputs.
    """
    x = np.asarray(x, np.float64)
    H = x.shape[1]
    hs = np.arange(H) if heads is None else np.asarray(heads)
    x = x[:, hs]
    f = np.asarray(f, np.float64)[:, hs]
    beta_logit = np.asarray(beta_logit, np.float64)[:, hs]
    g = np.asarray(g, np.float64)[:, hs]
    conv_w = np.asarray(conv_w, np.float64)[hs]
    A_log = np.asarray(A_log, np.float64)[hs]
    dt_bias = np.asarray(dt_bias, np.float64)[hs]
    cu = [int(c) for c in cu_seqlens]
    N = len(cu) - 1
    Ttot, Hs, C3 = x.shape
    d = C3 // 3
    K = conv_w.shape[-1]
    y = np.zeros((Ttot, Hs, d))
    o_all = np.zeros((Ttot, Hs, d))
    q_all = np.zeros((Ttot, Hs, d)); k_all = np.zeros((Ttot, Hs, d)); v_all = np.zeros((Ttot, Hs, d))
    la_all = np.zeros((Ttot, Hs, d)); b_all = np.zeros((Ttot, Hs))
    state = np.zeros((N, Hs, d, d))
    hist_out = np.zeros((N, K - 1, Hs, C3))
    for s in range(N):
        a, b = cu[s], cu[s + 1]
        h0 = None if conv_hist is None else np.asarray(conv_hist, np.float64)[s][:, hs]
        p = prep(x[a:b], f[a:b], beta_logit[a:b], conv_w, A_log, dt_bias, h0, lb, l2_eps)
        s0 = None if S0 is None else np.asarray(S0, np.float64)[s][hs]
        o, S = recurrence(p['q'], p['k'], p['v'], p['loga'], p['beta'], s0, q_scale)
        y[a:b] = gated_rmsnorm(o, g[a:b], norm_w, norm_eps)
        o_all[a:b] = o
        q_all[a:b], k_all[a:b], v_all[a:b] = p['q'], p['k'], p['v']
        la_all[a:b], b_all[a:b] = p['loga'], p['beta']
        state[s] = S
        hist_out[s] = p['conv_hist']
    return dict(y=y, o=o_all, state=state, conv_hist=hist_out, q=q_all, k=k_all,
                v=v_all, loga=la_all, beta=b_all)


# ---------------------------------------------------------------------------
# the steps either side: the fused input projection and the low-rank output gate
# ---------------------------------------------------------------------------
def projections(hidden, W_in, W_gb, H, d, gate_rank):
    """The layer's inputs from the hidden states, float64.

    glm53-flash-mlx README, quantization recipe: the runtime fuses the six KDA input
    projections into one matmul (they share the hidden width).  PR #27754, KDA commit:
    f, g and beta are read from the pre-conv hidden states, and the output gate is low
    rank, g_b(g_a(x)).  Reading taken (the pages name the pieces, not their layout): the
    six projections are q, k, v, f, beta and g_a, stacked as the rows of one weight
    W_in [3Hd + Hd + H + r, hidden] in the order q|k|v per head (the pre-conv x of the
    layer, [T, H, 3d]), f ([T, H, d]), the beta logit ([T, H]) and g_a ([T, r]); then
    g = g_a W_gb^T with W_gb [H d, r].  No bias.

    hidden: [T, hidden]; returns dict x, f, beta_logit, g_a, g.
    """
    hidden = np.asarray(hidden, np.float64)
    T = hidden.shape[0]
    Y = hidden @ np.asarray(W_in, np.float64).T
    nx, nf = 3 * H * d, H * d
    x = Y[:, :nx].reshape(T, H, 3 * d)
    f = Y[:, nx:nx + nf].reshape(T, H, d)
    beta_logit = Y[:, nx + nf:nx + nf + H]
    g_a = Y[:, nx + nf + H:nx + nf + H + gate_rank]
    g = (g_a @ np.asarray(W_gb, np.float64).T).reshape(T, H, d)
    return dict(x=x, f=f, beta_logit=beta_logit, g_a=g_a, g=g)


# ---------------------------------------------------------------------------
# speculative verify + rollback
# ---------------------------------------------------------------------------
def verify(q, k, v, loga, beta, g, norm_w, S0, q_scale=1.0, norm_eps=NORM_EPS):
    """Verify a block of draft tokens for one sequence without touching S0.

    Inputs are prep outputs for the block: q, k [Tb, H, d]; v, g [Tb, H, d];
    loga [Tb, H, d]; beta [Tb, H]; S0 [H, d, d].  Returns (y [Tb, H, d],
    tape [Tb, H, d, d]) with tape[j] the state after draft token j.
    dflash-mlx issue #63 (rollback for the KDA recurrent state) and PR #27754
    (recurrent-state rollback) motivate the tape; block size 8 is the DFlash2
    drafter's (issue #63, "Context").
    """
    o, _, states = recurrence(q, k, v, loga, beta, S0, q_scale, return_states=True)
    return gated_rmsnorm(o, g, norm_w, norm_eps), states


def rollback(S, conv_hist, tape, window, accepted):
    """Select the state after the accepted prefix of a verified block.

    S: [H, d, d]; conv_hist: [K-1, H, 3d]; tape: [Tb, H, d, d];
    window: [K-1+Tb, H, 3d] (old conv history followed by the block's
    pre-conv inputs); accepted L in 0..Tb.  L = 0 keeps S and conv_hist;
    otherwise S <- tape[L-1] and conv_hist <- window[L : L+K-1].
    """
    Km1 = conv_hist.shape[0]
    if accepted == 0:
        return np.array(S, copy=True), np.array(conv_hist, copy=True)
    return np.array(tape[accepted - 1], copy=True), np.array(window[accepted:accepted + Km1], copy=True)


# ---------------------------------------------------------------------------
# second spelling: chunkwise form of the same recurrence (float64)
# ---------------------------------------------------------------------------
def chunked_recurrence(q, k, v, loga, beta, S0=None, chunk=64, q_scale=1.0):
    """Chunkwise-parallel restatement of ``recurrence`` for ONE unit.

    q, k: [T, d_k]; v: [T, d_v]; loga: [T, d_k]; beta: [T]; S0: [d_k, d_v].
    Within a chunk with start state S and cumulative log decay
    G_r = sum_{i<=r} loga_i (per key channel):
        A[r,i] = b_r sum_c k_r k_i e^{G_r - G_i}   (i < r)
        M[r,i] = sum_c q_r k_i e^{G_r - G_i}       (i <= r)
        Tm = (I + A)^{-1} diag(b);  W = Tm (K * e^G);  U~ = Tm V
        U = U~ - W S;  O = (Q * e^G) S + M U
        S <- Diag(e^{G_last}) S + (K * e^{G_last - G})^T U
    This is the UT/WY form of the delta rule (DeltaNet chunkwise training,
    Yang et al. 2024) with the per-channel decay of gated linear attention.
    It exists only to check that algebra against the token loop.
    """
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64); loga = np.asarray(loga, np.float64)
    beta = np.asarray(beta, np.float64)
    T, dk = k.shape
    dv = v.shape[-1]
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, np.float64, copy=True)
    o = np.zeros((T, dv))
    for s in range(0, T, chunk):
        e = min(s + chunk, T)
        L = e - s
        G = np.cumsum(loga[s:e], axis=0)
        qc, kc, vc, bc = q[s:e], k[s:e], v[s:e], beta[s:e]
        A = np.zeros((L, L))
        M = np.zeros((L, L))
        for r in range(L):
            for i in range(r + 1):
                w = np.exp(G[r] - G[i])
                if i < r:
                    A[r, i] = bc[r] * np.sum(kc[r] * kc[i] * w)
                M[r, i] = np.sum(qc[r] * kc[i] * w)
        Tm = np.linalg.solve(np.eye(L) + A, np.diag(bc))
        W = Tm @ (kc * np.exp(G))
        Ut = Tm @ vc
        U = Ut - W @ S
        o[s:e] = q_scale * ((qc * np.exp(G)) @ S + M @ U)
        S = np.exp(G[-1])[:, None] * S + (kc * np.exp(G[-1][None, :] - G)).T @ U
    return o, S
