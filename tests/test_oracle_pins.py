"""Pins that tie the float64 oracle to facts outside itself.

Each check compares the oracle with something it does not contain: textbook
constants, hand-derived values (tests/golden/), closed forms, a brute-force
product of explicit transition matrices, invariants, and NumPy library
routines.  The mutation controls at the bottom plant a plausible mistake in
the oracle and require at least one pin to catch it (in the manner of the
negative control in the glm53-flash-mlx README's test list, where a deliberately
broken activation is shown to move the logits).
"""
import math
import os

import numpy as np
import pytest

from oracle import kda_oracle as ko

HERE = os.path.dirname(os.path.abspath(__file__))
SIG1 = 0.7310585786300049   # e / (1 + e)
SIG2 = 0.8807970779778823   # e^2 / (1 + e^2)


def _rng(seed):
    return np.random.default_rng(seed)


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# ---------------------------------------------------------------------------
# pin functions: each returns an error that must be tiny for a correct oracle
# ---------------------------------------------------------------------------
def pin_activations():
    err = 0.0
    err = max(err, abs(ko.sigmoid(np.array([0.0]))[0] - 0.5))
    err = max(err, abs(ko.sigmoid(np.array([1.0]))[0] - SIG1))
    err = max(err, abs(ko.sigmoid(np.array([-1.0]))[0] - (1 - SIG1)))
    err = max(err, abs(ko.silu(np.array([1.0]))[0] - SIG1))
    err = max(err, abs(ko.silu(np.array([-1.0]))[0] + (1 - SIG1)))
    err = max(err, abs(ko.silu(np.array([2.0]))[0] - 2 * SIG2))
    big = ko.sigmoid(np.array([-1e4, 1e4]))
    err = max(err, abs(big[0]) + abs(big[1] - 1.0))
    return err


def pin_log_decay():
    """Closed forms of lb * sigmoid(exp(A_log) (f + dt_bias))."""
    H, d = 2, 3
    dtb = np.array([[0.3, -0.2, 0.1], [0.0, 0.5, -0.5]])
    A_log = np.array([math.log(2.0), 0.0])
    # f = -dt_bias -> sigmoid(0) = 1/2 -> lb/2
    e1 = np.abs(ko.log_decay(-dtb, A_log, dtb, -5.0) + 2.5).max()
    # head 0: exp(A_log) = 2, f + dt_bias = 0.5 -> -5 sigmoid(1)
    f = 0.5 - dtb
    e2 = abs(ko.log_decay(f, A_log, dtb, -5.0)[0, 0] + 5 * SIG1)
    # head 1: exp(A_log) = 1, f + dt_bias = 1 -> -5 sigmoid(1)
    e3 = abs(ko.log_decay(1.0 - dtb, A_log, dtb, -5.0)[1, 2] + 5 * SIG1)
    # saturation: lb for large f, exactly 0 for very negative f
    hi = ko.log_decay(np.full((H, d), 1e4), A_log, dtb, -5.0)
    lo = ko.log_decay(np.full((H, d), -1e4), A_log, dtb, -5.0)
    e4 = np.abs(hi + 5.0).max() + np.abs(lo).max()
    return max(e1, e2, e3, e4)


LN1PE = 1.3132616875182228   # ln(1 + e)


def pin_softplus_decay():
    """Closed forms of the softplus branch, -exp(A_log) * softplus(f + dt_bias), selected
    when the gate has no lower bound (lb None)."""
    H, d = 2, 3
    dtb = np.array([[0.3, -0.2, 0.1], [0.0, 0.5, -0.5]])
    A_log = np.array([math.log(2.0), 0.0])
    # f = -dt_bias: softplus(0) = ln 2 -> -exp(A_log) ln 2 per head
    g0 = ko.log_decay(-dtb, A_log, dtb, None)
    e1 = max(np.abs(g0[0] + 2 * math.log(2.0)).max(), np.abs(g0[1] + math.log(2.0)).max())
    # f + dt_bias = 1: softplus(1) = ln(1 + e)
    g1 = ko.log_decay(1.0 - dtb, A_log, dtb, None)
    e2 = max(np.abs(g1[0] + 2 * LN1PE).max(), np.abs(g1[1] + LN1PE).max())
    # large argument: softplus(x) = x + ln(1 + e^-x) -> x; very negative: -> e^x -> 0
    g2 = ko.log_decay(50.0 - dtb, A_log, dtb, None)
    e3 = max(np.abs(g2[0] + 100.0).max(), np.abs(g2[1] + 50.0).max())
    g3 = ko.log_decay(np.full((H, d), -800.0), A_log, dtb, None)
    e4 = np.abs(g3).max()
    # no lower bound: log a keeps growing with the gate (past -5 of the bounded branch)
    e5 = 0.0 if ko.log_decay(np.full((1, 1), 10.0), np.zeros(1), np.zeros((1, 1)), None)[0, 0] < -9.9 else 1.0
    return max(e1, e2, e3, e4, e5)


def pin_q_scale():
    """o = q_scale S^T q: the hand example's outputs at q_scale = 2 are twice those at
    1 and the state is unchanged; through the layer with a huge RMSNorm eps (so y is
    proportional to o) y doubles too."""
    gv = _read_golden('recurrence_d2_hand.txt')
    q = np.stack([gv['q1'], gv['q2']])
    k = np.stack([gv['k1'], gv['k2']])
    v = np.stack([gv['v1'], gv['v2']])
    loga = np.log(np.stack([gv['a1'], gv['a2']]))
    beta = np.array([gv['b1'][0], gv['b2'][0]])
    o2, S2 = ko.recurrence(q, k, v, loga, beta, q_scale=2.0)
    e1 = max(np.abs(o2[0] - 2 * gv['o1']).max(), np.abs(o2[1] - 2 * gv['o2']).max(),
             np.abs(S2.reshape(-1) - gv['S2']).max())
    inp = _layer_inputs(19, 9)
    y1 = ko.layer(cu_seqlens=[0, 9], **inp, norm_eps=1e12)['y']
    y2 = ko.layer(cu_seqlens=[0, 9], **inp, norm_eps=1e12, q_scale=2.0)['y']
    e2 = np.abs(y2 - 2 * y1).max() / np.abs(y1).max()
    return max(e1, e2)


def pin_projections():
    """The fused projection against a brute-force triple loop on a tiny case, and the
    routing of its rows by hand: with W_in the identity on the first rows, x, f, the
    beta logit and g_a are consecutive slices of the hidden state."""
    rng = _rng(20)
    T, H, d, r = 3, 2, 2, 2
    n = 3 * H * d + H * d + H + r            # 12 + 4 + 2 + 2 = 20
    hid = n + 3
    hidden = rng.standard_normal((T, hid))
    W_in = rng.standard_normal((n, hid))
    W_gb = rng.standard_normal((H * d, r))
    p = ko.projections(hidden, W_in, W_gb, H, d, r)
    Y = np.zeros((T, n))
    for t in range(T):
        for j in range(n):
            acc = 0.0
            for c in range(hid):
                acc += hidden[t, c] * W_in[j, c]
            Y[t, j] = acc
    G = np.zeros((T, H * d))
    for t in range(T):
        for j in range(H * d):
            G[t, j] = sum(Y[t, 16 + H + c] * W_gb[j, c] for c in range(r))
    e1 = max(np.abs(p['x'].reshape(T, -1) - Y[:, :12]).max(),
             np.abs(p['f'].reshape(T, -1) - Y[:, 12:16]).max(),
             np.abs(p['beta_logit'] - Y[:, 16:18]).max(), np.abs(p['g_a'] - Y[:, 18:20]).max(),
             np.abs(p['g'].reshape(T, -1) - G).max())
    eye = np.zeros((n, hid))
    eye[:, :n] = np.eye(n)
    q = ko.projections(hidden, eye, W_gb, H, d, r)
    # x[t, h, :] = q_h | k_h | v_h: head 1's k is hidden columns 6 + 2 .. 6 + 3
    e2 = max(np.abs(q['x'][:, 1, 2:4] - hidden[:, 8:10]).max(),
             np.abs(q['f'][:, 0, :] - hidden[:, 12:14]).max(),
             np.abs(q['beta_logit'] - hidden[:, 16:18]).max(),
             np.abs(q['g_a'] - hidden[:, 18:20]).max())
    return max(e1, e2)


def pin_conv_library():
    """Conv against numpy.convolve with the kernel reversed (cross-correlation)."""
    rng = _rng(1)
    T, C, K = 9, 5, 4
    x = rng.standard_normal((T, C))
    w = rng.standard_normal((C, K))
    hist = rng.standard_normal((K - 1, C))
    out, new_hist = ko.causal_depthwise_conv(x, w, hist)
    xp = np.concatenate([hist, x], 0)
    ref = np.stack([np.convolve(xp[:, c], w[c, ::-1], mode='valid') for c in range(C)], 1)
    return max(np.abs(out - ref).max(), np.abs(new_hist - xp[-(K - 1):]).max())


def pin_conv_orientation():
    """Impulse response: tap K-1 multiplies the current token."""
    w = np.array([[1.0, 2.0, 3.0, 4.0]])
    x = np.zeros((6, 1))
    x[0, 0] = 1.0
    out, _ = ko.causal_depthwise_conv(x, w, None)
    return np.abs(out[:, 0] - np.array([4.0, 3.0, 2.0, 1.0, 0.0, 0.0])).max()


def pin_prep_composition():
    """conv (identity tap) -> SiLU -> L2 for q, SiLU only for v, by hand."""
    d, K = 4, 4
    w = np.zeros((1, 3 * d, K))
    w[..., K - 1] = 1.0
    xq = np.array([1.0, -1.0, 0.0, 2.0])
    xv = np.array([1.0, -1.0, 2.0, 0.0])
    x = np.concatenate([xq, xq, xv])[None, None, :]
    p = ko.prep(x, np.zeros((1, 1, d)), np.zeros((1, 1)), w, np.zeros(1), np.zeros((1, d)))
    sq = np.array([SIG1, -(1 - SIG1), 0.0, 2 * SIG2])
    qn = sq / math.sqrt(SIG1 ** 2 + (1 - SIG1) ** 2 + 4 * SIG2 ** 2)
    sv = np.array([SIG1, -(1 - SIG1), 2 * SIG2, 0.0])
    return max(np.abs(p['q'][0, 0] - qn).max(), np.abs(p['k'][0, 0] - qn).max(),
               np.abs(p['v'][0, 0] - sv).max(), abs(p['beta'][0, 0] - 0.5),
               abs(p['loga'][0, 0, 0] + 2.5))


def pin_l2_library():
    rng = _rng(2)
    x = rng.standard_normal((7, 3, 16))
    ref = x / np.linalg.norm(x, axis=-1, keepdims=True)
    small = np.full((1, 4), 1e-9)          # norm 2e-9 < eps: divided by eps
    e_small = np.abs(ko.l2_normalize(small, 1e-6) - small / 1e-6).max()
    zero = np.abs(ko.l2_normalize(np.zeros((1, 4)), 1e-6)).max()
    return max(np.abs(ko.l2_normalize(x, 1e-6) - ref).max(), e_small, zero)


def pin_rmsnorm():
    rng = _rng(3)
    o = rng.standard_normal((5, 2, 16))
    g = rng.standard_normal((5, 2, 16))
    w = 1 + 0.3 * rng.standard_normal(16)
    rms = np.linalg.norm(o, axis=-1, keepdims=True) / math.sqrt(16)
    sg = 1.0 / (1.0 + np.exp(-g))
    ref = o / np.sqrt(rms ** 2 + 1e-5) * w * sg
    e1 = np.abs(ko.gated_rmsnorm(o, g, w, 1e-5) - ref).max()
    # constant o = c, g = 0: y = c / sqrt(c^2 + eps) * w / 2
    c = 0.7
    y = ko.gated_rmsnorm(np.full(8, c), np.zeros(8), np.ones(8), 1e-5)
    e2 = np.abs(y - c / math.sqrt(c * c + 1e-5) * 0.5).max()
    return max(e1, e2)


def _read_golden(name):
    vals = {}
    with open(os.path.join(HERE, 'golden', name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith('#'):
                continue
            key, *nums = line.split()
            vals[key] = np.array([float(t) for t in nums])
    return vals


def pin_hand_example():
    gv = _read_golden('recurrence_d2_hand.txt')
    q = np.stack([gv['q1'], gv['q2']])
    k = np.stack([gv['k1'], gv['k2']])
    v = np.stack([gv['v1'], gv['v2']])
    loga = np.log(np.stack([gv['a1'], gv['a2']]))
    beta = np.array([gv['b1'][0], gv['b2'][0]])
    o, S = ko.recurrence(q, k, v, loga, beta)
    y = ko.gated_rmsnorm(o[1], np.zeros(2), np.ones(2), 1e-5)
    y_ref = gv['o2'] / math.sqrt(gv['ms2'][0] + 1e-5) * 0.5
    return max(np.abs(o[0] - gv['o1']).max(), np.abs(o[1] - gv['o2']).max(),
               np.abs(S.reshape(-1) - gv['S2']).max(), np.abs(y - y_ref).max())


def _brute_force(q, k, v, loga, beta, S0):
    """S_T and o_t from explicit transition matrices M_t = (I - b k k^T) Diag(a_t)."""
    T, dk = k.shape
    I = np.eye(dk)
    Ms = [(I - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(loga[t])) for t in range(T)]
    o = []
    for t in range(T):
        S_t = np.zeros_like(S0)
        for s in range(t + 1):
            P = I.copy()
            for u in range(s + 1, t + 1):
                P = Ms[u] @ P
            S_t = S_t + P @ (beta[s] * np.outer(k[s], v[s]))
        P = I.copy()
        for u in range(t + 1):
            P = Ms[u] @ P
        S_t = S_t + P @ S0
        o.append(S_t.T @ q[t])
    return np.array(o), S_t


def pin_brute_force(dk=8, dv=12, T=6, seed=4):
    rng = _rng(seed)
    q = _unit_rows(rng.standard_normal((T, dk)))
    k = _unit_rows(rng.standard_normal((T, dk)))
    v = rng.standard_normal((T, dv))
    loga = -5.0 * rng.uniform(0, 1, (T, dk))
    beta = rng.uniform(0, 1, T)
    S0 = rng.standard_normal((dk, dv))
    o, S = ko.recurrence(q, k, v, loga, beta, S0)
    o_ref, S_ref = _brute_force(q, k, v, loga, beta, S0)
    return max(np.abs(o - o_ref).max(), np.abs(S - S_ref).max())


def pin_beta_zero():
    """b = 0: S_T = Diag(prod_t a_t) S_0 and o_t = S_t^T q_t."""
    rng = _rng(5)
    T, d = 7, 6
    q = _unit_rows(rng.standard_normal((T, d)))
    k = _unit_rows(rng.standard_normal((T, d)))
    v = rng.standard_normal((T, d))
    loga = -5.0 * rng.uniform(0, 1, (T, d))
    S0 = rng.standard_normal((d, d))
    o, S = ko.recurrence(q, k, v, loga, np.zeros(T), S0)
    S_ref = np.exp(loga.sum(0))[:, None] * S0
    o_ref = np.array([(np.exp(loga[:t + 1].sum(0))[:, None] * S0).T @ q[t] for t in range(T)])
    return max(np.abs(S - S_ref).max(), np.abs(o - o_ref).max())


def pin_retrieval():
    """a = 1, b = 1, orthonormal keys: querying k_j returns v_j; overwrite keeps the last v."""
    rng = _rng(6)
    d = 8
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm.T                      # rows orthonormal
    v = rng.standard_normal((d, 5))
    o, S = ko.recurrence(keys, keys, v, np.zeros((d, d)), np.ones(d))
    e1 = np.abs(S.T @ keys.T - v.T).max()           # S^T k_j = v_j for all j
    e2 = np.abs(o[-1] - v[-1]).max()                 # read after write
    v2 = rng.standard_normal((2, 5))
    kk = np.stack([keys[0], keys[0]])
    o2, S2 = ko.recurrence(kk, kk, v2, np.zeros((2, d)), np.ones(2))
    e3 = np.abs(S2.T @ keys[0] - v2[1]).max()
    return max(e1, e2, e3)


# ---------------------------------------------------------------------------
# tests
# ---------------------------------------------------------------------------
def test_activations_textbook():
    assert pin_activations() < 1e-15


def test_log_decay_closed_forms():
    assert pin_log_decay() < 1e-14
    lo = ko.log_decay(np.full((1, 2), -1e4), np.zeros(1), np.zeros((1, 2)), -5.0)
    assert np.all(np.exp(lo) == 1.0)    # a = 1 exactly


def test_softplus_decay_closed_forms():
    assert pin_softplus_decay() < 1e-12


def test_q_scale_doubles_outputs():
    assert pin_q_scale() < 1e-10


def test_projections_brute_force_and_routing():
    assert pin_projections() < 1e-12


def test_conv_matches_numpy_convolve():
    assert pin_conv_library() < 1e-13


def test_conv_orientation():
    assert pin_conv_orientation() == 0.0


def test_prep_composition_by_hand():
    assert pin_prep_composition() < 1e-15


def test_l2_norm_library_and_eps():
    assert pin_l2_library() < 1e-14


def test_rmsnorm_textbook():
    assert pin_rmsnorm() < 1e-14


def test_hand_example_golden():
    assert pin_hand_example() < 1e-14


@pytest.mark.parametrize('dk,dv', [(8, 12), (8, 8), (3, 5)])
def test_brute_force_transition_products(dk, dv):
    assert pin_brute_force(dk, dv) < 1e-12


def test_beta_zero_pure_decay():
    assert pin_beta_zero() < 1e-13


def test_exact_retrieval_orthonormal_keys():
    assert pin_retrieval() < 1e-12


def _layer_inputs(seed, T, H=2, d=8, K=4):
    rng = _rng(seed)
    return dict(
        x=rng.standard_normal((T, H, 3 * d)), f=rng.standard_normal((T, H, d)),
        beta_logit=rng.standard_normal((T, H)), g=rng.standard_normal((T, H, d)),
        conv_w=0.5 * rng.standard_normal((H, 3 * d, K)), A_log=rng.uniform(0, math.log(16), H),
        dt_bias=math.sqrt(0.1) * rng.standard_normal((H, d)),
        norm_w=1 + math.sqrt(0.1) * rng.standard_normal(d))


def test_beta_zero_no_decay_state_bit_unchanged():
    """beta logit and f at -1e4 give b = 0 and a = 1 exactly: S is bit-unchanged."""
    inp = _layer_inputs(7, 9)
    inp['beta_logit'][:] = -1e4
    inp['f'][:] = -1e4
    inp['dt_bias'][:] = 0.0
    S0 = _rng(8).standard_normal((1, 2, 8, 8))
    out = ko.layer(cu_seqlens=[0, 9], S0=S0, **inp)
    assert np.array_equal(out['state'], S0)


def test_split_invariance_5_plus_7_bit_exact():
    """glm53-flash-mlx README test [5]: chunked prefill 5+7 equals single-shot."""
    inp = _layer_inputs(9, 12)
    S0 = 0.1 * _rng(10).standard_normal((1, 2, 8, 8))
    full = ko.layer(cu_seqlens=[0, 12], S0=S0, **inp)
    a = {k: (v[:5] if k in ('x', 'f', 'beta_logit', 'g') else v) for k, v in inp.items()}
    b = {k: (v[5:] if k in ('x', 'f', 'beta_logit', 'g') else v) for k, v in inp.items()}
    p1 = ko.layer(cu_seqlens=[0, 5], S0=S0, **a)
    p2 = ko.layer(cu_seqlens=[0, 7], S0=p1['state'], conv_hist=p1['conv_hist'], **b)
    assert np.array_equal(np.concatenate([p1['y'], p2['y']]), full['y'])
    assert np.array_equal(p2['state'], full['state'])
    assert np.array_equal(p2['conv_hist'], full['conv_hist'])


def test_varlen_sequences_independent():
    """Packed sequences equal separate runs (state and conv history reset)."""
    inp = _layer_inputs(11, 10)
    S0 = 0.1 * _rng(12).standard_normal((2, 2, 8, 8))
    packed = ko.layer(cu_seqlens=[0, 4, 10], S0=S0, **inp)
    for s, (a, b) in enumerate([(0, 4), (4, 10)]):
        one = {k: (v[a:b] if k in ('x', 'f', 'beta_logit', 'g') else v) for k, v in inp.items()}
        ref = ko.layer(cu_seqlens=[0, b - a], S0=S0[s:s + 1], **one)
        assert np.array_equal(packed['y'][a:b], ref['y'])
        assert np.array_equal(packed['state'][s], ref['state'][0])


def test_norm_bound_every_step():
    """||S_t||_F <= ||S_{t-1}||_F + b ||v||: the transition is non-expansive."""
    rng = _rng(13)
    T, d = 40, 16
    q = _unit_rows(rng.standard_normal((T, d)))
    k = _unit_rows(rng.standard_normal((T, d)))
    v = rng.standard_normal((T, d))
    loga = -5.0 * rng.uniform(0, 1, (T, d)) * (rng.uniform(0, 1, (T, d)) < 0.5)
    beta = rng.uniform(0, 1, T)
    S0 = rng.standard_normal((d, d))
    _, _, states = ko.recurrence(q, k, v, loga, beta, S0, return_states=True)
    prev = S0
    for t in range(T):
        assert np.linalg.norm(states[t]) <= np.linalg.norm(prev) + beta[t] * np.linalg.norm(v[t]) + 1e-12
        prev = states[t]


@pytest.mark.parametrize('chunk', [4, 16, 64])
def test_chunked_form_matches_token_loop(chunk):
    rng = _rng(14)
    T, d = 70, 16
    q = _unit_rows(rng.standard_normal((T, d)))
    k = _unit_rows(rng.standard_normal((T, d)))
    v = rng.standard_normal((T, d))
    loga = -5.0 / (1 + np.exp(-3 * rng.standard_normal((T, d))))
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    S0 = 0.1 * rng.standard_normal((d, d))
    o, S = ko.recurrence(q, k, v, loga, beta, S0)
    oc, Sc = ko.chunked_recurrence(q, k, v, loga, beta, S0, chunk)
    scale = max(np.abs(o).max(), np.abs(S).max())
    assert np.abs(o - oc).max() / scale < 1e-10
    assert np.abs(S - Sc).max() / scale < 1e-10


def test_verify_then_rollback_equals_prefix():
    """Rollback to L accepted drafts equals running only those L tokens."""
    inp = _layer_inputs(15, 8)
    S0 = 0.1 * _rng(16).standard_normal((2, 8, 8))
    hist0 = _rng(17).standard_normal((3, 2, 24))
    p = ko.prep(inp['x'], inp['f'], inp['beta_logit'], inp['conv_w'], inp['A_log'],
                inp['dt_bias'], hist0)
    y, tape = ko.verify(p['q'], p['k'], p['v'], p['loga'], p['beta'], inp['g'],
                        inp['norm_w'], S0)
    for L in range(0, 9):
        S_rb, h_rb = ko.rollback(S0, hist0, tape, p['window'], L)
        if L == 0:
            assert np.array_equal(S_rb, S0) and np.array_equal(h_rb, hist0)
            continue
        pp = ko.prep(inp['x'][:L], inp['f'][:L], inp['beta_logit'][:L], inp['conv_w'],
                     inp['A_log'], inp['dt_bias'], hist0)
        _, S_ref = ko.recurrence(pp['q'], pp['k'], pp['v'], pp['loga'], pp['beta'], S0)
        assert np.array_equal(S_rb, S_ref)
        assert np.array_equal(h_rb, pp['conv_hist'])


# ---------------------------------------------------------------------------
# mutation controls: a planted mistake must fail at least one pin
# ---------------------------------------------------------------------------
def _all_pins():
    pins = {
        'activations': pin_activations, 'log_decay': pin_log_decay,
        'conv_library': pin_conv_library, 'conv_orientation': pin_conv_orientation,
        'prep': pin_prep_composition, 'l2': pin_l2_library, 'rmsnorm': pin_rmsnorm,
        'hand': pin_hand_example, 'brute_square': lambda: pin_brute_force(8, 8),
        'beta_zero': pin_beta_zero, 'retrieval': pin_retrieval,
        'softplus': pin_softplus_decay, 'q_scale': pin_q_scale,
        'projections': pin_projections,
    }
    out = {}
    for name, fn in pins.items():
        try:
            out[name] = float(fn())
        except (ValueError, FloatingPointError):   # a shape mismatch is a detection too
            out[name] = float('inf')
    return out


def _mut_no_silu(x):
    return np.asarray(x, np.float64)


def _mut_reversed_taps(x, w, hist=None):
    return ko.__dict__['_orig_conv'](x, np.asarray(w)[:, ::-1], hist)


def _mut_softplus_decay(f, A_log, dt_bias, lb=-5.0):
    A = np.exp(np.asarray(A_log))[:, None]
    return -A * np.logaddexp(0.0, np.asarray(f) + dt_bias)


def _mut_softplus_bias_sign(f, A_log, dt_bias, lb=-5.0):
    """Mutation of the softplus branch only: the bias subtracted instead of added."""
    if lb is not None:
        return ko.__dict__['_orig_log_decay'](f, A_log, dt_bias, lb)
    A = np.exp(np.asarray(A_log))[:, None]
    return -A * np.logaddexp(0.0, np.asarray(f) - dt_bias)


def _mut_softplus_no_rate(f, A_log, dt_bias, lb=-5.0):
    """Mutation of the softplus branch only: the per-head rate exp(A_log) dropped."""
    if lb is not None:
        return ko.__dict__['_orig_log_decay'](f, A_log, dt_bias, lb)
    return -np.logaddexp(0.0, np.asarray(f) + dt_bias)


def _mut_q_scale_squared(q, k, v, loga, beta, S0=None, q_scale=1.0, return_states=False):
    return ko.__dict__['_orig_recurrence'](q, k, v, loga, beta, S0, q_scale * q_scale,
                                           return_states)


def _mut_layer_drops_q_scale(*args, q_scale=1.0, **kw):
    return ko.__dict__['_orig_layer'](*args, **kw)


def _mut_proj_transposed_gate(hidden, W_in, W_gb, H, d, gate_rank):
    """Mutation: g_b applied with the gate weight's layout transposed (rank-major)."""
    p = ko.__dict__['_orig_projections'](hidden, W_in, W_gb, H, d, gate_rank)
    T = p['g_a'].shape[0]
    W = np.asarray(W_gb, np.float64).reshape(gate_rank, H * d).T
    p['g'] = (p['g_a'] @ W.T).reshape(T, H, d)
    return p


def _mut_proj_beta_gate_swapped(hidden, W_in, W_gb, H, d, gate_rank):
    """Mutation: the beta logit taken from the end of the fused rows (after g_a)."""
    p = ko.__dict__['_orig_projections'](hidden, W_in, W_gb, H, d, gate_rank)
    Y = np.asarray(hidden, np.float64) @ np.asarray(W_in, np.float64).T
    nx, nf = 3 * H * d, H * d
    p['beta_logit'] = Y[:, nx + nf + gate_rank:nx + nf + gate_rank + H]
    return p


def _mut_value_axis(S, a):
    return S * a[..., None, :]


def _mut_no_gate(o, g, w, eps=1e-5):
    o = np.asarray(o, np.float64)
    return o / np.sqrt(np.mean(o * o, -1, keepdims=True) + eps) * w


def _mut_sqrt_sum_eps(x, eps=1e-6):
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.sum(x * x, -1, keepdims=True) + eps)


def _mut_decay_after_update(q, k, v, loga, beta, S0=None, q_scale=1.0, return_states=False):
    """Mutation: write first, decay afterwards (wrong recurrence ordering)."""
    T = q.shape[0]
    S = np.zeros(k.shape[1:-1] + (k.shape[-1], v.shape[-1])) if S0 is None else np.array(S0, float)
    o = np.zeros((T,) + v.shape[1:])
    states = []
    for t in range(T):
        r = np.einsum('...kv,...k->...v', S, k[t])
        u = beta[t][..., None] * (v[t] - r)
        S = S + k[t][..., :, None] * u[..., None, :]
        S = np.exp(loga[t])[..., :, None] * S
        o[t] = q_scale * np.einsum('...kv,...k->...v', S, q[t])
        states.append(S)
    if return_states:
        return o, S, np.array(states)
    return o, S


MUTATIONS = {
    'no_silu': ('silu', _mut_no_silu),
    'reversed_taps': ('causal_depthwise_conv', _mut_reversed_taps),
    'softplus_decay': ('log_decay', _mut_softplus_decay),
    'value_axis_decay': ('apply_key_decay', _mut_value_axis),
    'missing_output_gate': ('gated_rmsnorm', _mut_no_gate),
    'decay_after_update': ('recurrence', _mut_decay_after_update),
    'softplus_bias_sign': ('log_decay', _mut_softplus_bias_sign),
    'softplus_no_rate': ('log_decay', _mut_softplus_no_rate),
    'q_scale_squared': ('recurrence', _mut_q_scale_squared),
    'layer_drops_q_scale': ('layer', _mut_layer_drops_q_scale),
    'proj_transposed_gate': ('projections', _mut_proj_transposed_gate),
    'proj_beta_gate_swapped': ('projections', _mut_proj_beta_gate_swapped),
}


@pytest.mark.parametrize('name', sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setitem(ko.__dict__, '_orig_conv', ko.causal_depthwise_conv)
    monkeypatch.setitem(ko.__dict__, '_orig_log_decay', ko.log_decay)
    monkeypatch.setitem(ko.__dict__, '_orig_recurrence', ko.recurrence)
    monkeypatch.setitem(ko.__dict__, '_orig_layer', ko.layer)
    monkeypatch.setitem(ko.__dict__, '_orig_projections', ko.projections)
    monkeypatch.setattr(ko, attr, fn)
    pins = _all_pins()
    failing = [k for k, e in pins.items() if not (e < 1e-10)]
    assert failing, f'mutation {name} passed every pin'


def test_sqrt_sum_eps_l2_is_documented_insensitive(monkeypatch):
    """PR #27754: max(sqrt(sum), eps) vs sqrt(sum + eps) differ by ~eps/(2 sum).

    The form is not distinguishable at the parity tolerance on ordinary inputs;
    only the small-norm pin (norm below eps) separates them.
    """
    monkeypatch.setattr(ko, 'l2_normalize', _mut_sqrt_sum_eps)
    rng = _rng(18)
    x = rng.standard_normal((5, 128))
    ref = x / np.linalg.norm(x, axis=-1, keepdims=True)
    assert np.abs(ko.l2_normalize(x) - ref).max() < 1e-6
    assert pin_l2_library() > 1e-4
