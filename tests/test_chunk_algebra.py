"""CPU check, in float64, of a regrouped chunk algebra for the inter-chunk pass.

Carrying the state through a chunk as S' = gamma * S + K'^T U~ - (K'^T W) S and forming
O = (Q~ - M W) S + M U~ puts one product per chunk on the serial chain instead of two;
it is a regrouping of U = U~ - W S, S' = gamma * S + K'^T U, O = Q~ S + M U.  Written
here from those equations, with the chunk tiles built from their definitions, and
compared with the oracle's token loop on every chunk of a few sequences.
"""
import math

import numpy as np
import pytest

from oracle import kda_oracle as ko


def _tiles(q, k, v, loga, beta):
    """The chunk's tiles from their definitions (W, U~, Q~, K', M, gamma)."""
    L, dk = k.shape
    G = np.cumsum(loga, axis=0)
    A = np.zeros((L, L))
    M = np.zeros((L, L))
    for r in range(L):
        for i in range(r + 1):
            w = np.exp(G[r] - G[i])
            if i < r:
                A[r, i] = beta[r] * np.sum(k[r] * k[i] * w)
            M[r, i] = np.sum(q[r] * k[i] * w)
    Tm = np.linalg.solve(np.eye(L) + A, np.diag(beta))
    W = Tm @ (k * np.exp(G))
    Ut = Tm @ v
    Qt = q * np.exp(G)
    Kp = k * np.exp(G[-1][None, :] - G)
    return W, Ut, Qt, Kp, M, np.exp(G[-1])


@pytest.mark.parametrize('T,chunk,dk,dv', [(40, 16, 8, 12), (70, 32, 16, 16), (64, 64, 6, 5)])
def test_regrouped_chain_matches_token_loop(T, chunk, dk, dv):
    rng = np.random.default_rng(T + chunk)
    q = rng.standard_normal((T, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    loga = -5.0 / (1.0 + np.exp(-rng.standard_normal((T, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    S0 = 0.1 * rng.standard_normal((dk, dv))
    o_ref, S_ref = ko.recurrence(q, k, v, loga, beta, S0)
    S = S0.copy()
    o = np.zeros((T, dv))
    for s in range(0, T, chunk):
        e = min(s + chunk, T)
        W, Ut, Qt, Kp, M, gamma = _tiles(q[s:e], k[s:e], v[s:e], loga[s:e], beta[s:e])
        P, B = Kp.T @ W, Kp.T @ Ut            # formed off the chain
        Qp, R = Qt - M @ W, M @ Ut
        o[s:e] = Qp @ S + R                   # output product on top of R
        S = gamma[:, None] * S + (B - P @ S)  # the one product on the chain, on top of B
    scale = np.abs(o_ref).max()
    assert np.abs(o - o_ref).max() <= 1e-10 * max(1.0, scale)
    assert np.abs(S - S_ref).max() <= 1e-10 * max(1.0, np.abs(S_ref).max())
    assert math.isfinite(scale)
