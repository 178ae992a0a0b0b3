"""Seeded synthetic inputs for the KDA layer.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic, so both the CUDA path (through the binding) and the CPU
oracle can be fed from it.  Every tensor is drawn on the CPU from its own
``torch.Generator`` keyed by (seed, tensor name, sequence, token block), so any
sequence can be regenerated on its own and the values never depend on the
device.

Distributions (the tiny fp32 workload's recipe, used for every workload):
pre-conv q|k|v ~ N(0, 1); f, g ~ N(0, 1); beta logit ~ N(0, 1) (beta is its
sigmoid); conv w ~ N(0, 1/4); A_log ~ U(0, ln 16); dt_bias ~ N(0, 0.1);
norm w = 1 + N(0, 0.1); initial state N(0, s) when requested.  N(0, s) means
variance s.  Activations are drawn in fp32 and rounded once to the activation
dtype; parameters and states stay fp32.
"""
from __future__ import annotations

import hashlib
import math

import numpy as np
import torch

_TOKEN_BLOCK = 4096


def _key(*parts) -> int:
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], 'little') & ((1 << 63) - 1)


def _gen(*parts) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(_key(*parts))
    return g


def _normal(shape, std, *key):
    return torch.randn(*shape, generator=_gen(*key), dtype=torch.float32) * std


def _normal_tokens(name, seed, seq, L, tail, dtype):
    """N(0,1) tensor [L, *tail] for one sequence, drawn per 4096-token block."""
    out = torch.empty((L,) + tuple(tail), dtype=dtype)
    for b0 in range(0, L, _TOKEN_BLOCK):
        b1 = min(L, b0 + _TOKEN_BLOCK)
        out[b0:b1] = _normal((b1 - b0,) + tuple(tail), 1.0, seed, name, seq, b0).to(dtype)
    return out


def layer_params(seed, H, d, K=4):
    """fp32 parameters: conv w [H,3d,K], A_log [H], dt_bias [H,d], norm w [d]."""
    conv_w = _normal((H, 3 * d, K), 0.5, seed, 'conv_w')
    A_log = torch.rand(H, generator=_gen(seed, 'A_log'), dtype=torch.float32) * math.log(16.0)
    dt_bias = _normal((H, d), math.sqrt(0.1), seed, 'dt_bias')
    norm_w = 1.0 + _normal((d,), math.sqrt(0.1), seed, 'norm_w')
    return dict(conv_w=conv_w, A_log=A_log, dt_bias=dt_bias, norm_w=norm_w)


def layer_activations(seed, seqlens, H, d, dtype=torch.bfloat16, tag='act'):
    """Packed activations for sequences of the given lengths.

    Returns x [Ttot,H,3d], f [Ttot,H,d], beta_logit [Ttot,H], g [Ttot,H,d] in
    ``dtype`` and cu_seqlens int32 [N+1].
    """
    seqlens = [int(n) for n in seqlens]
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    parts = {k: [] for k in ('x', 'f', 'beta_logit', 'g')}
    for s, L in enumerate(seqlens):
        parts['x'].append(_normal_tokens('x', (seed, tag), s, L, (H, 3 * d), dtype))
        parts['f'].append(_normal_tokens('f', (seed, tag), s, L, (H, d), dtype))
        parts['beta_logit'].append(_normal_tokens('beta', (seed, tag), s, L, (H,), dtype))
        parts['g'].append(_normal_tokens('g', (seed, tag), s, L, (H, d), dtype))
    out = {k: (torch.cat(v, 0) if v else torch.empty(0)) for k, v in parts.items()}
    out['cu_seqlens'] = torch.from_numpy(cu)
    return out


def proj_weights(seed, hidden, H, d, gate_rank, dtype=torch.bfloat16):
    """Random-init projection weights of one layer: the fused input weight W_in
    [3Hd + Hd + H + gate_rank, hidden] ~ N(0, 1/hidden) (so that x, f, the beta logit and
    g_a come out ~ N(0, 1) for N(0, 1) hidden states, the activations' recipe) and the
    gate's second factor W_gb [H d, gate_rank] ~ N(0, 1/gate_rank)."""
    n = 4 * H * d + H + gate_rank
    W_in = _normal((n, hidden), 1.0 / math.sqrt(hidden), seed, 'W_in').to(dtype)
    W_gb = _normal((H * d, gate_rank), 1.0 / math.sqrt(gate_rank), seed, 'W_gb').to(dtype)
    return dict(W_in=W_in, W_gb=W_gb)


def hidden_states(seed, T, hidden, dtype=torch.bfloat16, tag='hidden'):
    """Hidden states [T, hidden] ~ N(0, 1), drawn per 4096-token block."""
    return _normal_tokens('hidden', (seed, tag), 0, T, (hidden,), dtype)


def initial_state(seed, n, H, d, variance):
    """fp32 recurrent states [n,H,d,d] ~ N(0, variance); zeros if variance is 0."""
    if variance == 0:
        return torch.zeros(n, H, d, d)
    return _normal((n, H, d, d), math.sqrt(variance), seed, 'state0')


def conv_history(seed, n, H, d, K, dtype, std=1.0):
    """Pre-conv history rows [n,K-1,H,3d] ~ N(0, std^2), in ``dtype``."""
    return _normal((n, K - 1, H, 3 * d), std, seed, 'conv_hist').to(dtype)


def varlen_lengths(seed, n=8, lo=1024, hi=32768):
    """n lengths floor(exp(U(ln lo, ln hi))) (log-uniform), seeded."""
    u = torch.rand(n, generator=_gen(seed, 'lengths'), dtype=torch.float64)
    return [int(math.floor(math.exp(math.log(lo) + float(t) * (math.log(hi) - math.log(lo)))))
            for t in u]


def accepted_lengths(seed, rounds, batch, block):
    """Accepted prefix lengths ~ U{0..block}, int32 [rounds, batch]."""
    return torch.randint(0, block + 1, (rounds, batch), generator=_gen(seed, 'accept'),
                         dtype=torch.int32)


# Workloads: sizes and recipes, named by what they are.
WORKLOADS = {
    'tiny_fp32': dict(seed=0, batch=1, heads=2, seqlen=64, head_dim=16, chunk=16, conv=4,
                      dtype='f32', state_variance=0.0),
    'prefill_8k': dict(seed=1, batch=1, heads=32, seqlen=8192, head_dim=128, chunk=64, conv=4,
                       dtype='bf16', state_variance=0.0),
    'decode_b64': dict(seed=2, batch=64, heads=32, prefill=512, steps=1024, head_dim=128,
                       chunk=64, conv=4, dtype='bf16', state_variance=0.0),
    'verify_b16': dict(seed=3, batch=16, heads=32, context=4096, block=8, rounds=256,
                       head_dim=128, chunk=64, conv=4, dtype='bf16', state_variance=0.0),
    'varlen_long': dict(seed=4, n_seqs=8, lo=1024, hi=32768, long_seqlen=131072, heads=32,
                        head_dim=128, chunk=64, conv=4, dtype='bf16', state_variance=0.01),
    'layer_8k_projections': dict(seed=6, batch=1, heads=32, seqlen=8192, head_dim=128,
                                 hidden=4096, gate_rank=128, chunk=64, conv=4, dtype='bf16'),
}
