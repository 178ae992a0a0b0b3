"""Parity at the benchmark workloads' full sizes, in the launch configuration the
bench uses, on sampled (sequence, head) units the oracle can compute one by one.

Every (sequence, head) unit of the layer is independent, so the oracle run on a
subset of units is exact evidence for those units.  Bar: max|GPU - oracle| /
max|oracle| <= 1e-2 (bf16 inputs, fp32 state); rollback bit-exact.
"""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_09_b200 import kda, synth
from tests.kda_cases import np64, oracle_layer, rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-2
H, D, K = 32, 128, 4


def _cfg():
    return kda.Config(num_heads=H, head_dim=D, conv_size=K, dtype=torch.bfloat16, chunk_size=64)


def _dev(d):
    return {k: v.cuda() for k, v in d.items()}


def _sub(acts, a, b):
    out = {k: acts[k][a:b] for k in ('x', 'f', 'beta_logit', 'g')}
    out['cu_seqlens'] = torch.tensor([0, b - a], dtype=torch.int32)
    return out


def test_prefill_8k_full_size():
    """B=1, H=32, T=8192, d=128, chunk 64 (the headline prefill), heads 0, 17, 31."""
    cfg = _cfg()
    P = synth.layer_params(1, H, D, K)
    A = synth.layer_activations(1, [8192], H, D, torch.bfloat16)
    state = torch.empty(1, H, D, D, device='cuda')
    y = kda.layer_prefill(cfg, _dev(P), _dev(A), state_out=state)
    torch.cuda.synchronize()
    heads = [0, 17, 31]
    ref = oracle_layer(cfg, P, A, heads=heads)
    assert rel_err(np64(y)[:, heads], ref['y']) <= TOL
    assert rel_err(np64(state)[:, heads], ref['state']) <= TOL


def test_decode_b64_full_size():
    """B=64, H=32: 512-token prefill then 1,024 decode steps; units (b, h) sampled."""
    cfg = _cfg()
    B, T0, steps = 64, 512, 1024
    P = synth.layer_params(2, H, D, K)
    Pd = _dev(P)
    A = synth.layer_activations(2, [T0] * B, H, D, torch.bfloat16)
    state = torch.zeros(B, H, D, D, device='cuda')
    conv = torch.zeros(B, K - 1, H, 3 * D, dtype=cfg.dtype, device='cuda')
    kda.layer_prefill(cfg, Pd, _dev(A), state_in=state, state_out=state, conv_state=conv)
    S = synth.layer_activations(2, [steps] * B, H, D, torch.bfloat16, tag='decode_steps')
    X = {k: S[k].view(B, steps, *S[k].shape[1:]).transpose(0, 1).contiguous().cuda()
         for k in ('x', 'f', 'beta_logit', 'g')}
    cu = torch.arange(B + 1, dtype=torch.int32, device='cuda')
    ys = torch.empty(steps, B, H, D, dtype=cfg.dtype, device='cuda')
    for i in range(steps):
        p = kda.kda_prep(cfg, cu, X['x'][i], X['f'][i], X['beta_logit'][i], Pd['conv_w'],
                         Pd['A_log'], Pd['dt_bias'], conv_state=conv, max_seqlen=1)
        kda.kda_decode(cfg, p['q'], p['k'], p['v'], p['log_a'], p['beta'], X['g'][i],
                       Pd['norm_w'], state, y=ys[i])
    torch.cuda.synchronize()
    ys = ys.cpu()
    for b, h in [(0, 0), (37, 21), (63, 31)]:
        seq = {k: torch.cat([A[k][b * T0:(b + 1) * T0], S[k][b * steps:(b + 1) * steps]])
               for k in ('x', 'f', 'beta_logit', 'g')}
        seq['cu_seqlens'] = torch.tensor([0, T0 + steps], dtype=torch.int32)
        ref = oracle_layer(cfg, P, seq, heads=[h])
        assert rel_err(np64(ys[:, b, h]), ref['y'][T0:, 0]) <= TOL, (b, h)
        assert rel_err(np64(state[b, h]), ref['state'][0, 0]) <= TOL, (b, h)


def test_verify_b16_full_size():
    """B=16, H=32, 4,096-token context, blocks of 8 with rollback; 32 rounds checked."""
    cfg = _cfg()
    B, T0, Tb, rounds = 16, 4096, 8, 32
    P = synth.layer_params(3, H, D, K)
    Pd = _dev(P)
    A = synth.layer_activations(3, [T0] * B, H, D, torch.bfloat16)
    state = torch.zeros(B, H, D, D, device='cuda')
    conv = torch.zeros(B, K - 1, H, 3 * D, dtype=cfg.dtype, device='cuda')
    kda.layer_prefill(cfg, Pd, _dev(A), state_in=state, state_out=state, conv_state=conv)
    Dr = synth.layer_activations(3, [256 * Tb] * B, H, D, torch.bfloat16, tag='drafts')
    acc = synth.accepted_lengths(3, 256, B, Tb)[:rounds]
    cu = torch.arange(B + 1, dtype=torch.int32, device='cuda') * Tb
    v4 = lambda t, *tail: t.view(B, Tb, *tail)
    for r in range(rounds):
        blk = {k: torch.stack([Dr[k][b * 256 * Tb + r * Tb: b * 256 * Tb + (r + 1) * Tb]
                               for b in range(B)]).reshape(B * Tb, *Dr[k].shape[1:]).cuda()
               for k in ('x', 'f', 'beta_logit', 'g')}
        p = kda.kda_prep(cfg, cu, blk['x'], blk['f'], blk['beta_logit'], Pd['conv_w'],
                         Pd['A_log'], Pd['dt_bias'], conv_state=conv,
                         conv_mode=kda.KDA_CONV_TAPE, max_seqlen=Tb)
        y, tape = kda.kda_verify(cfg, v4(p['q'], H, D), v4(p['k'], H, D), v4(p['v'], H, D),
                                 v4(p['log_a'], H, D), v4(p['beta'], H),
                                 v4(blk['g'], H, D), Pd['norm_w'], state)
        kda.kda_rollback(cfg, acc[r].cuda(), tape, state, conv_window=p['window'],
                         conv_state=conv)
        torch.cuda.synchronize()
        for b in (0, 9):
            L = int(acc[r, b])
            if L > 0:
                assert torch.equal(state[b], tape[b, L - 1])
    y_last = y.cpu()
    for b, h in [(0, 5), (9, 30)]:
        parts = [A[k][b * T0:(b + 1) * T0] for k in ('x',)]
        seq = {}
        for key in ('x', 'f', 'beta_logit', 'g'):
            chunks = [A[key][b * T0:(b + 1) * T0]]
            for r in range(rounds):
                base = b * 256 * Tb + r * Tb
                n = Tb if r == rounds - 1 else int(acc[r, b])
                chunks.append(Dr[key][base:base + n])
            seq[key] = torch.cat(chunks)
        total = seq['x'].shape[0]
        seq['cu_seqlens'] = torch.tensor([0, total], dtype=torch.int32)
        ref = oracle_layer(cfg, P, seq, heads=[h])
        assert rel_err(np64(y_last[b, :, h]), ref['y'][total - Tb:, 0]) <= TOL, (b, h)
        del parts


def test_varlen_and_131k_full_size():
    """8 packed sequences (log-uniform 1K-32K) and one 131,072-token sequence,
    nonzero initial state N(0, 0.01); sampled heads per sequence."""
    cfg = _cfg()
    P = synth.layer_params(4, H, D, K)
    Pd = _dev(P)
    lens = synth.varlen_lengths(4)
    A = synth.layer_activations(4, lens, H, D, torch.bfloat16)
    S0 = synth.initial_state(4, len(lens), H, D, 0.01)
    state = S0.cuda()
    y = kda.layer_prefill(cfg, Pd, _dev(A), state_in=state, state_out=state)
    torch.cuda.synchronize()
    y = y.cpu()
    cu = A['cu_seqlens'].tolist()
    longest = int(np.argmax(lens))
    for s, h in [(0, 3), (longest, 12)]:
        a, b = cu[s], cu[s + 1]
        ref = oracle_layer(cfg, P, _sub(A, a, b), S0=S0[s:s + 1], heads=[h])
        assert rel_err(np64(y[a:b, h]), ref['y'][:, 0]) <= TOL, s
        assert rel_err(np64(state[s, h]), ref['state'][0, 0]) <= TOL, s
    del A, y
    # one long sequence
    T = 131072
    L1 = synth.layer_activations(4, [T], H, D, torch.bfloat16, tag='long')
    S1 = synth.initial_state(5, 1, H, D, 0.01)
    st1 = S1.cuda()
    y1 = kda.layer_prefill(cfg, Pd, _dev(L1), state_in=st1, state_out=st1)
    torch.cuda.synchronize()
    h = 7
    ref = oracle_layer(cfg, P, L1, S0=S1, heads=[h])
    assert rel_err(np64(y1[:, h]), ref['y'][:, 0]) <= TOL
    assert rel_err(np64(st1[0, h]), ref['state'][0, 0]) <= TOL
