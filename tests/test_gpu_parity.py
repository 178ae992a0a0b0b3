"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Bar: max|GPU - oracle| / max|oracle| <= 1e-4 for fp32 inputs and <= 1e-2 for
bf16 inputs with an fp32 state; rollback and the verify tape are bit-exact.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

from linear_attention_recurrence_09_b200 import kda, synth
from oracle import kda_oracle as ko
from tests.kda_cases import (TOL, compare_layer, gpu_layer, make_case, np64, oracle_layer,
                             rel_err)

pytestmark = pytest.mark.gpu


def _assert(errs, tol):
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f'errors above {tol}: {errs}'


def test_tiny_fp32_layer():
    """Tiny fp32 workload: B=1, H=2, T=64, d=16, chunk 16, conv 4, zero state."""
    w = synth.WORKLOADS['tiny_fp32']
    cfg, P, A, S0, hist = make_case(w['seed'], [w['seqlen']], w['heads'], w['head_dim'],
                                    w['conv'], torch.float32, chunk=w['chunk'])
    _assert(compare_layer(cfg, P, A, S0, hist), 1e-4)


@pytest.mark.parametrize('dtype', [torch.float32, torch.bfloat16])
@pytest.mark.parametrize('d,K', [(16, 4), (64, 2), (128, 4), (32, 8)])
def test_prep_matches_oracle(dtype, d, K):
    seqlens = [0, 1, 5, 17, 40]
    cfg, P, A, _, hist = make_case(3, seqlens, 3, d, K, dtype, conv_hist=True)
    _, _, cs, p = gpu_layer(cfg, P, A, None, hist, fused=False)
    ref = oracle_layer(cfg, P, A, None, hist)
    tol = 1e-5
    for name, rname in [('q', 'q'), ('k', 'k'), ('v', 'v'), ('log_a', 'loga'), ('beta', 'beta')]:
        assert rel_err(np64(p[name]), ref[rname]) <= tol, name
    assert np.array_equal(np64(cs), ref['conv_hist'])


@pytest.mark.parametrize('dtype', [torch.float32, torch.bfloat16])
def test_prep_tape_window(dtype):
    cfg, P, A, _, hist = make_case(4, [8, 8, 8], 2, 32, 4, dtype, conv_hist=True)
    dev = 'cuda'
    cs = hist.to(dev)
    before = cs.clone()
    p = kda.kda_prep(cfg, A['cu_seqlens'].to(dev), A['x'].to(dev), A['f'].to(dev),
                     A['beta_logit'].to(dev), P['conv_w'].to(dev), P['A_log'].to(dev),
                     P['dt_bias'].to(dev), conv_state=cs, conv_mode=kda.KDA_CONV_TAPE,
                     max_seqlen=8)
    torch.cuda.synchronize()
    assert torch.equal(cs, before)          # TAPE mode never writes the conv state
    win = p['window'].cpu().view(3, 3 + 8, 2, 96)
    x = A['x'].view(3, 8, 2, 96)
    for s in range(3):
        assert torch.equal(win[s, :3], hist[s])
        assert torch.equal(win[s, 3:], x[s])


@pytest.mark.parametrize('fused', [True, False])
@pytest.mark.parametrize('d,chunk', [(32, 16), (64, 32), (128, 64), (128, 16)])
def test_prefill_varlen_ragged_bf16(d, chunk, fused):
    """kda_layer_prefill (fused prep at d=128, chunk 64) and kda_prep + kda_prefill."""
    seqlens = [0, 1, chunk - 1, chunk, chunk + 1, 3 * chunk + 7]
    cfg, P, A, S0, hist = make_case(5, seqlens, 4, d, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True, chunk=chunk)
    _assert(compare_layer(cfg, P, A, S0, hist, fused=fused), 1e-2)


@pytest.mark.parametrize('fused', [True, False])
@pytest.mark.parametrize('seqlens', [[1000], [0, 700, 1, 64, 1500, 0, 65], [8192],
                                     [3000, 17, 1500, 64, 2100]])
def test_cosched_launch_equals_separate_passes(seqlens, fused):
    """The tensor-core prefill as one co-scheduled launch (a full-width inter-chunk chain per
    head, walking the batch's sequences in order beside the intra-chunk pass, handing over
    through per-tile ready words) equals the two separate launches bit for bit: the chain
    takes each state element and each token's norm through the same operations in the same
    order.  Both meet the oracle bar on two of the heads (checked on the smaller cases; the
    8,192-token one is the headline shape)."""
    H = 32
    cfg, P, A, S0, hist = make_case(23, seqlens, H, 128, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True, chunk=64)
    sep = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_SEPARATE_PASSES)
    n0 = kda.kda_launch_count()
    y1, s1, c1, _ = gpu_layer(cfg, P, A, S0, hist, fused=fused)
    n1 = kda.kda_launch_count()
    y2, s2, c2, _ = gpu_layer(sep, P, A, S0, hist, fused=fused)
    n2 = kda.kda_launch_count()
    assert n2 - n1 == (n1 - n0) + 1          # the co-scheduled form is one launch fewer
    assert torch.equal(y1, y2)
    assert torch.equal(s1, s2)
    assert torch.equal(c1, c2)
    if sum(seqlens) <= 2400:
        _assert(compare_layer(cfg, P, A, S0, hist, heads=[0, 21], fused=fused), 1e-2)


@pytest.mark.parametrize('K', [2, 4])
def test_layer_prefill_conv_sizes(K):
    """Fused (K = 4) and fallback (K = 2) layer prefill, conv history carried."""
    cfg, P, A, S0, hist = make_case(16, [3, 130], 2, 128, K, torch.bfloat16, state_var=0.01,
                                    conv_hist=True, chunk=64)
    _assert(compare_layer(cfg, P, A, S0, hist), 1e-2)


@pytest.mark.parametrize('d,chunk', [(16, 16), (64, 32), (128, 64)])
def test_prefill_fp32(d, chunk):
    cfg, P, A, S0, hist = make_case(6, [37, 2 * chunk + 3], 2, d, 4, torch.float32,
                                    state_var=0.01, conv_hist=True, chunk=chunk)
    _assert(compare_layer(cfg, P, A, S0, hist), 1e-4)


def test_prefill_no_tokens_copies_state():
    cfg, P, A, S0, _ = make_case(7, [0, 0], 2, 64, 4, torch.bfloat16, state_var=0.01)
    y, s_out, _, _ = gpu_layer(cfg, P, A, S0, None)
    assert torch.equal(s_out.cpu(), S0)


def test_beta_zero_no_decay_keeps_state_bit_exact():
    """b = 0 and a = 1 (logits at -1e4): prefill and decode leave S bit-unchanged."""
    cfg, P, A, S0, _ = make_case(8, [70], 2, 64, 4, torch.bfloat16, state_var=0.01)
    A['beta_logit'][:] = -1e4
    A['f'][:] = -1e4
    _, s_out, _, p = gpu_layer(cfg, P, A, S0, None, fused=False)
    assert torch.equal(s_out.cpu(), S0)
    _, s_f, _, _ = gpu_layer(cfg, P, A, S0, None, fused=True)
    assert torch.equal(s_f.cpu(), S0)
    st = S0.cuda().clone()
    one = lambda t: t[:1].clone()
    kda.kda_decode(cfg, one(p['q']), one(p['k']), one(p['v']), one(p['log_a']), one(p['beta']),
                   one(A['g'].cuda()), P['norm_w'].cuda(), st, pool_size=1)
    torch.cuda.synchronize()
    assert torch.equal(st.cpu()[:1], S0[:1])


@pytest.mark.parametrize('dtype,d,chunk', [(torch.bfloat16, 128, 64), (torch.float32, 64, 32)])
def test_split_invariance_5_plus_7(dtype, d, chunk):
    """glm53-flash-mlx README test [5]: prefill 5 then 7 equals prefill 12.

    Both spellings are held to the oracle bar and leave a bit-identical conv
    history.  In fp32 they must also agree with each other to 1e-5 (the two differ
    only in where fp32 rounding falls).  In bf16 each spelling rounds its chunk
    tiles to bf16 at different places, so their mutual difference is bounded only
    by the two oracle bars together; no tighter self-comparison is asserted."""
    cfg, P, A, S0, hist = make_case(9, [12], 2, d, 4, dtype, state_var=0.01,
                                    conv_hist=True, chunk=chunk)
    y_full, s_full, c_full, _ = gpu_layer(cfg, P, A, S0, hist)
    a1 = {k: v[:5] for k, v in A.items() if k != 'cu_seqlens'}
    a1['cu_seqlens'] = torch.tensor([0, 5], dtype=torch.int32)
    a2 = {k: v[5:] for k, v in A.items() if k != 'cu_seqlens'}
    a2['cu_seqlens'] = torch.tensor([0, 7], dtype=torch.int32)
    y1, s1, c1, _ = gpu_layer(cfg, P, a1, S0, hist)
    y2, s2, c2, _ = gpu_layer(cfg, P, a2, s1.cpu(), c1.cpu())
    y_split = torch.cat([y1, y2]).cpu()
    ref = oracle_layer(cfg, P, A, S0, hist)
    tol = TOL[dtype]
    for y, s in ((y_full, s_full), (y_split, s2)):
        assert rel_err(np64(y), ref['y']) <= tol
        assert rel_err(np64(s), ref['state']) <= tol
    if dtype == torch.float32:
        assert rel_err(np64(y_split), np64(y_full)) <= 1e-5
        assert rel_err(np64(s2), np64(s_full)) <= 1e-5
    assert torch.equal(c2.cpu(), c_full.cpu())


def _decode_run(cfg, P, steps_acts, state, conv_state, dev='cuda', fused=False):
    """T decode steps: prep (T=1, COMMIT) + decode, or kda_layer_decode (fused).
    Returns y [T, B, H, d]."""
    ys = []
    for a in steps_acts:
        if fused:
            ys.append(kda.kda_layer_decode(cfg, a['x'].to(dev), a['f'].to(dev),
                                           a['beta_logit'].to(dev), a['g'].to(dev),
                                           P['conv_w'].to(dev), P['A_log'].to(dev),
                                           P['dt_bias'].to(dev), P['norm_w'].to(dev), state,
                                           conv_state=conv_state))
            continue
        p = kda.kda_prep(cfg, a['cu_seqlens'].to(dev), a['x'].to(dev), a['f'].to(dev),
                         a['beta_logit'].to(dev), P['conv_w'].to(dev), P['A_log'].to(dev),
                         P['dt_bias'].to(dev), conv_state=conv_state, max_seqlen=1)
        ys.append(kda.kda_decode(cfg, p['q'], p['k'], p['v'], p['log_a'], p['beta'],
                                 a['g'].to(dev), P['norm_w'].to(dev), state))
    torch.cuda.synchronize()
    return torch.stack(ys)


def _step_acts(seed, B, H, d, dtype, n):
    return [synth.layer_activations(seed, [1] * B, H, d, dtype, tag=('step', i)) for i in range(n)]


def _cat_seq(parts, b):
    """Token rows of sequence b across a list of activation dicts (one token per seq each)."""
    out = {}
    for key in ('x', 'f', 'beta_logit', 'g'):
        out[key] = torch.cat([p[key][p['cu_seqlens'][b]:p['cu_seqlens'][b + 1]] for p in parts])
    out['cu_seqlens'] = torch.tensor([0, out['x'].shape[0]], dtype=torch.int32)
    return out


def test_decode_matches_oracle():
    B, H, d, T0, steps = 3, 4, 128, 40, 6
    cfg, P, A, S0, hist = make_case(10, [T0] * B, H, d, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True)
    _, s_out, cs, _ = gpu_layer(cfg, P, A, S0, hist)
    sa = _step_acts(10, B, H, d, torch.bfloat16, steps)
    ys = _decode_run(cfg, P, sa, s_out, cs).cpu()
    for b in range(B):
        seq = _cat_seq([A] + sa, b)
        ref = oracle_layer(cfg, P, seq, S0[b:b + 1], hist[b:b + 1])
        assert rel_err(np64(ys[:, b]), ref['y'][T0:]) <= 1e-2
        assert rel_err(np64(s_out[b]), ref['state'][0]) <= 1e-2
        assert np.array_equal(np64(cs[b]), ref['conv_hist'][0])


def test_decode_equals_prefill_on_gpu():
    """glm53-flash-mlx README test [5]: token-by-token decode equals one forward."""
    B, H, d, T = 2, 2, 128, 20
    cfg, P, A, S0, hist = make_case(11, [1] * B, H, d, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True)
    sa = _step_acts(11, B, H, d, torch.bfloat16, T)
    st = S0.cuda().clone()
    cs = hist.cuda().clone()
    ys = _decode_run(cfg, P, sa, st, cs).cpu()
    for b in range(B):
        seq = _cat_seq(sa, b)
        y, s_out, c_out, _ = gpu_layer(cfg, P, seq, S0[b:b + 1], hist[b:b + 1])
        assert rel_err(np64(ys[:, b]), np64(y)) <= 1e-2
        assert rel_err(np64(st[b]), np64(s_out[0])) <= 1e-2
        assert torch.equal(cs[b].cpu(), c_out[0].cpu())


def test_verify_tape_equals_repeated_decode_bit_exact():
    B, H, d, Tb = 3, 2, 128, 8
    cfg, P, A, S0, hist = make_case(12, [Tb] * B, H, d, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True)
    dev = 'cuda'
    Pd = {k: v.to(dev) for k, v in P.items()}
    cs = hist.to(dev)
    p = kda.kda_prep(cfg, A['cu_seqlens'].to(dev), A['x'].to(dev), A['f'].to(dev),
                     A['beta_logit'].to(dev), Pd['conv_w'], Pd['A_log'], Pd['dt_bias'],
                     conv_state=cs, conv_mode=kda.KDA_CONV_TAPE, max_seqlen=Tb)
    shp = lambda t, *tail: t.view(B, Tb, *tail)
    st = S0.to(dev)
    y_v, tape = kda.kda_verify(cfg, shp(p['q'], H, d), shp(p['k'], H, d), shp(p['v'], H, d),
                               shp(p['log_a'], H, d), shp(p['beta'], H),
                               shp(A['g'].to(dev), H, d), Pd['norm_w'], st)
    torch.cuda.synchronize()
    assert torch.equal(st.cpu(), S0)                    # live state untouched
    st2 = S0.to(dev)
    for j in range(Tb):
        sel = lambda t: t.view(B, Tb, *t.shape[1:])[:, j].contiguous()
        y_d = kda.kda_decode(cfg, sel(p['q']), sel(p['k']), sel(p['v']), sel(p['log_a']),
                             sel(p['beta']), sel(A['g'].to(dev)), Pd['norm_w'], st2)
        torch.cuda.synchronize()
        assert torch.equal(tape[:, j], st2), j
        assert torch.equal(y_v[:, j], y_d), j
    # and against the oracle
    for b in range(B):
        seq = {k: v[b * Tb:(b + 1) * Tb] for k, v in A.items() if k != 'cu_seqlens'}
        seq['cu_seqlens'] = torch.tensor([0, Tb], dtype=torch.int32)
        ref = oracle_layer(cfg, P, seq, S0[b:b + 1], hist[b:b + 1])
        assert rel_err(np64(y_v[b]), ref['y']) <= 1e-2
        assert rel_err(np64(tape[b, -1]), ref['state'][0]) <= 1e-2


def test_rollback_bit_exact():
    B, H, d, Tb, K = 9, 2, 64, 8, 4
    cfg, P, A, S0, hist = make_case(13, [Tb] * B, H, d, K, torch.bfloat16, state_var=0.01,
                                    conv_hist=True)
    dev = 'cuda'
    Pd = {k: v.to(dev) for k, v in P.items()}
    cs = hist.to(dev)
    p = kda.kda_prep(cfg, A['cu_seqlens'].to(dev), A['x'].to(dev), A['f'].to(dev),
                     A['beta_logit'].to(dev), Pd['conv_w'], Pd['A_log'], Pd['dt_bias'],
                     conv_state=cs, conv_mode=kda.KDA_CONV_TAPE, max_seqlen=Tb)
    shp = lambda t, *tail: t.view(B, Tb, *tail)
    st = S0.to(dev)
    _, tape = kda.kda_verify(cfg, shp(p['q'], H, d), shp(p['k'], H, d), shp(p['v'], H, d),
                             shp(p['log_a'], H, d), shp(p['beta'], H),
                             shp(A['g'].to(dev), H, d), Pd['norm_w'], st)
    acc = torch.arange(B, dtype=torch.int32) % (Tb + 1)          # 0..8 all present
    kda.kda_rollback(cfg, acc.to(dev), tape, st, conv_window=p['window'], conv_state=cs)
    torch.cuda.synchronize()
    win = p['window'].view(B, K - 1 + Tb, H, 3 * d)
    for b in range(B):
        L = int(acc[b])
        if L == 0:
            assert torch.equal(st[b].cpu(), S0[b])
            assert torch.equal(cs[b].cpu(), hist[b])
        else:
            assert torch.equal(st[b], tape[b, L - 1])
            assert torch.equal(cs[b], win[b, L:L + K - 1])


def test_state_pool_slots():
    """decode with state_slots into a larger pool touches only the mapped rows."""
    B, H, d, pool = 3, 2, 32, 7
    cfg, P, A, _, _ = make_case(14, [1] * B, H, d, 4, torch.bfloat16)
    dev = 'cuda'
    pool_state = synth.initial_state(14, pool, H, d, 0.01).to(dev)
    before = pool_state.clone()
    slots = torch.tensor([5, 0, 3], dtype=torch.int32, device=dev)
    p = kda.kda_prep(cfg, A['cu_seqlens'].to(dev), A['x'].to(dev), A['f'].to(dev),
                     A['beta_logit'].to(dev), P['conv_w'].to(dev), P['A_log'].to(dev),
                     P['dt_bias'].to(dev))
    y = kda.kda_decode(cfg, p['q'], p['k'], p['v'], p['log_a'], p['beta'], A['g'].to(dev),
                       P['norm_w'].to(dev), pool_state, state_slots=slots)
    torch.cuda.synchronize()
    for r in (1, 2, 4, 6):
        assert torch.equal(pool_state[r], before[r])
    for b, r in enumerate([5, 0, 3]):
        st = before[r:r + 1].clone()
        one = lambda t: t[b:b + 1].clone()    # fresh, 16-byte aligned allocations
        y1 = kda.kda_decode(cfg, one(p['q']), one(p['k']), one(p['v']), one(p['log_a']),
                            one(p['beta']), one(A['g'].to(dev)), P['norm_w'].to(dev), st)
        torch.cuda.synchronize()
        assert torch.equal(st[0], pool_state[r])
        assert torch.equal(y1[0], y[b])


def test_bounded_wait_times_out_and_context_survives():
    """A wait that nothing completes gives up, reports KDA_ERR_TIMEOUT, and the
    context keeps working (failure detection without a GPU fault)."""
    ws = torch.empty(4096, dtype=torch.uint8, device='cuda')
    kda.kda_selftest_wait_timeout(ws)
    assert kda.kda_workspace_status(ws) == kda.KDA_ERR_TIMEOUT
    cfg, P, A, S0, hist = make_case(15, [20], 2, 64, 4, torch.bfloat16, state_var=0.01)
    _assert(compare_layer(cfg, P, A, S0, hist), 1e-2)
    w2 = torch.empty(kda.kda_layer_prefill_workspace_size(cfg, 1, 20), dtype=torch.uint8,
                     device='cuda')
    kda.layer_prefill(cfg, {k: v.cuda() for k, v in P.items()},
                      {k: v.cuda() for k, v in A.items()}, workspace=w2)
    assert kda.kda_workspace_status(w2) == kda.KDA_OK


@pytest.mark.parametrize('H,seqlens,one_launch', [(4, [300, 264], False), (32, [300, 264], True),
                                                  (32, [100, 64, 30], False)])
def test_layer_prefill_launches_and_fused_norm(H, seqlens, one_launch):
    """bf16, d = 128, chunk 64, conv 4: prep runs inside the intra-chunk pass and the gated
    norm inside the inter-chunk pass.  With H between a fifth and a quarter of the SMs (32 on
    a B200) and sequences of 4 chunks or more on average, both passes share one co-scheduled
    launch; otherwise (and with KDA_LAUNCH_SEPARATE_PASSES) they are two kernels.  The
    conv-state commit adds one launch when a conv state is given."""
    cfg, P, A, S0, hist = make_case(21, seqlens, H, 128, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True, chunk=64)
    N = len(seqlens)
    sep = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_SEPARATE_PASSES)
    Pd = {k: v.cuda() for k, v in P.items()}
    Ad = {k: v.cuda() for k, v in A.items()}
    one = 1 if one_launch else 2
    for c, n_pass in ((cfg, one), (sep, 2)):
        n0 = kda.kda_launch_count()
        kda.layer_prefill(c, Pd, Ad, state_out=torch.empty(N, H, 128, 128, device='cuda'))
        assert kda.kda_launch_count() - n0 == n_pass
    n0 = kda.kda_launch_count()
    y, s_out, cs, _ = gpu_layer(cfg, P, A, S0, hist, fused=True)
    assert kda.kda_launch_count() - n0 == one + 1
    heads = [0, H - 1]
    ref = oracle_layer(cfg, P, A, S0, hist, heads)
    assert rel_err(np64(y)[:, heads], ref['y']) <= 1e-2
    assert rel_err(np64(s_out)[:, heads], ref['state']) <= 1e-2


@pytest.mark.parametrize('dtype,d', [(torch.bfloat16, 128), (torch.bfloat16, 32),
                                     (torch.float32, 64), (torch.float32, 16)])
def test_layer_decode_fused_prep(dtype, d):
    """kda_layer_decode (prep inside the step kernel) against kda_prep + kda_decode and the
    oracle: same y and state to rounding, the same conv state bit for bit."""
    B, H, T0, steps = 3, 4, 40, 6
    cfg, P, A, S0, hist = make_case(12, [T0] * B, H, d, 4, dtype, state_var=0.01,
                                    conv_hist=True, chunk=16)
    _, s0, c0, _ = gpu_layer(cfg, P, A, S0, hist)
    sa = _step_acts(12, B, H, d, dtype, steps)
    s_a, c_a = s0.clone(), c0.clone()
    s_b, c_b = s0.clone(), c0.clone()
    n0 = kda.kda_launch_count()
    ys_f = _decode_run(cfg, P, sa, s_a, c_a, fused=True).cpu()
    assert kda.kda_launch_count() - n0 == steps
    ys_u = _decode_run(cfg, P, sa, s_b, c_b).cpu()
    assert torch.equal(c_a.cpu(), c_b.cpu())
    tol = TOL[dtype]
    assert rel_err(np64(ys_f), np64(ys_u)) <= tol
    assert rel_err(np64(s_a), np64(s_b)) <= tol
    for b in range(B):
        seq = _cat_seq([A] + sa, b)
        ref = oracle_layer(cfg, P, seq, S0[b:b + 1], hist[b:b + 1])
        assert rel_err(np64(ys_f[:, b]), ref['y'][T0:]) <= tol
        assert rel_err(np64(s_a[b]), ref['state'][0]) <= tol


@pytest.mark.parametrize('dtype', [torch.bfloat16, torch.float32])
def test_layer_verify_fused_prep_and_rollback(dtype):
    """kda_layer_verify against kda_prep (TAPE) + kda_verify: y and tape to rounding, the
    conv window bit for bit; rolling back with it equals the unfused rollback exactly."""
    B, H, d, Tb = 3, 4, 64, 8
    cfg, P, A, S0, hist = make_case(13, [1] * B, H, d, 4, dtype, state_var=0.01,
                                    conv_hist=True, chunk=16)
    D = synth.layer_activations(13, [Tb] * B, H, d, dtype, tag='drafts')
    dev = 'cuda'
    Pd = {k: v.to(dev) for k, v in P.items()}
    st = S0.to(dev)
    cs = hist.to(dev)
    v4 = lambda t, *tail: t.to(dev).reshape(B, Tb, *tail).contiguous()
    y_f, tape_f, win_f = kda.kda_layer_verify(
        cfg, v4(D['x'], H, 3 * d), v4(D['f'], H, d), v4(D['beta_logit'], H), v4(D['g'], H, d),
        Pd['conv_w'], Pd['A_log'], Pd['dt_bias'], Pd['norm_w'], st, conv_state=cs)
    p = kda.kda_prep(cfg, D['cu_seqlens'].to(dev), D['x'].to(dev), D['f'].to(dev),
                     D['beta_logit'].to(dev), Pd['conv_w'], Pd['A_log'], Pd['dt_bias'],
                     conv_state=cs, conv_mode=kda.KDA_CONV_TAPE, max_seqlen=Tb)
    y_u, tape_u = kda.kda_verify(cfg, p['q'].view(B, Tb, H, d), p['k'].view(B, Tb, H, d),
                                 p['v'].view(B, Tb, H, d), p['log_a'].view(B, Tb, H, d),
                                 p['beta'].view(B, Tb, H), v4(D['g'], H, d), Pd['norm_w'], st)
    torch.cuda.synchronize()
    assert torch.equal(win_f.cpu().reshape(p['window'].shape), p['window'].cpu())
    assert torch.equal(st.cpu(), S0) and torch.equal(cs.cpu(), hist)   # read only
    tol = TOL[dtype]
    assert rel_err(np64(y_f), np64(y_u)) <= tol
    assert rel_err(np64(tape_f), np64(tape_u)) <= tol
    acc = torch.tensor([0, 3, 8], dtype=torch.int32, device=dev)
    s1, c1 = st.clone(), cs.clone()
    kda.kda_rollback(cfg, acc, tape_f, s1, conv_window=win_f, conv_state=c1)
    torch.cuda.synchronize()
    assert torch.equal(s1[0].cpu(), S0[0]) and torch.equal(c1[0].cpu(), hist[0])
    for b, L in ((1, 3), (2, 8)):
        assert torch.equal(s1[b], tape_f[b, L - 1])
        assert torch.equal(c1[b], win_f[b, L:L + 3])


@pytest.mark.parametrize('fused', [True, False])
def test_maximal_decay_gate_bf16(fused):
    """Every gate at its lower bound (f large: log a = lb = -5 per token and channel), the
    widest exponent range inside a chunk (G spans -320 over 64 tokens): the reference-row
    split of the tcgen05 gram must stay exact, and the state forgets at e^-5 per token."""
    cfg, P, A, S0, hist = make_case(14, [64, 130, 7], 4, 128, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True, chunk=64)
    A['f'] = torch.full_like(A['f'], 30.0)
    _assert(compare_layer(cfg, P, A, S0, hist, fused=fused), 1e-2)


def test_mixed_decay_gate_bf16():
    """Gates alternating between no decay and the lower bound along the chunk and across
    channels (G jumps by 5 between neighbouring tokens on half the channels)."""
    cfg, P, A, S0, hist = make_case(15, [200], 4, 128, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True, chunk=64)
    f = torch.full_like(A['f'], -30.0)
    f[::2, :, ::2] = 30.0
    A['f'] = f
    _assert(compare_layer(cfg, P, A, S0, hist), 1e-2)


@pytest.mark.parametrize('q_scale', [128 ** -0.5, 2.0])
@pytest.mark.parametrize('dtype,d,chunk,fused', [(torch.bfloat16, 128, 64, True),
                                                 (torch.bfloat16, 128, 64, False),
                                                 (torch.float32, 64, 32, True)])
def test_q_scale(q_scale, dtype, d, chunk, fused):
    """q_scale != 1 (folded into the q normalisation on the fused path).  The RMSNorm eps
    is set to 1e3, far above mean(o^2), so y is proportional to o and a q_scale that is
    dropped, squared or applied on some tiles only moves y by its full factor (with the
    usual eps the norm would cancel it)."""
    cfg, P, A, S0, hist = make_case(16, [90, 33], 4, d, 4, dtype, state_var=0.01,
                                    conv_hist=True, chunk=chunk)
    cfg.q_scale = q_scale
    cfg.norm_eps = 1e3
    _assert(compare_layer(cfg, P, A, S0, hist, fused=fused), TOL[dtype])


def test_q_scale_decode_and_verify():
    """q_scale through the step kernel (kda_layer_decode, kda_layer_verify, kda_decode),
    with the same large RMSNorm eps so that y is proportional to o."""
    B, H, d, T0, steps = 2, 4, 128, 20, 5
    cfg, P, A, S0, hist = make_case(17, [T0] * B, H, d, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True)
    cfg.q_scale = 2.0
    cfg.norm_eps = 1e3
    _, s0, c0, _ = gpu_layer(cfg, P, A, S0, hist)
    sa = _step_acts(17, B, H, d, torch.bfloat16, steps)
    for fused in (True, False):
        st, cs = s0.clone(), c0.clone()
        ys = _decode_run(cfg, P, sa, st, cs, fused=fused).cpu()
        for b in range(B):
            ref = oracle_layer(cfg, P, _cat_seq([A] + sa, b), S0[b:b + 1], hist[b:b + 1])
            assert rel_err(np64(ys[:, b]), ref['y'][T0:]) <= 1e-2, (fused, b)
    Tb = 6
    D = synth.layer_activations(17, [Tb] * B, H, d, torch.bfloat16, tag='drafts')
    v4 = lambda t, *tail: t.cuda().reshape(B, Tb, *tail).contiguous()
    Pd = {k: v.cuda() for k, v in P.items()}
    y_v, _, _ = kda.kda_layer_verify(cfg, v4(D['x'], H, 3 * d), v4(D['f'], H, d),
                                     v4(D['beta_logit'], H), v4(D['g'], H, d), Pd['conv_w'],
                                     Pd['A_log'], Pd['dt_bias'], Pd['norm_w'], s0,
                                     conv_state=c0)
    torch.cuda.synchronize()
    for b in range(B):
        seq = {k: torch.cat([A[k][b * T0:(b + 1) * T0], D[k][b * Tb:(b + 1) * Tb]])
               for k in ('x', 'f', 'beta_logit', 'g')}
        seq['cu_seqlens'] = torch.tensor([0, T0 + Tb], dtype=torch.int32)
        ref = oracle_layer(cfg, P, seq, S0[b:b + 1], hist[b:b + 1])
        assert rel_err(np64(y_v[b]), ref['y'][T0:]) <= 1e-2, b


# ---------------------------------------------------------------------------
# the L2 norm's eps: q / max(||q||, eps) on rows whose norm is zero or below eps
# ---------------------------------------------------------------------------
# (head, channel segment 0 = q / 1 = k, first token, last token, scale): the
# pre-conv inputs of that segment are multiplied by `scale` on those tokens; the
# conv mixes K = 4 tokens, so rows from first + 3 on are exactly zero (scale 0)
# or have a norm far below 1e-6 (scale 1e-9) after the conv, and the
# 1e-4 rows stay above eps (normalised to unit length as usual)
EDGE_ROWS = [(0, 0, 10, 40, 0.0), (1, 1, 45, 75, 0.0), (2, 0, 70, 110, 1e-9),
             (3, 1, 100, 140, 1e-9), (3, 0, 145, 175, 1e-4)]


def _edge_case(dtype, d, chunk, T=200, seed=31):
    cfg, P, A, S0, _ = make_case(seed, [T], 4, d, 4, dtype, state_var=0.01, chunk=chunk)
    x = A['x'].clone()
    for h, seg, t0, t1, sc in EDGE_ROWS:
        x[t0:t1, h, seg * d:(seg + 1) * d] *= sc
    A['x'] = x
    return cfg, P, A, S0


def _edge_regions(T_off=0):
    """(head, rows) of the layer's output whose q or k was zero / below eps."""
    return [(h, slice(T_off + t0 + 3, T_off + t1)) for h, _, t0, t1, _ in EDGE_ROWS]


@pytest.mark.parametrize('dtype,d,chunk,fused', [(torch.bfloat16, 128, 64, True),
                                                 (torch.bfloat16, 128, 64, False),
                                                 (torch.float32, 64, 32, True),
                                                 (torch.bfloat16, 64, 16, False)])
def test_l2_eps_zero_and_tiny_rows_prefill(dtype, d, chunk, fused):
    """Rows of q or k that are exactly zero or whose norm is below the 1e-6 eps (PR
    #27754: ggml's max(sqrt(sum), eps) form): kda_layer_prefill (prep fused into the
    tcgen05 pass at bf16 d = 128) and kda_prep + kda_prefill against the oracle, on the
    whole output and on each edge region by itself."""
    cfg, P, A, S0 = _edge_case(dtype, d, chunk)
    y, s_out, _, p = gpu_layer(cfg, P, A, S0, None, fused=fused)
    ref = oracle_layer(cfg, P, A, S0)
    tol = TOL[dtype]
    assert rel_err(np64(y), ref['y']) <= tol
    assert rel_err(np64(s_out), ref['state']) <= tol
    yg = np64(y)
    for h, rows in _edge_regions():
        assert rel_err(yg[rows, h], ref['y'][rows, h]) <= tol, (h, rows)
    if p is not None:
        # kda_prep's normalised q / k on the edge rows themselves: 0, or x / eps
        for h, seg, t0, t1, _ in EDGE_ROWS:
            name = 'qk'[seg]
            got = np64(p[name])[t0 + 3:t1, h]
            want = ref[name][t0 + 3:t1, h]
            assert rel_err(got, want) <= 1e-5, (name, h)


@pytest.mark.parametrize('dtype,d', [(torch.bfloat16, 128), (torch.float32, 64)])
def test_l2_eps_zero_and_tiny_rows_decode_verify(dtype, d):
    """The same edge rows through the step kernel: kda_layer_decode (fused prep),
    kda_prep + kda_decode, and kda_layer_verify, after a prefill of the first 40 tokens."""
    T = 200
    cfg, P, A, S0 = _edge_case(dtype, d, 16, T=T)
    T0 = 40
    head = {k: A[k][:T0] for k in ('x', 'f', 'beta_logit', 'g')}
    head['cu_seqlens'] = torch.tensor([0, T0], dtype=torch.int32)
    _, s0, c0, _ = gpu_layer(cfg, P, head, S0, None)
    ref = oracle_layer(cfg, P, A, S0)
    tol = TOL[dtype]
    steps = [{k: A[k][t:t + 1] for k in ('x', 'f', 'beta_logit', 'g')} for t in range(T0, T)]
    for st_ in steps:
        st_['cu_seqlens'] = torch.tensor([0, 1], dtype=torch.int32)
    for fused in (True, False):
        st, cs = s0.clone(), c0.clone()
        ys = np64(_decode_run(cfg, P, steps, st, cs, fused=fused))[:, 0]   # [T - T0, H, d]
        assert rel_err(ys, ref['y'][T0:]) <= tol, fused
        assert rel_err(np64(st), ref['state']) <= tol, fused
        for h, rows in _edge_regions():
            r = slice(max(rows.start, T0) - T0, rows.stop - T0)
            assert rel_err(ys[r, h], ref['y'][T0:][r, h]) <= tol, (fused, h)
    # verify: blocks of 8 drafts over tokens 40..199, each verified from the state
    # after the tokens before it (rolled forward by accepting every draft)
    Pd = {k: v.cuda() for k, v in P.items()}
    st, cs = s0.clone(), c0.clone()
    yv = []
    for t in range(T0, T, 8):
        blk = lambda key, *tail: A[key][t:t + 8].cuda().reshape(1, 8, *tail).contiguous()
        y_b, tape, win = kda.kda_layer_verify(cfg, blk('x', 4, 3 * d), blk('f', 4, d),
                                              blk('beta_logit', 4), blk('g', 4, d),
                                              Pd['conv_w'], Pd['A_log'], Pd['dt_bias'],
                                              Pd['norm_w'], st, conv_state=cs)
        kda.kda_rollback(cfg, torch.tensor([8], dtype=torch.int32, device='cuda'), tape, st,
                         conv_window=win, conv_state=cs)
        yv.append(y_b[0])
    torch.cuda.synchronize()
    yv = np64(torch.cat(yv))
    assert rel_err(yv, ref['y'][T0:]) <= tol
    for h, rows in _edge_regions():
        r = slice(max(rows.start, T0) - T0, rows.stop - T0)
        assert rel_err(yv[r, h], ref['y'][T0:][r, h]) <= tol, h


# ---------------------------------------------------------------------------
# the softplus decay gate (no lower bound): PR #27754, "Metadata and tensor loading"
# ---------------------------------------------------------------------------
@pytest.mark.parametrize('fused', [True, False])
@pytest.mark.parametrize('dtype,d,chunk', [(torch.bfloat16, 128, 64), (torch.float32, 64, 32),
                                           (torch.bfloat16, 32, 16), (torch.float32, 16, 16)])
def test_softplus_gate_prefill(dtype, d, chunk, fused):
    """kda_layer_prefill and kda_prep + kda_prefill with log a = -exp(A_log) softplus(f +
    dt_bias): decays far below the bounded gate's -5 per token, so a chunk's cumulative
    decay spans hundreds of nats (the SIMT passes, exact inside each 16-token block)."""
    seqlens = [chunk - 3, 2 * chunk + 5, 1]
    cfg, P, A, S0, hist = make_case(41, seqlens, 3, d, 4, dtype, state_var=0.01,
                                    conv_hist=True, chunk=chunk)
    cfg.gate_lower_bound = None
    P['A_log'][0] = math.log(16.0)            # the recipe's largest rate on one head
    y, s_out, cs, p = gpu_layer(cfg, P, A, S0, hist, fused=fused)
    ref = oracle_layer(cfg, P, A, S0, hist)
    assert ref['loga'].min() < -20.0          # the workload reaches well past -5 per token
    tol = TOL[dtype]
    assert rel_err(np64(y), ref['y']) <= tol
    assert rel_err(np64(s_out), ref['state']) <= tol
    assert np.array_equal(np64(cs), ref['conv_hist'])
    if p is not None:
        assert rel_err(np64(p['log_a']), ref['loga']) <= 1e-5


@pytest.mark.parametrize('dtype,d', [(torch.bfloat16, 128), (torch.float32, 64)])
def test_softplus_gate_decode_verify(dtype, d):
    """The softplus gate through the step kernel: kda_layer_decode (gate computed in the
    kernel), kda_prep + kda_decode, and kda_layer_verify + rollback."""
    B, H, T0, steps = 2, 4, 30, 6
    cfg, P, A, S0, hist = make_case(42, [T0] * B, H, d, 4, dtype, state_var=0.01,
                                    conv_hist=True, chunk=16)
    cfg.gate_lower_bound = None
    _, s0, c0, _ = gpu_layer(cfg, P, A, S0, hist)
    sa = _step_acts(42, B, H, d, dtype, steps)
    tol = TOL[dtype]
    for fused in (True, False):
        st, cs = s0.clone(), c0.clone()
        ys = _decode_run(cfg, P, sa, st, cs, fused=fused).cpu()
        for b in range(B):
            ref = oracle_layer(cfg, P, _cat_seq([A] + sa, b), S0[b:b + 1], hist[b:b + 1])
            assert rel_err(np64(ys[:, b]), ref['y'][T0:]) <= tol, (fused, b)
            assert rel_err(np64(st[b]), ref['state'][0]) <= tol, (fused, b)
    Tb = 8
    D = synth.layer_activations(42, [Tb] * B, H, d, dtype, tag='drafts')
    v4 = lambda t, *tail: t.cuda().reshape(B, Tb, *tail).contiguous()
    Pd = {k: v.cuda() for k, v in P.items()}
    st, cs = s0.clone(), c0.clone()
    y_v, tape, win = kda.kda_layer_verify(cfg, v4(D['x'], H, 3 * d), v4(D['f'], H, d),
                                          v4(D['beta_logit'], H), v4(D['g'], H, d),
                                          Pd['conv_w'], Pd['A_log'], Pd['dt_bias'],
                                          Pd['norm_w'], st, conv_state=cs)
    acc = torch.tensor([3, 8], dtype=torch.int32, device='cuda')
    kda.kda_rollback(cfg, acc, tape, st, conv_window=win, conv_state=cs)
    torch.cuda.synchronize()
    for b, L in ((0, 3), (1, 8)):
        seq = {k: torch.cat([A[k][b * T0:(b + 1) * T0], D[k][b * Tb:b * Tb + L]])
               for k in ('x', 'f', 'beta_logit', 'g')}
        seq['cu_seqlens'] = torch.tensor([0, T0 + L], dtype=torch.int32)
        ref = oracle_layer(cfg, P, seq, S0[b:b + 1], hist[b:b + 1])
        assert rel_err(np64(y_v[b, :L]), ref['y'][T0:]) <= tol, b
        assert rel_err(np64(st[b]), ref['state'][0]) <= tol, b
        assert np.array_equal(np64(cs[b]), ref['conv_hist'][0])


# ---------------------------------------------------------------------------
# compact verify tape (k, u, a per step) and rollback by replay
# ---------------------------------------------------------------------------
@pytest.mark.parametrize('dtype,d', [(torch.bfloat16, 128), (torch.float32, 64),
                                     (torch.bfloat16, 32)])
def test_replay_rollback_equals_full_tape_bit_exact(dtype, d):
    """dflash-mlx issue #63 (tape-replay rollback): kda_verify_compact + kda_rollback_replay
    against kda_verify + kda_rollback on the same block, for every accepted length 0..8:
    the same y, and the replayed state equal to the full tape's entry bit for bit."""
    B, H, Tb, K = 9, 3, 8, 4
    cfg, P, A, S0, hist = make_case(43, [Tb] * B, H, d, K, dtype, state_var=0.01,
                                    conv_hist=True, chunk=16)
    dev = 'cuda'
    Pd = {k: v.to(dev) for k, v in P.items()}
    p = kda.kda_prep(cfg, A['cu_seqlens'].to(dev), A['x'].to(dev), A['f'].to(dev),
                     A['beta_logit'].to(dev), Pd['conv_w'], Pd['A_log'], Pd['dt_bias'],
                     conv_state=hist.to(dev), conv_mode=kda.KDA_CONV_TAPE, max_seqlen=Tb)
    shp = lambda t, *tail: t.view(B, Tb, *tail)
    args = (shp(p['q'], H, d), shp(p['k'], H, d), shp(p['v'], H, d), shp(p['log_a'], H, d),
            shp(p['beta'], H), shp(A['g'].to(dev), H, d), Pd['norm_w'])
    st_full, st_rep = S0.to(dev), S0.to(dev)
    y_full, tape = kda.kda_verify(cfg, *args, st_full)
    y_rep, kua = kda.kda_verify_compact(cfg, *args, st_rep)
    acc = torch.arange(B, dtype=torch.int32, device=dev) % (Tb + 1)     # 0..8
    cs_full, cs_rep = hist.to(dev), hist.to(dev)
    kda.kda_rollback(cfg, acc, tape, st_full, conv_window=p['window'], conv_state=cs_full)
    kda.kda_rollback_replay(cfg, acc, kua, st_rep, conv_window=p['window'], conv_state=cs_rep)
    torch.cuda.synchronize()
    assert torch.equal(y_full, y_rep)
    assert torch.equal(st_rep, st_full)
    assert torch.equal(cs_rep, cs_full)
    for b in range(B):
        L = int(acc[b])
        assert torch.equal(st_rep[b], tape[b, L - 1] if L else S0[b].to(dev)), b
    # the compact tape holds the step's k and a as prep produced them
    assert torch.equal(kua[:, :, :, 0], shp(p['k'], H, d))
    assert torch.allclose(kua[:, :, :, 2], torch.exp(shp(p['log_a'], H, d)), rtol=1e-6, atol=0)


@pytest.mark.parametrize('dtype', [torch.bfloat16, torch.float32])
def test_layer_verify_compact_and_replay(dtype):
    """kda_layer_verify_compact (prep in the step kernel) + kda_rollback_replay equals
    kda_layer_verify + kda_rollback bit for bit, and the oracle's accepted prefix."""
    B, H, d, Tb = 3, 4, 64, 8
    cfg, P, A, S0, hist = make_case(44, [1] * B, H, d, 4, dtype, state_var=0.01,
                                    conv_hist=True, chunk=16)
    D = synth.layer_activations(44, [Tb] * B, H, d, dtype, tag='drafts')
    dev = 'cuda'
    Pd = {k: v.to(dev) for k, v in P.items()}
    v4 = lambda t, *tail: t.to(dev).reshape(B, Tb, *tail).contiguous()
    args = (v4(D['x'], H, 3 * d), v4(D['f'], H, d), v4(D['beta_logit'], H), v4(D['g'], H, d),
            Pd['conv_w'], Pd['A_log'], Pd['dt_bias'], Pd['norm_w'])
    s1, c1 = S0.to(dev), hist.to(dev)
    s2, c2 = S0.to(dev), hist.to(dev)
    y1, tape, w1 = kda.kda_layer_verify(cfg, *args, s1, conv_state=c1)
    y2, kua, w2 = kda.kda_layer_verify_compact(cfg, *args, s2, conv_state=c2)
    acc = torch.tensor([0, 5, 8], dtype=torch.int32, device=dev)
    kda.kda_rollback(cfg, acc, tape, s1, conv_window=w1, conv_state=c1)
    kda.kda_rollback_replay(cfg, acc, kua, s2, conv_window=w2, conv_state=c2)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(w1, w2)
    assert torch.equal(s1, s2) and torch.equal(c1, c2)
    for b, L in enumerate([0, 5, 8]):
        # the block starts from S0 and the conv history: the oracle runs the L accepted drafts
        blk = {k: D[k][b * Tb:b * Tb + L] for k in ('x', 'f', 'beta_logit', 'g')}
        blk['cu_seqlens'] = torch.tensor([0, L], dtype=torch.int32)
        ref = oracle_layer(cfg, P, blk, S0[b:b + 1], hist[b:b + 1])
        assert rel_err(np64(s2[b]), ref['state'][0]) <= TOL[dtype], b
        assert np.array_equal(np64(c2[b]), ref['conv_hist'][0]), b


# ---------------------------------------------------------------------------
# KDA_LAUNCH_EARLY_STATE: the step and replay kernels stream the state before the
# kernel ahead of them on the stream has finished (programmatic dependent launch)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize('dtype,d', [(torch.bfloat16, 128), (torch.float32, 64)])
def test_early_state_launch_bit_exact(dtype, d):
    """Decode steps after kda_prep, and verify rounds (kda_prep, kda_verify_compact,
    kda_rollback_replay), with KDA_LAUNCH_EARLY_STATE, eager and replayed from a CUDA
    graph, equal the default launches bit for bit (y, state, conv state)."""
    B, H, Tb, steps, rounds = 5, 4, 8, 6, 3
    cfg, P, _, S0, hist = make_case(45, [1] * B, H, d, 4, dtype, state_var=0.01,
                                    conv_hist=True, chunk=16)
    early = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_EARLY_STATE)
    dev = 'cuda'
    Pd = {k: v.to(dev) for k, v in P.items()}
    sa = [{k: v.to(dev) for k, v in a.items()} for a in _step_acts(45, B, H, d, dtype, steps)]
    blocks = [{k: v.to(dev) for k, v in
               synth.layer_activations(46, [Tb] * B, H, d, dtype, tag=('round', r)).items()}
              for r in range(rounds)]
    acc = [torch.tensor([(3 * r + b) % (Tb + 1) for b in range(B)], dtype=torch.int32,
                        device=dev) for r in range(rounds)]

    def run(c, st, cs):
        ys = []
        for a in sa:
            p = kda.kda_prep(c, a['cu_seqlens'], a['x'], a['f'], a['beta_logit'], Pd['conv_w'],
                             Pd['A_log'], Pd['dt_bias'], conv_state=cs, max_seqlen=1)
            ys.append(kda.kda_decode(c, p['q'], p['k'], p['v'], p['log_a'], p['beta'], a['g'],
                                     Pd['norm_w'], st))
        shp = lambda t, *tail: t.view(B, Tb, *tail)
        for r, a in enumerate(blocks):
            p = kda.kda_prep(c, a['cu_seqlens'], a['x'], a['f'], a['beta_logit'], Pd['conv_w'],
                             Pd['A_log'], Pd['dt_bias'], conv_state=cs,
                             conv_mode=kda.KDA_CONV_TAPE, max_seqlen=Tb)
            y, kua = kda.kda_verify_compact(c, shp(p['q'], H, d), shp(p['k'], H, d),
                                            shp(p['v'], H, d), shp(p['log_a'], H, d),
                                            shp(p['beta'], H), shp(a['g'], H, d), Pd['norm_w'],
                                            st)
            kda.kda_rollback_replay(c, acc[r], kua, st, conv_window=p['window'], conv_state=cs)
            ys.append(y.reshape(B * Tb, H, d)[:B])
        return torch.stack(ys)

    ref_st, ref_cs = S0.to(dev), hist.to(dev)
    ref_y = run(cfg, ref_st, ref_cs)
    st, cs = S0.to(dev), hist.to(dev)
    y = run(early, st, cs)
    torch.cuda.synchronize()
    assert torch.equal(y, ref_y) and torch.equal(st, ref_st) and torch.equal(cs, ref_cs)

    g_st, g_cs = S0.to(dev), hist.to(dev)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        g_y = run(early, g_st, g_cs)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(g_y, ref_y) and torch.equal(g_st, ref_st) and torch.equal(g_cs, ref_cs)
    del g


# ---------------------------------------------------------------------------
# kda_prep with max_seqlen <= 16: the kernel for short sequences
# ---------------------------------------------------------------------------
@pytest.mark.parametrize('dtype', [torch.float32, torch.bfloat16])
@pytest.mark.parametrize('d,K,hint,softplus', [(128, 4, 1, False), (128, 4, 16, False),
                                               (64, 2, 8, False), (32, 8, 16, False),
                                               (16, 4, 8, False), (128, 4, 8, True)])
def test_prep_short_matches_oracle(dtype, d, K, hint, softplus):
    """The short-sequence prep (one CTA per sequence and head) against the oracle's prep:
    q, k, v, log a, beta to 1e-5 of max, the committed conv state and the TAPE window bit
    for bit.  One sequence is longer than the hint (taken in blocks, still exact); one case
    takes the softplus gate."""
    seqlens = [0, 1, hint, 3, hint + 21]
    cfg, P, A, _, hist = make_case(47, seqlens, 3, d, K, dtype, conv_hist=True)
    if softplus:
        cfg = dataclasses.replace(cfg, gate_lower_bound=None)
    dev = 'cuda'
    Pd = {k: v.to(dev) for k, v in P.items()}
    args = (A['cu_seqlens'].to(dev), A['x'].to(dev), A['f'].to(dev), A['beta_logit'].to(dev),
            Pd['conv_w'], Pd['A_log'], Pd['dt_bias'])
    cs = hist.to(dev)
    p = kda.kda_prep(cfg, *args, conv_state=cs, max_seqlen=hint)
    cs_t = hist.to(dev)
    pt = kda.kda_prep(cfg, *args, conv_state=cs_t, conv_mode=kda.KDA_CONV_TAPE,
                      max_seqlen=hint)
    torch.cuda.synchronize()
    ref = oracle_layer(cfg, P, A, None, hist)
    for name, rname in [('q', 'q'), ('k', 'k'), ('v', 'v'), ('log_a', 'loga'), ('beta', 'beta')]:
        assert rel_err(np64(p[name]), ref[rname]) <= 1e-5, name
        assert torch.equal(p[name], pt[name]), name          # TAPE mode: the same outputs
    assert np.array_equal(np64(cs), ref['conv_hist'])
    assert torch.equal(cs_t, hist.to(dev))                   # TAPE never writes the state
    Km1, cu = K - 1, A['cu_seqlens'].tolist()
    win = pt['window'].cpu()
    for s, T in enumerate(seqlens):
        base = cu[s] + s * Km1
        assert torch.equal(win[base:base + Km1], hist[s])
        assert torch.equal(win[base + Km1:base + Km1 + T], A['x'][cu[s]:cu[s + 1]])


def test_pool_slots_short_prep_and_early_state():
    """Decode and verify rounds through a state pool (slots, including a skipped -1) with
    the short prep (conv state in the pool too) and KDA_LAUNCH_EARLY_STATE: the mapped
    rows equal a run on the rows alone, bit for bit, and the other rows are untouched."""
    B, H, d, Tb, pool = 3, 2, 128, 8, 6
    cfg, P, _, _, _ = make_case(48, [1] * B, H, d, 4, torch.bfloat16, chunk=16)
    early = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_EARLY_STATE)
    dev = 'cuda'
    Pd = {k: v.to(dev) for k, v in P.items()}
    pool_state = synth.initial_state(48, pool, H, d, 0.01).to(dev)
    pool_conv = synth.conv_history(48, pool, H, d, 4, torch.bfloat16).to(dev)
    st0, cs0 = pool_state.clone(), pool_conv.clone()
    slots_l = [4, -1, 1]
    slots = torch.tensor(slots_l, dtype=torch.int32, device=dev)
    step = {k: v.to(dev) for k, v in synth.layer_activations(48, [1] * B, H, d, torch.bfloat16,
                                                              tag='pool_step').items()}
    blk = {k: v.to(dev) for k, v in synth.layer_activations(48, [Tb] * B, H, d, torch.bfloat16,
                                                             tag='pool_blk').items()}
    acc = torch.tensor([5, 0, 8], dtype=torch.int32, device=dev)

    def run(c, st, cs, sl, a_step, a_blk, acc_):
        p = kda.kda_prep(c, a_step['cu_seqlens'], a_step['x'], a_step['f'], a_step['beta_logit'],
                         Pd['conv_w'], Pd['A_log'], Pd['dt_bias'], conv_state=cs, state_slots=sl,
                         max_seqlen=1)
        y = kda.kda_decode(c, p['q'], p['k'], p['v'], p['log_a'], p['beta'], a_step['g'],
                           Pd['norm_w'], st, state_slots=sl)
        nb = a_step['x'].shape[0]
        shp = lambda t, *tail: t.view(nb, Tb, *tail)
        p = kda.kda_prep(c, a_blk['cu_seqlens'], a_blk['x'], a_blk['f'], a_blk['beta_logit'],
                         Pd['conv_w'], Pd['A_log'], Pd['dt_bias'], conv_state=cs, state_slots=sl,
                         conv_mode=kda.KDA_CONV_TAPE, max_seqlen=Tb)
        yv, kua = kda.kda_verify_compact(c, shp(p['q'], H, d), shp(p['k'], H, d),
                                         shp(p['v'], H, d), shp(p['log_a'], H, d),
                                         shp(p['beta'], H), shp(a_blk['g'], H, d), Pd['norm_w'],
                                         st, state_slots=sl)
        kda.kda_rollback_replay(c, acc_, kua, st, conv_window=p['window'], conv_state=cs,
                                state_slots=sl)
        return y, yv

    y, yv = run(early, pool_state, pool_conv, slots, step, blk, acc)
    torch.cuda.synchronize()
    for r in (0, 2, 3, 5):
        assert torch.equal(pool_state[r], st0[r]) and torch.equal(pool_conv[r], cs0[r]), r
    for b, r in enumerate(slots_l):
        if r < 0:
            continue
        st, cs = st0[r:r + 1].clone(), cs0[r:r + 1].clone()
        one = lambda a, T: {'cu_seqlens': torch.tensor([0, T], dtype=torch.int32, device=dev),
                            **{k: a[k][b * T:(b + 1) * T].clone() for k in ('x', 'f', 'beta_logit', 'g')}}
        y1, yv1 = run(cfg, st, cs, None, one(step, 1), one(blk, Tb), acc[b:b + 1].clone())
        torch.cuda.synchronize()
        assert torch.equal(st[0], pool_state[r]) and torch.equal(cs[0], pool_conv[r]), b
        assert torch.equal(y1[0], y[b]) and torch.equal(yv1[0], yv[b]), b


def test_cosched_pool_slots_with_a_skipped_sequence():
    """The co-scheduled launch with a state pool: a sequence mapped to slot -1 is skipped
    (its chain CTA returns, the intra-chunk role skips its tiles) and the pool rows no
    sequence maps to stay as they were; everything equals the separate launches bit for bit."""
    seqlens, H, d, pool = [600, 70, 331], 32, 128, 6
    cfg, P, A, _, _ = make_case(31, seqlens, H, d, 4, torch.bfloat16, chunk=64)
    sep = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_SEPARATE_PASSES)
    dev = 'cuda'
    Pd = {k: v.to(dev) for k, v in P.items()}
    Ad = {k: v.to(dev) for k, v in A.items()}
    slots = torch.tensor([4, -1, 1], dtype=torch.int32, device=dev)
    s0 = synth.initial_state(31, pool, H, d, 0.01).to(dev)
    c0 = (torch.randn(pool, 3, H, 3 * d, generator=torch.Generator().manual_seed(31)) * 0.5
          ).to(cfg.dtype).to(dev)
    outs = []
    for c in (cfg, sep):
        st, cs = s0.clone(), c0.clone()
        y = torch.full((sum(seqlens), H, d), 7.0, dtype=cfg.dtype, device=dev)
        kda.kda_layer_prefill(c, Ad['cu_seqlens'], Ad['x'], Ad['f'], Ad['beta_logit'], Ad['g'],
                              Pd['conv_w'], Pd['A_log'], Pd['dt_bias'], Pd['norm_w'],
                              conv_state=cs, state_in=st, state_out=st, state_slots=slots,
                              pool_size=pool, y=y, max_seqlen=max(seqlens))
        torch.cuda.synchronize()
        outs.append((y.clone(), st.clone(), cs.clone()))
    (y1, s1, c1), (y2, s2, c2) = outs
    assert torch.equal(y1, y2) and torch.equal(s1, s2) and torch.equal(c1, c2)
    skipped = slice(seqlens[0], seqlens[0] + seqlens[1])
    assert torch.all(y1[skipped] == 7.0)
    for r in (0, 2, 3, 5):
        assert torch.equal(s1[r], s0[r]) and torch.equal(c1[r], c0[r])
    assert not torch.equal(s1[4], s0[4]) and not torch.equal(s1[1], s0[1])


def test_cosched_launch_in_a_cuda_graph():
    """The co-scheduled (cooperative) launch captured in a CUDA graph with the call's
    workspace clear: two replays give the eager result bit for bit."""
    seqlens, H = [1000], 32
    cfg, P, A, S0, hist = make_case(33, seqlens, H, 128, 4, torch.bfloat16, state_var=0.01,
                                    chunk=64)
    dev = 'cuda'
    Pd = {k: v.to(dev) for k, v in P.items()}
    Ad = {k: v.to(dev) for k, v in A.items()}
    s_in = S0.to(dev)
    ws = torch.empty(kda.kda_layer_prefill_workspace_size(cfg, 1, sum(seqlens)),
                     dtype=torch.uint8, device=dev)
    y_ref = torch.empty(sum(seqlens), H, 128, dtype=cfg.dtype, device=dev)
    st_ref = torch.empty_like(s_in)
    kda.layer_prefill(cfg, Pd, Ad, state_in=s_in, state_out=st_ref, workspace=ws, y=y_ref)
    torch.cuda.synchronize()
    y = torch.empty_like(y_ref)
    st = torch.empty_like(st_ref)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        kda.layer_prefill(cfg, Pd, Ad, state_in=s_in, state_out=st, workspace=ws, y=y)
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(g):
        kda.layer_prefill(cfg, Pd, Ad, state_in=s_in, state_out=st, workspace=ws, y=y)
    for _ in range(2):
        y.zero_()
        st.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref) and torch.equal(st, st_ref)
    del g


def test_cosched_many_empty_sequences_pass_their_state_through():
    """The co-scheduled launch with more empty sequences than the chain's list holds (they
    are then found by walking the batch): every empty sequence's state row is copied from
    state_in to state_out, and the states equal the separate launches' bit for bit.  With
    2,304 (sequence, head) chains the separate form runs the gated norm as its own kernel
    (exact sigmoid, another sum order), so y agrees to rounding there."""
    n_empty, H, d = 70, 32, 128
    seqlens = [9300] + [0] * n_empty + [9250]
    N, T = len(seqlens), sum(seqlens)
    assert T >= 4 * 64 * N                      # long enough on average for one launch
    cfg = kda.Config(num_heads=H, head_dim=d, conv_size=4, dtype=torch.bfloat16, chunk_size=64)
    sep = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_SEPARATE_PASSES)
    dev = 'cuda'
    P = {k: v.to(dev) for k, v in synth.layer_params(41, H, d, 4).items()}
    A = {k: v.to(dev) for k, v in synth.layer_activations(41, seqlens, H, d, torch.bfloat16).items()}
    s0 = synth.initial_state(41, N, H, d, 0.01).to(dev)
    outs = []
    for c in (cfg, sep):
        st = torch.full_like(s0, float('nan'))
        n0 = kda.kda_launch_count()
        y = kda.layer_prefill(c, P, A, state_in=s0, state_out=st)
        torch.cuda.synchronize()
        outs.append((y, st, kda.kda_launch_count() - n0))
    (y1, s1, n1), (y2, s2, n2) = outs
    assert n1 == 1 and n2 == 3
    assert torch.equal(s1, s2)
    assert rel_err(np64(y1), np64(y2)) <= 5e-3
    assert torch.equal(s1[1:1 + n_empty], s0[1:1 + n_empty])


def test_cosched_without_initial_or_final_state():
    """The co-scheduled launch with no state_in (zeros) and with no state_out (only y):
    the same y as the separate launches, bit for bit."""
    seqlens, H = [700, 900], 32
    cfg, P, A, _, _ = make_case(43, seqlens, H, 128, 4, torch.bfloat16, chunk=64)
    sep = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_SEPARATE_PASSES)
    Pd = {k: v.cuda() for k, v in P.items()}
    Ad = {k: v.cuda() for k, v in A.items()}
    for with_out in (True, False):
        ys, states = [], []
        for c in (cfg, sep):
            st = torch.empty(len(seqlens), H, 128, 128, device='cuda') if with_out else None
            n0 = kda.kda_launch_count()
            ys.append(kda.layer_prefill(c, Pd, Ad, state_out=st))
            torch.cuda.synchronize()
            assert kda.kda_launch_count() - n0 == (1 if c is cfg else 2)
            states.append(st)
        assert torch.equal(ys[0], ys[1])
        if with_out:
            assert torch.equal(states[0], states[1])


@pytest.mark.parametrize('fused', [True, False])
def test_l2_eps_edge_rows_cosched(fused):
    """The zero / below-eps q and k rows at 32 heads, where both passes run in one
    co-scheduled launch: heads 0-3 (the edge rows) against the oracle, on the whole output
    of those heads and on each edge region by itself."""
    T, H, d = 300, 32, 128
    cfg, P, A, S0, _ = make_case(35, [T], H, d, 4, torch.bfloat16, state_var=0.01, chunk=64)
    x = A['x'].clone()
    for h, seg, t0, t1, sc in EDGE_ROWS:
        x[t0:t1, h, seg * d:(seg + 1) * d] *= sc
    A['x'] = x
    n0 = kda.kda_launch_count()
    y, s_out, _, _ = gpu_layer(cfg, P, A, S0, None, fused=fused)
    # one co-scheduled launch, plus the conv-state commit (and, unfused, the prep itself)
    assert kda.kda_launch_count() - n0 == (2 if fused else 3)
    heads = [0, 1, 2, 3]
    ref = oracle_layer(cfg, P, A, S0, None, heads)
    yg = np64(y)[:, heads]
    assert rel_err(yg, ref['y']) <= 1e-2
    assert rel_err(np64(s_out)[:, heads], ref['state']) <= 1e-2
    for h, rows in _edge_regions():
        assert rel_err(yg[rows, h], ref['y'][rows, h]) <= 1e-2, (h, rows)


@pytest.mark.parametrize('q_scale', [128 ** -0.5, 2.0])
def test_q_scale_cosched(q_scale):
    """q_scale != 1 at 32 heads, through the co-scheduled launch, with the RMSNorm eps at
    1e3 so that y is proportional to o (a lost or doubled q_scale moves y by its factor);
    two heads against the oracle."""
    cfg, P, A, S0, hist = make_case(17, [300, 270], 32, 128, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True, chunk=64)
    cfg.q_scale = q_scale
    cfg.norm_eps = 1e3
    n0 = kda.kda_launch_count()
    errs = compare_layer(cfg, P, A, S0, hist, heads=[5, 30], fused=True)
    assert kda.kda_launch_count() - n0 == 2        # one co-scheduled launch + conv commit
    _assert(errs, 1e-2)


def test_maximal_decay_gate_cosched():
    """Every gate at its lower bound (log a = -5 per token and channel) at 32 heads, through
    the co-scheduled launch: the widest exponent range inside a chunk; two heads against
    the oracle, and the same bits as the separate launches."""
    cfg, P, A, S0, hist = make_case(15, [300, 130], 32, 128, 4, torch.bfloat16, state_var=0.01,
                                    conv_hist=True, chunk=64)
    A['f'] = torch.full_like(A['f'], 30.0)
    sep = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_SEPARATE_PASSES)
    y1, s1, c1, _ = gpu_layer(cfg, P, A, S0, hist)
    y2, s2, c2, _ = gpu_layer(sep, P, A, S0, hist)
    assert torch.equal(y1, y2) and torch.equal(s1, s2) and torch.equal(c1, c2)
    _assert(compare_layer(cfg, P, A, S0, hist, heads=[0, 17]), 1e-2)
