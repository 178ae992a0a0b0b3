"""GPU parity of the projections either side of the recurrence (kda_proj_gemm, the
tcgen05 GEMM) and of the whole layer from hidden states to y, against the float64 oracle.

The GEMM's bar follows from its arithmetic: bf16 operands are exact in fp32, products
accumulate in fp32 (relative error ~K 2^-24) and the result is rounded once to bf16
(2^-9 of each element), so max|GPU - oracle| / max|oracle| <= 4e-3 per output tensor.
"""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_09_b200 import kda, synth
from oracle import kda_oracle as ko
from tests.kda_cases import np64, rel_err

pytestmark = pytest.mark.gpu
GEMM_TOL = 4e-3


def _bf16_rounded(a):
    """float64 values rounded to bf16 (round to nearest even), as float64."""
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize('M,N,K', [(1, 256, 64), (300, 520, 200), (128, 768, 1024),
                                   (517, 256 * 5 + 8, 320)])
def test_proj_gemm_matches_oracle_with_ranges(M, N, K):
    """Ragged M (rows past the last 128-row tile), N (a partial 256-column tile) and K (a
    tail past the last 64-wide slice); three output ranges with padded row strides, and the
    columns outside every range left untouched."""
    g = torch.Generator().manual_seed(M * 7 + N + K)
    A = (torch.randn(M, K, generator=g) / K ** 0.25).to(torch.bfloat16)
    B = (torch.randn(N, K, generator=g) / K ** 0.25).to(torch.bfloat16)
    ref = np64(A) @ np64(B).T
    cuts = [0, 8 * (N // 24), 8 * (N // 12) + 8, N]
    outs, bufs = [], []
    for i in range(3):
        w = cuts[i + 1] - cuts[i]
        buf = torch.full((M, w + 8 * i), float('nan'), dtype=torch.bfloat16, device='cuda')
        bufs.append(buf)
        outs.append((buf, cuts[i], cuts[i + 1]))
    kda.kda_proj_gemm(A.cuda(), B.cuda(), outs)
    torch.cuda.synchronize()
    for i, buf in enumerate(bufs):
        w = cuts[i + 1] - cuts[i]
        got = np64(buf)
        assert rel_err(got[:, :w], ref[:, cuts[i]:cuts[i + 1]]) <= GEMM_TOL, i
        assert np.isnan(got[:, w:]).all(), i      # padding past the range untouched


def test_proj_gemm_status_and_rejections():
    st = torch.zeros(4, dtype=torch.int32, device='cuda')
    A = torch.randn(64, 64, device='cuda').to(torch.bfloat16)
    B = torch.randn(256, 64, device='cuda').to(torch.bfloat16)
    out = torch.empty(64, 256, dtype=torch.bfloat16, device='cuda')
    kda.kda_proj_gemm(A, B, [(out, 0, 256)], status=st)
    assert kda.kda_workspace_status(st) == kda.KDA_OK
    assert rel_err(np64(out), np64(A) @ np64(B).T) <= GEMM_TOL
    with pytest.raises(kda.KdaError):                 # overlapping ranges
        kda.kda_proj_gemm(A, B, [(out, 0, 136), (out, 128, 256)])
    with pytest.raises(kda.KdaError):                 # range end not a multiple of 8
        kda.kda_proj_gemm(A, B, [(out, 0, 250)])


@pytest.mark.parametrize('T,H,d,hidden,r', [(200, 8, 64, 384, 64), (131, 8, 128, 512, 128)])
def test_layer_from_hidden_states(T, H, d, hidden, r):
    """The full layer from hidden states: fused input projection -> low-rank gate -> KDA
    layer (prep, chunked recurrence, gated RMSNorm).  The projections are checked against
    the oracle's float64 products; the layer's output against the oracle layer run on
    those products rounded to the bf16 activations the layer takes (the boundary dtype)."""
    cfg = kda.Config(num_heads=H, head_dim=d, conv_size=4, dtype=torch.bfloat16, chunk_size=64)
    W = synth.proj_weights(51, hidden, H, d, r)
    P = synth.layer_params(51, H, d, 4)
    hs = synth.hidden_states(51, T, hidden)
    p = kda.layer_projections(cfg, hs.cuda(), W['W_in'].cuda(), W['W_gb'].cuda(), r)
    cu = torch.tensor([0, T], dtype=torch.int32)
    Pd = {k: v.cuda() for k, v in P.items()}
    state = torch.empty(1, H, d, d, device='cuda')
    y = kda.kda_layer_prefill(cfg, cu.cuda(), p['x'], p['f'], p['beta_logit'], p['g'],
                              Pd['conv_w'], Pd['A_log'], Pd['dt_bias'], Pd['norm_w'],
                              state_out=state)
    torch.cuda.synchronize()
    ref_p = ko.projections(np64(hs), np64(W['W_in']), np64(W['W_gb']), H, d, r)
    for name in ('x', 'f', 'beta_logit', 'g_a'):
        assert rel_err(np64(p[name]), ref_p[name]) <= GEMM_TOL, name
    # g is a product of the bf16-rounded g_a (the GEMM's own output) with W_gb
    g_ref = (np64(p['g_a']) @ np64(W['W_gb']).T).reshape(T, H, d)
    assert rel_err(np64(p['g']), g_ref) <= GEMM_TOL
    acts = {k: _bf16_rounded(ref_p[k]) for k in ('x', 'f', 'beta_logit', 'g')}
    ref = ko.layer(x=acts['x'], f=acts['f'], beta_logit=acts['beta_logit'],
                   g=_bf16_rounded(g_ref), conv_w=np64(P['conv_w']), A_log=np64(P['A_log']),
                   dt_bias=np64(P['dt_bias']), norm_w=np64(P['norm_w']), cu_seqlens=[0, T])
    assert rel_err(np64(y), ref['y']) <= 1e-2
    assert rel_err(np64(state), ref['state']) <= 1e-2
