"""Helpers shared by the GPU parity tests: run the CUDA path through the binding
and the float64 oracle on the same seeded inputs, and compare.

The oracle receives the activations exactly as the GPU does (bf16-rounded
values upcast to float64), so a difference measures kernel error, not input
quantisation.  The error metric is max|GPU - oracle| / max|oracle| per tensor.
"""
import numpy as np
import torch

from linear_attention_recurrence_09_b200 import kda, synth
from oracle import kda_oracle as ko

TOL = {torch.float32: 1e-4, torch.bfloat16: 1e-2}


def np64(t):
    return t.detach().to('cpu').to(torch.float64).numpy()


def rel_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max() if ref.size else 0.0
    if scale == 0.0:
        return float(np.abs(got).max()) if got.size else 0.0
    return float(np.abs(got - ref).max() / scale)


def make_case(seed, seqlens, H, d, K=4, dtype=torch.bfloat16, state_var=0.0, conv_hist=False,
              chunk=64):
    cfg = kda.Config(num_heads=H, head_dim=d, conv_size=K, dtype=dtype, chunk_size=chunk)
    params = synth.layer_params(seed, H, d, K)
    acts = synth.layer_activations(seed, seqlens, H, d, dtype)
    N = len(seqlens)
    S0 = synth.initial_state(seed, N, H, d, state_var) if state_var > 0 else None
    hist = synth.conv_history(seed, N, H, d, K, dtype) if conv_hist else None
    return cfg, params, acts, S0, hist


def gpu_layer(cfg, params, acts, S0=None, hist=None, dev='cuda', fused=True):
    """The layer on the GPU: kda_layer_prefill (fused=True) or kda_prep + kda_prefill.
    Returns y, final states, conv history, prep outputs (None when fused)."""
    N = acts['cu_seqlens'].numel() - 1
    H, d, K = cfg.num_heads, cfg.head_dim, cfg.conv_size
    P = {k: v.to(dev) for k, v in params.items()}
    Ad = {k: v.to(dev) for k, v in acts.items()}
    s_in = S0.to(dev) if S0 is not None else None
    s_out = torch.empty(N, H, d, d, device=dev)
    cs = (hist.clone() if hist is not None else
          torch.zeros(N, K - 1, H, 3 * d, dtype=cfg.dtype)).to(dev)
    if fused:
        y = kda.layer_prefill(cfg, P, Ad, state_in=s_in, state_out=s_out, conv_state=cs)
        p = None
    else:
        y, p = kda.prep_then_prefill(cfg, P, Ad, state_in=s_in, state_out=s_out, conv_state=cs)
    torch.cuda.synchronize()
    return y, s_out, cs, p


def oracle_layer(cfg, params, acts, S0=None, hist=None, heads=None):
    return ko.layer(
        x=np64(acts['x']), f=np64(acts['f']), beta_logit=np64(acts['beta_logit']),
        g=np64(acts['g']), conv_w=np64(params['conv_w']), A_log=np64(params['A_log']),
        dt_bias=np64(params['dt_bias']), norm_w=np64(params['norm_w']),
        cu_seqlens=acts['cu_seqlens'].numpy(),
        S0=None if S0 is None else np64(S0), conv_hist=None if hist is None else np64(hist),
        lb=cfg.gate_lower_bound, l2_eps=cfg.l2_eps, norm_eps=cfg.norm_eps,
        q_scale=cfg.q_scale, heads=heads)


def compare_layer(cfg, params, acts, S0=None, hist=None, heads=None, fused=True):
    """Run both sides; return dict of relative errors (y, state, conv history)."""
    y, s_out, cs, _ = gpu_layer(cfg, params, acts, S0, hist, fused=fused)
    ref = oracle_layer(cfg, params, acts, S0, hist, heads)
    hs = slice(None) if heads is None else list(heads)
    errs = {
        'y': rel_err(np64(y)[:, hs], ref['y']),
        'state': rel_err(np64(s_out)[:, hs], ref['state']),
        'conv_hist': rel_err(np64(cs)[:, :, hs], ref['conv_hist']),
    }
    return errs
