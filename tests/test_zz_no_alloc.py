"""kda_prefill_noalloc against kda_prefill, through the C ABI.

kda_prefill_noalloc serves callers that cannot allocate device memory (a host
framework that owns all of HBM, or a path that must not pay cudaMalloc's
latency and synchronisation): it keeps its scratch in a fixed 64 MiB device
array inside the library instead of a caller-provided workspace.  This file is
collected last so that a run stopping at the first failure has already run
every other test; it passes alone in a fresh process (whose first call does
the per-device set-up) and after the other tests.
"""
import pytest
import torch

from linear_attention_recurrence_09_b200 import kda, synth

pytestmark = pytest.mark.gpu


def _prep(cfg, P, A):
    return kda.kda_prep(cfg, A['cu_seqlens'], A['x'], A['f'], A['beta_logit'], P['conv_w'],
                        P['A_log'], P['dt_bias'])


@pytest.mark.parametrize('dtype,d,chunk', [(torch.bfloat16, 128, 64), (torch.float32, 64, 32)])
def test_noalloc_matches_prefill_on_two_calls_in_a_row(dtype, d, chunk):
    H, K = 4, 4
    lens = [150, 77]
    cfg = kda.Config(num_heads=H, head_dim=d, conv_size=K, dtype=dtype, chunk_size=chunk)
    N, T = len(lens), sum(lens)
    assert kda.kda_prefill_workspace_size(cfg, N, T) <= kda.NOALLOC_SCRATCH_BYTES
    P = {k: v.cuda() for k, v in synth.layer_params(21, H, d, K).items()}
    S0 = synth.initial_state(21, N, H, d, 0.01).cuda()
    s_ref, s_na = S0.clone(), S0.clone()
    for call in range(2):
        A = {k: v.cuda() for k, v in
             synth.layer_activations(21, lens, H, d, dtype, tag=('call', call)).items()}
        p = _prep(cfg, P, A)
        y_ref = torch.empty(T, H, d, dtype=dtype, device='cuda')
        y_na = torch.full((T, H, d), float('nan'), dtype=dtype, device='cuda')
        kda.kda_prefill(cfg, A['cu_seqlens'], p['q'], p['k'], p['v'], p['log_a'], p['beta'],
                        A['g'], P['norm_w'], state_in=s_ref, state_out=s_ref, y=y_ref)
        kda.kda_prefill_noalloc(cfg, A['cu_seqlens'], p['q'], p['k'], p['v'], p['log_a'],
                                p['beta'], A['g'], P['norm_w'], state_in=s_na, state_out=s_na,
                                y=y_na)
        torch.cuda.synchronize()
        # the same deterministic kernels on the same inputs: any byte of stale scratch
        # that leaked into the result would show as a difference
        assert torch.equal(y_na, y_ref), call
        assert torch.equal(s_na, s_ref), call
        assert not torch.isnan(y_na.float()).any()


def test_noalloc_rejects_problems_beyond_its_scratch():
    cfg = kda.Config(num_heads=32, head_dim=128, conv_size=4, dtype=torch.bfloat16, chunk_size=64)
    T = 8192
    assert kda.kda_prefill_workspace_size(cfg, 1, T) > kda.NOALLOC_SCRATCH_BYTES
    f32 = lambda *s: torch.empty(*s, device='cuda')
    cu = torch.tensor([0, T], dtype=torch.int32, device='cuda')
    with pytest.raises(kda.KdaError) as e:
        kda.kda_prefill_noalloc(cfg, cu, f32(T, 32, 128), f32(T, 32, 128), f32(T, 32, 128),
                                f32(T, 32, 128), f32(T, 32),
                                torch.empty(T, 32, 128, dtype=torch.bfloat16, device='cuda'),
                                f32(128))
    assert e.value.status == kda.KDA_ERR_SCRATCH_LIMIT
