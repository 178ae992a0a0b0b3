"""CPU tests of the C ABI: the library loads, exports every declared symbol, and
rejects invalid arguments on the host before anything is launched.

Every call here fails validation, so no CUDA work is ever enqueued (the fake
device pointers are never dereferenced).
"""
import ctypes
import os
import random
import re

import pytest
import torch

from linear_attention_recurrence_09_b200 import build as kbuild
from linear_attention_recurrence_09_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope='module')
def L():
    kbuild.build()
    return kda.lib()


def _declared():
    src = open(os.path.join(ROOT, 'include', 'kda.h')).read()
    return sorted(set(re.findall(r'KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(', src)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert set(names) == set(kda.ENTRY_POINTS)
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings(L):
    assert kda.kda_abi_version() == kda.ABI_VERSION == 2
    for code in range(8):
        assert kda.kda_status_string(code).startswith('KDA_')
    assert 'unknown' in kda.kda_status_string(99)


def _cfg(**kw):
    base = dict(num_heads=2, head_dim=16, conv_size=4, dtype=torch.float32, chunk_size=16)
    base.update(kw)
    return kda.Config(**base).c()


A = 0x10000      # fake 16-byte aligned device addresses (never dereferenced)
MIS = 0x10004    # fake misaligned address


def _prep(L, cfg, **over):
    args = dict(n=1, T=4, cu=A, maxlen=0, x=A, f=A, bl=A, cw=A, al=A, dtb=A, cs=None, slots=None,
                pool=1, mode=0, win=None, q=A, k=A, v=A, la=A, b=A)
    args.update(over)
    return L.kda_prep(ctypes.byref(cfg) if cfg is not None else None, args['n'], args['T'],
                      args['cu'], args['maxlen'], args['x'], args['f'], args['bl'], args['cw'],
                      args['al'], args['dtb'], args['cs'], args['slots'], args['pool'],
                      args['mode'], args['win'], args['q'], args['k'], args['v'], args['la'],
                      args['b'], None)


def test_prep_rejects_bad_arguments(L):
    assert _prep(L, None) == kda.KDA_ERR_INVALID_ARG
    assert _prep(L, _cfg(head_dim=48)) == kda.KDA_ERR_UNSUPPORTED
    assert _prep(L, _cfg(chunk_size=128)) == kda.KDA_ERR_UNSUPPORTED
    assert _prep(L, _cfg(gate_lower_bound=-6.0)) == kda.KDA_ERR_UNSUPPORTED
    assert _prep(L, _cfg(gate_lower_bound=0.0)) == kda.KDA_ERR_UNSUPPORTED
    # the softplus gate ignores the lower bound: validation goes on to the pointers
    sp = _cfg(gate_lower_bound=None)
    assert sp.gate_kind == kda.KDA_GATE_SOFTPLUS
    assert _prep(L, sp, cu=None) == kda.KDA_ERR_INVALID_ARG
    sp.gate_lower_bound = -6.0
    assert _prep(L, sp, cu=MIS) == kda.KDA_ERR_MISALIGNED
    bad = _cfg()
    bad.gate_kind = 2
    assert _prep(L, bad) == kda.KDA_ERR_INVALID_ARG
    bad = _cfg()
    bad.launch_flags = 4                              # bits 0 and 1 are the defined flags
    assert _prep(L, bad) == kda.KDA_ERR_INVALID_ARG
    ok = _cfg()
    ok.launch_flags = kda.KDA_LAUNCH_EARLY_STATE
    assert _prep(L, ok, cu=None) == kda.KDA_ERR_INVALID_ARG   # accepted: on to the pointers
    assert _prep(L, _cfg(conv_size=9)) == kda.KDA_ERR_INVALID_ARG
    assert _prep(L, _cfg(num_heads=0)) == kda.KDA_ERR_INVALID_ARG
    assert _prep(L, _cfg(l2_eps=0.0)) == kda.KDA_ERR_INVALID_ARG
    assert _prep(L, _cfg(), n=-1) == kda.KDA_ERR_INVALID_ARG
    assert _prep(L, _cfg(), mode=2) == kda.KDA_ERR_INVALID_ARG
    assert _prep(L, _cfg(), cu=None) == kda.KDA_ERR_INVALID_ARG
    assert _prep(L, _cfg(), cu=MIS) == kda.KDA_ERR_MISALIGNED
    assert _prep(L, _cfg(), x=MIS) == kda.KDA_ERR_MISALIGNED
    assert _prep(L, _cfg(), x=None) == kda.KDA_ERR_INVALID_ARG
    assert _prep(L, _cfg(), mode=1, win=None) == kda.KDA_ERR_INVALID_ARG
    assert _prep(L, _cfg(), cs=A, pool=0) == kda.KDA_ERR_INVALID_ARG
    assert _prep(L, _cfg(), n=0) == kda.KDA_OK      # nothing to do, nothing launched


def test_prefill_rejects_bad_workspace(L):
    cfg = _cfg()
    need = L.kda_prefill_workspace_size(ctypes.byref(cfg), 1, 64)
    assert need > 0

    def call(ws, nbytes, **kw):
        a = dict(q=A, y=A, cu=A)
        a.update(kw)
        return L.kda_prefill(ctypes.byref(cfg), 1, 64, a['cu'], a['q'], A, A, A, A, A, A,
                             None, None, None, 1, a['y'], ws, nbytes, None)

    assert call(None, need) == kda.KDA_ERR_WORKSPACE
    assert call(A, need - 1) == kda.KDA_ERR_WORKSPACE
    assert call(A + 16, need) == kda.KDA_ERR_WORKSPACE     # not 256-byte aligned
    assert call(A, need, q=MIS) == kda.KDA_ERR_MISALIGNED
    assert call(A, need, y=None) == kda.KDA_ERR_INVALID_ARG
    assert call(A, need, cu=None) == kda.KDA_ERR_INVALID_ARG


def test_layer_prefill_validates_and_sizes_workspace(L):
    fused = _cfg(head_dim=128, chunk_size=64, dtype=torch.bfloat16, num_heads=4)
    plain = _cfg(head_dim=64, chunk_size=64, dtype=torch.bfloat16, num_heads=4)
    for cfg in (fused, plain):
        c = ctypes.byref(cfg)
        base = L.kda_prefill_workspace_size(c, 1, 100)
        lay = L.kda_layer_prefill_workspace_size(c, 1, 100)
        # the fallback adds fp32 q, k, v, log a (4 x T H d) and beta (T H) for the separate prep
        extra = 0 if cfg is fused else 100 * 4 * (4 * 64 * 4 + 4)
        assert lay >= base + extra and lay - base - extra < 256
    cfg = fused
    need = L.kda_layer_prefill_workspace_size(ctypes.byref(cfg), 1, 64)

    def call(ws, nbytes, **kw):
        a = dict(x=A, y=A, cu=A, cw=A)
        a.update(kw)
        return L.kda_layer_prefill(ctypes.byref(cfg), 1, 64, a['cu'], 64, a['x'], A, A, A,
                                   a['cw'], A, A, A, None, None, None, None, 1, a['y'], ws,
                                   nbytes, None)

    assert call(None, need) == kda.KDA_ERR_WORKSPACE
    assert call(A, need - 1) == kda.KDA_ERR_WORKSPACE
    assert call(A + 16, need) == kda.KDA_ERR_WORKSPACE
    assert call(A, need, x=MIS) == kda.KDA_ERR_MISALIGNED
    assert call(A, need, y=None) == kda.KDA_ERR_INVALID_ARG
    assert call(A, need, cw=None) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_layer_prefill(ctypes.byref(cfg), 0, 0, None, 0, None, None, None, None, None,
                               None, None, None, None, None, None, None, 0, None, None, 0,
                               None) == kda.KDA_OK      # nothing to do, nothing launched


def test_step_entry_points_reject_bad_arguments(L):
    cfg = _cfg()
    c = ctypes.byref(cfg)
    assert L.kda_decode(c, 0, None, None, None, None, None, None, None, None, None, 0, None,
                        None) == kda.KDA_OK
    assert L.kda_decode(c, 2, A, A, A, A, A, A, A, A, None, 1, A, None) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_decode(c, 2, A, A, MIS, A, A, A, A, A, None, 2, A, None) == kda.KDA_ERR_MISALIGNED
    assert L.kda_verify(c, 2, 17, A, A, A, A, A, A, A, A, None, 2, A, A, None) == \
        kda.KDA_ERR_INVALID_ARG
    assert L.kda_verify(c, 2, 8, A, A, A, A, A, A, A, A, None, 2, None, A, None) == \
        kda.KDA_ERR_INVALID_ARG
    assert L.kda_rollback(c, 2, 0, A, A, None, A, None, None, 2, None) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_rollback(c, 2, 8, A, A, A, A, None, None, 2, None) == kda.KDA_ERR_INVALID_ARG
    assert L.kda_workspace_status(None, None) == kda.KDA_ERR_INVALID_ARG
    # compact tape: the tape_kua pointer is required, the block length bounded
    assert L.kda_verify_compact(c, 2, 8, A, A, A, A, A, A, A, A, None, 2, None, A, None) == \
        kda.KDA_ERR_INVALID_ARG
    assert L.kda_verify_compact(c, 2, 8, A, A, A, A, A, A, A, A, None, 2, MIS, A, None) == \
        kda.KDA_ERR_MISALIGNED
    assert L.kda_verify_compact(c, 2, 0, A, A, A, A, A, A, A, A, None, 2, A, A, None) == \
        kda.KDA_ERR_INVALID_ARG
    assert L.kda_rollback_replay(c, 2, 17, A, A, None, A, None, None, 2, None) == \
        kda.KDA_ERR_INVALID_ARG
    assert L.kda_rollback_replay(c, 2, 8, A, None, None, A, None, None, 2, None) == \
        kda.KDA_ERR_INVALID_ARG
    assert L.kda_rollback_replay(c, 2, 8, A, A, A, A, None, None, 2, None) == \
        kda.KDA_ERR_INVALID_ARG
    assert L.kda_rollback_replay(c, 0, 8, None, None, None, None, None, None, 0, None) == kda.KDA_OK
    lv = [c, 2, 8, A, A, A, A, A, A, A, A, None, A, None, 2, None, A, A, None]
    assert L.kda_layer_verify_compact(*lv) == kda.KDA_ERR_INVALID_ARG      # tape_kua NULL


def test_workspace_size_grows_with_tokens(L):
    cfg = _cfg(head_dim=128, chunk_size=64, dtype=torch.bfloat16, num_heads=32)
    c = ctypes.byref(cfg)
    s1 = L.kda_prefill_workspace_size(c, 1, 8192)
    s2 = L.kda_prefill_workspace_size(c, 1, 16384)
    per_tok_min = 32 * 128 * (4 * 2 + 4)     # W, U~, Q~, K' in bf16 and o in fp32
    assert s1 >= 8192 * per_tok_min
    assert s2 - s1 >= 8192 * per_tok_min
    assert L.kda_prefill_workspace_size(None, 1, 8) == 0
    assert L.kda_prefill_workspace_size(c, -1, 8) == 0


def test_binding_rejects_host_tensors():
    cfg = kda.Config(num_heads=2, head_dim=16, dtype=torch.float32, chunk_size=16)
    x = torch.zeros(4, 2, 48)
    with pytest.raises(ValueError):
        kda._ptr(x, torch.float32, 'x')
    del cfg


@pytest.mark.parametrize('tile', [16, 64])
def test_slot_map_never_collides(tile):
    """slot(s, c) = floor(cu[s]/tile) + s + c is injective and below total/tile + N + 1."""
    rnd = random.Random(tile)
    for _ in range(200):
        n = rnd.randint(1, 9)
        lens = [rnd.choice([0, 1, tile - 1, tile, tile + 1, rnd.randint(0, 5 * tile)])
                for _ in range(n)]
        cu = [0]
        for ln in lens:
            cu.append(cu[-1] + ln)
        total = cu[-1]
        seen = set()
        for s in range(n):
            for c in range((lens[s] + tile - 1) // tile):
                slot = cu[s] // tile + s + c
                assert slot not in seen
                assert slot < total // tile + n + 1
                seen.add(slot)
