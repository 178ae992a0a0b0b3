"""Thin ctypes binding over libkda.so (C ABI in include/kda.h).

Argument marshalling only: every step of the layer runs in the CUDA library.
Tensors must be contiguous CUDA tensors of the documented dtype; outputs left
as ``None`` are allocated here with torch (PyTorch supplies device memory and
the current stream, nothing else).  A missing library raises at first use:
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, 'libkda.so')

KDA_OK = 0
KDA_ERR_INVALID_ARG = 1
KDA_ERR_MISALIGNED = 2
KDA_ERR_UNSUPPORTED = 3
KDA_ERR_CUDA = 4
KDA_ERR_TIMEOUT = 5
KDA_ERR_WORKSPACE = 6
KDA_ERR_SCRATCH_LIMIT = 7
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024
KDA_F32 = 0
KDA_BF16 = 1
KDA_CONV_COMMIT = 0
KDA_CONV_TAPE = 1
KDA_GATE_BOUNDED_SIGMOID = 0
KDA_GATE_SOFTPLUS = 1
KDA_LAUNCH_EARLY_STATE = 1
KDA_LAUNCH_SEPARATE_PASSES = 2
ABI_VERSION = 2

ENTRY_POINTS = ('kda_status_string', 'kda_abi_version', 'kda_prep',
                'kda_prefill_workspace_size', 'kda_prefill', 'kda_decode', 'kda_verify',
                'kda_rollback', 'kda_workspace_status', 'kda_selftest_wait_timeout',
                'kda_prefill_noalloc', 'kda_layer_prefill_workspace_size', 'kda_layer_prefill',
                'kda_set_phase_events', 'kda_launch_count', 'kda_last_cuda_error',
                'kda_layer_decode', 'kda_layer_verify', 'kda_verify_compact',
                'kda_layer_verify_compact', 'kda_rollback_replay', 'kda_proj_gemm')


class KdaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = f'{where}: {kda_status_string(status)} ({status})'
        if status == KDA_ERR_CUDA:
            msg += ': ' + lib().kda_last_cuda_error().decode()
        super().__init__(msg)


class CConfig(ctypes.Structure):
    _fields_ = [('num_heads', ctypes.c_int32), ('head_dim', ctypes.c_int32),
                ('conv_size', ctypes.c_int32), ('dtype', ctypes.c_int32),
                ('chunk_size', ctypes.c_int32), ('gate_lower_bound', ctypes.c_float),
                ('l2_eps', ctypes.c_float), ('norm_eps', ctypes.c_float),
                ('q_scale', ctypes.c_float), ('gate_kind', ctypes.c_int32),
                ('launch_flags', ctypes.c_int32)]


@dataclass
class Config:
    """Layer configuration; mirrors ``kda_config``.  ``gate_lower_bound=None`` selects
    the softplus decay gate (KDA_GATE_SOFTPLUS), as an absent lower bound does.
    ``launch_flags``: KDA_LAUNCH_EARLY_STATE lets the token-step calls and the replay
    rollback stream the recurrent state before the kernel ahead of them on the stream
    has finished; set it only when that kernel writes neither the state nor the slots
    (kda_prep, or kda_verify_compact before kda_rollback_replay).
    KDA_LAUNCH_SEPARATE_PASSES keeps the tensor-core prefill's two passes in separate
    launches where one co-scheduled launch would otherwise carry both."""
    num_heads: int
    head_dim: int
    conv_size: int = 4
    dtype: torch.dtype = torch.bfloat16
    chunk_size: int = 64
    gate_lower_bound: Optional[float] = -5.0
    l2_eps: float = 1e-6
    norm_eps: float = 1e-5
    q_scale: float = 1.0
    launch_flags: int = 0

    def c(self) -> CConfig:
        if self.dtype not in (torch.float32, torch.bfloat16):
            raise ValueError('activation dtype must be float32 or bfloat16')
        softplus = self.gate_lower_bound is None
        return CConfig(self.num_heads, self.head_dim, self.conv_size,
                       KDA_BF16 if self.dtype == torch.bfloat16 else KDA_F32,
                       self.chunk_size, 0.0 if softplus else self.gate_lower_bound,
                       self.l2_eps, self.norm_eps, self.q_scale,
                       KDA_GATE_SOFTPLUS if softplus else KDA_GATE_BOUNDED_SIGMOID,
                       self.launch_flags)


class CProjOut(ctypes.Structure):
    _fields_ = [('out', ctypes.c_void_p), ('ld', ctypes.c_int64), ('col_begin', ctypes.c_int32),
                ('col_end', ctypes.c_int32)]


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32


def lib() -> ctypes.CDLL:
    """Load libkda.so from this package directory (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f'{LIB_PATH} is missing: build it with '
                               '`python -m linear_attention_recurrence_09_b200.build`')
        L = ctypes.CDLL(LIB_PATH)
        L.kda_status_string.restype = ctypes.c_char_p
        L.kda_status_string.argtypes = [ctypes.c_int]
        L.kda_abi_version.restype = ctypes.c_int
        L.kda_abi_version.argtypes = []
        L.kda_prep.restype = ctypes.c_int
        L.kda_prep.argtypes = [ctypes.POINTER(CConfig), _I, _I, _P, _I, _P, _P, _P, _P, _P, _P,
                               _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _P]
        L.kda_prefill_workspace_size.restype = ctypes.c_size_t
        L.kda_prefill_workspace_size.argtypes = [ctypes.POINTER(CConfig), _I, _I]
        L.kda_prefill.restype = ctypes.c_int
        L.kda_prefill.argtypes = [ctypes.POINTER(CConfig), _I, _I, _P, _P, _P, _P, _P, _P, _P,
                                  _P, _P, _P, _P, _I, _P, _P, ctypes.c_size_t, _P]
        L.kda_decode.restype = ctypes.c_int
        L.kda_decode.argtypes = [ctypes.POINTER(CConfig), _I, _P, _P, _P, _P, _P, _P, _P, _P,
                                 _P, _I, _P, _P]
        L.kda_verify.restype = ctypes.c_int
        L.kda_verify.argtypes = [ctypes.POINTER(CConfig), _I, _I, _P, _P, _P, _P, _P, _P, _P,
                                 _P, _P, _I, _P, _P, _P]
        L.kda_rollback.restype = ctypes.c_int
        L.kda_rollback.argtypes = [ctypes.POINTER(CConfig), _I, _I, _P, _P, _P, _P, _P, _P,
                                   _I, _P]
        L.kda_workspace_status.restype = ctypes.c_int
        L.kda_workspace_status.argtypes = [_P, _P]
        L.kda_selftest_wait_timeout.restype = ctypes.c_int
        L.kda_selftest_wait_timeout.argtypes = [_P, _P]
        L.kda_layer_prefill_workspace_size.restype = ctypes.c_size_t
        L.kda_layer_prefill_workspace_size.argtypes = [ctypes.POINTER(CConfig), _I, _I]
        L.kda_layer_prefill.restype = ctypes.c_int
        L.kda_layer_prefill.argtypes = [ctypes.POINTER(CConfig), _I, _I, _P, _I, _P, _P, _P, _P,
                                        _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P,
                                        ctypes.c_size_t, _P]
        L.kda_layer_decode.restype = ctypes.c_int
        L.kda_layer_decode.argtypes = [ctypes.POINTER(CConfig), _I, _P, _P, _P, _P, _P, _P, _P,
                                       _P, _P, _P, _P, _I, _P, _P]
        L.kda_layer_verify.restype = ctypes.c_int
        L.kda_layer_verify.argtypes = [ctypes.POINTER(CConfig), _I, _I, _P, _P, _P, _P, _P, _P,
                                       _P, _P, _P, _P, _P, _I, _P, _P, _P, _P]
        L.kda_verify_compact.restype = ctypes.c_int
        L.kda_verify_compact.argtypes = L.kda_verify.argtypes
        L.kda_layer_verify_compact.restype = ctypes.c_int
        L.kda_layer_verify_compact.argtypes = L.kda_layer_verify.argtypes
        L.kda_rollback_replay.restype = ctypes.c_int
        L.kda_rollback_replay.argtypes = L.kda_rollback.argtypes
        L.kda_proj_gemm.restype = ctypes.c_int
        L.kda_proj_gemm.argtypes = [_I, _I, _I, _P, _P, ctypes.POINTER(CProjOut), _I, _P, _P]
        L.kda_last_cuda_error.restype = ctypes.c_char_p
        L.kda_last_cuda_error.argtypes = []
        L.kda_launch_count.restype = ctypes.c_longlong
        L.kda_launch_count.argtypes = []
        L.kda_set_phase_events.restype = ctypes.c_int
        L.kda_set_phase_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), _I]
        L.kda_prefill_noalloc.restype = ctypes.c_int
        L.kda_prefill_noalloc.argtypes = [ctypes.POINTER(CConfig), _I, _I, _P, _P, _P, _P, _P,
                                          _P, _P, _P, _P, _P, _P, _I, _P, _P]
        _lib = L
    return _lib


def kda_status_string(status: int) -> str:
    return lib().kda_status_string(int(status)).decode()


def kda_abi_version() -> int:
    return lib().kda_abi_version()


def _check(status, where):
    if status != KDA_OK:
        raise KdaError(status, where)


def _ptr(t, dtype=None, name='tensor', shape=None):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f'{name} must be a CUDA tensor')
    if not t.is_contiguous():
        raise ValueError(f'{name} must be contiguous')
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f'{name} must be {dtype}, got {t.dtype}')
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f'{name} must have shape {tuple(shape)}, got {tuple(t.shape)}')
    return t.data_ptr() if t.numel() > 0 else None


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def kda_prep(cfg: Config, cu_seqlens, x, f, beta_logit, conv_w, A_log, dt_bias,
             conv_state=None, state_slots=None, pool_size=None, conv_mode=KDA_CONV_COMMIT,
             conv_window=None, max_seqlen=0, out=None, stream=None):
    """Conv + SiLU + L2 + decay gate + beta.  Returns dict q, k, v, log_a, beta (+ window)."""
    H, d, K = cfg.num_heads, cfg.head_dim, cfg.conv_size
    T = x.shape[0]
    N = cu_seqlens.numel() - 1
    dev = x.device
    o = dict(out or {})
    for name in ('q', 'k', 'v'):
        if o.get(name) is None:
            o[name] = _empty((T, H, d), torch.float32, dev)
    if o.get('log_a') is None:
        o['log_a'] = _empty((T, H, d), torch.float32, dev)
    if o.get('beta') is None:
        o['beta'] = _empty((T, H), torch.float32, dev)
    if conv_mode == KDA_CONV_TAPE and conv_window is None:
        conv_window = _empty((T + N * (K - 1), H, 3 * d), cfg.dtype, dev)
    if pool_size is None:
        pool_size = conv_state.shape[0] if conv_state is not None else N
    c = cfg.c()
    st = lib().kda_prep(
        ctypes.byref(c), N, T, _ptr(cu_seqlens, torch.int32, 'cu_seqlens'), int(max_seqlen),
        _ptr(x, cfg.dtype, 'x', (T, H, 3 * d)), _ptr(f, cfg.dtype, 'f', (T, H, d)),
        _ptr(beta_logit, cfg.dtype, 'beta_logit', (T, H)),
        _ptr(conv_w, torch.float32, 'conv_w', (H, 3 * d, K)),
        _ptr(A_log, torch.float32, 'A_log', (H,)),
        _ptr(dt_bias, torch.float32, 'dt_bias', (H, d)),
        _ptr(conv_state, cfg.dtype, 'conv_state'), _ptr(state_slots, torch.int32, 'state_slots'),
        int(pool_size), int(conv_mode), _ptr(conv_window, cfg.dtype, 'conv_window'),
        _ptr(o['q'], torch.float32, 'q'), _ptr(o['k'], torch.float32, 'k'),
        _ptr(o['v'], torch.float32, 'v'),
        _ptr(o['log_a'], torch.float32, 'log_a'), _ptr(o['beta'], torch.float32, 'beta'),
        _stream(stream))
    _check(st, 'kda_prep')
    if conv_mode == KDA_CONV_TAPE:
        o['window'] = conv_window
    return o


def kda_prefill_workspace_size(cfg: Config, n_seqs: int, total_tokens: int) -> int:
    c = cfg.c()
    return int(lib().kda_prefill_workspace_size(ctypes.byref(c), int(n_seqs), int(total_tokens)))


def prefill_workspace(cfg: Config, n_seqs: int, total_tokens: int, device='cuda'):
    """A uint8 device buffer of kda_prefill_workspace_size bytes (256-aligned by torch)."""
    return torch.empty(kda_prefill_workspace_size(cfg, n_seqs, total_tokens), dtype=torch.uint8,
                       device=device)


def kda_prefill(cfg: Config, cu_seqlens, q, k, v, log_a, beta, g, norm_w, state_in=None,
                state_out=None, state_slots=None, pool_size=None, y=None, workspace=None,
                stream=None):
    """Chunked prefill.  Returns y; the final states go to ``state_out``."""
    H, d = cfg.num_heads, cfg.head_dim
    T = q.shape[0]
    N = cu_seqlens.numel() - 1
    if y is None:
        y = _empty((T, H, d), cfg.dtype, q.device)
    if workspace is None:
        workspace = prefill_workspace(cfg, N, T, q.device)
    if pool_size is None:
        ref = state_in if state_in is not None else state_out
        pool_size = ref.shape[0] if ref is not None else N
    c = cfg.c()
    st = lib().kda_prefill(
        ctypes.byref(c), N, T, _ptr(cu_seqlens, torch.int32, 'cu_seqlens'),
        _ptr(q, torch.float32, 'q', (T, H, d)), _ptr(k, torch.float32, 'k', (T, H, d)),
        _ptr(v, torch.float32, 'v', (T, H, d)), _ptr(log_a, torch.float32, 'log_a', (T, H, d)),
        _ptr(beta, torch.float32, 'beta', (T, H)), _ptr(g, cfg.dtype, 'g', (T, H, d)),
        _ptr(norm_w, torch.float32, 'norm_w', (d,)),
        _ptr(state_in, torch.float32, 'state_in'), _ptr(state_out, torch.float32, 'state_out'),
        _ptr(state_slots, torch.int32, 'state_slots'), int(pool_size),
        _ptr(y, cfg.dtype, 'y', (T, H, d)), _ptr(workspace, None, 'workspace'),
        int(workspace.numel() * workspace.element_size()), _stream(stream))
    _check(st, 'kda_prefill')
    return y


def kda_prefill_noalloc(cfg: Config, cu_seqlens, q, k, v, log_a, beta, g, norm_w,
                        state_in=None, state_out=None, state_slots=None, pool_size=None, y=None,
                        stream=None):
    """kda_prefill with the library's fixed device scratch (the entry point itself
    allocates nothing; pass ``y`` to avoid the one torch allocation made here)."""
    H, d = cfg.num_heads, cfg.head_dim
    T = q.shape[0]
    N = cu_seqlens.numel() - 1
    if y is None:
        y = _empty((T, H, d), cfg.dtype, q.device)
    if pool_size is None:
        ref = state_in if state_in is not None else state_out
        pool_size = ref.shape[0] if ref is not None else N
    c = cfg.c()
    st = lib().kda_prefill_noalloc(
        ctypes.byref(c), N, T, _ptr(cu_seqlens, torch.int32, 'cu_seqlens'),
        _ptr(q, torch.float32, 'q', (T, H, d)), _ptr(k, torch.float32, 'k', (T, H, d)),
        _ptr(v, torch.float32, 'v', (T, H, d)), _ptr(log_a, torch.float32, 'log_a', (T, H, d)),
        _ptr(beta, torch.float32, 'beta', (T, H)), _ptr(g, cfg.dtype, 'g', (T, H, d)),
        _ptr(norm_w, torch.float32, 'norm_w', (d,)),
        _ptr(state_in, torch.float32, 'state_in'), _ptr(state_out, torch.float32, 'state_out'),
        _ptr(state_slots, torch.int32, 'state_slots'), int(pool_size),
        _ptr(y, cfg.dtype, 'y', (T, H, d)), _stream(stream))
    _check(st, 'kda_prefill_noalloc')
    return y


def kda_decode(cfg: Config, q, k, v, log_a, beta, g, norm_w, state, state_slots=None,
               pool_size=None, y=None, stream=None):
    """One token per sequence; ``state`` [pool, H, d, d] is updated in place.  Returns y."""
    H, d = cfg.num_heads, cfg.head_dim
    B = q.shape[0]
    if y is None:
        y = _empty((B, H, d), cfg.dtype, q.device)
    if pool_size is None:
        pool_size = state.shape[0]
    c = cfg.c()
    st = lib().kda_decode(
        ctypes.byref(c), B, _ptr(q, torch.float32, 'q', (B, H, d)),
        _ptr(k, torch.float32, 'k', (B, H, d)),
        _ptr(v, torch.float32, 'v', (B, H, d)), _ptr(log_a, torch.float32, 'log_a', (B, H, d)),
        _ptr(beta, torch.float32, 'beta', (B, H)), _ptr(g, cfg.dtype, 'g', (B, H, d)),
        _ptr(norm_w, torch.float32, 'norm_w', (d,)), _ptr(state, torch.float32, 'state'),
        _ptr(state_slots, torch.int32, 'state_slots'), int(pool_size),
        _ptr(y, cfg.dtype, 'y', (B, H, d)), _stream(stream))
    _check(st, 'kda_decode')
    return y


def kda_verify(cfg: Config, q, k, v, log_a, beta, g, norm_w, state, state_slots=None,
               pool_size=None, tape=None, y=None, stream=None):
    """Verify [B, Tb] draft tokens from ``state`` (unchanged).  Returns (y, tape)."""
    H, d = cfg.num_heads, cfg.head_dim
    B, Tb = q.shape[0], q.shape[1]
    if y is None:
        y = _empty((B, Tb, H, d), cfg.dtype, q.device)
    if tape is None:
        tape = _empty((B, Tb, H, d, d), torch.float32, q.device)
    if pool_size is None:
        pool_size = state.shape[0]
    c = cfg.c()
    st = lib().kda_verify(
        ctypes.byref(c), B, Tb, _ptr(q, torch.float32, 'q', (B, Tb, H, d)),
        _ptr(k, torch.float32, 'k', (B, Tb, H, d)), _ptr(v, torch.float32, 'v', (B, Tb, H, d)),
        _ptr(log_a, torch.float32, 'log_a', (B, Tb, H, d)),
        _ptr(beta, torch.float32, 'beta', (B, Tb, H)), _ptr(g, cfg.dtype, 'g', (B, Tb, H, d)),
        _ptr(norm_w, torch.float32, 'norm_w', (d,)), _ptr(state, torch.float32, 'state'),
        _ptr(state_slots, torch.int32, 'state_slots'), int(pool_size),
        _ptr(tape, torch.float32, 'tape', (B, Tb, H, d, d)),
        _ptr(y, cfg.dtype, 'y', (B, Tb, H, d)), _stream(stream))
    _check(st, 'kda_verify')
    return y, tape


def kda_verify_compact(cfg: Config, q, k, v, log_a, beta, g, norm_w, state, state_slots=None,
                       pool_size=None, tape_kua=None, y=None, stream=None):
    """Verify [B, Tb] draft tokens from ``state`` (unchanged), recording each step's
    (k, u, a) instead of the state.  Returns (y, tape_kua [B, Tb, H, 3, d])."""
    H, d = cfg.num_heads, cfg.head_dim
    B, Tb = q.shape[0], q.shape[1]
    if y is None:
        y = _empty((B, Tb, H, d), cfg.dtype, q.device)
    if tape_kua is None:
        tape_kua = _empty((B, Tb, H, 3, d), torch.float32, q.device)
    if pool_size is None:
        pool_size = state.shape[0]
    c = cfg.c()
    st = lib().kda_verify_compact(
        ctypes.byref(c), B, Tb, _ptr(q, torch.float32, 'q', (B, Tb, H, d)),
        _ptr(k, torch.float32, 'k', (B, Tb, H, d)), _ptr(v, torch.float32, 'v', (B, Tb, H, d)),
        _ptr(log_a, torch.float32, 'log_a', (B, Tb, H, d)),
        _ptr(beta, torch.float32, 'beta', (B, Tb, H)), _ptr(g, cfg.dtype, 'g', (B, Tb, H, d)),
        _ptr(norm_w, torch.float32, 'norm_w', (d,)), _ptr(state, torch.float32, 'state'),
        _ptr(state_slots, torch.int32, 'state_slots'), int(pool_size),
        _ptr(tape_kua, torch.float32, 'tape_kua', (B, Tb, H, 3, d)),
        _ptr(y, cfg.dtype, 'y', (B, Tb, H, d)), _stream(stream))
    _check(st, 'kda_verify_compact')
    return y, tape_kua


def kda_rollback_replay(cfg: Config, accepted, tape_kua, state, conv_window=None,
                        conv_state=None, state_slots=None, pool_size=None, stream=None):
    """Commit accepted prefixes by replaying the compact tape on the live state."""
    H, d = cfg.num_heads, cfg.head_dim
    B, Tb = tape_kua.shape[0], tape_kua.shape[1]
    if pool_size is None:
        pool_size = state.shape[0]
    c = cfg.c()
    st = lib().kda_rollback_replay(
        ctypes.byref(c), B, Tb, _ptr(accepted, torch.int32, 'accepted', (B,)),
        _ptr(tape_kua, torch.float32, 'tape_kua', (B, Tb, H, 3, d)),
        _ptr(conv_window, cfg.dtype, 'conv_window'), _ptr(state, torch.float32, 'state'),
        _ptr(conv_state, cfg.dtype, 'conv_state'), _ptr(state_slots, torch.int32, 'state_slots'),
        int(pool_size), _stream(stream))
    _check(st, 'kda_rollback_replay')


def kda_rollback(cfg: Config, accepted, tape, state, conv_window=None, conv_state=None,
                 state_slots=None, pool_size=None, stream=None):
    """Commit accepted prefixes: state <- tape[L-1], conv state <- window[L:L+K-1]."""
    H, d = cfg.num_heads, cfg.head_dim
    B, Tb = tape.shape[0], tape.shape[1]
    if pool_size is None:
        pool_size = state.shape[0]
    c = cfg.c()
    st = lib().kda_rollback(
        ctypes.byref(c), B, Tb, _ptr(accepted, torch.int32, 'accepted', (B,)),
        _ptr(tape, torch.float32, 'tape', (B, Tb, H, d, d)),
        _ptr(conv_window, cfg.dtype, 'conv_window'), _ptr(state, torch.float32, 'state'),
        _ptr(conv_state, cfg.dtype, 'conv_state'), _ptr(state_slots, torch.int32, 'state_slots'),
        int(pool_size), _stream(stream))
    _check(st, 'kda_rollback')


def kda_workspace_status(workspace, stream=None) -> int:
    """Synchronise the stream and return the prefill workspace status code."""
    return int(lib().kda_workspace_status(_ptr(workspace, None, 'workspace'), _stream(stream)))


def kda_selftest_wait_timeout(workspace, stream=None):
    """Run the bounded-wait self-test on ``workspace`` (enqueue only)."""
    _check(lib().kda_selftest_wait_timeout(_ptr(workspace, None, 'workspace'), _stream(stream)),
           'kda_selftest_wait_timeout')


def kda_layer_decode(cfg: Config, x, f, beta_logit, g, conv_w, A_log, dt_bias, norm_w, state,
                     conv_state=None, state_slots=None, pool_size=None, y=None, stream=None):
    """One token per sequence from the raw layer inputs (prep fused).  Returns y."""
    H, d, K = cfg.num_heads, cfg.head_dim, cfg.conv_size
    B = x.shape[0]
    if y is None:
        y = _empty((B, H, d), cfg.dtype, x.device)
    if pool_size is None:
        pool_size = state.shape[0]
    c = cfg.c()
    _check(lib().kda_layer_decode(
        ctypes.byref(c), B, _ptr(x, cfg.dtype, 'x', (B, H, 3 * d)),
        _ptr(f, cfg.dtype, 'f', (B, H, d)), _ptr(beta_logit, cfg.dtype, 'beta_logit', (B, H)),
        _ptr(g, cfg.dtype, 'g', (B, H, d)), _ptr(conv_w, torch.float32, 'conv_w', (H, 3 * d, K)),
        _ptr(A_log, torch.float32, 'A_log', (H,)), _ptr(dt_bias, torch.float32, 'dt_bias', (H, d)),
        _ptr(norm_w, torch.float32, 'norm_w', (d,)), _ptr(conv_state, cfg.dtype, 'conv_state'),
        _ptr(state, torch.float32, 'state'), _ptr(state_slots, torch.int32, 'state_slots'),
        int(pool_size), _ptr(y, cfg.dtype, 'y', (B, H, d)), _stream(stream)), 'kda_layer_decode')
    return y


def kda_layer_verify(cfg: Config, x, f, beta_logit, g, conv_w, A_log, dt_bias, norm_w, state,
                     conv_state=None, state_slots=None, pool_size=None, tape=None, window=None,
                     y=None, stream=None):
    """A block of draft tokens per sequence from the raw inputs (prep fused).
    x is [B, T_b, H, 3d].  Returns (y, tape, window)."""
    H, d, K = cfg.num_heads, cfg.head_dim, cfg.conv_size
    B, Tb = x.shape[0], x.shape[1]
    if y is None:
        y = _empty((B, Tb, H, d), cfg.dtype, x.device)
    if tape is None:
        tape = _empty((B, Tb, H, d, d), torch.float32, x.device)
    if window is None:
        window = _empty((B, K - 1 + Tb, H, 3 * d), cfg.dtype, x.device)
    if pool_size is None:
        pool_size = state.shape[0]
    c = cfg.c()
    _check(lib().kda_layer_verify(
        ctypes.byref(c), B, Tb, _ptr(x, cfg.dtype, 'x', (B, Tb, H, 3 * d)),
        _ptr(f, cfg.dtype, 'f', (B, Tb, H, d)),
        _ptr(beta_logit, cfg.dtype, 'beta_logit', (B, Tb, H)),
        _ptr(g, cfg.dtype, 'g', (B, Tb, H, d)), _ptr(conv_w, torch.float32, 'conv_w', (H, 3 * d, K)),
        _ptr(A_log, torch.float32, 'A_log', (H,)), _ptr(dt_bias, torch.float32, 'dt_bias', (H, d)),
        _ptr(norm_w, torch.float32, 'norm_w', (d,)), _ptr(conv_state, cfg.dtype, 'conv_state'),
        _ptr(state, torch.float32, 'state'), _ptr(state_slots, torch.int32, 'state_slots'),
        int(pool_size), _ptr(tape, torch.float32, 'tape', (B, Tb, H, d, d)),
        _ptr(window, cfg.dtype, 'window', (B, K - 1 + Tb, H, 3 * d)),
        _ptr(y, cfg.dtype, 'y', (B, Tb, H, d)), _stream(stream)), 'kda_layer_verify')
    return y, tape, window


def kda_layer_verify_compact(cfg: Config, x, f, beta_logit, g, conv_w, A_log, dt_bias, norm_w,
                             state, conv_state=None, state_slots=None, pool_size=None,
                             tape_kua=None, window=None, y=None, stream=None):
    """kda_layer_verify recording each step's (k, u, a).  Returns (y, tape_kua, window)."""
    H, d, K = cfg.num_heads, cfg.head_dim, cfg.conv_size
    B, Tb = x.shape[0], x.shape[1]
    if y is None:
        y = _empty((B, Tb, H, d), cfg.dtype, x.device)
    if tape_kua is None:
        tape_kua = _empty((B, Tb, H, 3, d), torch.float32, x.device)
    if window is None:
        window = _empty((B, K - 1 + Tb, H, 3 * d), cfg.dtype, x.device)
    if pool_size is None:
        pool_size = state.shape[0]
    c = cfg.c()
    _check(lib().kda_layer_verify_compact(
        ctypes.byref(c), B, Tb, _ptr(x, cfg.dtype, 'x', (B, Tb, H, 3 * d)),
        _ptr(f, cfg.dtype, 'f', (B, Tb, H, d)),
        _ptr(beta_logit, cfg.dtype, 'beta_logit', (B, Tb, H)),
        _ptr(g, cfg.dtype, 'g', (B, Tb, H, d)), _ptr(conv_w, torch.float32, 'conv_w', (H, 3 * d, K)),
        _ptr(A_log, torch.float32, 'A_log', (H,)), _ptr(dt_bias, torch.float32, 'dt_bias', (H, d)),
        _ptr(norm_w, torch.float32, 'norm_w', (d,)), _ptr(conv_state, cfg.dtype, 'conv_state'),
        _ptr(state, torch.float32, 'state'), _ptr(state_slots, torch.int32, 'state_slots'),
        int(pool_size), _ptr(tape_kua, torch.float32, 'tape_kua', (B, Tb, H, 3, d)),
        _ptr(window, cfg.dtype, 'window', (B, K - 1 + Tb, H, 3 * d)),
        _ptr(y, cfg.dtype, 'y', (B, Tb, H, d)), _stream(stream)), 'kda_layer_verify_compact')
    return y, tape_kua, window


def kda_proj_gemm(A, B, outs, status=None, stream=None):
    """C = A B^T (bf16 in, fp32 accumulate, bf16 out) with column ranges of C routed to
    separate tensors.  A [M, K] and B [N, K] are bf16 CUDA tensors; ``outs`` is a list of
    (tensor, col_begin, col_end): columns [col_begin, col_end) of C go to ``tensor``, a
    contiguous bf16 CUDA tensor read as M rows of numel / M elements, each row starting
    with the range."""
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError('A and B must share K')
    arr = (CProjOut * max(1, len(outs)))()
    for i, (t, c0, c1) in enumerate(outs):
        if t.numel() % max(M, 1):
            raise ValueError('output tensor size must be a multiple of M rows')
        ld = t.numel() // max(M, 1)
        arr[i] = CProjOut(_ptr(t, torch.bfloat16, f'outs[{i}]'), ld, int(c0), int(c1))
    _check(lib().kda_proj_gemm(int(M), int(N), int(K), _ptr(A, torch.bfloat16, 'A'),
                               _ptr(B, torch.bfloat16, 'B'), arr, len(outs),
                               _ptr(status, torch.int32, 'status'), _stream(stream)),
           'kda_proj_gemm')


def kda_launch_count() -> int:
    """Kernels the library launched from this thread so far (cumulative)."""
    return int(lib().kda_launch_count())


def kda_set_phase_events(events=()):
    """Record up to three ``torch.cuda.Event`` after the intra-chunk, inter-chunk and
    output-norm passes of the following prefills on this thread; ``()`` clears.
    Each event must already have been recorded once (torch creates it lazily)."""
    events = list(events)
    if len(events) > 3:
        raise ValueError('at most three phase events')
    handles = []
    for e in events:
        h = 0 if e is None else int(e.cuda_event)
        if e is not None and h == 0:
            raise ValueError('record the event once before passing it (created lazily)')
        handles.append(h)
    arr = (ctypes.c_void_p * max(1, len(handles)))(*handles)
    _check(lib().kda_set_phase_events(arr if handles else None, len(handles)),
           'kda_set_phase_events')


# ---------------------------------------------------------------------------
# compositions of the entry points
# ---------------------------------------------------------------------------
def kda_layer_prefill_workspace_size(cfg: Config, n_seqs: int, total_tokens: int) -> int:
    c = cfg.c()
    return int(lib().kda_layer_prefill_workspace_size(ctypes.byref(c), int(n_seqs),
                                                      int(total_tokens)))


def kda_layer_prefill(cfg: Config, cu_seqlens, x, f, beta_logit, g, conv_w, A_log, dt_bias,
                      norm_w, conv_state=None, state_in=None, state_out=None, state_slots=None,
                      pool_size=None, y=None, workspace=None, max_seqlen=0, stream=None):
    """The whole layer from raw inputs (prep fused where supported).  Returns y."""
    H, d, K = cfg.num_heads, cfg.head_dim, cfg.conv_size
    T = x.shape[0]
    N = cu_seqlens.numel() - 1
    if y is None:
        y = _empty((T, H, d), cfg.dtype, x.device)
    if workspace is None:
        workspace = torch.empty(kda_layer_prefill_workspace_size(cfg, N, T), dtype=torch.uint8,
                                device=x.device)
    if pool_size is None:
        ref = next((t for t in (state_in, state_out, conv_state) if t is not None), None)
        pool_size = ref.shape[0] if ref is not None else N
    c = cfg.c()
    st = lib().kda_layer_prefill(
        ctypes.byref(c), N, T, _ptr(cu_seqlens, torch.int32, 'cu_seqlens'), int(max_seqlen),
        _ptr(x, cfg.dtype, 'x', (T, H, 3 * d)), _ptr(f, cfg.dtype, 'f', (T, H, d)),
        _ptr(beta_logit, cfg.dtype, 'beta_logit', (T, H)), _ptr(g, cfg.dtype, 'g', (T, H, d)),
        _ptr(conv_w, torch.float32, 'conv_w', (H, 3 * d, K)),
        _ptr(A_log, torch.float32, 'A_log', (H,)), _ptr(dt_bias, torch.float32, 'dt_bias', (H, d)),
        _ptr(norm_w, torch.float32, 'norm_w', (d,)), _ptr(conv_state, cfg.dtype, 'conv_state'),
        _ptr(state_in, torch.float32, 'state_in'), _ptr(state_out, torch.float32, 'state_out'),
        _ptr(state_slots, torch.int32, 'state_slots'), int(pool_size),
        _ptr(y, cfg.dtype, 'y', (T, H, d)), _ptr(workspace, None, 'workspace'),
        int(workspace.numel() * workspace.element_size()), _stream(stream))
    _check(st, 'kda_layer_prefill')
    return y


def prep_then_prefill(cfg: Config, params, acts, state_in=None, state_out=None, conv_state=None,
                      workspace=None, prep_out=None, y=None, stream=None):
    """kda_prep + kda_prefill as two calls; returns (y, prep outputs)."""
    p = kda_prep(cfg, acts['cu_seqlens'], acts['x'], acts['f'], acts['beta_logit'],
                 params['conv_w'], params['A_log'], params['dt_bias'], conv_state=conv_state,
                 out=prep_out, stream=stream)
    y = kda_prefill(cfg, acts['cu_seqlens'], p['q'], p['k'], p['v'], p['log_a'], p['beta'],
                    acts['g'], params['norm_w'], state_in=state_in, state_out=state_out,
                    y=y, workspace=workspace, stream=stream)
    return y, p


def layer_prefill(cfg: Config, params, acts, state_in=None, state_out=None, conv_state=None,
                  workspace=None, y=None, stream=None):
    """kda_layer_prefill on dicts of parameters and activations; returns y."""
    return kda_layer_prefill(cfg, acts['cu_seqlens'], acts['x'], acts['f'], acts['beta_logit'],
                             acts['g'], params['conv_w'], params['A_log'], params['dt_bias'],
                             params['norm_w'], conv_state=conv_state, state_in=state_in,
                             state_out=state_out, y=y, workspace=workspace, stream=stream)


def layer_projections(cfg: Config, hidden, W_in, W_gb, gate_rank, out=None, stream=None):
    """The layer's inputs from the hidden states: kda_proj_gemm with the fused input
    weight (x = q|k|v pre-conv, f, beta logit, g_a, each into its own dense tensor),
    then kda_proj_gemm with the gate's second factor (g = g_a W_gb^T).  bf16 only; the
    head count and gate rank must be multiples of 8 (the output ranges are 16-byte
    aligned).  Returns dict x, f, beta_logit, g_a, g."""
    H, d = cfg.num_heads, cfg.head_dim
    T = hidden.shape[0]
    dev = hidden.device
    nx, nf = 3 * H * d, H * d
    o = dict(out or {})
    shapes = {'x': (T, H, 3 * d), 'f': (T, H, d), 'beta_logit': (T, H),
              'g_a': (T, gate_rank), 'g': (T, H, d)}
    for name, shp in shapes.items():
        if o.get(name) is None:
            o[name] = _empty(shp, torch.bfloat16, dev)
    kda_proj_gemm(hidden, W_in, [(o['x'], 0, nx), (o['f'], nx, nx + nf),
                                 (o['beta_logit'], nx + nf, nx + nf + H),
                                 (o['g_a'], nx + nf + H, nx + nf + H + gate_rank)],
                  stream=stream)
    kda_proj_gemm(o['g_a'], W_gb, [(o['g'], 0, H * d)], stream=stream)
    return o
