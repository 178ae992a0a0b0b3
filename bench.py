#!/usr/bin/env python
"""Throughput of the KDA layer hot path on B200, one JSON line on rank 0.

Headline workload (one step): prep + chunked prefill of one packed batch,
B = 1, H = 32, T = 8192, d = 128, chunk 64, bf16 activations, fp32 state,
A_log and dt_bias, seeded synthetic inputs resident in HBM.  Metric: prefill
tokens/s.  At N = 1 the same line also carries the batched decode workload
(B = 64, H = 32, d = 128, 1,024 steps after a 512-token prefill, CUDA graph),
the speculative verify + rollback workload (B = 16, blocks of 8 drafts after a
4,096-token context, 256 rounds, CUDA graph) and the long / varlen prefill (one
131,072-token sequence; 8 packed sequences of 1K-32K tokens).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kda|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch of the
same workload (weak scaling, no collective in the data path); the timing is
the max over ranks.  ``--impl reference`` times the float64 CPU oracle.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = 'KDA prefill tokens/s & decode tokens/s (1 B200) + % of TC / HBM roofline'
SMI_FIELDS = ('index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,'
              'clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,'
              'clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap')


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument('--gpus', type=int, default=1)
    ap.add_argument('--steps', type=int, default=200)
    ap.add_argument('--warmup', type=int, default=5)
    ap.add_argument('--impl', default='kda', choices=['kda', 'reference'])
    ap.add_argument('--tokens', type=int, default=8192, help='prefill length (8192 = headline)')
    ap.add_argument('--no-extras', action='store_true', help='skip decode / verify workloads')
    ap.add_argument('--no-cpu', action='store_true', help='skip the CPU oracle baseline')
    ap.add_argument('--only', default='',
                    help='prefill|decode|verify|long|layer_full: run one workload only')
    ap.add_argument('--no-long', action='store_true', help='skip the long / varlen workload')
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; no data-path collective)
# ---------------------------------------------------------------------------
class Dist:
    def __init__(self):
        import torch
        self.world = int(os.environ.get('WORLD_SIZE', '1'))
        self.rank = int(os.environ.get('RANK', '0'))
        self.local = int(os.environ.get('LOCAL_RANK', '0'))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            backend = 'nccl' if torch.cuda.is_available() else 'gloo'
            if backend == 'nccl':
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch
        dev = 'cuda' if torch.cuda.is_available() else 'cpu'
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    def __init__(self, gpu_index: int):
        self.proc = None
        import tempfile
        # the raw samples go to KDA_CLOCKS_DIR (default: the system temp directory)
        folder = os.environ.get('KDA_CLOCKS_DIR') or tempfile.gettempdir()
        self.path = os.path.join(folder, f'kda_bench_clocks_rank{gpu_index}_{os.getpid()}.csv')
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, 'w')
            self.proc = subprocess.Popen(
                ['nvidia-smi', '-i', str(gpu_index), f'--query-gpu={SMI_FIELDS}',
                 '--format=csv,noheader,nounits', '-lms', '50'],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(',')]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace('.', '').isdigit()]
        loaded = [float(r[3]) for r in rows if r[3].replace('.', '').isdigit()]
        names = ['hw_slowdown', 'hw_thermal_slowdown', 'sw_thermal_slowdown', 'sw_power_cap']
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == 'Active'})
        return {'sm_mhz': statistics.median(sm) if sm else None,
                'sm_max_mhz': float(rows[0][2]) if rows[0][2].replace('.', '').isdigit() else None,
                'reasons': reasons, 'samples': len(rows),
                'power_w_max': max(loaded) if loaded else None}


def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, 'measured' | 'fallback')."""
    try:
        with open(os.path.join(ROOT, 'MEASURED_PEAKS.json')) as fh:
            p = json.load(fh)
        return (p['hbm_gbs'], p['bf16_tflops'], p.get('bf16_tflops_sustained', p['bf16_tflops']),
                'measured')
    except Exception:
        return 6650.0, 1590.0, 1400.0, 'fallback'


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) comes from the
# committed ncu summaries; a summary records the sha256 of the kernel's source file at
# capture time, and the sha256 of its code (comments and blank lines removed), and counts
# only while that code is unchanged.
PROFILED = {
    'prefill_cosched': ('profiles/prefill_cosched_sm100_8k.md',
                        ('linear_attention_recurrence_09_b200/csrc/kda_intra_sm100.cu',
                         'linear_attention_recurrence_09_b200/csrc/kda_chain_sm100.cuh')),
    'intra_chunk': ('profiles/intra_chunk_sm100_prefill_8k.md',
                    'linear_attention_recurrence_09_b200/csrc/kda_intra_sm100.cu'),
    'inter_chunk': ('profiles/interchunk_sm100_prefill_8k.md',
                    'linear_attention_recurrence_09_b200/csrc/kda_prefill_sm100.cu'),
    'proj_gemm': ('profiles/proj_gemm_layer_8k.md',
                  'linear_attention_recurrence_09_b200/csrc/kda_gemm_sm100.cu'),
    'kda_decode': ('profiles/step_decode_b64.md',
                   'linear_attention_recurrence_09_b200/csrc/kda_step.cu'),
    'kda_verify_compact': ('profiles/step_verify_compact_b16.md',
                           'linear_attention_recurrence_09_b200/csrc/kda_step.cu'),
    'prep_short': ('profiles/prep_short_decode_b64.md',
                   'linear_attention_recurrence_09_b200/csrc/kda_prep.cu'),
}


def code_text(src):
    """C/C++/CUDA source without comments, trailing blanks and blank lines (string and
    character literals kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in '"\'':
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == '\\' else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith('//', i):
            while i < n and src[i] != '\n':
                i += 1
        elif src.startswith('/*', i):
            j = src.find('*/', i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (line.rstrip() for line in ''.join(out).split('\n'))
    return '\n'.join(line for line in lines if line)


def code_sha256(path):
    """sha256 of the code of one source file, or of several joined by newlines."""
    import hashlib
    paths = [path] if isinstance(path, str) else list(path)
    texts = []
    for p in paths:
        with open(p, encoding='utf-8') as fh:
            texts.append(code_text(fh.read()))
    return hashlib.sha256('\n'.join(texts).encode()).hexdigest()


def profiled_traffic(kernel):
    import re
    if kernel not in PROFILED:
        return None
    summary, source = PROFILED[kernel]
    summary = os.path.join(ROOT, summary)
    source = (os.path.join(ROOT, source) if isinstance(source, str)
              else [os.path.join(ROOT, f) for f in source])
    try:
        text = open(summary).read()
        digest = code_sha256(source)
    except OSError:
        return None
    m_hash = re.search(r'code_sha256:\s*([0-9a-f]{64})', text)
    m_traffic = re.search(r'traffic_bytes_per_launch:\s*([0-9]+)', text)
    if not (m_hash and m_traffic) or m_hash.group(1) != digest:
        return None
    return int(m_traffic.group(1))


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
def prefill_workload(torch, kda, synth, T, seed, dev):
    H, d, K = 32, 128, 4
    cfg = kda.Config(num_heads=H, head_dim=d, conv_size=K, dtype=torch.bfloat16, chunk_size=64)
    P = {k: v.to(dev) for k, v in synth.layer_params(seed, H, d, K).items()}
    A_cpu = synth.layer_activations(seed, [T], H, d, torch.bfloat16)
    A = {k: v.to(dev) for k, v in A_cpu.items()}
    N = 1
    y = torch.empty(T, H, d, dtype=cfg.dtype, device=dev)
    state = torch.empty(N, H, d, d, device=dev)
    ws = torch.empty(kda.kda_layer_prefill_workspace_size(cfg, N, T), dtype=torch.uint8,
                     device=dev)
    return dict(cfg=cfg, P=P, A=A, A_cpu=A_cpu, y=y, state=state, ws=ws, T=T, H=H, d=d)


PHASES = ('intra_chunk', 'inter_chunk', 'gated_norm')


def prefill_config(T, H, d, world):
    """The headline workload's description, shared by both arms."""
    return {'workload': f'prefill B=1 H={H} T={T} d={d} chunk=64 conv=4 (one KDA layer: prep, '
                        'chunked recurrence, gated RMSNorm)',
            'global_batch': world, 'seq_len': T, 'heads': H, 'head_dim': d,
            'parallelism': f'replicas x{world} (independent batches per GPU)',
            'l2': f'inputs larger than L2 (x alone is {T * H * 3 * d * 2 / 1e6:.0f} MB)'}


def prefill_bytes(T, H, d, C=64, K=4, fused_norm=True):
    """Algorithmic HBM bytes per launch of each pass of kda_layer_prefill (bf16
    activations, fp32 state, bf16 chunk tiles), and of the layer as a whole (inputs x,
    f, beta logit, g read once, y and the final state written once).  With the norm
    fused into the inter-chunk pass that pass reads g and writes y; otherwise it writes
    o (fp32) and the gated-norm pass reads o and g and writes y."""
    th = T * H
    nch = -(-T // C)
    tiles = th * (4 * d * 2 + C * 2) + nch * H * d * 4          # W, U~, Q~, K', M; e^{G_C}
    intra = th * (3 * d * 2 + d * 2 + 2) + tiles + H * (3 * d * K + 1 + d) * 4
    layer = th * (3 * d * 2 + d * 2 + 2 + d * 2 + d * 2) + H * d * d * 4
    if fused_norm:
        inter = tiles + th * d * 2 + d * 4 + th * d * 2 + H * d * d * 4   # + g, norm_w in; y out
        return {'intra_chunk': intra, 'inter_chunk': inter, 'layer': layer,
                'prefill_cosched': intra + inter}
    inter = tiles + th * d * 4 + H * d * d * 4                  # tiles in, o and state out
    norm = th * d * 4 + th * d * 2 + d * 4 + th * d * 2         # o, g, norm_w in; y out
    return {'intra_chunk': intra, 'inter_chunk': inter, 'gated_norm': norm, 'layer': layer}


def layer_method_bytes(total_tokens, n_seqs, H, d):
    """The method's own HBM bytes for one layer call (the per-unit figure of the
    hot-path measurement: 1,538 B per (token, head) at d = 128 with bf16 activations):
    x (3d), f (d), g (d) and the beta logit (1) read once, y (d) written once, plus the
    final fp32 state of every (sequence, head) written once.  Everything else the
    passes move (the chunk tiles handed from pass 1 to pass 2) is design traffic."""
    th = total_tokens * H
    return th * (3 * d * 2 + d * 2 + 2 + d * 2 + d * 2) + n_seqs * H * d * d * 4


def prefill_dense_flops(T, H, d, C=64):
    """Flops of the chunk form's dense tiles per step: per (chunk, head) the grams A and
    M (2 C^2 d MAC), W = T (K e^G) and U~ = T V (2 C^2 d), U = U~ - W S, Q~ S and the
    state increment K'^T U (3 C d^2), and M U (C^2 d): 2 (5 C d + 3 d^2) flops per
    (token, head), 47.2 GFLOP at B = 1, H = 32, T = 8192, d = 128, C = 64.  Issued MMA
    work (hi/lo splits, padding, the unused part of the 128 x 128 gram) is not counted."""
    return 2 * (5 * C * d + 3 * d * d) * (-(-T // C) * C) * H


# nominal dense tensor-core rates on B200 (PFLOP/s): tf32 1.1, bf16 2.25; a tf32 MMA is timed
# against the measured bf16 peak scaled by this ratio
TF32_PER_BF16 = 1.1 / 2.25


def prefill_mma_flops(T, H, d, C=64):
    """Tensor-core work the two passes issue per step (flops of the MMAs as issued, padding
    included), by operand type.  Pass 1 per (chunk, head): the tf32 gram (M = N = 2C,
    K = d) and the bf16 W/U~ products (three + two MMAs of M = d, N = K = C).  Pass 2 per
    (chunk, head): [W; Q~] S (M = 2C, K = d), K'^T U (M = d, K = C) and [0; M] U (M = 2C,
    K = C), each over the d value columns."""
    tiles = -(-T // C) * H
    intra_tf32 = tiles * 2 * (2 * C) * (2 * C) * d
    intra_bf16 = tiles * 5 * 2 * d * C * C
    inter_bf16 = tiles * (2 * (2 * C) * d * d + 2 * d * d * C + 2 * (2 * C) * d * C)
    return {'intra_chunk': {'tf32': intra_tf32, 'bf16': intra_bf16},
            'inter_chunk': {'tf32': 0, 'bf16': inter_bf16},
            'prefill_cosched': {'tf32': intra_tf32, 'bf16': intra_bf16 + inter_bf16}}


def issued_mma_view(flops, ms_phase, bf16_tflops):
    """Per pass: the time the tensor pipe needs for the MMAs it issues at peak (bf16 at
    the measured peak, tf32 at that times the nominal ratio) as a fraction of the pass's
    duration.  A view of the design, not the roofline (see tensor_roofline)."""
    out = {}
    for ph, f in flops.items():
        if ph not in ms_phase:
            continue
        t_peak = f['bf16'] / (bf16_tflops * 1e12) + f['tf32'] / (bf16_tflops * TF32_PER_BF16 * 1e12)
        out[ph] = {'issued_mma_gflop': (f['bf16'] + f['tf32']) / 1e9,
                   'ms_at_peak': t_peak * 1e3,
                   'frac': t_peak * 1e3 / ms_phase[ph]}
    return out


def tensor_roofline(dense_flops, ms_step, burst_tflops, sustained_tflops):
    """Dense-tile flops of one step over (step time x bf16 dense peak)."""
    achieved = dense_flops / (ms_step / 1e3) / 1e12
    return {'bound': 'tensor', 'dense_tile_gflop': dense_flops / 1e9, 'achieved': achieved,
            'peak': burst_tflops, 'unit': 'TFLOP/s', 'frac': achieved / burst_tflops,
            'frac_sustained': achieved / sustained_tflops,
            'ms_at_peak': dense_flops / (burst_tflops * 1e12) * 1e3}


def run_prefill(args, dist, torch, kda, synth, dev):
    W = prefill_workload(torch, kda, synth, args.tokens, 1 + 1000 * dist.rank, dev)
    cfg, P, A, y, state, ws = (W[k] for k in ('cfg', 'P', 'A', 'y', 'state', 'ws'))
    stream = torch.cuda.current_stream()

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)            # torch creates the CUDA event on first record
        return e

    # beside the headline: the same layer with the two passes as separate launches
    cfg_sep = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_SEPARATE_PASSES)

    def step(e=None, c=cfg):
        # one pass of the layer: fused prep + intra-chunk, inter-chunk, gated norm (one
        # co-scheduled launch, or separate launches)
        if e:
            e[0].record(stream)
            kda.kda_set_phase_events(e[1:])
        kda.kda_layer_prefill(c, A['cu_seqlens'], A['x'], A['f'], A['beta_logit'], A['g'],
                              P['conv_w'], P['A_log'], P['dt_bias'], P['norm_w'],
                              state_out=state, y=y, workspace=ws, max_seqlen=W['T'])
        if e:
            kda.kda_set_phase_events(())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dist.barrier()
    sampler = ClockSampler(torch.cuda.current_device()) if dist.rank == 0 else None
    torch.cuda.synchronize()
    per = [[ev() for _ in range(4)] for _ in range(args.steps)]
    t_start, t_end = ev(), ev()
    wall0 = time.perf_counter()
    n_launch0 = kda.kda_launch_count()
    t_start.record(stream)
    for i in range(args.steps):
        step(per[i])
    t_end.record(stream)
    launches = kda.kda_launch_count() - n_launch0
    torch.cuda.synchronize()
    dist.barrier()
    ms = t_start.elapsed_time(t_end)
    # keep the GPU loaded (untimed) so the clock sampler sees at least ~1 s under load
    while time.perf_counter() - wall0 < 1.0:
        step()
        torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    one_launch = launches == args.steps          # both passes (and the norm) co-scheduled
    fused_norm = one_launch or launches == 2 * args.steps   # norm inside the inter pass
    phases = (('prefill_cosched',) if one_launch else PHASES[:2] if fused_norm else PHASES)
    # per-step statistic: the median of the K per-step event durations (the timed region's
    # mean is kept beside it); per pass likewise
    step_ms = [p[0].elapsed_time(p[3]) for p in per]
    ms_phase = {ph: statistics.median(p[i].elapsed_time(p[i + 1]) for p in per)
                for i, ph in enumerate(phases)}
    # the separate launches, timed the same way (untimed warm-up first)
    for _ in range(args.warmup):
        step(c=cfg_sep)
    per_sep = [[ev() for _ in range(4)] for _ in range(args.steps)]
    for i in range(args.steps):
        step(per_sep[i], c=cfg_sep)
    torch.cuda.synchronize()
    separate = {'ms_per_step': dist.max(statistics.median(p[0].elapsed_time(p[3])
                                                          for p in per_sep)),
                'breakdown_ms': {ph: statistics.median(p[i].elapsed_time(p[i + 1])
                                                       for p in per_sep)
                                 for i, ph in enumerate(PHASES[:2])},
                'launches_per_step': 2}
    ms_step = dist.max(statistics.median(step_ms))
    ms_mean = dist.max(ms) / args.steps
    T, H, d = W['T'], W['H'], W['d']
    value = dist.world * T / (ms_step / 1e3)

    # end to end through the same entry point with host buffers (pinned).  Steps are
    # pipelined the way a serving loop runs them: step i+1's inputs are copied in on one
    # copy stream while step i computes, and step i's y and final state are copied out on
    # another while step i+1 computes (inputs and outputs double-buffered; the workspace is
    # shared, the compute being serial).  Every step's own copies are inside the region.
    hx = {k: W['A_cpu'][k].pin_memory() for k in ('x', 'f', 'beta_logit', 'g')}
    hy = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    hs = torch.empty(state.shape, dtype=state.dtype).pin_memory()
    n_e2e = max(3, min(20, args.steps))
    bufs = [{'A': {k: A[k] for k in hx}, 'y': y, 'state': state},
            {'A': {k: torch.empty_like(A[k]) for k in hx}, 'y': torch.empty_like(y),
             'state': torch.empty_like(state)}]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    for e in in_done + comp_done + out_done:
        e.record(stream)

    def e2e_step(i):
        b, j = bufs[i & 1], i & 1
        s_in.wait_event(comp_done[j])        # step i-2 has read this input buffer
        with torch.cuda.stream(s_in):
            for k, h in hx.items():
                b['A'][k].copy_(h, non_blocking=True)
        in_done[j].record(s_in)
        stream.wait_event(in_done[j])
        stream.wait_event(out_done[j])       # step i-2's outputs have left this buffer
        kda.kda_layer_prefill(cfg, A['cu_seqlens'], b['A']['x'], b['A']['f'],
                              b['A']['beta_logit'], b['A']['g'], P['conv_w'], P['A_log'],
                              P['dt_bias'], P['norm_w'], state_out=b['state'], y=b['y'],
                              workspace=ws, max_seqlen=W['T'], stream=stream)
        comp_done[j].record(stream)
        s_out.wait_event(comp_done[j])
        with torch.cuda.stream(s_out):
            hy.copy_(b['y'], non_blocking=True)
            hs.copy_(b['state'], non_blocking=True)
        out_done[j].record(s_out)

    def e2e_run(n):
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for i in range(n):
            e2e_step(i)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    e2e_run(2)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = ev(), ev()
    e0.record(stream)
    e2e_run(n_e2e)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = dist.max(e0.elapsed_time(e1)) / n_e2e
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = hy.numel() * hy.element_size() + hs.numel() * hs.element_size()

    hbm, tc, tc_sus, peak_kind = measured_peaks()
    nb = prefill_bytes(T, H, d, fused_norm=fused_norm)
    method = layer_method_bytes(T, 1, H, d)
    achieved = method / (ms_step / 1e3) / 1e9
    pass_traffic = [profiled_traffic(ph) for ph in phases]
    res = {
        'metric': METRIC, 'value': value, 'unit': 'tokens/s', 'n_gpus': dist.world,
        'steps': args.steps, 'warmup': args.warmup, 'ms_per_step': ms_step,
        'ms_per_step_mean': ms_mean, 'timing': 'median of per-step CUDA-event durations',
        'higher_is_better': True, 'scaling': 'weak', 'vs_baseline': None, 'dtype': 'bf16',
        'data': 'synthetic (seeded N(0,1) activations, random-init layer parameters)',
        'config': prefill_config(T, H, d, dist.world),
        'e2e': {'value': dist.world * T / (e2e_ms / 1e3), 'unit': 'tokens/s',
                'h2d_bytes_per_step': h2d, 'd2h_bytes_per_step': d2h,
                'ms_per_step': e2e_ms,
                'pipelining': 'copies in / compute / copies out on three streams, inputs '
                              'and outputs double-buffered; every step copies its own '
                              'inputs in and its y and final state out'},
        'gpu_launches': launches,
        # the method's bytes (x, f, g, beta logit in; y, final state out) over the step, i.e.
        # over the one kda_layer_prefill call whose two launches are the dominant work
        'roofline': {'bound': 'hbm', 'kernel': ('kda_layer_prefill (one co-scheduled launch: '
                     'the intra-chunk pass beside the inter-chunk chains)' if one_launch else
                     'kda_layer_prefill (intra-chunk + inter-chunk launches)'),
                     'achieved': achieved, 'peak': hbm, 'unit': 'GB/s',
                     'frac': achieved / hbm,
                     'traffic': (sum(pass_traffic) if all(t is not None for t in pass_traffic)
                                 else None),
                     'peak_kind': peak_kind, 'algorithmic_bytes_per_launch': method,
                     'per_unit': '1,538 B per (token, head) + 64 KB state per head'},
        'breakdown_ms': ms_phase,
        'separate_passes': separate,
        # bytes this design moves per pass (incl. the chunk tiles handed from pass 1 to pass
        # 2, which the method itself does not need), with ncu DRAM traffic where profiled
        'design_traffic': {ph: {'bytes': nb[ph],
                                'achieved_gbs': nb[ph] / (ms_phase[ph] / 1e3) / 1e9,
                                'frac': nb[ph] / (ms_phase[ph] / 1e3) / 1e9 / hbm,
                                'ncu_dram_bytes': tr}
                           for ph, tr in zip(phases, pass_traffic)},
        'tensor_roofline': tensor_roofline(prefill_dense_flops(T, H, d), ms_step, tc, tc_sus),
        'issued_mma': issued_mma_view(prefill_mma_flops(T, H, d), ms_phase, tc),
        'clocks': clocks,
    }
    del W
    return res


def run_layer_full(torch, kda, synth, dev, steps=10, warmup=3):
    """The layer from hidden states (B = 1, T = 8192, H = 32, d = 128, hidden 4096, gate
    rank 128, random-init weights): the fused input projection and the low-rank gate as
    two kda_proj_gemm launches, then kda_layer_prefill.  Reports tokens/s for the whole
    x -> y layer and the projections' tensor-core fraction (GEMM flops over their
    event-timed duration at the measured bf16 dense peak)."""
    w = synth.WORKLOADS['layer_8k_projections']
    T, H, d, hidden, r = w['seqlen'], w['heads'], w['head_dim'], w['hidden'], w['gate_rank']
    cfg = kda.Config(num_heads=H, head_dim=d, conv_size=4, dtype=torch.bfloat16, chunk_size=64)
    W = {k: v.to(dev) for k, v in synth.proj_weights(w['seed'], hidden, H, d, r).items()}
    P = {k: v.to(dev) for k, v in synth.layer_params(w['seed'], H, d, 4).items()}
    hs = synth.hidden_states(w['seed'], T, hidden).to(dev)
    cu = torch.tensor([0, T], dtype=torch.int32, device=dev)
    o = {'x': torch.empty(T, H, 3 * d, dtype=cfg.dtype, device=dev),
         'f': torch.empty(T, H, d, dtype=cfg.dtype, device=dev),
         'beta_logit': torch.empty(T, H, dtype=cfg.dtype, device=dev),
         'g_a': torch.empty(T, r, dtype=cfg.dtype, device=dev),
         'g': torch.empty(T, H, d, dtype=cfg.dtype, device=dev)}
    y = torch.empty(T, H, d, dtype=cfg.dtype, device=dev)
    state = torch.empty(1, H, d, d, device=dev)
    ws = torch.empty(kda.kda_layer_prefill_workspace_size(cfg, 1, T), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    def step(e=None):
        if e:
            e[0].record(stream)
        kda.layer_projections(cfg, hs, W['W_in'], W['W_gb'], r, out=o)
        if e:
            e[1].record(stream)
        kda.kda_layer_prefill(cfg, cu, o['x'], o['f'], o['beta_logit'], o['g'], P['conv_w'],
                              P['A_log'], P['dt_bias'], P['norm_w'], state_out=state, y=y,
                              workspace=ws, max_seqlen=T)
        if e:
            e[2].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    evs = [[ev() for _ in range(3)] for _ in range(steps)]
    n0 = kda.kda_launch_count()
    for i in range(steps):
        step(evs[i])
    launches = (kda.kda_launch_count() - n0) // steps
    torch.cuda.synchronize()
    ms = statistics.median(e[0].elapsed_time(e[2]) for e in evs)
    ms_gemm = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    n_in = 4 * H * d + H + r
    flops = 2 * T * hidden * n_in + 2 * T * r * H * d
    _, tc, tc_sus, peak_kind = measured_peaks()
    ach = flops / (ms_gemm / 1e3) / 1e12
    return {'value': T / (ms / 1e3), 'unit': 'tokens/s',
            'workload': f'layer from hidden states: B=1 T={T} H={H} d={d} hidden={hidden} gate '
                        f'rank {r}; fused input projection [{n_in} x {hidden}] + g_b '
                        f'[{H * d} x {r}] (random-init bf16 weights) + KDA layer',
            'ms_per_step': ms, 'ms_projections': ms_gemm, 'ms_layer': ms - ms_gemm,
            'launches_per_step': launches,
            'tensor_roofline': {'bound': 'tensor', 'kernel': 'kda_proj_gemm (2 launches)',
                                'achieved': ach, 'peak': tc, 'unit': 'TFLOP/s',
                                'frac': ach / tc, 'frac_sustained': ach / tc_sus,
                                'gflop_per_step': flops / 1e9, 'peak_kind': peak_kind,
                                'traffic_fused_projection': profiled_traffic('proj_gemm')}}


def run_long(torch, kda, synth, dev, steps=5, warmup=3):
    """The long / varlen prefill workload: one B = 1, T = 131,072 sequence, and 8 packed
    sequences of log-uniform lengths in [1,024, 32,768]; H = 32, d = 128, bf16, initial
    state N(0, 0.01).  Inputs are drawn on the device from a seeded generator with the
    recipe's distributions (the timing does not depend on the values)."""
    H, d, K = 32, 128, 4
    cfg = kda.Config(num_heads=H, head_dim=d, conv_size=K, dtype=torch.bfloat16, chunk_size=64)
    P = {k: v.to(dev) for k, v in synth.layer_params(4, H, d, K).items()}
    hbm, _, _, peak_kind = measured_peaks()
    gen = torch.Generator(device=dev)
    gen.manual_seed(4)
    out = {}
    for name, lens in (('single_131k', [131072]), ('packed_8', synth.varlen_lengths(4))):
        N, T = len(lens), sum(lens)
        cu = torch.tensor([0] + list(__import__('itertools').accumulate(lens)),
                          dtype=torch.int32, device=dev)
        rnd = lambda *shape: torch.randn(*shape, generator=gen, device=dev).to(cfg.dtype)
        x, f, bl, g = rnd(T, H, 3 * d), rnd(T, H, d), rnd(T, H), rnd(T, H, d)
        s0 = torch.randn(N, H, d, d, generator=gen, device=dev) * 0.1
        state = torch.empty_like(s0)
        y = torch.empty(T, H, d, dtype=cfg.dtype, device=dev)
        ws = torch.empty(kda.kda_layer_prefill_workspace_size(cfg, N, T), dtype=torch.uint8,
                         device=dev)
        stream = torch.cuda.current_stream()

        def ev():
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)            # torch creates the CUDA event on first record
            return e

        evs = [[ev() for _ in range(4)] for _ in range(steps)]

        def step(e=None, c=cfg):
            if e:
                e[0].record(stream)
                kda.kda_set_phase_events(e[1:])
            kda.kda_layer_prefill(c, cu, x, f, bl, g, P['conv_w'], P['A_log'], P['dt_bias'],
                                  P['norm_w'], state_in=s0, state_out=state, y=y, workspace=ws,
                                  max_seqlen=max(lens))
            if e:
                kda.kda_set_phase_events(())

        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        n0 = kda.kda_launch_count()
        for i in range(steps):
            step(evs[i])
        launches = (kda.kda_launch_count() - n0) // steps
        torch.cuda.synchronize()
        ms = statistics.median(e[0].elapsed_time(e[3]) for e in evs)
        method = layer_method_bytes(T, N, H, d)
        ach = method / (ms / 1e3) / 1e9

        def breakdown(ev_list, n_launch):
            if n_launch == 1:
                return {'prefill_cosched': statistics.median(e[0].elapsed_time(e[1])
                                                             for e in ev_list)}
            return {'intra_chunk': statistics.median(e[0].elapsed_time(e[1]) for e in ev_list),
                    'inter_chunk': statistics.median(e[1].elapsed_time(e[2]) for e in ev_list)}

        rec = {'value': T / (ms / 1e3), 'unit': 'tokens/s', 'tokens': T, 'n_seqs': N,
               'max_seqlen': max(lens), 'ms_per_step': ms,
               'breakdown_ms': breakdown(evs, launches),
               'launches_per_step': launches,
               'roofline': {'bound': 'hbm', 'achieved': ach, 'peak': hbm, 'unit': 'GB/s',
                            'frac': ach / hbm, 'peak_kind': peak_kind,
                            'algorithmic_bytes_per_launch': method}}
        if launches == 1:
            # beside it: the two passes as separate launches (for one sequence, the inter-chunk
            # pass over the serial chunks gives the 4-slice chain period)
            c_sep = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_SEPARATE_PASSES)
            for _ in range(warmup):
                step(c=c_sep)
            evs2 = [[ev() for _ in range(4)] for _ in range(steps)]
            for i in range(steps):
                step(evs2[i], c=c_sep)
            torch.cuda.synchronize()
            bd = breakdown(evs2, 2)
            rec['separate_passes'] = {
                'ms_per_step': statistics.median(e[0].elapsed_time(e[3]) for e in evs2),
                'breakdown_ms': bd}
            if N == 1:
                rec['separate_passes']['chain_us_per_chunk'] = bd['inter_chunk'] * 1e3 / (-(-T // 64))
            # the co-scheduled chains run one CTA per head, all value columns; the step is
            # bound by the intra-chunk pass on the remaining SMs, not by the chain
        elif N == 1:
            rec['chain_us_per_chunk'] = rec['breakdown_ms']['inter_chunk'] * 1e3 / (-(-T // 64))
        out[name] = rec
        del x, f, bl, g, y, ws, state, s0
        torch.cuda.empty_cache()
    out['workload'] = ('long/varlen prefill: one B=1 T=131072 sequence, and 8 packed sequences '
                       'of log-uniform lengths in [1024, 32768]; H=32 d=128 chunk 64 bf16, '
                       'initial state N(0, 0.01)')
    return out


def hbm_roofline(kernel, alg_bytes, ms_launch, hbm, peak_kind, note=None):
    """HBM roofline of a state-streaming kernel.  `frac` uses the ncu DRAM bytes of the
    committed summary while the kernel's code is unchanged (the state can partly hit in
    the 126 MB L2 between launches, so bytes / time alone can overstate), otherwise the
    algorithmic bytes; `frac_basis` says which.  Both figures are given."""
    traffic = profiled_traffic(kernel)
    alg = alg_bytes / (ms_launch / 1e3) / 1e9
    dram = traffic / (ms_launch / 1e3) / 1e9 if traffic else None
    out = {'bound': 'hbm', 'kernel': kernel, 'achieved': dram if dram else alg, 'peak': hbm,
           'unit': 'GB/s', 'frac': (dram if dram else alg) / hbm,
           'frac_basis': 'ncu DRAM bytes' if dram else 'algorithmic bytes',
           'frac_algorithmic': alg / hbm, 'frac_dram': dram / hbm if dram else None,
           'traffic': traffic, 'peak_kind': peak_kind,
           'algorithmic_bytes_per_launch': alg_bytes, 'ms_per_launch': ms_launch}
    if note:
        out['note'] = note
    return out


def run_decode(torch, kda, synth, dev, steps=1024):
    """Batched decode: B=64, H=32, d=128, 512-token prefill then `steps` single-token steps."""
    B, H, d, K, T0 = 64, 32, 128, 4, 512
    cfg = kda.Config(num_heads=H, head_dim=d, conv_size=K, dtype=torch.bfloat16, chunk_size=64)
    P = {k: v.to(dev) for k, v in synth.layer_params(2, H, d, K).items()}
    A = {k: v.to(dev) for k, v in synth.layer_activations(2, [T0] * B, H, d, torch.bfloat16).items()}
    state = torch.zeros(B, H, d, d, device=dev)
    conv = torch.zeros(B, K - 1, H, 3 * d, dtype=cfg.dtype, device=dev)
    kda.layer_prefill(cfg, P, A, state_in=state, state_out=state, conv_state=conv)
    # step inputs: sequence b's `steps` tokens drawn as one sequence, laid out [step, b]
    S = synth.layer_activations(2, [steps] * B, H, d, torch.bfloat16, tag='decode_steps')
    X = {k: S[k].view(B, steps, *S[k].shape[1:]).transpose(0, 1).contiguous().to(dev)
         for k in ('x', 'f', 'beta_logit', 'g')}
    cu = torch.arange(B + 1, dtype=torch.int32, device=dev)
    o = {'q': torch.empty(B, H, d, device=dev), 'k': torch.empty(B, H, d, device=dev),
         'v': torch.empty(B, H, d, device=dev),
         'log_a': torch.empty(B, H, d, device=dev), 'beta': torch.empty(B, H, device=dev)}
    y = torch.empty(steps, B, H, d, dtype=cfg.dtype, device=dev)

    def fused(i):
        # one launch: conv against the conv state (advanced in place), SiLU, norms, gate,
        # beta and the state step
        kda.kda_layer_decode(cfg, X['x'][i], X['f'][i], X['beta_logit'][i], X['g'][i],
                             P['conv_w'], P['A_log'], P['dt_bias'], P['norm_w'], state,
                             conv_state=conv, y=y[i])

    # beside it: the decode kernel streaming the state while kda_prep (which never writes
    # it) finishes (KDA_LAUNCH_EARLY_STATE)
    cfg_early = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_EARLY_STATE)

    def two_call(i, c_step=cfg):
        kda.kda_prep(cfg, cu, X['x'][i], X['f'][i], X['beta_logit'][i], P['conv_w'], P['A_log'],
                     P['dt_bias'], conv_state=conv, max_seqlen=1, out=o)
        kda.kda_decode(c_step, o['q'], o['k'], o['v'], o['log_a'], o['beta'], X['g'][i],
                       P['norm_w'], state, y=y[i])

    def graph_ms(one):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            one(0)                  # warm (also loads the kernels)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                one(i)
        g.replay()                  # warm
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1)

    # the two-call step (kda_prep, then kda_decode) is timed first and is the headline: on
    # B200 it is faster than the one-launch kda_layer_decode, timed beside it
    ms = graph_ms(two_call)
    ms_early = graph_ms(lambda i: two_call(i, cfg_early))
    ms_fused = graph_ms(fused)
    # the decode kernel alone: back-to-back launches on resident inputs
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 200
    dec = lambda: kda.kda_decode(cfg, o['q'], o['k'], o['v'], o['log_a'], o['beta'], X['g'][0],
                                 P['norm_w'], state, y=y[0])
    for _ in range(3):
        dec()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(n):
        dec()
    e1.record()
    torch.cuda.synchronize()
    ms_k = e0.elapsed_time(e1) / n
    # per (b, h): state read + written; q, k, v, log a (fp32), beta in; g in, y out (bf16)
    bytes_k = B * H * (2 * d * d * 4 + 4 * d * 4 + 4 + d * 2 + d * 2)
    hbm, _, _, peak_kind = measured_peaks()
    return {'value': B * steps / (ms / 1e3), 'unit': 'tokens/s',
            'workload': f'decode B={B} H={H} d={d}, {steps} steps after a {T0}-token prefill '
                        '(kda_prep + kda_decode per step, CUDA graph)',
            'ms_per_step': ms / steps, 'gpu_launches': 2 * steps,
            'early_state_ms_per_step': ms_early / steps,
            'fused_ms_per_step': ms_fused / steps,
            'roofline': hbm_roofline('kda_decode', bytes_k, ms_k, hbm, peak_kind,
                                     'state 134 MB is just above L2 (126 MB)')}


def run_verify(torch, kda, synth, dev, rounds=256):
    """Speculative verify: B=16, H=32, d=128, 4,096-token context, blocks of 8, `rounds` rounds."""
    B, H, d, K, T0, Tb = 16, 32, 128, 4, 4096, 8
    cfg = kda.Config(num_heads=H, head_dim=d, conv_size=K, dtype=torch.bfloat16, chunk_size=64)
    P = {k: v.to(dev) for k, v in synth.layer_params(3, H, d, K).items()}
    A = {k: v.to(dev) for k, v in synth.layer_activations(3, [T0] * B, H, d, torch.bfloat16).items()}
    state = torch.zeros(B, H, d, d, device=dev)
    conv = torch.zeros(B, K - 1, H, 3 * d, dtype=cfg.dtype, device=dev)
    kda.layer_prefill(cfg, P, A, state_in=state, state_out=state, conv_state=conv)
    D = synth.layer_activations(3, [rounds * Tb] * B, H, d, torch.bfloat16, tag='drafts')
    X = {k: D[k].view(B, rounds, Tb, *D[k].shape[1:]).transpose(0, 1).contiguous().to(dev)
         for k in ('x', 'f', 'beta_logit', 'g')}
    acc = synth.accepted_lengths(3, rounds, B, Tb).to(dev)
    cu = (torch.arange(B + 1, dtype=torch.int32, device=dev) * Tb)
    o = {'q': torch.empty(B * Tb, H, d, device=dev), 'k': torch.empty(B * Tb, H, d, device=dev),
         'v': torch.empty(B * Tb, H, d, device=dev),
         'log_a': torch.empty(B * Tb, H, d, device=dev), 'beta': torch.empty(B * Tb, H, device=dev)}
    win = torch.empty(B * (Tb + K - 1), H, 3 * d, dtype=cfg.dtype, device=dev)
    tape = torch.empty(B, Tb, H, d, d, device=dev)
    kua = torch.empty(B, Tb, H, 3, d, device=dev)
    y = torch.empty(B, Tb, H, d, dtype=cfg.dtype, device=dev)
    v4 = lambda t, *tail: t.view(B, Tb, *tail)
    vargs = lambda r: (v4(o['q'], H, d), v4(o['k'], H, d), v4(o['v'], H, d),
                       v4(o['log_a'], H, d), v4(o['beta'], H), X['g'][r], P['norm_w'], state)

    win4 = win.view(B, Tb + K - 1, H, 3 * d)
    xb = lambda r, key, *tail: X[key][r].view(B, Tb, *tail)

    # verify and the replay stream the state while the kernel before them (kda_prep,
    # kda_verify_compact; neither writes it) finishes
    cfg_early = dataclasses.replace(cfg, launch_flags=kda.KDA_LAUNCH_EARLY_STATE)

    def one(r, mode):
        ce = cfg if mode == 'compact_wait' else cfg_early
        if mode == 'fused':
            # one launch for prep + verify (compact tape), then the replay rollback
            kda.kda_layer_verify_compact(cfg, xb(r, 'x', H, 3 * d), xb(r, 'f', H, d),
                                         xb(r, 'beta_logit', H), X['g'][r], P['conv_w'],
                                         P['A_log'], P['dt_bias'], P['norm_w'], state,
                                         conv_state=conv, tape_kua=kua, window=win4, y=y)
            kda.kda_rollback_replay(ce, acc[r], kua, state, conv_window=win4, conv_state=conv)
            return
        # prep (conv window for the rollback), verify, rollback to the accepted prefix
        kda.kda_prep(cfg, cu, X['x'][r].view(B * Tb, H, 3 * d), X['f'][r].view(B * Tb, H, d),
                     X['beta_logit'][r].view(B * Tb, H), P['conv_w'], P['A_log'], P['dt_bias'],
                     conv_state=conv, conv_mode=kda.KDA_CONV_TAPE, conv_window=win,
                     max_seqlen=Tb, out=o)
        if mode in ('compact', 'compact_wait'):
            kda.kda_verify_compact(ce, *vargs(r), tape_kua=kua, y=y)
            kda.kda_rollback_replay(ce, acc[r], kua, state, conv_window=win, conv_state=conv)
        else:
            kda.kda_verify(ce, *vargs(r), tape=tape, y=y)
            kda.kda_rollback(cfg, acc[r], tape, state, conv_window=win, conv_state=conv)

    def graph_ms(mode):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            one(0, mode)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(rounds):
                one(r, mode)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1)

    def launch_ms(fn, n=100):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    # the three-call round (kda_prep, kda_verify_compact, kda_rollback_replay) is timed first
    # and is the headline: on B200 it is faster than the two-call round with the prep fused
    # (kda_layer_verify_compact), timed beside it with the full-state tape round
    ms = graph_ms('compact')
    ms_wait = graph_ms('compact_wait')
    ms_fused = graph_ms('fused')
    ms_full = graph_ms('full')
    ms_k = launch_ms(lambda: kda.kda_verify_compact(cfg, *vargs(0), tape_kua=kua, y=y))
    ms_r = launch_ms(lambda: kda.kda_rollback_replay(cfg, acc[0], kua, state, conv_window=win,
                                                     conv_state=conv))
    # per (b, h): the state in; per draft q, k, v, log a (fp32), beta, g in; y and the
    # compact tape (3 d fp32) out
    io = Tb * (4 * d * 4 + 4 + d * 2 + d * 2 + 3 * d * 4)
    bytes_k = B * H * (d * d * 4 + io)
    n_acc = int((acc[0] > 0).sum())
    bytes_r = n_acc * H * (2 * d * d * 4) + int(acc[0].sum()) * H * 3 * d * 4
    hbm, _, _, peak_kind = measured_peaks()
    return {'value': B * Tb * rounds / (ms / 1e3), 'unit': 'verified draft tokens/s',
            'workload': f'verify+rollback B={B} H={H} d={d}, blocks of {Tb} after a {T0}-token '
                        f'context, {rounds} rounds, accepted ~ U{{0..{Tb}}} (CUDA graph; '
                        'kda_prep, kda_verify_compact with the compact (k, u, a) tape, '
                        'kda_rollback_replay; verify and replay stream the state while the '
                        'kernel before them finishes)',
            'ms_per_round': ms / rounds, 'gpu_launches': 3 * rounds,
            'state_after_previous_ms_per_round': ms_wait / rounds,
            'fused_prep_ms_per_round': ms_fused / rounds,
            'full_state_tape_ms_per_round': ms_full / rounds,
            'roofline': hbm_roofline('kda_verify_compact', bytes_k, ms_k, hbm, peak_kind),
            'rollback_replay': {'ms_per_launch': ms_r, 'algorithmic_bytes_per_launch': bytes_r,
                                'frac': bytes_r / (ms_r / 1e3) / 1e9 / hbm}}


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(torch, synth, heads=32, tokens=2048, seed=1):
    """Units for the oracle: each head of the headline workload over a token prefix."""
    H, d, K = 32, 128, 4
    P = synth.layer_params(seed, H, d, K)
    A = synth.layer_activations(seed, [tokens], H, d, torch.bfloat16)
    np64 = lambda t: t.to(torch.float64).numpy()
    units = []
    for h in range(heads):
        units.append((np64(A['x'][:, h:h + 1]), np64(A['f'][:, h:h + 1]),
                      np64(A['beta_logit'][:, h:h + 1]), np64(A['g'][:, h:h + 1]),
                      np64(P['conv_w'][h:h + 1]), np64(P['A_log'][h:h + 1]),
                      np64(P['dt_bias'][h:h + 1]), np64(P['norm_w']),
                      A['cu_seqlens'].numpy()))
    return units


def cpu_baseline(torch, synth, heads=32, tokens=4096):
    from oracle import baseline
    units = oracle_sample(torch, synth, heads, tokens)
    wall, workers = baseline.time_units(units)
    token_heads = heads * tokens
    return {'value': token_heads / 32 / wall, 'unit': 'tokens/s', 'cores': workers,
            'kind': 'oracle',
            'sample': f'float64 oracle layer (prep + token loop + gated RMSNorm) on {heads} of 32 '
                      f'heads x the first {tokens} tokens of the headline workload, one head per '
                      f'process; value scaled to whole tokens (all 32 heads)',
            'wall_s': wall, 'cpu_s': wall * workers}


def run_reference(args, dist):
    if dist.rank != 0:
        return None
    import torch
    from linear_attention_recurrence_09_b200 import synth
    from oracle import baseline
    units = oracle_sample(torch, synth, heads=32, tokens=256)
    wall, workers = baseline.time_units(units[:1])          # warm
    walls = []
    for i in range(args.warmup + args.steps):
        w, workers = baseline.time_units(units)
        if i >= args.warmup:
            walls.append(w)
    tps = 256 / statistics.mean(walls)
    cb = {'value': tps, 'unit': 'tokens/s', 'cores': workers, 'kind': 'oracle',
          'sample': 'float64 oracle on all 32 heads x the first 256 tokens of the headline '
                    'workload per step, one head per process'}
    return {'impl': 'reference', 'metric': METRIC, 'value': tps, 'unit': 'tokens/s',
            'n_gpus': dist.world, 'steps': args.steps, 'warmup': args.warmup,
            'ms_per_step': statistics.mean(walls) * 1e3, 'higher_is_better': True,
            'scaling': 'weak', 'vs_baseline': None, 'dtype': 'f64', 'data': 'synthetic',
            'config': prefill_config(8192, 32, 128, dist.world),
            'cpu_baseline': cb,
            'e2e': {'value': tps, 'unit': 'tokens/s', 'h2d_bytes_per_step': 0,
                    'd2h_bytes_per_step': 0}}


def main():
    args = parse_args()
    dist = Dist()
    try:
        if args.impl == 'reference':
            res = run_reference(args, dist)
            if res is not None:
                print(json.dumps(res))
            return
        import torch
        from linear_attention_recurrence_09_b200 import kda, synth
        if not torch.cuda.is_available():
            raise SystemExit('bench.py needs a CUDA GPU (there is no CPU fallback)')
        dev = torch.device('cuda', dist.local)
        torch.cuda.set_device(dev)
        kda.lib()
        res = {}
        if args.only in ('', 'prefill'):
            res = run_prefill(args, dist, torch, kda, synth, dev)
        if dist.world == 1 and not args.no_extras:
            if args.only in ('', 'decode'):
                res['decode'] = run_decode(torch, kda, synth, dev)
            if args.only in ('', 'verify'):
                res['verify'] = run_verify(torch, kda, synth, dev)
            if args.only in ('', 'long') and not args.no_long:
                res['long'] = run_long(torch, kda, synth, dev)
            if args.only in ('', 'layer_full'):
                res['layer_full'] = run_layer_full(torch, kda, synth, dev)
        if dist.rank == 0 and dist.world == 1 and not args.no_cpu and args.only in ('', 'prefill'):
            res['cpu_baseline'] = cpu_baseline(torch, synth)
        if dist.rank == 0:
            print(json.dumps(res))
    finally:
        dist.close()


if __name__ == '__main__':
    main()
