"""Build libkda.so (the C-ABI library) in-tree with nvcc for sm_100a.

Each CUDA source compiles to its own object under ``_build/`` (in parallel,
skipped when up to date); the objects link into ``libkda.so`` next to this file.
"""
from __future__ import annotations

import glob
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, 'csrc')
LIB = os.path.join(PKG, 'libkda.so')
OBJDIR = os.path.join(ROOT, '_build')

ARCH = ['-gencode', 'arch=compute_100a,code=sm_100a']
CFLAGS = ['-O3', '-lineinfo', '-std=c++17', '--expt-relaxed-constexpr',
          '-Xcompiler', '-fPIC,-O3,-fvisibility=hidden', '-Xptxas', '-warn-spills']


def _nvcc() -> str:
    home = os.environ.get('CUDA_HOME', '/usr/local/cuda')
    cand = os.path.join(home, 'bin', 'nvcc')
    return cand if os.path.exists(cand) else 'nvcc'


def sources():
    return sorted(glob.glob(os.path.join(CSRC, '*.cu')))


def _headers():
    return (glob.glob(os.path.join(CSRC, '*.cuh')) + glob.glob(os.path.join(CSRC, '*.h')) +
            [os.path.join(ROOT, 'include', 'kda.h'), os.path.abspath(__file__)])


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in deps)


def up_to_date() -> bool:
    return not _stale(LIB, sources() + _headers())


def _compile(src, force, extra, verbose):
    obj = os.path.join(OBJDIR, os.path.basename(src)[:-3] + '.o')
    if not force and not _stale(obj, [src] + _headers()):
        return obj, ''
    cmd = [_nvcc(), *ARCH, *CFLAGS, *extra, '-I', os.path.join(ROOT, 'include'),
           '-c', src, '-o', obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError('nvcc failed on %s:\n%s%s' % (src, res.stdout, res.stderr))
    return obj, (' '.join(cmd) + '\n' if verbose else '') + res.stdout + res.stderr


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile every CUDA source and link libkda.so next to this file; return its path."""
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    with ThreadPoolExecutor(max_workers=max(1, min(len(sources()), os.cpu_count() or 1))) as ex:
        results = list(ex.map(lambda s: _compile(s, force, extra, verbose), sources()))
    for _, log in results:
        if log.strip() and verbose:
            print(log)
    tmp = LIB + '.tmp'
    cmd = [_nvcc(), *ARCH, '-shared', '-Xcompiler', '-fPIC', '-o', tmp,
           *[o for o, _ in results]]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError('nvcc link failed:\n' + res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == '__main__':
    import sys
    print(build(force='--force' in sys.argv, verbose=True))
