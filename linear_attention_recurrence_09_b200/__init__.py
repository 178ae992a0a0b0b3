"""KDA (Kimi Delta Attention) layer hot path for NVIDIA B200 (sm_100a).

The compute lives in ``libkda.so`` (CUDA C++, C ABI declared in
``include/kda.h``); :mod:`.kda` is a thin ctypes binding over it.
"""
