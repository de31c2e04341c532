"""Hybrid-precision attention (HyQuant's hot path) for NVIDIA B200 (sm_100a).

The compute lives in ``libhq.so`` (hand-written CUDA, C ABI declared in
``include/hq.h``); :mod:`.hq` is the thin Python binding over it and
:mod:`.synth` draws the seeded synthetic workloads.
"""
__all__ = ["hq", "synth"]
