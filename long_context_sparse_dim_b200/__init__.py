"""B200-native RTPurbo sparse attention: 16-dim indexer, dynamic top-p, sparse and window attention.

The compute runs in ``librtp.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/rtp.h``); :mod:`.rtp` is the thin ctypes binding and
:mod:`.workloads` draws seeded synthetic inputs.
"""
__all__ = ["rtp", "workloads"]
