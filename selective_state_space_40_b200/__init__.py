"""B200-native (sm_100a) Mamba selective scan and selective state update.

The compute lives in ``libmambascan.so`` (hand-written CUDA behind a C ABI,
declared in ``include/mambascan.h``); ``binding`` is a thin ctypes layer with
the same entry-point names. The library is loaded on first use and a missing
or unloadable library raises: there is no CPU fallback.
"""
__all__ = ["binding", "synthetic"]
