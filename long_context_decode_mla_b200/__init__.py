"""B200-native decode-context-parallel (DCP) absorbed-MLA decode.

The compute path lives in ``libdcpmla.so`` (hand-written sm_100a kernels
behind a C ABI, see ``include/dcpmla.h``); :mod:`.dcpmla` is the thin ctypes
binding with the same entry-point names, and :mod:`.workload` draws seeded
synthetic inputs.  Importing the package does not load the library; the first
call into :mod:`.dcpmla` does, and raises if it is missing.
"""
__all__ = ["dcpmla", "workload"]
