"""B200-native forward scan of a recurrent associative memory written by a gain-weighted residual.

The compute path is the C-ABI library ``libkdn.so`` (hand-written sm_100a CUDA
kernels, declared in ``include/kdn.h``); ``delta_rule_recurrent_scan_b200.kdn``
is the thin ctypes binding over it.  Importing this package loads nothing:
the library is opened on the first call, and a missing library is an error,
never a fallback.
"""

__all__ = ["kdn", "workloads"]
