"""B200-native ClusterKV-style semantic cluster recall.

The compute path lives in ``libckv.so`` (CUDA for sm_100a behind a C ABI,
declared in ``include/ckv.h``); :mod:`semantic_cluster_recall_b200.ckv` is
its thin ctypes binding. Importing the package loads nothing: the library is
loaded on first use of the binding and fails loudly if it is missing.
"""
__all__ = ["ckv", "synth"]
