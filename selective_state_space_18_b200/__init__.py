"""B200-native Mamba-1 selective scan (S6) forward and decode state update.

The compute path lives in the CUDA library ``libssscan.so`` (sources under
``csrc/``, C declarations in ``include/ss_scan.h``).  ``ssscan`` is the thin ctypes
binding over it; ``inputs`` holds the seeded synthetic workload generators.
Importing the package loads nothing; the library is loaded on the first call.
"""
__all__ = ["ssscan", "inputs"]
