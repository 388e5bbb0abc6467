"""Ragged paged attention for NVIDIA B200 (sm_100a).

The compute path is the native library ``librpa.so`` (C ABI declared in ``include/rpa.h``);
``api`` is a thin ctypes binding over it.  Importing this package does not load the library;
the first call into ``api`` does, and raises if the library is missing.
"""
__all__ = ["api", "workloads"]
