"""B200-native latent-KV chunk attention (VideoMLA hot path).

The compute path lives in ``libvmla.so`` (CUDA for sm_100a behind a C ABI,
declared in ``include/vmla.h``).  ``api`` is a thin ctypes binding over it;
the library is loaded on first use and its absence is an error.
"""
__all__ = ["api", "synth"]
