"""B200-native Mamba-2 SSD forward scan.

The compute lives in ``libssd.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/ssd.h``).  This package is the thin Python binding:
``forward`` marshals torch tensors into the C call and nothing else.  Importing
the package does not load the library; the first call does, and fails loudly if
the library is missing.
"""
from __future__ import annotations

__all__ = ["forward", "forward_ws", "workspace_bytes", "workspace_layout", "lib_path",
           "SSDError"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
