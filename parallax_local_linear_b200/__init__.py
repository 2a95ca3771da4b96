"""Parallax attention (parameterized Local Linear Attention) for B200.

The compute lives in ``libparallax.so`` (hand-written sm_100a CUDA behind a
C ABI, declared in ``include/parallax.h``); ``binding`` marshals torch
tensors into that ABI.  Importing the package does not load the library;
the first use of ``decode`` / ``prefill`` does, and raises if it is missing.
"""

__all__ = ["decode", "prefill", "decode_workspace_size", "last_device_error",
           "decode_noalloc", "lib"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
