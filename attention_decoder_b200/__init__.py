"""LFM3-1.7B hybrid decoder forward (prefill + batched decode) on one NVIDIA B200.

The compute path is liblfm3.so (hand-written sm_100a kernels behind the C ABI of
include/lfm3.h); this package only loads it and marshals arguments. Importing the package does
not load the library; the first call does, and fails loudly if it has not been built.
"""
from ._lib import SYMBOLS, Lfm3Error, lib  # noqa: F401


def __getattr__(name):
    if name in ("Lfm3Model", "Lfm3State"):
        from . import model
        return getattr(model, name)
    raise AttributeError(name)
