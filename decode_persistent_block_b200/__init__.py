"""Persistent batch-1 decode megakernel for one B200 (sm_100a).

The product is `libmk.so`, a C-ABI library (include/mk.h) whose CUDA kernels
run the whole decode step; `mk` is its thin ctypes binding.
"""
from . import mk
from .build import build
from .mk import Decoder, MkError, load, plan, simulate, to_device

__all__ = ["mk", "build", "Decoder", "MkError", "load", "plan", "simulate", "to_device"]
