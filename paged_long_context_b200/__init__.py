"""B200 (sm_100a) paged decode attention behind a small C ABI.

    from paged_long_context_b200 import binding, synth
    bufs = binding.paged_decode(case)       # case: synth.DecodeCase on a CUDA device

The CUDA library libcfr_paged.so is built in-tree by
``python -m paged_long_context_b200.build``; the binding loads it on first
use and refuses to run without it (there is no CPU fallback).
"""
from . import accounting, binding, synth  # noqa: F401

__all__ = ["accounting", "binding", "synth"]
