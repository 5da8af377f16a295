"""Recurrent gated-delta-rule decode step (and long-prompt prefill) for B200 (sm_100a).

The compute path is the C-ABI library ``libgdr.so`` built from ``csrc/``; the
Python functions here only marshal torch tensors into it. Importing the
package does not load the library: the first use of ``decode``,
``decode_gated``, ``prefill``, ``prefill_gated``, ``linear_attention_gate`` or
``lib`` does, and raises if it is missing (there is no CPU fallback).
"""
from __future__ import annotations

__all__ = ["decode", "decode_gated", "prefill", "prefill_gated", "linear_attention_gate",
           "device_error", "GdrError", "lib", "library_path", "last_launch", "kernel_forms"]

_LAZY = {"decode", "decode_gated", "prefill", "prefill_gated", "linear_attention_gate",
         "device_error", "GdrError", "lib", "library_path", "STATUS_NAMES", "last_launch",
         "kernel_forms"}


def __getattr__(name):
    if name in _LAZY:
        from . import binding

        return getattr(binding, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
