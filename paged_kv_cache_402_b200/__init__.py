"""Paged KV-cache decode path for B200 (sm_100a).

The public names (``pa_append_kv``, ``pa_decode``, ``pa_copy_blocks``,
``Allocator``, ``KVCache``, ...) live in :mod:`.binding`, the ctypes binding of
libpagedattn.so; they are loaded on first use, so that ``.build`` (which
compiles the library) and ``.synth`` (seeded inputs) can be imported without
it.  Using any binding name without the built library raises ImportError.
"""
from __future__ import annotations

import importlib


def __getattr__(name):
    if name.startswith("__"):
        raise AttributeError(name)
    binding = importlib.import_module(".binding", __name__)
    try:
        return getattr(binding, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
