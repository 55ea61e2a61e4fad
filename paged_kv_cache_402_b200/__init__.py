"""Paged KV-cache decode path for B200 (sm_100a).

The public names (``pa_append_kv``, ``pa_decode``, ``pa_copy_blocks``,
``Allocator``, ``KVCache``, ...) live in :mod:`.binding`, the ctypes binding of
libpagedattn.so; they are loaded on first use, so that ``.build`` (which
compiles the library), ``.synth`` (seeded inputs) and ``.trace`` can be
imported without it.  Using any binding name without the built library raises
ImportError.
"""
from __future__ import annotations

import importlib

# Submodules that never load the library.  `from package import build` asks
# this module's __getattr__ first; for these names it must answer
# AttributeError so that Python imports the submodule itself instead of
# loading the binding.
_SUBMODULES = frozenset({"build", "synth", "trace", "binding"})


def __getattr__(name):
    if name.startswith("__") or name in _SUBMODULES:
        raise AttributeError(name)
    binding = importlib.import_module(".binding", __name__)
    try:
        return getattr(binding, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
