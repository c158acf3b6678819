"""B200-native Memory Sparse Attention (MSA) hot path.

The C-ABI libraries (``lib/libmsa_{pool,route,gather,decode,prefill,bank}.so``, declared in
``include/*.h``) are bound in ``abi``; their entry points are re-exported here under the
same names and loaded on first use.  There is no CPU fallback: the first access raises
ImportError if the libraries have not been built (``python top_kv_routing_b200/build.py``).
"""
from __future__ import annotations

import importlib

_SUBMODULES = {"abi", "build", "engine"}


def __getattr__(name: str):
    if name.startswith("__") or name in _SUBMODULES:
        raise AttributeError(name)
    return getattr(importlib.import_module(__name__ + ".abi"), name)
