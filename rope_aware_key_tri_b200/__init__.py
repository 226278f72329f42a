"""B200 (sm_100a) TriAttention KV-cache scoring-and-pruning pass.

The compute lives in the CUDA library ``lib/libtri_b200.so`` behind the C ABI of
``include/tri.h``; :mod:`rope_aware_key_tri_b200.tri` is its ctypes binding and
loads the library on import (it raises if the library is missing: there is no
fallback path). Attribute access on this package imports the binding lazily so
that ``build.py`` can run before the library exists.
"""

__all__ = ["TriContext", "TriError", "make_kv", "tri"]


def __getattr__(name):
    import importlib
    if name in ("TriContext", "TriError", "make_kv"):
        return getattr(importlib.import_module(".tri", __name__), name)
    if name == "tri":
        return importlib.import_module(".tri", __name__)
    raise AttributeError(name)
