"""SAS gated block-sparse attention for B200 (sm_100a).

The compute lives in ``libsas.so`` (hand-written CUDA behind a C ABI declared in
``include/sas.h``).  ``trainable_block_sparse_sas_b200.api`` is the thin ctypes
binding with the same entry-point names; importing it loads the library and
raises if it has not been built.  ``synthetic`` draws the seeded inputs.
"""
import importlib

__all__ = ["api", "synthetic"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
