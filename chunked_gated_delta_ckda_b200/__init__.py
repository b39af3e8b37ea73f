"""B200 (sm_100a) implementation of the Complex KDA (CKDA) recurrence.

The library is ``lib/libckda.so`` (C ABI in include/ckda.h, built by
``python -m chunked_gated_delta_ckda_b200.build``).  ``_abi`` binds it with
the same function names; ``api`` adds tensor-level helpers; ``workloads``
holds the seeded synthetic input generators.
"""
from . import workloads  # noqa: F401

__all__ = ["workloads", "api", "_abi"]


def __getattr__(name):
    # the CUDA binding loads lazily so CPU-only users of ``workloads`` need no library
    if name in ("api", "_abi"):
        import importlib
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
