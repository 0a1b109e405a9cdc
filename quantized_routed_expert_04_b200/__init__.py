"""Routed int4 expert (MoE) layer for one B200: C-ABI library + thin binding.

Importing the package loads nothing native; the CUDA library is loaded on the
first use of a ``strata_moe_*`` call (see ``binding``), and that load fails
loudly if the library has not been built.
"""
from . import synth  # noqa: F401


def __getattr__(name):
    if name.startswith("strata_") or name in ("StrataError", "load_library", "Status", "StrataMoE"):
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
