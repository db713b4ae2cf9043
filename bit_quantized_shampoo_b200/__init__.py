"""B200 4-bit Shampoo preconditioner (libshampoo4.so + a thin PyTorch binding)."""
from . import _lib  # noqa: F401

__all__ = ["Shampoo4", "quant4_pack", "quant4_unpack", "quant4_tables", "update_stats_noalloc"]


def __getattr__(name):
    if name in __all__:
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
