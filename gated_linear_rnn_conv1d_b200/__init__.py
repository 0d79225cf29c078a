"""B200-native RG-LRU temporal core: Conv1D(4) → RG-LRU, prefill scan and decode step.

The kernels live in librglru.so (C ABI, include/rglru.h); `rglru` is its Python binding.
Importing the package does not load the library; the first call does, and raises if it
has not been built (there is no fallback path)."""
from . import inputs  # noqa: F401
from . import rglru  # noqa: F401

__all__ = ["inputs", "rglru"]
