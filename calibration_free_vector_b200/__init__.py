"""NSNQuant KV-cache hot path for B200 (sm_100a): a C-ABI CUDA library
(include/nsn.h, libnsn.so) and its thin Python binding (`nsn`)."""
from . import nsn  # noqa: F401  (the library itself is loaded lazily on first use)

__all__ = ["nsn"]
