"""B200-native absorbed Multi-Head Latent Attention decode over a paged latent KV cache.

The compute path is hand-written CUDA for sm_100a behind the C-ABI library
``libmla.so`` (declared in ``include/mla.h``); this package is the thin Python
binding (argument marshalling only) plus the seeded input generator and host
size helpers.  The binding loads the library lazily on first use and raises
if it is missing: there is no fallback path.
"""
from . import layout  # noqa: F401

__all__ = ["layout"]
