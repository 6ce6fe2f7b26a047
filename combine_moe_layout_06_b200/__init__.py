"""B200-native MoE expert-parallel dispatch and combine fused with layout.

The compute path is libmoe_layout.so (CUDA, sm_100a) behind the C ABI in
include/moe_layout.h; :mod:`.capi` is its Python binding, :mod:`.buffers`
allocates device buffers with torch, :mod:`.inputs` draws seeded synthetic
workloads and :mod:`.build` compiles the library.
"""
from . import capi  # noqa: F401  (loads the shared library lazily)

__all__ = ["capi"]
