"""B200-native hot path of Veda block-sparse attention.

The six steps run in ``libveda.so`` (CUDA kernels for sm_100a behind the C ABI of
``include/veda.h``); ``veda`` is its ctypes binding. Build the library with
``python -m block_sparse_attention_max_b200.build``.
"""
from . import veda  # noqa: F401
from .veda import (  # noqa: F401
    VedaError, block_scores, block_sparse_attn_fwd, build_tile_map, check_device_status,
    geometry_sizes, permute_tiles, select_blocks, sparse_attention, tile_pool, unpermute,
)
