"""ZHA (Zyphra Hierarchical Attention) decode on NVIDIA B200: Python binding of libzha.so.

The compute path is the CUDA library built from csrc/ (see include/zha.h);
this package only marshals arguments to it.
"""
from .zha import (  # noqa: F401
    DenseDecoder, LevelLayout, ZhaConfig, ZhaError, ZhaTree, dense_decode, dense_scratch_bytes, lib,
    make_config, tree_bytes, tree_layout, launch_count, LIB_PATH, ZHA_BF16, ZHA_F32, STAT_NODES_SCORED,
    STAT_LEAVES_KEPT, STAT_KEYS, STAT_STEPS,
)
