"""B200-native (sm_100a) Video Sparse Attention forward.

The compute lives in ``libvsa.so`` (CUDA, C ABI in ``include/vsa.h``); this
package is its Python binding plus the seeded input generator
(:mod:`.inputs`).  Build the library with
``python -m block_sparse_attention_15_b200.build``.
"""
from .binding import (  # noqa: F401
    VSAError,
    block_sparse_attn,
    block_sparse_attn_backward,
    block_sparse_attn_from_indices,
    block_sparse_attn_varlen,
    block_sparse_attn_varlen_backward,
    build_vsa_metadata,
    check_device_status,
    gather_tokens,
    get_device_status,
    lib,
    scatter_tokens,
    vsa_forward,
    vsa_forward_host,
    video_sparse_attn_bshd,
)

__all__ = [
    "VSAError", "block_sparse_attn", "block_sparse_attn_backward",
    "block_sparse_attn_from_indices", "block_sparse_attn_varlen_backward", "block_sparse_attn_varlen", "build_vsa_metadata",
    "check_device_status", "gather_tokens", "get_device_status", "lib", "scatter_tokens",
    "vsa_forward", "vsa_forward_host", "video_sparse_attn_bshd",
]
