"""B200 (sm_100a) hot path of context-parallel attention for diffusion transformers.

Ring attention over K/V chunks with an fp32 log-sum-exp merge, the Ulysses
sequence <-> head all-to-all as an on-GPU permutation, and their unified
composition, all running in the hand-written CUDA kernels of libcpattn.so
(C-ABI in include/cpattn.h).  This package is the thin Python binding.
"""
from .binding import (  # noqa: F401
    CpError, attn_partial, attn_partial_merge, lse_merge, ring_attention, ring_attention_gathered,
    ring_chunk_offsets, ulysses_permute,
    usp_attention, usp_workspace_bytes, last_device_error, selftest_wait_timeout,
    selftest_bounds_check, is_debug_build,
    ulysses_anything_permute, ulysses_anything_attention,
    attention_flops, SEQ_TO_HEAD, HEAD_TO_SEQ,
)
