"""Branch attention for speculative-draft training, B200-native (sm_100a).

Causal main-sequence attention over a packed, load-balanced zigzag split (R
virtual ranks on one GPU), rank-local branch attention and their online-softmax
(log-sum-exp) merge, forward and backward, in hand-written tcgen05/TMA CUDA
kernels behind the C ABI of include/ba.h (libba_b200.so).  This package is the
thin ctypes binding; PyTorch supplies device memory and streams.
"""
from ._abi import (BA_MASK_BITMASK, BA_MASK_BLOCK, BA_MASK_CHAIN, BA_WS_BWD, BA_WS_FWD, BAError,  # noqa: F401
                   EXPORTED, LIB_PATH, clear_cache, error_word_fields, lib, plan_cache_stats,
                   profile_collect, profile_enable, set_wait_limit, status_string)
from .api import BranchAttention, lse_merge, sync_status  # noqa: F401
