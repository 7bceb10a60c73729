"""VideoMLA latent-window attention for B200 (sm_100a): libmla.so and its ctypes binding.

The compute path lives in csrc/ (CUDA kernels behind the C ABI of include/mla.h); binding.py
marshals torch tensors and streams into those calls.  Build with build.py.
"""
from .binding import (  # noqa: F401
    EXPORTED, LatentWindowCache, MLAError, load_library, make_config, mla_cache_append, mla_cache_commit, mla_commit_plan,
    mla_cache_copy_buffer, mla_cache_create, mla_cache_debug_buffers, mla_cache_destroy,
    mla_cache_device_bytes, mla_cache_profile_enable, mla_cache_profile_read, mla_cache_read,
    mla_cache_state, mla_cache_sync, mla_config, mla_config_check, mla_ring_bytes, mla_ring_slot, mla_cache_slot, mla_cache_bytes,
    mla_window_attention, mla_window_attention_noalloc, mla_dense_attention, mla_dense_sync,
    mla_cache_selftest_timeout, mla_cache_selftest_bounds,
    mla_dense_workspace_bytes, MLA_OK, MLA_ERR_INVALID_ARGUMENT, MLA_ERR_UNSUPPORTED,
    MLA_ERR_OUT_OF_MEMORY, MLA_ERR_CUDA, MLA_ERR_DEVICE_TIMEOUT, MLA_ERR_STATE, MLA_ERR_RANGE, MLA_ERR_BOUNDS,
)
