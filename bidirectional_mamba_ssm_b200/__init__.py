"""B200 (sm_100a) bidirectional Mamba-2 mixer core behind a small C ABI.

The kernels live in libbimamba.so (built in-tree from csrc/ by
``python -m bidirectional_mamba_ssm_b200.build``); ``_lib`` is the ctypes
binding with the same entry-point names as include/bimamba.h.  The binding
is loaded on first attribute access so that ``inputs`` can be used without
the shared library.
"""
__all__ = ["bimamba_version", "bimamba_launch_count", "bimamba_set_timing_events", "bimamba_strerror", "bimamba_get_error", "bimamba_conv_silu",
           "bimamba_workspace_bytes", "bimamba_ssd_fwd_rev", "bimamba_block_decode",
           "make_dims", "new_workspace", "BimambaError",
           "bimamba_noalloc_scratch_bytes", "bimamba_block_decode_noalloc"]


def __getattr__(name):
    if name in __all__:
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)
