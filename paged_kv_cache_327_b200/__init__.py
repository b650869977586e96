"""Paged KV-cache decode attention for B200 (sm_100a).

The hot path -- copy_blocks, reshape_and_cache and split-K paged decode attention --
runs in hand-written CUDA kernels behind the C ABI declared in ``include/pa.h``
(``libpa.so``).  The names below marshal torch tensors into that ABI; importing them
fails loudly when the library has not been built.  ``block_manager`` (refcounted
block pool and tables) and ``workload`` (seeded synthetic decode steps) are host-only.
"""
from . import block_manager, workload  # noqa: F401

_BINDING_NAMES = (
    "pa_decode", "pa_reshape_and_cache", "pa_copy_blocks", "pa_decode_workspace_size",
    "pa_strerror", "pa_get_device_error", "PAError", "DecodeWorkspace", "load_library",
    "device_workload", "run_step",
)


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
