"""B200-native (sm_100a) tiled, IO-aware exact attention.

The kernels and their C ABI live in ``libfa.so`` (sources under ``csrc/``,
declarations in ``include/fa.h``); ``fa`` is the thin ctypes binding;
``host_pipeline`` runs forward + backward on pinned host tensors with the
PCIe copies overlapped with the kernels.
"""
from .fa import (FaError, attention, backward, forward, last_error_word, load_library, selftest_wait_timeout,
                 status_string, sync_status, workspace_bytes)

__all__ = ["FaError", "attention", "backward", "forward", "last_error_word", "load_library",
           "selftest_wait_timeout", "status_string", "sync_status", "workspace_bytes"]
