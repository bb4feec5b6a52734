"""Attention forward + backward on inputs in host memory, with the PCIe copies
overlapped with the kernels: the Python face of the C entry point
fa_fwd_bwd_host (argument marshalling only; the pipeline -- head groups
through copy-in, kernels and copy-out on the library's own streams -- runs in
the library).
"""
from __future__ import annotations

from .fa import forward_backward_host, host_workspace_bytes

__all__ = ["forward_backward_host", "host_workspace_bytes"]
