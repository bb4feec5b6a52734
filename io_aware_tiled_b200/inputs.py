"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws random tensors.
Recipe (the pages name no generator; this is the plainest reading of
"i.i.d. N(0, sigma^2) from seed s"):

  * ``torch.Generator("cpu").manual_seed(seed)``;
  * draw float32 ``randn`` tensors of shape [B, H, N, d] in the order
    Q, K, V, dO (dO only when requested);
  * multiply Q and K by ``sigma_qk`` (V and dO keep sigma 1);
  * round to bf16 (round to nearest even).

Drawing on the CPU makes the values independent of the device.
"""
from __future__ import annotations

import torch


def attention_inputs(B: int, H: int, N: int, d: int, seed: int = 0, sigma_qk: float = 1.0,
                     with_do: bool = True):
    """Return (q, k, v, do) as contiguous bf16 CPU tensors ([B, H, N, d]);
    ``do`` is None when ``with_do`` is False."""
    if min(B, H, N, d) <= 0:
        raise ValueError("B, H, N and d must be positive")
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32) if with_do else None
    if sigma_qk != 1.0:
        q = q * sigma_qk
        k = k * sigma_qk
    out = [t.to(torch.bfloat16).contiguous() if t is not None else None for t in (q, k, v, do)]
    return tuple(out)
