"""The five named workloads of this attention path (shapes and value spread).

Each entry is a plain description; nothing here computes attention.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal_modes: tuple
    backward: bool
    sigma_qk: float = 1.0
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    def fwd_flops(self, causal: bool) -> float:
        """4*B*H*N^2*d, halved for causal (the conventional count)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if causal else f

    def bwd_flops(self, causal: bool) -> float:
        """2.5x the forward count."""
        return 2.5 * self.fwd_flops(causal)


WORKLOADS = {
    # single-head small forward, non-causal
    "pr1_b1h1n256d64": Workload("pr1_b1h1n256d64", 1, 1, 256, 64, (False,), False),
    # headline forward shape, both masks
    "fwd_b2h16n4096d128": Workload("fwd_b2h16n4096d128", 2, 16, 4096, 128, (False, True), False),
    # training step, causal
    "train_b4h32n2048d128": Workload("train_b4h32n2048d128", 4, 32, 2048, 128, (True,), True),
    # long sequence, causal (materialised S would be 8 GiB in bf16)
    "long_b1h16n16384d128": Workload("long_b1h16n16384d128", 1, 16, 16384, 128, (True,), True),
    # stability and ragged tails: logits reach hundreds; N not a tile multiple
    "ragged_b8h12n1000d64": Workload("ragged_b8h12n1000d64", 8, 12, 1000, 64, (False, True), True,
                                     sigma_qk=8.0),
}
