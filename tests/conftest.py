import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The largest errors the parity checks measured in this session, beside
    their bounds: O max-abs against the oracle rounded to bf16 (no allowance)
    and beyond half a bf16 spacing (the bound's reading), LSE max-abs,
    gradient relative Frobenius errors."""
    try:
        from tests.parity import GRAD_REL_FROB, LSE_ABS, O_MAX_ABS, O_REL_FROB, RECORD
    except ImportError:
        return
    if not RECORD:
        return
    tr = terminalreporter
    tr.section("parity errors (largest measured in this session)")

    def worst(kinds, key):
        rows = [(m[key], what) for k, what, m in RECORD if k in kinds and key in m]
        return max(rows) if rows else None

    lines = [
        ("O max-abs vs bf16(oracle)", worst(("O",), "max_abs_vs_bf16_oracle"), None),
        ("O max-abs beyond half a bf16 spacing", worst(("O",), "max_abs_beyond_half_ulp"), O_MAX_ABS),
        ("O rel-frob vs bf16(oracle)", worst(("O",), "rel_frob"), O_REL_FROB),
        ("LSE max-abs", worst(("LSE",), "max_abs"), LSE_ABS),
        ("dQ rel-frob", worst(("dq",), "rel_frob"), GRAD_REL_FROB),
        ("dK rel-frob", worst(("dk",), "rel_frob"), GRAD_REL_FROB),
        ("dV rel-frob", worst(("dv",), "rel_frob"), GRAD_REL_FROB),
    ]
    for label, w, bound in lines:
        if w is None:
            continue
        b = f" (bound {bound:g})" if bound is not None else ""
        tr.write_line(f"{label}: {w[0]:.3e}{b} at {w[1]}")
    tr.write_line(f"{len(RECORD)} comparisons")
