import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


# Per-configuration statistics that parity tests record (near-tie counts,
# tolerated code differences, Gram errors), printed after the run even under
# -q, where passing tests' output is captured.
PARITY_STATS = []


def record_stat(config_name, **values):
    PARITY_STATS.append((config_name, values))


def pytest_terminal_summary(terminalreporter):
    if not PARITY_STATS:
        return
    terminalreporter.write_sep("-", "parity statistics per configuration")
    for name, values in PARITY_STATS:
        terminalreporter.write_line(
            "%s: %s" % (name, ", ".join("%s=%s" % kv for kv in values.items())))


def bf16_bits(t):
    """uint16 numpy view of a bf16 torch tensor (any device)."""
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(u16):
    u = np.asarray(u16, np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):
        return u.view(np.float32).astype(np.float64)


def f32_to_bf16_bits(a):
    """Round fp32 values to bf16 (nearest even) and return the bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.lib()
    return oracle
