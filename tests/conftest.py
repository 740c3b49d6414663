import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU test")


@pytest.fixture(scope="session")
def golden():
    import json
    with open(os.path.join(ROOT, "tests", "golden", "pages.json")) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- shared helpers
import numpy as np


def rel_l2(a, b):
    """||a - b|| / ||b|| in float64 (b is the oracle)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def to64(t):
    """Device/host tensor -> float64 numpy (exact widening)."""
    import torch
    t = t.detach().to("cpu")
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.numpy().astype(np.float64)


# Tolerances: fp32 ops rel-L2 <= 1e-5; bf16 per-op outputs are rounded to bf16
# (relative 2^-9 per element, so rel-L2 ~ 3e-3) -> 1e-2; bf16 end-to-end hidden
# states 2e-2; Sinkhorn matrices 1e-6 absolute.
#
# GDN state (fp32) of a bf16 op: every product that updates the state takes exact bf16
# inputs (k, q) or operands carried as two bf16 terms, hi + lo (the state copy, the chunk's
# left factor and the update's left factor; relative error ~2^-17), so the state is kept at
# fp32-grade accuracy: 1e-4 (the short-chunk case T = 1 and decays near 1 included).
TOL = {"fp32": 1e-5, "bf16": 1e-2, "bf16_e2e": 2e-2, "sinkhorn": 1e-6, "gdn_state": 1e-4}


@pytest.fixture(scope="session")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import looped_hybrid_attention_b200 as L   # noqa: F401  (fails loudly if the library is missing)
    return torch.device("cuda:0")
