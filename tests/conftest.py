import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (minutes of CPU time)")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if gpu_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


# ----------------------------------------------------------------- helpers
def tolerance_violations(y: np.ndarray, y_ref: np.ndarray, rel: float = 1e-2,
                         abs_rms: float = 1e-3, rms_of: np.ndarray = None) -> np.ndarray:
    """Boolean mask of elements breaking |y - y_ref| <= rel*|y_ref| + abs_rms*rms.

    rms is taken over the whole output tensor of the GEMM (rms_of, default
    y_ref); for sampled rows pass the rms of the full reference if known.
    """
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    ref_for_rms = y_ref if rms_of is None else np.asarray(rms_of, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref_for_rms ** 2))) if ref_for_rms.size else 0.0
    return np.abs(y - y_ref) > rel * np.abs(y_ref) + abs_rms * rms


def frob_rel_err(y: np.ndarray, y_ref: np.ndarray) -> float:
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    den = np.linalg.norm(y_ref)
    return float(np.linalg.norm(y - y_ref) / den) if den > 0 else float(np.linalg.norm(y))
