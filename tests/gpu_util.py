"""Shared helpers of the GPU parity tests (imported by tests only)."""
import numpy as np
import torch


def rel_err(got, want) -> float:
    """Normwise relative error max|g - w| / max|w| (elementwise relative error is
    undefined near zero)."""
    g = np.asarray(got, np.float64)
    w = np.asarray(want, np.float64)
    den = np.max(np.abs(w))
    return float(np.max(np.abs(g - w)) / (den if den > 0 else 1.0))


def bits(a):
    return np.ascontiguousarray(np.asarray(a, np.float32)).view(np.uint32)


def cuda_ok() -> bool:
    return torch.cuda.is_available()


# the tolerance the workload states for fp32-accumulated hidden states and logits
TOL = 2e-3
# argmax tokens must agree whenever the oracle's top-2 margin exceeds this
MARGIN = 1e-2
