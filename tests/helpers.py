"""Shared test helpers: numpy <-> torch marshalling and the tolerance rule."""
import numpy as np
import torch

# |y - y_ref| <= REL * (|y_ref| + rms(y_ref)) elementwise, fp32 accumulation, fp16 output.
REL_TOL = 1e-2


def to_dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_np(t: torch.Tensor) -> np.ndarray:
    a = t.detach().cpu().numpy()
    if a.dtype == np.int32:
        a = a.view(np.uint32)
    return a


def assert_linear_close(y: np.ndarray, y_ref: np.ndarray, rel: float = REL_TOL):
    y = y.astype(np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    err = np.abs(y - y_ref)
    bound = rel * (np.abs(y_ref) + rms)
    bad = err > bound
    assert np.all(np.isfinite(y)), "non-finite outputs"
    assert not bad.any(), (f"{int(bad.sum())} of {y.size} outside tolerance; worst err "
                           f"{float((err / np.maximum(bound, 1e-300)).max()):.3g} x bound")
