"""Shared test helpers: numpy <-> torch marshalling, the linear tolerance rule and the
scale-search agreement rule."""
import numpy as np
import torch

from oracle import awq_oracle as O

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


# Scale-search agreement (the method's rule for the chosen alpha; losses as stated in
# tests/test_parity_search.py).
LOSS_REL = 5e-5


def check_search_result(X, got, ref, loss_rel=LOSS_REL, s_exact=None):
    """got = (s fp16 [K], losses fp64 [n], best index) from the GPU, ref = the oracle's
    scale_search(...) tuple.  The index equals the oracle's, or is one grid step away
    where the oracle's two losses differ by less than 1e-6 relative; s* is bit-exact when
    the index agrees (up to the fp16-midpoint exception of pow: s_exact(alpha) gives the
    fp64 value before rounding, pow(m, alpha) by default); every loss agrees within
    loss_rel relative.  Returns the GPU's best index."""
    s, losses, best = got
    rb, ralpha, rs, rlosses = ref
    if best != rb:
        assert abs(best - rb) == 1, (best, rb)
        assert abs(rlosses[best] - rlosses[rb]) <= 1e-6 * rlosses[rb], (best, rb)
    else:
        diff = s.view(np.uint16) != rs.view(np.uint16)
        if diff.any():
            if s_exact is None:
                p = np.power(O.act_absmean(X), ralpha)[diff]
            else:
                p = s_exact(ralpha)[diff]
            lo = rs[diff].astype(np.float64)
            hi = s[diff].astype(np.float64)
            mid = (lo + hi) / 2
            assert np.all(np.abs(p - mid) <= 1e-12 * np.abs(mid)), "s* differs"
    rel = np.abs(losses - rlosses) / np.maximum(rlosses, 1e-300)
    assert rel.max() <= loss_rel, f"loss rel err {rel.max():.3g}"
    return best
