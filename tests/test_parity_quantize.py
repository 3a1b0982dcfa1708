"""GPU parity: awq_quantize_pack and awq_fold_inverse_scale against the CPU oracle.
Codes, zeros and scales must match bit for bit."""
import numpy as np
import pytest

import inputs
from helpers import to_dev, to_np
from oracle import awq_oracle as O

pytestmark = pytest.mark.gpu

SHAPES = [(8, 128), (37, 256), (64, 1024), (5, 2048 + 256), (130, 4096), (3, 14336)]


def _check(lib, W, s, G, zp):
    q, sc, z = lib.quantize_pack(to_dev(W), None if s is None else to_dev(s), G, zp)
    rq, rs, rz = O.quantize_pack(W, s, G, zp)
    assert np.array_equal(to_np(q), rq), "qweight differs"
    assert np.array_equal(to_np(sc).view(np.uint16), rs.view(np.uint16)), "scales differ"
    if zp:
        assert np.array_equal(to_np(z), rz), "qzeros differ"
    else:
        assert z is None


@pytest.mark.parametrize("G", O.GROUP_SIZES)
@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
def test_quantize_pack_bit_exact(lib, G, zp, shape):
    N, K = shape
    if K % G:
        pytest.skip("K not a multiple of G")
    W = inputs.weights(N, K, 0.02, seed=100 + N + K)
    _check(lib, W, None, G, zp)
    X = inputs.activations(32, K, seed=101 + K)
    s = O.scales_for_alpha(O.act_absmean(X), 0.65)
    _check(lib, W, s, G, zp)


def test_quantize_pack_edge_values(lib):
    """Constant groups (scale floor), exact grid values, zeros, all-negative groups."""
    K = 256
    rows = [np.zeros(K), np.full(K, 0.25), np.full(K, -3.0), np.linspace(-1, 1, K),
            np.where(np.arange(K) % 2 == 0, 1.375, -0.5), np.linspace(0.1, 0.9, K)]
    W = np.stack(rows).astype(np.float16)
    for G in O.GROUP_SIZES:
        for zp in (True, False):
            _check(lib, W, None, G, zp)


def test_quantize_pack_round_half_even_ties(lib):
    """Quotients w/scale that land exactly on half-integers (the scale is 2^-7, every
    weight an odd multiple of 2^-8): the codes must follow round-half-to-even of the IEEE
    quotient, which the kernel decides with an exact division near rounding boundaries."""
    K = 256
    u = 2.0 ** -7
    ties_zp = np.array([0.0, 15 * u] + [(k % 15 + 0.5) * u for k in range(K - 2)])
    ties_sym = np.array([-7 * u, 7 * u] + [((k % 15) - 7.5) * u for k in range(K - 2)])
    ties_sym = np.clip(ties_sym, -7 * u, 7 * u)
    for G in O.GROUP_SIZES:
        # every group holds the extremes that fix the scale at 2^-7, then the ties
        def grouped(base):
            out = np.empty(K)
            for g0 in range(0, K, G):
                out[g0:g0 + G] = np.concatenate([base[:2], base[2:2 + G - 2]])
            return out
        W = np.stack([grouped(ties_zp), grouped(ties_zp)[::-1].copy(), grouped(ties_sym)]).astype(np.float16)
        for zp in (True, False):
            _check(lib, W, None, G, zp)


def test_quantize_pack_full_layer_4096(lib):
    """The 4096 x 4096 layer of the single-GEMV workload, every element."""
    W = inputs.weights(4096, 4096, 0.02, seed=inputs.SEED_W)
    _check(lib, W, None, 128, True)


def test_fold_inverse_scale_bit_exact(lib):
    X = inputs.activations(33, 1024, seed=102)
    s = O.scales_for_alpha(O.act_absmean(X), 0.8)
    got = to_np(lib.fold_inverse_scale(to_dev(X), to_dev(s)))
    want = O.fold_inverse_scale(X, s)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))
