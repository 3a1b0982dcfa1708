"""GPU parity: awq_apply_clip against the oracle's clip search.

Rules:
  * every error err[n, g, j] agrees with the oracle's within ERR_REL relative (derived from
    the arithmetic of the kernel: dW carries a 22-bit significand and X is exact, so the
    products are exact; the error of E is the fp32 accumulation of the tensor cores over
    2 G / 16 steps per group (at most 32 steps; about 2^-25 per step, measured on the
    scale search), i.e. at most ~1e-6 relative in E and ~2e-6 in E^2, plus the fp32 sums of
    16 squares (< 1e-6); ERR_REL = 1e-5 holds that with a margin);
  * the chosen index equals the oracle's, or is one step away where the oracle's two
    errors differ by less than 2 ERR_REL relative (the kernel cannot order them closer);
  * the packed weights are bit-exact against the oracle's packing at the GPU's indices.
"""
import numpy as np
import pytest
import torch

import inputs
from helpers import to_dev, to_np
from oracle import awq_oracle as O

pytestmark = pytest.mark.gpu

ERR_REL = 1e-5


def _check(lib, X, W, s, G, zp, n_grid=20, n_clip=10):
    q, sc, z, idx, err = lib.apply_clip(to_dev(X), to_dev(W), None if s is None else to_dev(s), G, zp, n_grid,
                                        n_clip, errors=True)
    lib.device_error()
    idx, err = to_np(idx).astype(np.int64), err.cpu().numpy()
    s_np = np.ones(W.shape[1], dtype=np.float16) if s is None else s
    ridx, rerr, _ = O.clip_search(X, W, s_np, G, zp, n_grid, n_clip)
    rel = np.abs(err - rerr) / np.maximum(rerr, 1e-300)
    worst = float(rel[rerr > 0].max()) if np.any(rerr > 0) else 0.0
    assert worst <= ERR_REL, f"clip error rel diff {worst:.3g}"
    d = idx != ridx
    if d.any():
        assert np.all(np.abs(idx[d] - ridx[d]) == 1)
        a = np.take_along_axis(rerr[d], idx[d][:, None], axis=1)[:, 0]
        b = np.take_along_axis(rerr[d], ridx[d][:, None], axis=1)[:, 0]
        assert np.all(np.abs(a - b) <= 2 * ERR_REL * b)
    ref = O.quantize_pack_clipped(W, s_np, G, zp, idx, n_grid)
    assert np.array_equal(to_np(q), ref[0]), "qweight differs"
    assert np.array_equal(to_np(sc).view(np.uint16), ref[1].view(np.uint16)), "scales differ"
    if zp:
        assert np.array_equal(to_np(z), ref[2]), "qzeros differ"
    return idx, worst


SHAPES = [(64, 256, 128), (300, 512, 200), (40, 1024, 130), (512, 256, 64), (700, 512, 200)]


@pytest.mark.parametrize("G", O.GROUP_SIZES)
@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("mkn", SHAPES, ids=lambda t: "x".join(map(str, t)))
def test_apply_clip_parity(lib, G, zp, mkn):
    M, K, N = mkn
    if K % G:
        pytest.skip("K % G")
    X = inputs.activations(M, K, seed=600 + M + K)
    W = inputs.weights(N, K, 0.02, seed=601 + N + K)
    s = O.scales_for_alpha(O.act_absmean(X), 0.35)
    idx, _ = _check(lib, X, W, s, G, zp)
    assert np.any(idx > 0)


def test_apply_clip_one_ratio_is_quantize_pack(lib):
    """n_clip = 1: no clipping, the result is awq_quantize_pack of W s bit for bit."""
    X = inputs.activations(64, 512, seed=602)
    W = inputs.weights(96, 512, 0.02, seed=603)
    s = O.scales_for_alpha(O.act_absmean(X), 0.5)
    for zp in (True, False):
        q, sc, z, idx = lib.apply_clip(to_dev(X), to_dev(W), to_dev(s), 128, zp, 20, 1)
        qq, ss, zz = lib.quantize_pack(to_dev(W), to_dev(s), 128, zp)
        lib.device_error()
        assert torch.equal(q, qq) and torch.equal(sc, ss) and (not zp or torch.equal(z, zz))
        assert int(idx.max().item()) == 0


def test_apply_clip_without_scale_and_grid_variants(lib):
    """s = NULL (s = 1), other grids, a ragged K = 96 with G = 32, zero rows."""
    X = inputs.activations(100, 96, seed=604)
    W = inputs.weights(70, 96, 0.02, seed=605)
    W[5] = 0
    for n_grid, n_clip in ((20, 10), (10, 4), (32, 32)):
        _check(lib, X, W, None, 32, True, n_grid, n_clip)


def test_apply_clip_units_cross_channel_blocks(lib):
    """More (128-channel block, group) units than one wave of CTAs holds (1300 channels in
    11 blocks, the last ragged, x 16 groups = 176 units): CTAs take one or two units, some
    crossing from one block to the next; every error and index against the oracle."""
    M, K, N, G = 64, 1024, 1300, 64
    X = inputs.activations(M, K, seed=607)
    W = inputs.weights(N, K, 0.02, seed=608)
    s = O.scales_for_alpha(O.act_absmean(X), 0.4)
    _check(lib, X, W, s, G, True)


def test_apply_clip_layer_4096(lib):
    """The quantisation sweep's layer (4096 x 4096, 512 tokens) at its searched scale,
    G = 128 with zero point; errors and indices of 512 sampled output channels against the
    oracle, packing of every row at the GPU's indices."""
    M, K, N, G = 512, 4096, 4096, 128
    X = inputs.activations(M, K, inputs.SEED_X + 40, inputs.SEED_OUTLIER + 40)
    W = inputs.weights(N, K, 0.02, inputs.SEED_W + 40)
    s = O.scales_for_alpha(O.act_absmean(X), 0.35)
    q, sc, z, idx, err = lib.apply_clip(to_dev(X), to_dev(W), to_dev(s), G, True, 20, 10, errors=True)
    lib.device_error()
    idx, err = to_np(idx).astype(np.int64), err.cpu().numpy()
    rows = np.sort(np.random.Generator(np.random.PCG64(606)).choice(N, 512, replace=False))
    ridx, rerr, _ = O.clip_search(X, W[rows], s, G, True, 20, 10)
    rel = np.abs(err[rows] - rerr) / rerr
    assert rel.max() <= ERR_REL
    d = idx[rows] != ridx
    if d.any():
        assert np.all(np.abs(idx[rows][d] - ridx[d]) == 1)
    ref = O.quantize_pack_clipped(W, s, G, True, idx, 20)
    assert np.array_equal(to_np(q), ref[0]) and np.array_equal(to_np(z), ref[2])
    assert np.array_equal(to_np(sc).view(np.uint16), ref[1].view(np.uint16))
