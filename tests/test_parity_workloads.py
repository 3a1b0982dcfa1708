"""GPU parity at the full sizes of the measured workloads, launched as the benchmark
launches them:

* batched decode: the seven Mistral-7B-shaped linears (q/k/v 4096->4096/1024/1024,
  o 4096->4096, gate/up 4096->14336, down 14336->4096), group 128 with zero point, at
  M = 4, 8, 16 and 64 tokens: the GEMV (M <= 8, the TMA kernel since N % 16 = 0) and the
  GEMM at every M, 256 sampled output channels each, every token; the packed weights
  bit-exact against the oracle's over the whole matrix;
* the quantisation sweep: one 4096 x 4096 layer with 512 calibration tokens, for every
  group size in {32, 64, 128, 256} with and without zero point: scale search over 20
  alphas (the alpha rule, s*, every loss), then quantise/pack with s* (bit-exact), the
  activation fold X' = X / s* (bit-exact), the GEMV at M = 1 and the GEMM at M = 512 on
  X' (every output against the oracle's fp64 linear).

Tolerance of the linear (from the arithmetic): |y - y_ref| <= 1e-2 (|y_ref| + rms(y_ref)).
"""
import numpy as np
import pytest
import torch

import inputs
from helpers import assert_linear_close, check_search_result, to_dev, to_np
from oracle import awq_oracle as O

pytestmark = pytest.mark.gpu

BATCHED_M = (4, 8, 16, 64)
BATCHED_SEED_OFFSET = 20      # seeds of the batched-decode workload
SWEEP_SEED_OFFSET = 40        # seeds of the quantisation sweep


def _same_packed(gpu, ref, zp):
    q, sc, z = gpu
    rq, rs, rz = ref
    assert np.array_equal(to_np(q), rq), "qweight differs"
    assert np.array_equal(to_np(sc).view(np.uint16), rs.view(np.uint16)), "scales differ"
    if zp:
        assert np.array_equal(to_np(z), rz), "qzeros differ"


def test_batched_decode_mistral_layer(lib):
    rng = np.random.Generator(np.random.PCG64(21))
    for i, (name, K, N) in enumerate(inputs.MISTRAL_7B_LAYER):
        W = inputs.weights(N, K, 0.02, inputs.SEED_W + BATCHED_SEED_OFFSET + i)
        ref = O.quantize_pack(W, None, 128, True)
        dev = lib.quantize_pack(to_dev(W), None, 128, True)
        _same_packed(dev, ref, True)
        rows = np.sort(rng.choice(N, 256, replace=False))
        for M in BATCHED_M:
            X = inputs.activations(M, K, inputs.SEED_X + BATCHED_SEED_OFFSET + i,
                                   inputs.SEED_OUTLIER + BATCHED_SEED_OFFSET)
            y_ref = O.linear_rows(X, ref[0], ref[1], ref[2], K, 128, True, rows)
            Xd = to_dev(X)
            fns = ([lib.linear_gemv] if M <= 8 else []) + [lib.linear_gemm]
            for fn in fns:
                y = to_np(fn(Xd, *dev, 128, True))
                lib.device_error()
                assert_linear_close(y[:, rows], y_ref)


@pytest.mark.parametrize("G", O.GROUP_SIZES)
@pytest.mark.parametrize("zp", [True, False])
def test_quantization_sweep_4096(lib, G, zp):
    M, K, N = 512, 4096, 4096
    X = inputs.activations(M, K, inputs.SEED_X + SWEEP_SEED_OFFSET, inputs.SEED_OUTLIER + SWEEP_SEED_OFFSET)
    W = inputs.weights(N, K, 0.02, inputs.SEED_W + SWEEP_SEED_OFFSET)
    Xd, Wd = to_dev(X), to_dev(W)
    # 1. scale search
    s_dev, losses, best = lib.scale_search(Xd, Wd, G, zp, 20)
    lib.device_error()
    got = (to_np(s_dev), losses.cpu().numpy(), int(best.cpu().item()))
    check_search_result(X, got, O.scale_search(X, W, G, zp, 20))
    s = got[0]          # the downstream steps are compared on the GPU's s*
    # 2. quantise / pack with s*
    dev = lib.quantize_pack(Wd, s_dev, G, zp)
    ref = O.quantize_pack(W, s, G, zp)
    _same_packed(dev, ref, zp)
    # 3. the activation side s^-1 X
    Xp = lib.fold_inverse_scale(Xd, s_dev)
    Xp_ref = O.fold_inverse_scale(X, s)
    assert np.array_equal(to_np(Xp).view(np.uint16), Xp_ref.view(np.uint16))
    # 4. the linear on X': GEMV at M = 1, GEMM at M = 512, every output
    y1 = to_np(lib.linear_gemv(Xp[:1].contiguous(), *dev, G, zp))
    y2 = to_np(lib.linear_gemm(Xp, *dev, G, zp))
    lib.device_error()
    y_ref = O.linear(Xp_ref, ref[0], ref[1], ref[2], K, G, zp)
    assert_linear_close(y1, y_ref[:1])
    assert_linear_close(y2, y_ref)
