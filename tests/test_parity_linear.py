"""GPU parity: awq_linear_gemv / awq_linear_gemm against the oracle's fp64 linear.

Tolerance (from the arithmetic): |y - y_ref| <= 1e-2 (|y_ref| + rms(y_ref)) per element.
The kernels' own error is far smaller (exact fp16 products, fp32 accumulation, one fp16
rounding of the output; the GEMM adds one fp16 rounding of each dequantised weight)."""
import numpy as np
import pytest
import torch

import inputs
from helpers import assert_linear_close, to_dev, to_np
from bit_weight_only_linear_b200 import awq as _awq
from oracle import awq_oracle as O

pytestmark = pytest.mark.gpu


def _packed(W, G, zp, s=None):
    q, sc, z = O.quantize_pack(W, s, G, zp)
    return q, sc, z, (to_dev(q), to_dev(sc), to_dev(z) if zp else None)


def _run(lib, kind, X, dq, G, zp):
    fn = lib.linear_gemv if kind == "gemv" else lib.linear_gemm
    y = fn(to_dev(X), dq[0], dq[1], dq[2], G, zp)
    torch.cuda.synchronize()
    return to_np(y)


SMALL = [(1, 128, 8), (1, 256, 37), (2, 1024, 64), (3, 2048, 130), (4, 4096, 96), (8, 3072, 33),
         (1, 4096 + 1024, 257), (5, 256, 512), (1, 14336, 64)]


@pytest.mark.parametrize("G", O.GROUP_SIZES)
@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("mkn", SMALL, ids=lambda t: "x".join(map(str, t)))
def test_gemv_parity(lib, G, zp, mkn):
    M, K, N = mkn
    if K % G:
        pytest.skip("K % G")
    W = inputs.weights(N, K, 0.02, seed=200 + K + N)
    X = inputs.activations(M, K, seed=201 + M + K)
    q, sc, z, dq = _packed(W, G, zp)
    y = _run(lib, "gemv", X, dq, G, zp)
    assert_linear_close(y, O.linear(X, q, sc, z, K, G, zp))


def test_gemv_outputs_do_not_spill(lib):
    """Guard band around Y: the kernel writes exactly M x N values."""
    M, K, N, G = 3, 1024, 70, 64
    W = inputs.weights(N, K, seed=202)
    X = inputs.activations(M, K, seed=203)
    q, sc, z, dq = _packed(W, G, True)
    buf = torch.full((M * N + 64,), float("nan"), dtype=torch.float16, device="cuda")
    y = buf[32:32 + M * N].view(M, N)
    lib.linear_gemv(to_dev(X), dq[0], dq[1], dq[2], G, True, out=y)
    torch.cuda.synchronize()
    b = to_np(buf).astype(np.float64)
    assert np.all(np.isnan(b[:32])) and np.all(np.isnan(b[32 + M * N:]))
    assert_linear_close(b[32:32 + M * N].reshape(M, N), O.linear(X, q, sc, z, K, G, True))


@pytest.mark.parametrize("M,K,N,G,zp", [
    (1, 256, 47360, 128, True),     # one padded stage per row group, 10 row groups per CTA
    (3, 2176, 38400, 32, False),    # two stages per row group (the second partial), 9 per CTA
])
def test_gemv_more_row_groups_than_parameter_slots(lib, M, K, N, G, zp):
    """A CTA of the TMA GEMV keeps at most 8 row groups of raw scales/zeros in flight;
    with more row groups per CTA than that, the slots are refilled.  Checked on every
    output of 512 sampled rows (a spread of row groups) plus the last 16 rows."""
    W = inputs.weights(N, K, 0.02, seed=210 + K)
    X = inputs.activations(M, K, seed=211 + K)
    q, sc, z, dq = _packed(W, G, zp)
    y = _run(lib, "gemv", X, dq, G, zp)
    rows = np.unique(np.concatenate([np.random.default_rng(212).choice(N, 512, replace=False),
                                     np.arange(N - 16, N)]))
    assert_linear_close(y[:, rows], O.linear_rows(X, q, sc, z, K, G, zp, rows))


def test_gemv_single_workload_full(lib):
    """M=1, K=N=4096, G=128, zero point: every output against the oracle."""
    W = inputs.weights(4096, 4096, 0.02, seed=inputs.SEED_W)
    X = inputs.activations(1, 4096, seed=inputs.SEED_X)
    q, sc, z, dq = _packed(W, 128, True)
    assert_linear_close(_run(lib, "gemv", X, dq, 128, True), O.linear(X, q, sc, z, 4096, 128, True))


def test_gemv_mistral_layer_sampled(lib):
    """The seven Mistral-7B decode linears at M=1 (full size, launch as benchmarked):
    256 sampled output channels per linear against the oracle."""
    rng = np.random.Generator(np.random.PCG64(5))
    for name, W, X in inputs.layer_inputs(inputs.MISTRAL_7B_LAYER, 1, 0.02):
        N, K = W.shape
        q, sc, z, dq = _packed(W, 128, True)
        y = _run(lib, "gemv", X, dq, 128, True)
        rows = np.sort(rng.choice(N, 256, replace=False))
        ref = O.linear_rows(X, q, sc, z, K, 128, True, rows)
        assert_linear_close(y[:, rows], ref)


def test_gemv_mistral_layer_fused_sampled(lib):
    """The fused decode layer (q/k/v and gate/up concatenated) as benchmarked:
    256 sampled output channels per fused linear against the oracle."""
    rng = np.random.Generator(np.random.PCG64(6))
    for name, W, X in inputs.fused_layer_inputs(1, 0.02):
        N, K = W.shape
        q, sc, z, dq = _packed(W, 128, True)
        y = _run(lib, "gemv", X, dq, 128, True)
        rows = np.sort(rng.choice(N, 256, replace=False))
        assert_linear_close(y[:, rows], O.linear_rows(X, q, sc, z, K, 128, True, rows))


GEMM_SMALL = [(1, 128, 128), (4, 256, 130), (16, 1024, 256), (17, 512, 384), (33, 256, 128),
              (64, 2048, 256), (100, 1024, 200), (128, 512, 128), (200, 256, 384), (256, 1024, 256),
              (300, 512, 136), (513, 256, 128)]


@pytest.mark.parametrize("G", O.GROUP_SIZES)
@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("mkn", GEMM_SMALL, ids=lambda t: "x".join(map(str, t)))
def test_gemm_parity(lib, G, zp, mkn):
    M, K, N = mkn
    if K % G:
        pytest.skip("K % G")
    W = inputs.weights(N, K, 0.02, seed=300 + K + N)
    X = inputs.activations(M, K, seed=301 + M + K)
    q, sc, z, dq = _packed(W, G, zp)
    y = _run(lib, "gemm", X, dq, G, zp)
    assert_linear_close(y, O.linear(X, q, sc, z, K, G, zp))


def test_gemm_ragged_k_tail(lib):
    """K = 96 with G = 32: the last 64-channel k-block is half outside the matrix."""
    M, K, N, G = 40, 96, 130, 32
    W = inputs.weights(N, K, seed=302)
    X = inputs.activations(M, K, seed=303)
    for zp in (True, False):
        q, sc, z, dq = _packed(W, G, zp)
        assert_linear_close(_run(lib, "gemm", X, dq, G, zp), O.linear(X, q, sc, z, K, G, zp))


@pytest.mark.parametrize("M,K,N,G,zp", [
    (40, 4160, 384, 64, False),   # 65 k-blocks, split K: the last split is one k-block of a 4-block stage
    (130, 704, 1000, 64, True),   # 256-token tiles, 11 k-blocks in 2 splits: the second ends mid-stage
])
def test_gemm_split_k_partial_stage(lib, M, K, N, G, zp):
    """The 128-channel form loads packed weights 4 k-blocks per copy and splits K on whole
    copies; a split that ends inside one (K not a multiple of 256) uses part of it."""
    W = inputs.weights(N, K, 0.02, seed=304 + K)
    X = inputs.activations(M, K, seed=305 + K)
    q, sc, z, dq = _packed(W, G, zp)
    assert_linear_close(_run(lib, "gemm", X, dq, G, zp), O.linear(X, q, sc, z, K, G, zp))


def test_gemm_outputs_do_not_spill(lib):
    M, K, N, G = 70, 512, 136, 128
    W = inputs.weights(N, K, seed=304)
    X = inputs.activations(M, K, seed=305)
    q, sc, z, dq = _packed(W, G, True)
    buf = torch.full((M * N + 64,), float("nan"), dtype=torch.float16, device="cuda")
    y = buf[32:32 + M * N].view(M, N)
    lib.linear_gemm(to_dev(X), dq[0], dq[1], dq[2], G, True, out=y)
    torch.cuda.synchronize()
    lib.device_error()
    b = to_np(buf).astype(np.float64)
    assert np.all(np.isnan(b[:32])) and np.all(np.isnan(b[32 + M * N:]))
    assert_linear_close(b[32:32 + M * N].reshape(M, N), O.linear(X, q, sc, z, K, G, True))


def test_gemm_equals_gemv_at_small_batch(lib):
    """Both forms compute the same definition: at M = 4 they agree within the rule."""
    M, K, N, G = 4, 4096, 1024, 128
    W = inputs.weights(N, K, seed=306)
    X = inputs.activations(M, K, seed=307)
    q, sc, z, dq = _packed(W, G, True)
    a = _run(lib, "gemv", X, dq, G, True)
    b = _run(lib, "gemm", X, dq, G, True)
    assert_linear_close(b, a.astype(np.float64))


def test_gemm_llama70b_prefill_sampled(lib):
    """The four Llama-70B-shaped prefill linears at M = 2048, full size, launched as
    benchmarked: 128 sampled output channels each against the oracle."""
    rng = np.random.Generator(np.random.PCG64(9))
    for i, (name, K, N) in enumerate(inputs.LLAMA_70B_FUSED):
        W = inputs.weights(N, K, 0.015, inputs.SEED_W + 30 + i)
        X = inputs.activations(2048, K, inputs.SEED_X + 30 + i, inputs.SEED_OUTLIER + 30)
        Wd = to_dev(W)
        q, sc, z = lib.quantize_pack(Wd, None, 128, True)
        del Wd
        y = to_np(lib.linear_gemm(to_dev(X), q, sc, z, 128, True))
        lib.device_error()
        rows = np.sort(rng.choice(N, 128, replace=False))
        # the GPU's packing of the sampled rows, bit for bit against the oracle's
        rq, rs, rz = O.quantize_pack(W[rows], None, 128, True)
        assert np.array_equal(to_np(q)[rows], rq)
        assert np.array_equal(to_np(sc)[rows].view(np.uint16), rs.view(np.uint16))
        assert np.array_equal(to_np(z)[rows], rz)
        ref = O.linear_rows(X, rq, rs, rz, K, 128, True, np.arange(len(rows)))
        assert_linear_close(y[:, rows], ref)


def test_gemm_wide_two_waves_ragged(lib):
    """A prefill shape on the wide form with more 256 x 256 tiles (160) than one wave of
    SMs, ragged in M (300 tokens) and N (20440 channels): every output channel of the last
    7 channel tiles and a sample of the rest against the oracle, and a second call gives
    the same bits."""
    M, K, N, G = 300, 704, 20440, 64
    W = inputs.weights(N, K, 0.02, seed=320)
    X = inputs.activations(M, K, seed=321)
    q, sc, z, dq = _packed(W, G, True)
    Xd = to_dev(X)
    y1 = to_np(lib.linear_gemm(Xd, dq[0], dq[1], dq[2], G, True))
    y2 = to_np(lib.linear_gemm(Xd, dq[0], dq[1], dq[2], G, True))
    lib.device_error()
    assert np.array_equal(y1.view(np.uint16), y2.view(np.uint16))
    rng = np.random.Generator(np.random.PCG64(322))
    rows = np.concatenate([np.sort(rng.choice(74 * 256, 96, replace=False)), np.arange(74 * 256, N)])
    assert_linear_close(y1[:, rows], O.linear_rows(X, q, sc, z, K, G, True, rows))


def _edge_weights(K):
    """Rows of constant groups (scale at the 1e-5 floor), and rows of large magnitude
    (group ranges up to ~4e4: scale16 near 2700, the fp16 products (q - z) * scale16 up
    to ~4e4, still finite)."""
    g = np.random.Generator(np.random.PCG64(310))
    rows = [np.zeros(K), np.full(K, 0.25), np.full(K, -3.0),
            g.uniform(-20000, 20000, K), g.uniform(0, 30000, K), g.uniform(-40000, -100, K),
            np.where(np.arange(K) % 3 == 0, 18000.0, -21000.0)]
    return np.stack(rows).astype(np.float16)


@pytest.mark.parametrize("G", O.GROUP_SIZES)
@pytest.mark.parametrize("zp", [True, False])
def test_gemm_edge_magnitudes(lib, G, zp):
    """Constant groups and large-magnitude groups through both linear forms, against the
    oracle; the activations are small so that the outputs stay finite in fp16."""
    K, M = 512, 40
    W = np.concatenate([_edge_weights(K)] * 3)
    X = (inputs.activations(M, K, seed=311).astype(np.float32) * np.float32(1e-3)).astype(np.float16)
    q, sc, z, dq = _packed(W, G, zp)
    ref = O.linear(X, q, sc, z, K, G, zp)
    y = _run(lib, "gemm", X, dq, G, zp)
    lib.device_error()
    assert_linear_close(y, ref)
    assert_linear_close(_run(lib, "gemv", X[:3], dq, G, zp), ref[:3])


def test_gemm_reports_fp16_overflow(lib):
    """A group whose dequantised weights leave fp16 ((q - z) * scale16 = 15 * 5000) makes
    the GEMM flag AWQ_ERR_RANGE; the next call on valid weights runs clean."""
    N, K, G = 128, 256, 128
    codes = np.random.Generator(np.random.PCG64(312)).integers(0, 16, size=(N, K)).astype(np.uint8)
    codes[:, 0] = 15
    scales = np.full((N, K // G), 0.01, dtype=np.float16)
    scales[5, 1] = 5000.0
    zeros = np.zeros((N, K // G), dtype=np.uint8)
    dq = (to_dev(O.pack_codes(codes)), to_dev(scales), to_dev(O.pack_nibbles(zeros)))
    X = (inputs.activations(16, K, seed=313).astype(np.float32) * np.float32(1e-3)).astype(np.float16)
    lib.linear_gemm(to_dev(X), *dq, G, True)
    with pytest.raises(_awq.AWQError) as err:
        lib.device_error()
    assert err.value.status == _awq.AWQ_ERR_RANGE
    scales[5, 1] = 4000.0          # 15 * 4000 = 60000: finite
    dq = (dq[0], to_dev(scales), dq[2])
    y = _run(lib, "gemm", X, dq, G, True)
    lib.device_error()
    assert_linear_close(y, O.linear(X, O.pack_codes(codes), scales, O.pack_nibbles(zeros), K, G, True))


def test_gemv_directly_after_quantize_pack(lib):
    """The GEMV streams its weights before it waits for the previous kernel; a GEMV
    enqueued right after awq_quantize_pack into the same buffers (no synchronisation in
    between) must still see the new weights."""
    N, K, G = 4096, 4096, 128
    X = inputs.activations(1, K, seed=314)
    Xd = to_dev(X)
    W0 = to_dev(inputs.weights(N, K, 0.02, seed=315))
    bufs = lib.quantize_pack(W0, None, G, True)
    torch.cuda.synchronize()
    for i in range(3):
        W = inputs.weights(N, K, 0.02, seed=316 + i)
        Wd = to_dev(W)
        torch.cuda.synchronize()
        lib.quantize_pack(Wd, None, G, True, out=bufs)
        y = to_np(lib.linear_gemv(Xd, *bufs, G, True))
        q, sc, z = O.quantize_pack(W, None, G, True)
        assert_linear_close(y, O.linear(X, q, sc, z, K, G, True))
