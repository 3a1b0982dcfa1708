"""Failure detection on the GPU without a fault.

Every device-side wait of the library is bounded: a wait that runs out sets a device
error word and the kernel returns, so a stalled pipeline ends with a status the host
reads instead of a hang.  awq_check_bounded_wait enqueues a kernel whose mbarrier wait
can never complete (nothing arrives on the barrier); this test checks that it reports
AWQ_ERR_TIMEOUT after the 2 s limit and that the context stays usable afterwards.
"""
import time

import numpy as np
import pytest
import torch

import inputs
from helpers import assert_linear_close, to_dev, to_np
from oracle import awq_oracle as O

AWQ_ERR_TIMEOUT = 5


@pytest.mark.gpu
def test_stalled_wait_reports_timeout_and_context_survives(lib):
    lib.device_error()                                   # start from a clear error word
    t0 = time.perf_counter()
    lib.check_bounded_wait()
    with pytest.raises(lib.AWQError) as err:
        lib.device_error()                               # synchronises, reads, clears
    elapsed = time.perf_counter() - t0
    assert err.value.status == AWQ_ERR_TIMEOUT
    assert 1.5 < elapsed < 60.0, elapsed                 # the 2 s limit, not a hang
    lib.device_error()                                   # cleared by the read above

    # the context still runs kernels correctly
    M, K, N, G = 1, 1024, 64, 128
    W = inputs.weights(N, K, 0.02, seed=400)
    X = inputs.activations(M, K, seed=401)
    q, sc, z = O.quantize_pack(W, None, G, True)
    y = lib.linear_gemv(to_dev(X), to_dev(q), to_dev(sc), to_dev(z), G, True)
    torch.cuda.synchronize()
    lib.device_error()
    assert_linear_close(to_np(y), O.linear(X, q, sc, z, K, G, True))
    assert np.isfinite(to_np(y)).all()
