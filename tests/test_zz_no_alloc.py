"""awq_scale_search_noalloc: the scale search for callers that cannot allocate.

Some callers cannot allocate device memory at the point where they quantise a
layer: a runtime without an allocator of its own, a memory pool that has already
been carved up, or a process that must not grow its footprint after start-up.  For
them the library offers a scale search that takes no workspace and keeps its
scratch in a fixed device array inside the library.  These tests call it through
the C ABI and check it against awq_scale_search (which uses a caller workspace)
under the same rules as the other search tests: the same alpha index (or one grid
step apart where the two losses are within 1e-6 relative), the same s* when the
index agrees, and losses within 5e-5 relative.  Each configuration is called twice
in a row, since the array keeps the previous call's contents.

The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import inputs
from helpers import to_dev, to_np

LOSS_REL = 5e-5


def _compare(ref, got):
    s_ref, l_ref, b_ref = to_np(ref[0]), ref[1].cpu().numpy(), int(ref[2].cpu().item())
    s, l, b = to_np(got[0]), got[1].cpu().numpy(), int(got[2].cpu().item())
    rel = np.abs(l - l_ref) / np.maximum(l_ref, 1e-300)
    assert rel.max() <= LOSS_REL, f"loss rel diff {rel.max():.3g}"
    if b != b_ref:
        assert abs(b - b_ref) == 1 and abs(l_ref[b] - l_ref[b_ref]) <= 1e-6 * l_ref[b_ref], (b, b_ref)
    else:
        assert np.array_equal(s.view(np.uint16), s_ref.view(np.uint16))


@pytest.mark.gpu
@pytest.mark.parametrize("M,K,N,G,zp", [
    (256, 16384, 384, 128, True),    # three chunks of output channels
    (100, 1024, 130, 32, False),     # one ragged chunk, symmetric mode
])
def test_noalloc_matches_workspace_search(M, K, N, G, zp):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_weight_only_linear_b200 import awq, build
    build.build()
    X = to_dev(inputs.activations(M, K, seed=500 + K))
    W = to_dev(inputs.weights(N, K, 0.02, seed=501 + K))
    ref = awq.scale_search(X, W, G, zp, 20)
    torch.cuda.synchronize()
    out = (torch.empty(K, dtype=torch.float16, device="cuda"), torch.empty(20, dtype=torch.float64, device="cuda"),
           torch.empty(1, dtype=torch.int32, device="cuda"))
    for i in range(2):
        if i == 1:
            # the first call has loaded the module and looked up the array's address: from
            # here on nothing may be allocated, by the library or on its behalf
            free0, reserved0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()
        got = awq.scale_search_noalloc(X, W, G, zp, 20, out=out)
        torch.cuda.synchronize()
        awq.device_error()
        if i == 1:
            assert torch.cuda.mem_get_info()[0] == free0 and torch.cuda.memory_reserved() == reserved0
        _compare(ref, got)


def test_noalloc_rejects_sizes_beyond_the_fixed_scratch():
    """K above 16384 or M above 2^20 is refused on the host, before anything is launched
    (the pointers below are never dereferenced)."""
    from bit_weight_only_linear_b200 import awq, build
    build.build()
    lib = awq.load_library()
    fake = 0x10000
    cfg = awq.config(128, True)
    f = lib.awq_scale_search_noalloc
    assert f(fake, 16, fake, 64, 16384 + 128, cfg, 20, fake, 0, 0, None) == awq.AWQ_ERR_UNSUPPORTED
    assert f(fake, (1 << 20) + 1, fake, 64, 256, cfg, 20, fake, 0, 0, None) == awq.AWQ_ERR_UNSUPPORTED
    assert f(fake, 16, fake, 64, 256, cfg, 0, fake, 0, 0, None) == awq.AWQ_ERR_INVALID_ARG
