"""Host-side checks of the C ABI (no GPU): the library loads, exports every symbol the
header declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "awq.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(awq_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from bit_weight_only_linear_b200 import awq, build
    build.build()
    return awq.load_library()


def test_header_declares_the_boundary():
    names = header_functions()
    for n in ("awq_quantize_pack", "awq_scale_search", "awq_linear_gemv", "awq_linear_gemm",
              "awq_workspace_bytes", "awq_status_string", "awq_device_error", "awq_fold_inverse_scale"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from bit_weight_only_linear_b200 import awq
    for name in header_functions():
        assert hasattr(lib, name), name
        assert name in awq.SIGNATURES, f"binding lacks {name}"


def test_status_strings(lib):
    for code in range(7):
        s = lib.awq_status_string(code).decode()
        assert s.startswith("AWQ_")
    assert lib.awq_status_string(99).decode() == "AWQ_ERR_UNKNOWN"
    assert lib.awq_abi_version() == 2


def _cfg(g=128, zp=1, bits=4):
    from bit_weight_only_linear_b200.awq import QuantConfig
    return QuantConfig(bits, g, zp)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails its checks first


def test_quantize_pack_argument_errors(lib):
    f = lib.awq_quantize_pack
    assert f(FAKE, 0, 8, 128, _cfg(bits=3), FAKE, FAKE, FAKE, None) == 2      # w_bit != 4
    assert f(FAKE, 0, 8, 128, _cfg(g=48), FAKE, FAKE, FAKE, None) == 2        # group size
    assert f(FAKE, 0, 8, 100, _cfg(g=32), FAKE, FAKE, FAKE, None) == 1        # K % G
    assert f(FAKE, 0, 0, 128, _cfg(), FAKE, FAKE, FAKE, None) == 1            # N = 0
    assert f(FAKE, 0, 8, 128, _cfg(), FAKE, FAKE, 0, None) == 1               # zeros missing
    assert f(FAKE + 2, 0, 8, 128, _cfg(), FAKE, FAKE, FAKE, None) == 1        # misaligned W
    assert f(0, 0, 8, 128, _cfg(), FAKE, FAKE, FAKE, None) == 1               # null W
    assert f(FAKE, 0, 8, 128, _cfg(zp=2), FAKE, FAKE, FAKE, None) == 1        # bad zero_point


@pytest.mark.parametrize("name", ["awq_linear_gemv", "awq_linear_gemm"])
def test_linear_argument_errors(lib, name):
    f = getattr(lib, name)
    ok = dict(X=FAKE, M=1, q=FAKE, s=FAKE, z=FAKE, N=64, K=256, c=_cfg(), Y=FAKE)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["X"], a["M"], a["q"], a["s"], a["z"], a["N"], a["K"], a["c"], a["Y"], 0, 0, None)
    assert call(M=0) == 1
    assert call(N=-1) == 1
    assert call(K=200) == 1
    assert call(c=_cfg(bits=8)) == 2
    assert call(z=0) == 1
    assert call(Y=FAKE + 8) == 1
    assert call(X=0) == 1


def test_gemv_rejects_large_batch(lib):
    f = lib.awq_linear_gemv
    assert f(FAKE, 9, FAKE, FAKE, FAKE, 64, 256, _cfg(), FAKE, 0, 0, None) == 2


def test_scale_search_argument_errors(lib):
    f = lib.awq_scale_search
    need = lib.awq_workspace_bytes(1, 16, 64, 256, _cfg())
    assert need > 0
    assert f(FAKE, 16, FAKE, 64, 256, _cfg(), 0, FAKE, 0, 0, FAKE, need, None) == 1      # n_grid
    assert f(FAKE, 16, FAKE, 64, 256, _cfg(), 65, FAKE, 0, 0, FAKE, need, None) == 1
    assert f(FAKE, 16, FAKE, 64, 256, _cfg(), 20, FAKE, 0, 0, FAKE, need - 16, None) == 3  # workspace
    assert f(FAKE, 16, FAKE, 64, 256, _cfg(), 20, FAKE, 0, 0, 0, need, None) == 1          # null ws
    assert f(FAKE, 0, FAKE, 64, 256, _cfg(), 20, FAKE, 0, 0, FAKE, need, None) == 1        # M = 0


def test_workspace_sizes(lib):
    assert lib.awq_workspace_bytes(0, 1, 4096, 4096, _cfg()) == 0
    assert lib.awq_workspace_bytes(2, 1, 4096, 4096, _cfg()) == 0
    # the GEMM needs a workspace only to split K when its tiles leave SMs idle
    assert lib.awq_workspace_bytes(3, 2048, 8192, 8192, _cfg()) == 0
    small = lib.awq_workspace_bytes(3, 16, 4096, 4096, _cfg())
    assert small > 0 and small % (16 * 4096 * 4) == 0
    a = lib.awq_workspace_bytes(1, 512, 4096, 4096, _cfg())
    b = lib.awq_workspace_bytes(1, 512, 8192, 4096, _cfg())
    assert b > a > 0


def test_product_path_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "bit_weight_only_linear_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "oracle" not in src.lower(), f"{f} mentions the oracle"
    oracle_dir = os.path.join(ROOT, "oracle")
    for f in os.listdir(oracle_dir):
        if f.endswith(".py"):
            src = open(os.path.join(oracle_dir, f), encoding="utf-8").read()
            assert "bit_weight_only_linear_b200" not in src and "torch" not in src
