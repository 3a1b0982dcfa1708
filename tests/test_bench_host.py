"""Host-side pieces of bench.py (no GPU): the algorithmic byte counts behind `value` and
`roofline.achieved`, and the guard that reports a recorded DRAM traffic figure only
while the GEMV's code is the code it was measured on."""
import os

import pytest

import bench
import inputs


def test_linear_bytes_closed_form():
    # packed codes N*K/2, fp16 scales 2*N*K/G, zero words 4*N*ceil(K/G/8), x 2*M*K, y 2*M*N
    N, K, M, G = 4096, 14336, 1, 128
    ng = K // G
    want = N * K // 2 + 2 * N * ng + 4 * N * ((ng + 7) // 8) + 2 * M * K + 2 * M * N
    assert bench.linear_bytes(M, N, K) == want
    assert bench.packed_bytes(100, 256, 32, False) == 100 * 128 + 100 * 8 * 2


def test_decode_layer_bytes():
    """The headline step reads the fused layer's bytes once: 113,451,008 B; the seven
    unfused linears read 113,475,584 B (their inputs are not shared)."""
    fused = sum(bench.linear_bytes(1, n, k) for _, k, n, _ in inputs.MISTRAL_7B_LAYER_FUSED)
    assert fused == 113_451_008
    assert bench.layer_bytes(inputs.MISTRAL_7B_LAYER) == 113_475_584
    # the fusion only concatenates rows: the packed weights are the same bytes
    packed_fused = sum(bench.packed_bytes(n, k) for _, k, n, _ in inputs.MISTRAL_7B_LAYER_FUSED)
    packed_unfused = sum(bench.packed_bytes(n, k) for _, k, n in inputs.MISTRAL_7B_LAYER)
    assert packed_fused == packed_unfused


def test_source_digest_ignores_comments(tmp_path):
    a = tmp_path / "a.cuh"
    a.write_text("int f() {\n    return 1;  // one\n}\n")
    b = tmp_path / "b.cuh"
    b.write_text("/* a block\n   comment */\nint f() {\n\n    return 1;\n}\n// trailing\n")
    c = tmp_path / "c.cuh"
    c.write_text("int f() {\n    return 2;\n}\n")
    assert bench.source_digest([str(a)]) == bench.source_digest([str(b)])
    assert bench.source_digest([str(a)]) != bench.source_digest([str(c)])


def test_traffic_record_guarded_by_the_gemv_code(monkeypatch, tmp_path):
    assert bench.profile_traffic("no_such_kernel") is None
    # a record taken on other code is not reported
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.txt").write_text("# header\ngemv_mistral7b_layer 123 0000000000000000\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profile_traffic("gemv_mistral7b_layer") is None
    (prof / "traffic.txt").write_text(
        "gemv_mistral7b_layer 123 %s\n" % bench.source_digest(bench.gemv_sources()))
    assert bench.profile_traffic("gemv_mistral7b_layer") == pytest.approx(123.0)


def test_gemv_sources_are_the_gemv_files():
    names = sorted(os.path.basename(p) for p in bench.gemv_sources())
    assert names == ["common.cuh", "gemv.cuh", "gemv_launch.cuh", "launch.cuh", "sm100.cuh"]


def test_every_traffic_tag_names_existing_sources():
    for tag, names in bench.KERNEL_SOURCES.items():
        found = sorted(os.path.basename(p) for p in bench.kernel_sources(tag))
        assert found == sorted(names), tag


def test_rotations_exceed_twice_the_l2():
    for nbytes in (8_716_288, 113_451_008, 300_000_000):
        r = bench.rotations_for(nbytes)
        assert r * nbytes > 2 * bench.L2_BYTES and r >= 2
