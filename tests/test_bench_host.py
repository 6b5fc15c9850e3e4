"""Host arithmetic of bench.py, on CPU: the algorithmic bytes and FLOP
rooflines its fractions divide by, and the rule that a recorded DRAM traffic
is reported only while the GEMM source is the one it was captured on.
"""
import hashlib
import os

import pytest

import bench


def test_layout_bytes_attention_layer():
    # 4096 columns at (32, 960, 3104): 32 + 720 + 1552 code bytes and 128
    # scale bytes per row, plus the source bytes per element
    assert bench.layout_bytes(1, (32, 960, 3104), 0) == 32 + 720 + 1552 + 128
    assert bench.layout_bytes(4096, (32, 960, 3104), 2) == 4096 * (4096 * 2 + 2432)


def test_layout_bytes_pads_segments_to_blocks():
    # 1 eight-bit and 33 four-bit columns occupy one and two 32-position blocks
    assert bench.layout_bytes(1, (1, 0, 33), 0) == 32 + 64 // 2 + 3


def test_gemm_roofline_is_the_slower_of_compute_and_bytes():
    pk = {"hbm_gbs": 6548.8, "bf16_tflops": 1671.8, "fp8_tflops": 3343.6}
    M, N, counts = 2048, 4096, (32, 960, 3104)
    t_c = 2 * M * N * 3104 / 3343.6e12 + 2 * M * N * 992 / 1671.8e12
    assert bench.gemm_roofline_s(M, N, counts, pk) == pytest.approx(t_c, rel=1e-12)
    assert bench.gemm_roofline_s(M, N, counts, pk) == pytest.approx(25.53e-6, rel=1e-3)
    # one row: the packed W dominates, bytes-bound
    byts = bench.layout_bytes(1, counts, 0) + bench.layout_bytes(N, counts, 0) + N * 2
    assert bench.gemm_roofline_s(1, N, counts, pk) == pytest.approx(byts / 6548.8e9, rel=1e-12)


def test_attention_bytes():
    # K and V: 64 code bytes and 4 scale bytes per token and kv head, the bf16
    # query and the fp32 output
    assert bench.attn_bytes(8192, 8, 32) == 2 * 8192 * 8 * 68 + 32 * 128 * 2 + 32 * 128 * 4


def test_peaks_fall_back_to_twice_bf16_for_the_e4m3_peak():
    pk = bench.peaks()
    assert pk["fp8_tflops"] == 2.0 * pk["bf16_tflops"]
    assert "no fp8 measurement" in pk["fp8_source"]


def test_traffic_is_read_only_for_the_captured_source(tmp_path, monkeypatch):
    src = os.path.join(bench.ROOT, "mx_microscaling_mixed_b200", "csrc", "mxs_gemm.cu")
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "p.md").write_text(f"dram_bytes_per_call[mlp_down]: 1.5e9\nsource_sha256: {digest}\n")
    (prof / "stale.md").write_text("dram_bytes_per_call[mlp_down]: 1.5e9\nsource_sha256: " + "0" * 64 + "\n")
    # the bench resolves the GEMM source under ROOT; give it a tree whose
    # source is the real one
    csrc = tmp_path / "mx_microscaling_mixed_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "mxs_gemm.cu").write_bytes(open(src, "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profile("p.md", "mlp_down") == 1.5e9
    assert bench.traffic_from_profile("p.md", "mlp_up") is None          # no line for that layer
    assert bench.traffic_from_profile("stale.md", "mlp_down") is None    # source changed since
    assert bench.traffic_from_profile("missing.md", "mlp_down") is None
