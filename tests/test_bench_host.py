"""Host-side logic of bench.py that the timing rests on (CPU only): the rotating-copy count
that keeps every timed launch reading from HBM, the DRAM-capture gating by source hash, and
the roofline arithmetic helpers."""

import pytest

import bench


def test_rotating_copies_touch_more_than_twice_l2():
    l2 = 126 * 2 ** 20
    for footprint in (1 << 20, 13 << 20, 32 << 20, 100 << 20, 300 << 20):
        n = bench.n_sets(footprint, l2)
        assert 2 <= n <= 16
        assert n * footprint > 2 * l2 or n == 16      # 16 copies is the cap for tiny layers
    assert bench.n_sets(300 << 20, l2) == 2           # one copy already exceeds L2: two alternate


def _write_capture(path, sha, read=1000, write=24):
    path.write_text("# a capture\n"
                    f"sources_sha256: {sha}\n"
                    f"dram_bytes_read: {read}\n"
                    f"dram_bytes_write: {write}\n")


def test_traffic_is_used_only_for_the_sources_it_was_captured_on(tmp_path, monkeypatch):
    f = tmp_path / "capture.txt"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.captured_traffic() == (None, "no capture")
    _write_capture(f, bench.gemm_sources_sha())
    traffic, note = bench.captured_traffic()
    assert traffic == 1024 and "this build" in note
    _write_capture(f, "0" * 64)
    traffic, note = bench.captured_traffic()
    assert traffic is None and "stale" in note


def test_sources_hash_changes_with_any_gemm_source(tmp_path, monkeypatch):
    import os
    import shutil
    root = tmp_path / "root"
    csrc = root / "bit_diffusion_transformer_act_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.GEMM_SOURCES:
        shutil.copy(os.path.join(bench.ROOT, "bit_diffusion_transformer_act_b200", "csrc", name), csrc / name)
    monkeypatch.setattr(bench, "ROOT", str(root))
    h0 = bench.gemm_sources_sha()
    assert h0 == bench.gemm_sources_sha()
    (csrc / bench.GEMM_SOURCES[0]).write_text((csrc / bench.GEMM_SOURCES[0]).read_text() + "\n")
    assert bench.gemm_sources_sha() != h0


def test_flop_and_byte_counts_of_the_attention_layer():
    M, K, N = 4096, 3072, 3072
    assert bench.svdq_flops(M, K, N) == pytest.approx(2.0 * M * N * K)
    # kernel 1: X and U hi|lo in bf16, codes (4 bits), scales (one byte per 16), the smoothing
    # factors and the packed low-rank operand
    assert bench.k1_bytes(M, K) == pytest.approx(33167360.0)
