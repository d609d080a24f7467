"""The roofline numerator: algorithmic bytes of one decode launch (packed codes, one fp16
scale and zero per 32 elements, the bf16 residual of per-channel keys, bf16 q in and out),
checked against hand computations of that definition."""
import sys
import os

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_small_case_by_hand():
    # per-channel K4V2, B = Hkv = G = 1, D = 64, L = 37: one 32-token key group
    # (32*64*(4+1)/8 = 1280) + 5 residual rows (5*64*2 = 640); values 37*64*(2+1)/8 = 888;
    # q and out 2*1*64*2 = 256
    assert bench.decode_bytes(1, 1, 1, 64, 37, 4, 2, 0) == 1280 + 640 + 888 + 256
    # per-token keys: 37*64*5/8 = 1480 for the keys, no residual
    assert bench.decode_bytes(1, 1, 1, 64, 37, 4, 2, 1) == 1480 + 888 + 256


def test_context_4096_k4v2_layer():
    # 64 x 8 units; keys 128 groups x 32 x 128 x 5/8 = 327680; values 4096 x 128 x 3/8 =
    # 196608; q/out 2 x 4 x 128 x 2 = 2048: 526336 per unit, 269.5 MB per layer
    assert bench.decode_bytes(64, 8, 4, 128, 4096, 4, 2, 0) == 512 * 526336 == 269484032


def test_context_8192_k8v2_layer():
    # 32 x 4 units, GQA 7; keys 256 x 32 x 128 x 9/8 = 1179648; values 8192 x 128 x 3/8 =
    # 393216; q/out 2 x 7 x 128 x 2 = 3584: 1576448 per unit, 201.8 MB per layer
    assert bench.decode_bytes(32, 4, 7, 128, 8192, 8, 2, 0) == 128 * 1576448 == 201785344


def test_default_schedule_mean():
    # the default workload's 128 decode steps (L = 129..256), K8V4: 24.0 MB per layer on average
    mean = sum(bench.decode_bytes(64, 8, 4, 128, L, 8, 4, 0) for L in range(129, 257)) / 128
    assert mean == pytest.approx(24.0e6, rel=2e-3)


def test_decode_paths_entry():
    """Per-path launch time and roofline fraction: GB/s = algorithmic bytes / time."""
    d = bench.decode_paths_entry(18_395_136.0, 0.008, 0.032, 6558.7, "decode_split_kernel")
    assert d["mma_sync"]["kernel"] == "decode_split_kernel"
    assert d["mma_sync"]["avg_launch_us"] == pytest.approx(8.0)
    assert d["mma_sync"]["hbm_gbs"] == pytest.approx(18_395_136.0 / 8e-6 / 1e9)
    assert d["mma_sync"]["frac"] == pytest.approx(d["mma_sync"]["hbm_gbs"] / 6558.7)
    assert d["tcgen05"]["kernel"] == "decode_umma_kernel"
    assert d["tcgen05"]["frac"] == pytest.approx(d["mma_sync"]["frac"] / 4)
    assert "tcgen05" not in bench.decode_paths_entry(1e6, 0.01, None, 6558.7, "decode_paged_kernel")


def test_captured_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    """The committed traffic blocks are used only while their source hash matches, scaled
    to the caller's algorithmic bytes."""
    sha = bench.kernel_source_sha256()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "decode_split_traffic.txt").write_text(
        f"# test\nsource_sha256: {sha}\nworkload: w\nkernel: k\nL: 1\ndram_bytes: 104\nalgorithmic_bytes: 100\n\n"
        f"source_sha256: {'0' * 64}\nworkload: v\nkernel: k\nL: 1\ndram_bytes: 200\nalgorithmic_bytes: 100\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha256", lambda: sha)
    assert bench.captured_traffic("w", 1000.0) == pytest.approx(1040.0)
    assert bench.captured_traffic("v", 1000.0) is None      # stale hash
    assert bench.captured_traffic("x", 1000.0) is None      # no capture
