"""Host-side logic of bench.py that decides what its JSON line reports: the
tensor peak a GEMM fraction is divided by, and the kernel-version key that
ties the stored ncu traffic to the GEMM's code."""
import os
import shutil

import bench

PEAKS = {"hbm_gbs": 6549.0, "bf16_tflops": 1657.1, "bf16_tflops_sustained": 1394.4}


def test_short_unthrottled_region_uses_the_burst_peak():
    peak, which = bench.tensor_peak(PEAKS, 0.05, {"reasons": []})
    assert peak == PEAKS["bf16_tflops"] and which.startswith("bf16_tflops ")
    peak, _ = bench.tensor_peak(PEAKS, 0.05, None)  # no clock record
    assert peak == PEAKS["bf16_tflops"]


def test_power_capped_or_long_region_uses_the_sustained_peak():
    peak, which = bench.tensor_peak(PEAKS, 0.05, {"reasons": ["sw_power_cap"]})
    assert peak == PEAKS["bf16_tflops_sustained"] and "sw_power_cap" in which
    peak, which = bench.tensor_peak(PEAKS, 4.0, {"reasons": []})
    assert peak == PEAKS["bf16_tflops_sustained"] and which.startswith("bf16_tflops_sustained")


def test_missing_peaks_fall_back_to_the_stated_figures():
    peak, _ = bench.tensor_peak({}, 0.05, {"reasons": []})
    assert peak == bench.FALLBACK_PEAKS["bf16_tflops"]


def _copy_sources(tmp_path):
    src = os.path.join(bench.ROOT, "bit_nf4_quantized_blockwise_b200", "csrc")
    dst = tmp_path / "bit_nf4_quantized_blockwise_b200" / "csrc"
    dst.mkdir(parents=True)
    for name in ("pairgemm.cuh", "common.cuh"):
        shutil.copy(os.path.join(src, name), dst / name)
    return dst


def test_kernel_key_ignores_comments_and_blank_lines(tmp_path, monkeypatch):
    key = bench.kernel_source_hash()
    dst = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_source_hash() == key
    f = dst / "pairgemm.cuh"
    text = f.read_text()
    f.write_text("// a new header line\n\n" + text.replace("\n", "  // trailing remark\n", 3) + "\n\n")
    assert bench.kernel_source_hash() == key


def test_kernel_key_changes_with_the_code(tmp_path, monkeypatch):
    key = bench.kernel_source_hash()
    dst = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = dst / "pairgemm.cuh"
    text = f.read_text()
    assert "PG_STAGES = 3" in text
    f.write_text(text.replace("PG_STAGES = 3", "PG_STAGES = 4", 1))
    assert bench.kernel_source_hash() != key


def test_stored_traffic_is_dropped_for_another_kernel_version(tmp_path, monkeypatch):
    dst = _copy_sources(tmp_path)
    prof = tmp_path / "profiles"
    prof.mkdir()
    shutil.copy(os.path.join(bench.ROOT, bench.TRAFFIC_PROFILE), prof / os.path.basename(bench.TRAFFIC_PROFILE))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    stored = bench.stored_traffic()
    f = dst / "pairgemm.cuh"
    f.write_text(f.read_text().replace("PG_STAGES = 3", "PG_STAGES = 4", 1))
    assert bench.stored_traffic() is None
    if stored is not None:
        assert stored > 0
