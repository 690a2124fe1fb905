"""Host logic of bench.py that needs no GPU: the roofline's traffic figure is
taken from the committed ncu summary only while that summary was captured on
the kernel source as it stands."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_committed_decode_profile_is_plausible():
    # when the committed capture matches the decode sources, its DRAM bytes
    # per launch are at least the cache rows the step streams (37.76 MB) and
    # close to the step's algorithmic bytes (38.54 MB)
    traffic = bench.profiled_traffic()
    if traffic is not None:
        assert 37.76e6 <= traffic <= 1.1 * 38.54e6


def test_decode_step_bytes_of_the_b32_workload():
    # 16 sequences with 4097 tokens after the step (2049 rows at s = 2) and 16
    # with 4096 (2048 rows): the cache rows once, plus the per-sequence and
    # per-step terms the roofline counts
    import mtla_synth as synth
    d = synth.MAIN
    B = 32
    t_after = [4097 if b % 2 == 0 else 4096 for b in range(B)]
    rows = 16 * 2049 + 16 * 2048
    D = d.r + d.d_R
    expect = (rows * D * 2 + B * D * 2 + B * d.H * D * 2 + B * D * 2 + B * d.H * d.r * 4 + B * d.H * 4 +
              d.r * D * 4 + D * 4 + B * D * 4)
    assert bench.decode_step_bytes(t_after, d) == expect == 38538368


def test_traffic_is_dropped_when_the_source_changed(tmp_path, monkeypatch):
    summary = tmp_path / "summary.md"
    summary.write_text("# x\n\n- kernel_source_sha: `0000000000000000`\n"
                       "- dram_bytes_per_launch_full_size: `38088704`\n")
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(summary))
    assert bench.profiled_traffic() is None
    summary.write_text(f"# x\n\n- kernel_source_sha: `{bench.kernel_source_hash()}`\n"
                       "- dram_bytes_per_launch_full_size: `38088704`\n")
    assert bench.profiled_traffic() == 38088704.0


def test_traffic_is_dropped_without_a_summary(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(tmp_path / "missing.md"))
    assert bench.profiled_traffic() is None
