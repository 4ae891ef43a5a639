"""CPU tests of bench.py's measurement logic: the FLOP convention against a brute
count of visible (query, key) pairs, the workload table, the peak source, and the
rule that a committed ncu traffic figure is used only while the kernel sources it
was taken from are unchanged."""
import numpy as np
import pytest

import bench


def _visible_pairs(nq, nk, causal):
    """Brute force: key j visible to query i iff j <= i + (nk - nq) under the causal mask."""
    i = np.arange(nq)[:, None]
    j = np.arange(nk)[None, :]
    return int(np.sum(j <= i + (nk - nq))) if causal else nq * nk


@pytest.mark.parametrize("nq,nk", [(128, 128), (300, 300), (512, 8192), (1, 1000), (77, 300)])
def test_fwd_flops_counts_visible_pairs(nq, nk):
    B, H, d = 2, 3, 64
    assert bench.fwd_flops(B, H, nq, d, False, 1.0, nk) == 4.0 * B * H * d * _visible_pairs(nq, nk, False)
    # causal: the exact count minus the diagonal's half (N^2 / 2 for a square problem,
    # the convention of the pages' FLOP figures)
    assert bench.fwd_flops(B, H, nq, d, True, 1.0, nk) == 4.0 * B * H * d * (_visible_pairs(nq, nk, True) - nq / 2)


def test_fwd_flops_density_and_square_default():
    assert bench.fwd_flops(1, 16, 16384, 64, False, 0.25) == 0.25 * 4.0 * 16 * 16384 ** 2 * 64
    assert bench.fwd_flops(8, 16, 2048, 64, True) == 0.5 * bench.fwd_flops(8, 16, 2048, 64, False)


def test_workload_table():
    w = bench.workload("b8h16n2048d64")
    assert (w["B"], w["H"], w["N"], w["Nk"], w["d"]) == (8, 16, 2048, 2048, 64)
    assert [v[0] for v in w["variants"]] == ["noncausal", "causal"] and w["dropout_p"] == 0.0
    c = bench.workload("b4h16q512k8192d128_causal")
    assert (c["N"], c["Nk"], c["d"]) == (512, 8192, 128)
    s = bench.workload("sweep_N4096_d128_causal")
    assert (s["B"], s["H"], s["N"], s["d"]) == (4, 16, 4096, 128) and s["variants"][0][1] is True
    sp = bench.workload("b1h16n16384d64_sparse")
    assert sp["variants"] == [("blocksparse", False, 0.25)]
    dr = bench.workload("b8h16n2048d64_dropout")
    assert dr["dropout_p"] == 0.1


def test_peaks_come_from_the_measured_file():
    """The measured figures when the driver has written them on this machine, else
    the recipe's fallback figures, labelled as such."""
    import os
    p, kind = bench.peaks()
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert kind.startswith("measured")
    else:
        assert kind == "fallback" and p == bench.FALLBACK_PEAKS
    assert p["bf16_tflops"] > 1000 and p["hbm_gbs"] > 1000


def test_peaks_file_forms(tmp_path):
    """Every figure the bench divides by is present whatever the file holds: flat or
    nested keys are taken, missing or malformed ones fall back, and the label says so."""
    import json
    f = tmp_path / "peaks.json"
    full = {"hbm_gbs": 6529.4, "bf16_tflops": 1674.6, "bf16_tflops_sustained": 1388.6, "clocks": "1965 MHz"}
    f.write_text(json.dumps(full))
    assert bench.peaks(str(f)) == ({k: full[k] for k in bench.FALLBACK_PEAKS}, "measured")
    f.write_text(json.dumps({"gpu": "B200", "peaks": {k: full[k] for k in bench.FALLBACK_PEAKS}}))
    assert bench.peaks(str(f))[1] == "measured"
    f.write_text(json.dumps({"hbm_gbs": 6529.4, "bf16_tflops": "n/a", "bf16_tflops_sustained": True}))
    p, kind = bench.peaks(str(f))
    assert kind == "measured, partly fallback" and p["hbm_gbs"] == 6529.4
    assert p["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    assert p["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]
    for text in ("{not json", "[1, 2]", json.dumps({"other": 1})):
        f.write_text(text)
        assert bench.peaks(str(f)) == (bench.FALLBACK_PEAKS, "fallback")
    assert bench.peaks(str(tmp_path / "absent.json")) == (bench.FALLBACK_PEAKS, "fallback")


def test_traffic_only_while_sources_unchanged(tmp_path, monkeypatch):
    """A committed ncu figure is reported only while the kernel sources hash to the value
    stored with it."""
    h = bench.kernel_source_hash()
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "fa_bwd_dkdv_kernel_wl.txt").write_text(
        "# capture notes\nsource_hash: %s\ndram_bytes_per_launch: 123456789\n" % h)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: h)
    assert bench.profiled_traffic("fa_bwd_dkdv_kernel", "wl") == 123456789.0
    assert bench.profiled_traffic("fa_bwd_dkdv_kernel", "no_such_workload") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0000000000000000")
    assert bench.profiled_traffic("fa_bwd_dkdv_kernel", "wl") is None


def test_default_workload_is_the_long_context_config():
    """The default bench line is the largest single-GPU workload, the one the head-dim-128
    targets are stated on: B=2, H=16, N=8192, d=128, causal, forward + backward."""
    args = bench.build_parser().parse_args([])
    w = bench.workload(args.workload)
    assert (w["B"], w["H"], w["N"], w["d"]) == (2, 16, 8192, 128)
    assert [v[0] for v in w["variants"]] == ["causal"]
    assert args.gpus == 1 and args.warmup >= 3


def test_source_hash_covers_the_kernel_files(tmp_path, monkeypatch):
    import os
    import shutil
    csrc = tmp_path / "exact_tiled_attention_34_b200" / "csrc"
    csrc.mkdir(parents=True)
    for fn in bench.KERNEL_SOURCES:
        shutil.copy(os.path.join(bench.ROOT, "exact_tiled_attention_34_b200", "csrc", fn), csrc / fn)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    (csrc / "unrelated.cu").write_text("// not part of the profiled kernels\n")
    assert bench.kernel_source_hash() == h0
    with open(csrc / "fa_bwd.cuh", "a") as f:
        f.write("\n")
    assert bench.kernel_source_hash() != h0


def test_clock_samples_are_summarised():
    """The clock record that decides whether a run is kept: median SM clock, the largest
    maximum, and every throttle reason active in any sample."""
    na = "Not Active"
    rows = [f"0, 1965, 1965, 240.5, 0x0, {na}, {na}, {na}, {na}",
            f"0, 1665, 1965, 998.0, 0x4, {na}, {na}, {na}, Active",
            f"0, 1700, 1965, 990.1, 0x4, {na}, {na}, {na}, Active",
            "0, [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]",
            "garbage", ""]
    c = bench.parse_clock_lines(rows)
    assert c == {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    c = bench.parse_clock_lines([f"0, 1200, 1965, 700.0, 0x8, Active, {na}, Active, {na}"])
    assert c["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.parse_clock_lines(["[N/A]"]) is None and bench.parse_clock_lines([]) is None
    # with no samples the line is rated against the burst peak (no clock evidence of a cap)
    assert bench.ClockSampler(0).stop() is None
