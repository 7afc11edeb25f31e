"""bench.py's host-side arithmetic: the work model behind `roofline` and `step_roofline`,
the peaks it divides by, and the lookup of measured DRAM traffic (CPU only).

The expected numbers are worked out by hand for the benchmarked workload (4 layers of
1024 x 1024, r = 128, B = 64, T = 128, bf16 inputs): B*T = 8192 stacked rows.
"""
import json

import pytest

import bench
import workloads as W

MIB = 1 << 20


def test_step_work_of_the_bench_workload():
    flops, byts = bench.step_work(W.get("mlp4x1024"))
    # per layer: 2*8192*128*(1024+1024) for the two contractions of the projection and
    # 2*1024*128*1024 for the back-projection
    assert flops == 4 * (4_294_967_296 + 268_435_456) == 18_253_611_008
    # per layer: A and Gout once (8192 * 2048 * 2 B = 32 MiB), W read + written (8 MiB),
    # m and v read + written (16 * 128 * 1024 B = 2 MiB)
    assert byts == 4 * (32 + 8 + 2) * MIB == 176_160_768


def test_phase_work_of_the_tensor_core_path():
    w = W.get("mlp4x1024")
    work = bench.phase_work(w, "tc")
    # aggregation: Gout (16 MiB) + AP (2 MiB) + S written (0.5 MiB) per layer
    assert work["aggregate"]["bytes"] == 4 * (16 * MIB + 2 * MIB + MIB // 2) == 77_594_624
    assert work["aggregate"]["flops"] == 4 * 2 * 8192 * 128 * 1024
    # projection: A (16 MiB) + AP written (2 MiB) per layer
    assert work["project"]["bytes"] == 4 * 18 * MIB
    # back-projection: W read + written (8 MiB), P and dR in bf16 (0.25 MiB each)
    assert work["backproject"]["bytes"] == 4 * (8 * MIB + MIB // 2)
    # P in bf16: 1024 x 128 x 2 B per layer
    assert work["gen_P"]["bytes"] == 4 * 256 * 1024
    # fp32 P, AP and dR on the CUDA-core path
    assert bench.phase_work(w, "simt")["gen_P"]["bytes"] == 4 * 512 * 1024


def test_phase_work_with_the_stored_aggregation():
    w = W.get("mlp4x1024")
    work = bench.phase_work(w, "tc", "store")
    # each R_i in bf16: B * r * d_out * 2 B = 64 * 128 * 1024 * 2 = 16 MiB per layer
    r_bytes = 4 * 16 * MIB
    # the norm phase reads Gout (16 MiB) and AP (2 MiB) and writes the R_i
    assert work["norm"]["bytes"] == 4 * 18 * MIB + r_bytes
    assert work["norm"]["flops"] == 4 * 2 * 8192 * 128 * 1024
    # the aggregation alone: R_i read once, S written (0.5 MiB per layer), no contraction
    assert work["aggregate"] == {"bytes": r_bytes + 4 * MIB // 2, "flops": 0}
    # fused with noise + Adam: R_i read, S written, m and v read and written (16 B per
    # element), dR written in bf16: 128 * 1024 * (4 + 16 + 2) B per layer
    assert work["aggregate_adam"] == {"bytes": r_bytes + 4 * 128 * 1024 * 22, "flops": 0}
    # the recomputed aggregation has no fused phase
    assert "aggregate_adam" not in bench.phase_work(w, "tc")


def test_sqnorms_work_counts_both_contractions_and_the_outputs():
    w = W.get("mlp4x1024")
    flops, byts = bench.sqnorms_work(w)
    assert flops == 4 * 2 * 8192 * 128 * 2048
    assert byts == 4 * 32 * MIB + 4 * 64


def test_layer_summary():
    assert bench.layer_summary(W.get("mlp4x1024")) == "4x1024x1024"
    mixed = W.scaled(W.get("vit_b"), layers=((768, 2304), (3072, 768), (768, 2304)))
    assert bench.layer_summary(mixed) == "3 layers of 768x2304, 3072x768"


def test_peaks_fall_back_when_the_measured_file_is_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "absent.json"))
    pk = bench.peaks()
    assert pk["source"] == "fallback" and pk["hbm_gbs"] == 6650.0 and pk["bf16_tflops"] == 1590.0
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"hbm_gbs": 6500.5, "bf16_tflops": 1600.0}))
    monkeypatch.setattr(bench, "PEAKS_FILE", str(f))
    pk = bench.peaks()
    assert pk["source"] == "measured" and pk["hbm_gbs"] == 6500.5
    assert pk["bf16_tflops_sustained"] == 1600.0      # burst stands in when absent


def test_traffic_is_reported_only_for_the_code_it_was_measured_on(monkeypatch, tmp_path):
    sha = bench.kernel_source_sha("tc")
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps({
        "tc:aggregate:mlp4x1024": {"dram_bytes_per_launch": 8.89e6, "source_sha": sha},
        "tc:norm:mlp4x1024": {"dram_bytes_per_launch": 8.0e7, "source_sha": "0" * 16},
        "tc:norm:mlp4x1024:sqnorms": {"dram_bytes_per_launch": 7.0e7, "source_sha": sha},
    }))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.traffic_for("aggregate", "mlp4x1024", "tc") == 8.89e6
    assert bench.traffic_for("norm", "mlp4x1024", "tc") is None            # stale counters
    assert bench.traffic_for("norm", "mlp4x1024", "tc", "sqnorms") == 7.0e7
    assert bench.traffic_for("project", "mlp4x1024", "tc") is None         # never measured


def test_source_hash_ignores_comments_but_not_code(monkeypatch, tmp_path):
    csrc = tmp_path / "random_gradient_projection_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in ("simt.cu", "philox.cuh"):
        (csrc / n).write_text("int f() { return 1; }\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_source_sha("simt")
    (csrc / "simt.cu").write_text("// a comment\nint f() { return 1; }  /* another */\n\n")
    assert bench.kernel_source_sha("simt") == base
    (csrc / "philox.cuh").write_text("int f() { return 2; }\n")
    assert bench.kernel_source_sha("simt") != base


@pytest.mark.parametrize("name", sorted(W.WORKLOADS))
def test_every_workload_has_a_positive_step_roofline(name):
    w = W.get(name)
    flops, byts = bench.step_work(w)
    pk = bench.peaks()
    assert flops > 0 and byts > 0
    t = max(flops / (pk["bf16_tflops"] * 1e12), byts / (pk["hbm_gbs"] * 1e9))
    assert 0 < t < 1.0
