"""Host-side helpers of bench.py on CPU: the FLOP and byte counts the
reported throughputs divide by, the rule that a recorded DRAM traffic figure
is used only while the kernel's source is the one it was measured on, the
peak table's fallback, and the workload tables' shapes."""
import json

import pytest

import bench


def test_flop_convention():
    # 4 B H N^2 d per forward (two N x N x d products), half under the causal mask
    w = dict(B=2, H=16, N=8192, d=128, causal=True)
    assert bench.fwd_flops(w) == 0.5 * 4 * 2 * 16 * 8192 ** 2 * 128
    assert bench.fwd_flops(dict(w, causal=False)) == 2 * bench.fwd_flops(w)


def test_decode_bytes_count_every_cache_row_once():
    w = dict(B=3, H=4, Nq=2, Nk=100, d=64)
    kv = 2 * 3 * 4 * 100 * 64 * 2          # K and V, bf16
    qo = 2 * 3 * 4 * 2 * 64 * 2            # Q in, O out, bf16
    assert bench.decode_bytes(w) == kv + qo + 3 * 4 * 2 * 4   # + LSE fp32


def test_recorded_traffic_follows_the_kernel_source(monkeypatch):
    with open(bench.os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        rec = json.load(f)
    for kernel, per_workload in rec.items():
        if kernel.startswith("_"):
            continue
        for workload, ent in per_workload.items():
            got = bench.recorded_traffic(kernel, workload)
            if ent["sources_hash"] == bench.kernel_sources_hash(kernel):
                assert got == float(ent["dram_bytes_per_launch"])
            else:
                assert got is None
    # a different source hash (the kernel changed since the capture) voids it
    monkeypatch.setattr(bench, "kernel_sources_hash", lambda kernel: "0" * 16)
    assert bench.recorded_traffic("fa_bwd_main_kernel", bench.DEFAULT_WORKLOAD) is None
    assert bench.recorded_traffic("fa_bwd_main_kernel", "no_such_workload") is None


def test_peaks_fall_back_when_the_measured_file_is_absent(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback"
    assert p["hbm_gbs"] == bench.FALLBACK_PEAKS["hbm_gbs"]
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000, "bf16_tflops": 1600}))
    p = bench.load_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6000.0 and p["bf16_tflops"] == 1600.0


@pytest.mark.parametrize("table", ["WORKLOADS", "QK8_WORKLOADS", "BIAS_WORKLOADS", "RING_WORKLOADS"])
def test_attention_workloads_are_well_formed(table):
    for name, w in getattr(bench, table).items():
        assert w["d"] in (64, 128) and w["N"] >= 1 and w["B"] >= 1 and w["H"] >= 1, name
        assert w["dist"] in ("normal", "row_scaled"), name
        if "G" in w:
            assert w["N"] % w["G"] == 0, name       # ring shards must divide N
    assert bench.DEFAULT_WORKLOAD in bench.WORKLOADS


def test_decode_workloads_are_well_formed():
    for name, w in bench.DECODE_WORKLOADS.items():
        assert 1 <= w["Nq"] <= w["Nk"] and w["d"] in (64, 128), name
