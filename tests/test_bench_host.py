"""Host parts of bench.py (no GPU): the clock summary taken from nvidia-smi samples during the timed
region (median SM clock, throttle reasons that were active at any sample), and the DRAM traffic
record, which is reported only while the kernel sources match the ones it was measured on."""
import json
import os

import bench


def test_clock_summary_median_and_reasons():
    s = bench.ClockSampler(0)
    s.lines = [
        "0, 1965, 1965, 690.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 999.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 950.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    out = s.summary()
    assert out == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    s.lines = ["0, 1200, 1965, 500, 0x8, Not Active, Active, Not Active, Not Active"]
    assert s.summary()["reasons"] == ["hw_thermal_slowdown"]
    s.lines = []
    assert s.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_traffic_record_follows_the_kernel_sources(monkeypatch):
    import pathlib
    root = pathlib.Path(bench.ROOT) / "_build" / "bench_host"      # the ignored build folder
    prof = root / "profiles"
    prof.mkdir(parents=True, exist_ok=True)
    rec = {"some_kernel": {"source_hash": "abc", "bytes_per_launch": 123}}
    (prof / "dram_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench._traffic_record("some_kernel", "abc") == rec["some_kernel"]
    assert bench._traffic_record("some_kernel", "changed") is None
    assert bench._traffic_record("other_kernel", "abc") is None
    # the hash covers the listed sources byte for byte
    src = root / "k.cu"
    src.write_text("a")
    h1 = bench._kernel_hash(["k.cu"])
    src.write_text("b")
    assert bench._kernel_hash(["k.cu"]) != h1


def test_committed_traffic_record_names_the_decode_kernel():
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        rec = json.load(f)
    r = rec["gqa_tc_wide_kernel"]
    assert r["bytes_per_launch"] > 0 and 1.0 <= r["traffic_over_algorithmic"] < 1.1


def test_physical_gpu_and_rank_environment(monkeypatch):
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3,5")
    assert bench._physical_gpu(0) == 3 and bench._physical_gpu(1) == 5 and bench._physical_gpu(2) == 2
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-1234abcd")     # UUIDs: keep the local index
    assert bench._physical_gpu(0) == 0
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    assert bench._physical_gpu(1) == 1
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench._dist() == (1, 0, 0)
    monkeypatch.setenv("WORLD_SIZE", "4")
    monkeypatch.setenv("RANK", "2")
    monkeypatch.setenv("LOCAL_RANK", "2")
    assert bench._dist() == (4, 2, 2)


def test_kv_bytes_counts_k_and_v_once():
    from workloads import tiny_gqa_case
    c = tiny_gqa_case()
    # lengths {37, 128, 200, 256} x 2 KV heads x 64 dims x 2 bytes x (K, V)
    assert bench._kv_bytes(c) == (37 + 128 + 200 + 256) * 2 * 64 * 2 * 2
