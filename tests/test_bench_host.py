"""Host-side arithmetic of bench.py (no GPU): the algorithmic FLOP and byte counts that
every roofline fraction divides by, and the hash guard on the recorded DRAM traffic."""

import hashlib
import json
import os

import pytest

import bench
from hybrid_sliding_window_sink_b200 import workloads as wl


def _pairs_brute(n, window):
    if window <= 0 or window >= n:
        return sum(i + 1 for i in range(n))
    return sum(i - max(0, i - window + 1) + 1 for i in range(n))


@pytest.mark.parametrize("n", [1, 5, 130, 300])
@pytest.mark.parametrize("window", [0, 1, 7, 128, 129, 500])
def test_swa_pairs_matches_brute_force(n, window):
    assert bench.swa_pairs(n, window) == _pairs_brute(n, window)


def test_headline_prefill_work():
    """SWA layer, n=32768, 64 Q / 8 KV, W=128: 171.5 GFLOP and 1.518 GB algorithmic."""
    flops, nbytes = bench.prefill_work(wl.SWA_PREFILL)
    pairs = 32768 * 128 - 128 * 127 // 2
    assert flops == 2.0 * (192 + 128) * pairs * 64
    assert abs(flops / 171.5e9 - 1) < 1e-3
    q = 32768 * 64 * 192 * 2
    kv = 32768 * 8 * (192 + 128) * 2
    o = 32768 * 64 * 128 * 2
    lse = 64 * 32768 * 4
    assert nbytes == q + kv + o + lse + 64 * 4
    assert abs(nbytes / 1.518e9 - 1) < 1e-3


def test_decode_byte_counts():
    hq, hkv = 64, 8
    ring = bench.decode_layer_bytes([100, 300], hq, hkv, "ring", 128)
    lin = bench.decode_layer_bytes([100, 300], hq, hkv, "linear", 4096)
    per_tok = hkv * (192 + 128) * 2
    assert lin - ring == (300 - 128) * per_tok           # the ring holds only 128 slots
    # one-token multi-query decode counts exactly what decode counts
    assert bench.mtp_layer_bytes([100, 300], hq, hkv, "ring", 128, 1) == ring
    # FP8: 320 B of E4M3 + two fp32 scales per (token, KV head), same q / out / lse
    fp8 = bench.fp8_decode_layer_bytes([100, 300], hq, hkv, "linear", 4096)
    assert lin - fp8 == 400 * hkv * (640 - 328)


def test_roofline_fields():
    r = bench.roofline_hbm(6.5578e9, 1.0, {"hbm_gbs": 6557.8}, "measured", traffic=123)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] == 123
    assert r["achieved"] == 6557.8 and r["frac"] == 1.0
    t = bench.roofline_tensor(1.6637e12, 1.0, 1663.7, "measured")
    assert t["bound"] == "tensor" and abs(t["frac"] - 1.0) < 1e-9


def test_traffic_reported_only_while_sources_match(tmp_path, monkeypatch):
    csrc = tmp_path / "hybrid_sliding_window_sink_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_text("kernel v1\n")
    sha = hashlib.sha256(b"kernel v1\n").hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    rec = {"k": {"sources": ["k.cuh"], "sha": sha, "bytes_per_unit": 10.5}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("k", 4) == 42
    assert bench.traffic_for("missing", 4) is None
    (csrc / "k.cuh").write_text("kernel v2\n")             # the kernel changed: no traffic
    assert bench.traffic_for("k", 4) is None


def test_recorded_traffic_files_exist():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for key, r in rec.items():
        if key.startswith("_"):
            continue
        assert os.path.exists(os.path.join(bench.ROOT, r["capture"])), key
        for src in r["sources"]:
            assert os.path.exists(os.path.join(bench.ROOT, "hybrid_sliding_window_sink_b200", "csrc", src))


def _run_reference(monkeypatch, capsys, rank="0"):
    monkeypatch.setattr(bench, "REF_SECONDS", 0.5)
    monkeypatch.setattr(bench, "REF_CORES", 2)
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3"])
    monkeypatch.setenv("RANK", rank)
    monkeypatch.setenv("WORLD_SIZE", "2" if rank != "0" else "1")
    monkeypatch.setenv("LOCAL_RANK", rank)
    bench.main()
    return [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]


def test_reference_arm_json_contract(monkeypatch, capsys):
    """`bench.py --impl reference` (the float64 oracle on host cores, two processes and a
    short budget here): one JSON line with the contract's keys, the oracle as its cpu_baseline."""
    lines = _run_reference(monkeypatch, capsys)
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] >= 3 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["dtype"] == "f64" and d["data"] == "synthetic"
    assert d["config"]["workload"] == wl.SWA_PREFILL.name
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing(monkeypatch, capsys):
    assert _run_reference(monkeypatch, capsys, rank="1") == []


def _fake_workloads():
    hb = lambda f: {"bound": "hbm", "achieved": 4321.5, "peak": 6452.2, "unit": "GB/s", "frac": f,  # noqa: E731
                    "traffic": 123456789012, "peak_source": "measured"}
    step = {"value": 5123.4, "unit": "GB/s", "ms_per_step": 20.1234, "ga_layer": hb(0.8123),
            "swa_layer": hb(0.6123), "roofline": hb(0.7912), "ms_ga_layer": 2.1234, "ms_swa_layer": 0.01234}
    return {
        "tiny_prefill": {"ms": 0.01234, "tflops": 51.23, "frac": 0.0712, "device_error": 0},
        "ga_prefill": {"value": 1012.34, "ms_per_step": 21.7234, "device_error": 0,
                       "roofline": {"frac": 0.6123, "traffic": 1434567890}},
        "chunk_prefill": {"swa": {"ms": 0.2123, "roofline": hb(0.5123)},
                          "ga": {"ms": 16.1234, "tflops": 1012.34, "roofline": {"frac": 0.6123}}},
        "hybrid_decode_step": dict(step), "fp8_decode_step": dict(step), "mtp_decode_step": dict(step),
        "token_select": {"ms_per_call": 0.5812, "value": 5766.1, "roofline": hb(0.8812)},
        "sparse_decode": {"ms_per_call": 0.00812, "value": 2961.2, "roofline": hb(0.4512)},
    }


def test_bench_line_fits_the_driver_tail():
    """The whole JSON line, with every workload and the CPU baseline, stays well under the
    ~3000 characters of stdout the driver keeps, so every figure is recorded."""
    w = bench.compact_workloads(_fake_workloads())
    assert set(w) == {"tiny_prefill", "ga_prefill", "chunk_swa", "chunk_ga", "decode_step", "fp8_step",
                      "mtp_step", "select", "sparse"}
    line = {"metric": bench.METRIC, "value": 376.155, "unit": "TFLOP/s", "n_gpus": 1, "steps": 20,
            "warmup": 5, "ms_per_step": 0.45584, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.SWA_PREFILL.name, "global_batch": 1, "seq_len": 32768,
                       "parallelism": "dp1", "l2": "inputs > L2"},
            "roofline": {"bound": "hbm", "achieved": 3330.9, "peak": 6452.2, "unit": "GB/s", "frac": 0.5079,
                         "traffic": 1419895808}, "peaks": "measured",
            "tensor": {"achieved": 376.15, "frac": 0.2261}, "gpu_launches": 20,
            "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]},
            "device_error": 0,
            "e2e": {"value": 6.225, "unit": "TFLOP/s", "h2d_bytes_per_step": 973078784,
                    "d2h_bytes_per_step": 545259520, "ms_per_step": 27.545},
            "workloads": w,
            "cpu_baseline": {"value": 0.0123456789, "unit": "TFLOP/s", "cores": 224, "kind": "oracle",
                             "sample": "x" * 200,
                             "per_config": {k: [12345.67, "extra"] for k in
                                            ("tiny_prefill", "swa_prefill", "ga_prefill", "swa_decode",
                                             "ga_decode", "sparse_decode")}}}
    text = json.dumps(line, separators=(",", ":"))
    assert len(text) < 2600, len(text)
