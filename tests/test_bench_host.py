"""Host-side logic of bench.py: argument defaults, the timing rules it
enforces, the peak denominators and the recorded DRAM-traffic figure (which
must vanish as soon as the decode kernel's sources change)."""

import importlib.util
import json
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", ROOT / "bench.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_defaults_are_one_gpu_and_a_short_run(bench):
    a = bench.parse([])
    assert (a.gpus, a.impl, a.workload) == (1, "ours", bench.DEFAULT_WORKLOAD)
    assert a.warmup >= 3 and 0 < a.steps <= 1000


def test_warmup_is_raised_to_three(bench, monkeypatch):
    seen = {}

    def fake_run(args):
        seen["warmup"] = args.warmup
        return 0

    monkeypatch.setattr(bench, "run_ours", fake_run)
    bench.main(["--warmup", "1", "--steps", "2"])
    assert seen["warmup"] == 3


def test_peaks_come_from_the_measured_file_when_present(bench):
    peaks = bench.measured_peaks()
    if (ROOT / "MEASURED_PEAKS.json").exists():
        d = json.loads((ROOT / "MEASURED_PEAKS.json").read_text())
        assert peaks["source"] == "measured" and peaks["hbm_gbs"] == float(d["hbm_gbs"])
    else:
        assert peaks["source"] == "fallback"


def test_recorded_traffic_follows_the_decode_sources(bench, tmp_path, monkeypatch):
    rec = json.loads((ROOT / "profiles" / "decode_traffic.json").read_text())
    current = rec["source_hash"] == bench.kernel_source_hash()
    assert bench.recorded_traffic(rec["workload"]) == (rec["dram_bytes_per_launch"] if current else None)
    assert bench.recorded_traffic("no_such_workload") is None
    # the same record in a copy of the tree whose decode sources differ by one byte
    fake = tmp_path / "repo"
    (fake / "profiles").mkdir(parents=True)
    (fake / "mla_latent_kv_39_b200" / "csrc").mkdir(parents=True)
    for name in bench.DECODE_SOURCES:
        (fake / "mla_latent_kv_39_b200" / "csrc" / name).write_bytes(
            (ROOT / "mla_latent_kv_39_b200" / "csrc" / name).read_bytes())
    src = fake / "mla_latent_kv_39_b200" / "csrc" / bench.DECODE_SOURCES[-1]
    src.write_bytes(src.read_bytes() + b"\n")
    (fake / "profiles" / "decode_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", fake)
    assert bench.recorded_traffic(rec["workload"]) is None


def test_rank_seeds_differ_per_rank(bench):
    assert len({bench.rank_seed(0, r) for r in range(8)}) == 8


def test_percentiles_are_nearest_rank(bench):
    assert bench.percentiles([]) is None
    assert bench.percentiles([7.0]) == {"p50": 7.0, "p95": 7.0, "p99": 7.0}
    p = bench.percentiles([float(x) for x in range(200, 0, -1)])   # order does not matter
    assert p == {"p50": 100.0, "p95": 190.0, "p99": 198.0}


def test_reference_arm_reports_the_gpu_arms_metric(bench):
    import inspect
    src = inspect.getsource(bench.run_reference) + inspect.getsource(bench.run_ours)
    assert src.count('"metric": METRIC') == 2


def test_decode_roofline_counts_causal_rows_and_picks_the_larger_floor(bench):
    import torch
    from mla_synth import WORKLOADS, generate, reduced
    peaks = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}
    for n_q, bound in ((1, "hbm"), (64, "tensor")):
        wl = reduced(WORKLOADS["v3_prefill_b8_c64_ragged1k_4k"], lengths=[0, 5, 300], n_q=n_q)
        data = generate(wl)
        # visible rows, one query row at a time: sequence b's row j sees L_b + j + 1 rows
        visible = sum(int(data.cached_len[b]) + j + 1 for b in range(wl.batch) for j in range(n_q))
        sh = wl.shape
        assert bench.decode_flops(wl, data) == visible * (2 * sh.n_heads * (2 * sh.d_c + sh.d_r))
        cache = int(data.seq_lens.sum()) * sh.row * sh.elem_bytes
        r = bench.decode_roofline(wl, data, cache, 1e-4, peaks, None)
        assert r["bound"] == bound
        floor = max(r["hbm_floor_us"], r["tensor_floor_us"]) if bound == "tensor" else r["hbm_floor_us"]
        assert abs(r["frac"] - floor / 100.0) < 1e-9
