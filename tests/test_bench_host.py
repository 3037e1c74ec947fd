"""Host-side logic of bench.py, on CPU: the algorithmic units the roofline
divides by, the peak and traffic sources it reports, and the reference arm's
JSON line.

The units are pinned by brute force: the prefill's causal flops by counting
every visible (query row, head, key) one by one, the decode's bytes by summing
every cached token's K and V rows for every KV head.
"""
import hashlib
import json
import os

import numpy as np
import pytest

import bench
from paged_kv_cache_376_b200 import workloads as W


def test_prefill_flops_count_every_visible_key():
    wl = W.prefill_workload([0, 5, 16, 40], [1, 31, 33, 64], seed=501)
    qsl, ctx = wl.query_start_loc, wl.context_lens
    visible = 0
    for s in range(wl.num_seqs):
        T = int(qsl[s + 1] - qsl[s])
        prefix = int(ctx[s]) - T
        for i in range(T):               # row i sees keys 0 .. prefix + i
            for key in range(int(ctx[s])):
                visible += key <= prefix + i
    want = 4 * wl.head_dim * wl.num_q_heads * visible
    assert wl.prefill_flops() == want
    got = bench._sample_work(wl, "prefill", range(wl.num_seqs)) * 1e12
    assert got == pytest.approx(want, rel=1e-12)
    assert bench._units(wl, "prefill")[1] == "TFLOP/s"


def test_decode_bytes_count_every_cached_row():
    wl = W.tiny_decode()
    rows = 0
    for s in range(wl.num_seqs):
        for _ in range(int(wl.context_lens[s])):
            rows += 2 * wl.num_kv_heads      # one K and one V row per head
    want = rows * wl.head_dim * 2            # bf16
    assert wl.kv_bytes_read() == want
    assert bench._sample_work(wl, "tiny", range(wl.num_seqs)) * 1e9 == \
        pytest.approx(want, rel=1e-12)
    assert bench._units(wl, "tiny") == (want / 1e9, "GB/s", wl.num_seqs)


def test_peaks_come_from_the_measured_file_else_the_fallback(tmp_path,
                                                             monkeypatch):
    # the file is written per machine; a stand-in with the same keys
    measured = tmp_path / "measured"
    measured.mkdir()
    p = {"hbm_gbs": 6538.3, "bf16_tflops": 1637.9,
         "bf16_tflops_sustained": 1372.0}
    (measured / "MEASURED_PEAKS.json").write_text(json.dumps(p))
    monkeypatch.setattr(bench, "ROOT", str(measured))
    hbm, bf16, sustained, src = bench._peaks()
    assert (hbm, bf16, src) == (p["hbm_gbs"], p["bf16_tflops"], "measured")
    assert sustained == p["bf16_tflops_sustained"]
    del p["bf16_tflops_sustained"]      # burst figure only: used for both
    (measured / "MEASURED_PEAKS.json").write_text(json.dumps(p))
    assert bench._peaks()[2] == p["bf16_tflops"]
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._peaks() == (bench.FALLBACK_HBM_GBS,
                              bench.FALLBACK_BF16_TFLOPS,
                              bench.FALLBACK_BF16_TFLOPS, "fallback")


def test_traffic_is_reported_only_while_the_sources_are_unchanged(
        tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("__global__ void k() {}\n")
    (tmp_path / "profiles").mkdir()
    entry = {"dram_bytes_per_launch": 123456,
             "sources": {"k.cu": hashlib.sha256(src.read_bytes()).hexdigest()},
             "summary": "profiles/k.md"}
    (tmp_path / "profiles" / "traffic.json").write_text(
        json.dumps({"tv_k@wl": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("tv_k", "wl") == 123456
    assert bench._traffic("tv_k", "other-workload") is None
    src.write_text("__global__ void k() { /* changed */ }\n")
    assert bench._traffic("tv_k", "wl") is None


def test_committed_traffic_entries_name_existing_sources_and_summaries():
    with open(bench.ROOT + "/profiles/traffic.json") as f:
        entries = json.load(f)
    assert entries
    for key, e in entries.items():
        kernel, workload = key.split("@")
        assert kernel.startswith("tv_") and workload
        assert e["dram_bytes_per_launch"] > 0
        for path in e["sources"]:
            assert os.path.isfile(os.path.join(bench.ROOT, path)), path
        assert os.path.isfile(os.path.join(bench.ROOT, e["summary"]))


def test_reference_arm_prints_one_json_line(capsys):
    assert bench.main(["--impl", "reference", "--workload", "tiny",
                       "--steps", "3", "--warmup", "3"]) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    r = json.loads(lines[0])
    assert r["impl"] == "reference" and r["unit"] == "GB/s"
    assert r["steps"] == 3 and r["warmup"] == 3 and r["n_gpus"] == 1
    assert r["higher_is_better"] is True and r["value"] > 0
    assert r["config"]["workload"] == W.tiny_decode().name
    assert r["cpu_baseline"]["kind"] == "oracle"
    assert r["cpu_baseline"]["value"] == r["value"]
    assert r["e2e"] == {"value": r["value"], "unit": "GB/s",
                        "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_fewer_than_three_warmup_steps_are_refused():
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--workload", "tiny",
                    "--steps", "3", "--warmup", "2"])


def test_prefill_config_names_the_ordered_step():
    wl = W.prefill_workload([0, 7], [16, 9], seed=502)
    cfg = bench._config(wl, "prefill")
    assert "tv_paged_prefill" in cfg["step"] and "ordered" in cfg["step"]
    assert cfg["query_rows"] == int(np.asarray(wl.q).shape[0])


def test_cpu_baseline_reports_all_cores_and_one_core():
    import oracle
    wl = W.tiny_decode()
    cores = oracle.max_threads()
    r = bench.cpu_baseline(wl, "tiny", budget_s=0.3)
    assert r["kind"] == "oracle" and r["unit"] == "GB/s"
    assert r["cores"] == cores and r["value"] > 0
    one = r["single_core"]
    assert one["cores"] == 1 and one["value"] > 0 and one["unit"] == "GB/s"
    assert oracle.max_threads() == cores        # thread count restored


def test_roofline_peak_follows_the_bound_and_the_timed_region():
    hbm, burst, sus = 6538.3, 1637.9, 1372.1
    assert bench._roofline_peak("GB/s", 0.01, hbm, burst, sus) == \
        (hbm, "hbm", "hbm_gbs")
    assert bench._roofline_peak("GB/s", 30.0, hbm, burst, sus) == \
        (hbm, "hbm", "hbm_gbs")
    assert bench._roofline_peak("TFLOP/s", 0.006, hbm, burst, sus) == \
        (burst, "tensor", "bf16_tflops")
    assert bench._roofline_peak("TFLOP/s", bench.SUSTAINED_S, hbm, burst,
                                sus) == (sus, "tensor",
                                         "bf16_tflops_sustained")


def test_l2_is_flushed_only_where_the_working_set_could_stay_in_l2():
    """Steps whose touched bytes (cached K/V + q + out) are under twice the
    126 MB L2 are timed one by one with L2 flushed in between; the decode
    configurations stream more than that and run back to back."""
    tiny = W.tiny_decode()
    assert bench.working_set_bytes(tiny) == (tiny.kv_bytes_read()
                                             + 2 * tiny.q.nbytes)
    assert bench.flushes_l2(tiny)
    small_prefill = W.prefill_workload([100, 0], [64, 64], seed=3)
    assert bench.flushes_l2(small_prefill)
    # 64 x 2048 tokens x 2 KB = 268 MB of K/V: more than twice L2
    big = W.decode_workload([2048] * 64, num_pages=8192, seed=4)
    assert big.kv_bytes_read() == 268435456
    assert not bench.flushes_l2(big)
    assert bench.flushes_l2(big, l2_bytes=1 << 30)
    cfg = bench._config(tiny, "tiny")
    assert "flushed" in cfg["l2"]
