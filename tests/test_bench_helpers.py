"""CPU checks of the benchmark's bookkeeping: work accounting, clock parsing, the traffic record
and the peak fallback. These feed the numbers of the JSON line, so they are pinned here."""
import hashlib
import json

import bench
import oracle
import synth


def test_row_flops_sum_to_the_forward_flops():
    w = bench.workload(seq_len=1000, hq=3, hkv=1)
    w.update(B=2, block_size=96, topk=4, d=128)
    rows = [(b, h, t) for b in range(w["B"]) for h in range(w["Hq"]) for t in range(w["N"])]
    assert bench.rows_useful_flops(w, rows) == bench.useful_flops(w)


def test_row_flops_match_the_oracle_selection():
    """4 d x (keys a row attends), with the keys counted from the oracle's own selection."""
    B, N, Hq, Hkv, d, bs, k = 1, 700, 2, 1, 16, 64, 3
    q, kk, v = synth.inputs(B, N, Hq, Hkv, d, bs, 9)
    r = oracle.forward(q, kk, v, bs, k)
    keys = 0
    for (b, h, t), sel in zip(r["rows"], r["sel"]):
        c = t // bs
        for j in sel:
            if j < 0:
                continue
            keys += (t - c * bs + 1) if j == c else bs
    w = dict(B=B, N=N, Hq=Hq, Hkv=Hkv, d=d, block_size=bs, topk=k)
    assert bench.rows_useful_flops(w, r["rows"]) == 4.0 * d * keys


def test_clock_summary_ignores_idle_samples_and_collects_reasons():
    cs = bench.ClockSampler("0")
    cs.lines = [
        "1965, 1965, 120.5, Not Active, Not Active, Not Active, Not Active",   # idle: ignored
        "1600, 1965, 998.0, Not Active, Not Active, Not Active, Active",
        "1590, 1965, 1001.2, Not Active, Not Active, Not Active, Active",
        "1610, 1965, 990.0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    s = cs.summary()
    assert s == {"sm_mhz": 1600.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_summary_without_samples():
    cs = bench.ClockSampler("0")
    cs.lines = []
    assert cs.summary()["samples"] == 0


def test_traffic_record_is_ignored_once_the_kernel_sources_change(tmp_path, monkeypatch):
    src = [tmp_path / "a.cuh", tmp_path / "b.cuh"]
    src[0].write_text("kernel a")
    src[1].write_text("kernel b")
    h = hashlib.sha256(b"kernel a" + b"kernel b").hexdigest()
    rec = tmp_path / "traffic.json"
    rec.write_text(json.dumps({"source_sha256": h, "bytes_per_full_launch": 1.5e11}))
    monkeypatch.setattr(bench, "ATTN_SRC", [str(p) for p in src])
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.attention_traffic() == 1.5e11
    src[1].write_text("kernel b, changed")
    assert bench.attention_traffic() is None


def test_peaks_fall_back_when_the_measured_file_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, source = bench.read_peaks()
    assert source == "fallback" and peaks == bench.FALLBACK_PEAKS
