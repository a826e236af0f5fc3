"""Host logic of bench.py on CPU: the algorithmic units behind every roofline fraction, the
clock record, and the DRAM-traffic lookup."""
import json
import os
import tempfile

import numpy as np
import pytest

import bench
import synthetic


def brute_keys(T, D, W):
    """Number of (query, key) pairs of one head by explicit enumeration of the key set: the
    window (t - We, t] (We = max(W, 1)) and the chunk ends j = D-1 mod D older than it."""
    We = max(W, 1)
    t = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    causal = j <= t
    window = j > t - We
    chunk_end = (j % D) == D - 1
    return int(np.count_nonzero(causal & (window | chunk_end)))


def test_attended_keys_tiny_by_enumeration():
    # B1 H2 T256, D4, W0: 8,320 pairs per head, 16,640 in all
    w = synthetic.WORKLOADS["tiny_fp32"]
    u = bench.algorithmic(w)
    assert u["attended_keys"] == w.B * w.H * brute_keys(w.T, w.D, w.W) == 16640


def test_attended_keys_prefill_1p5b_by_enumeration():
    w = synthetic.WORKLOADS["prefill_1p5b"]
    u = bench.algorithmic(w)
    assert u["attended_keys"] == w.B * w.H * brute_keys(w.T, w.D, w.W)
    # 4 d FLOPs per attended pair: 17.2 GFLOP; the scan streams 5 N bytes: 335.5 MB
    assert u["attn_flops"] == 4 * w.d * u["attended_keys"]
    assert round(u["attn_flops"] / 1e9, 1) == 17.2
    assert u["recur_bytes"] == 5 * w.B * w.H * w.T * w.d * 2 == 335544320
    assert u["attn_bytes"] == 4 * w.B * w.H * w.T * w.d * 2


@pytest.mark.parametrize("name,keys_g,flops_g", [("window_2p6b", 0.1658, 84.9),
                                                  ("hybrid_7p6b", 4.55, 2327.0)])
def test_attended_keys_large_workloads(name, keys_g, flops_g):
    # the per-configuration totals: Σ_t |S(t)| and 4 d Σ_t |S(t)| to three significant digits
    w = synthetic.WORKLOADS[name]
    u = bench.algorithmic(w)
    assert u["attended_keys"] / 1e9 == pytest.approx(keys_g, rel=2e-3)
    assert u["attn_flops"] / 1e9 == pytest.approx(flops_g, rel=2e-3)


def test_attended_keys_with_sinks_by_enumeration():
    # sinks: the first n positions join every key set (counted once where a sink is a chunk end
    # or inside the window already)
    w = synthetic.Workload("s", B=1, H=1, d=64, T=300, D=8, W=16, dtype="f32")
    n = 5
    We = max(w.W, 1)
    t = np.arange(w.T)[:, None]
    j = np.arange(w.T)[None, :]
    keyset = (j <= t) & ((j > t - We) | ((j % w.D) == w.D - 1) | (j < n))
    assert bench.algorithmic(w, n_sink=n)["attended_keys"] == int(np.count_nonzero(keyset))


def test_clock_summary_reads_median_max_and_reasons():
    s = bench.ClockSampler(0)
    fd, s.path = tempfile.mkstemp(suffix=".csv")
    os.close(fd)
    lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1900, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 980.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    with open(s.path, "w") as f:
        f.write("\n".join(lines) + "\n")
    out = s.summary()
    assert out == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3}
    assert not os.path.exists(s.path)


def test_recorded_traffic_follows_the_source_hash():
    table = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for kernel_file, rows in table.items():
        for workload, e in rows.items():
            src = os.path.join(bench.ROOT, "recurrence_augmented_dilated_b200", "csrc", kernel_file)
            same = e["source_sha"] == bench.file_sha(src) and \
                e.get("headers_sha", bench.headers_sha()) == bench.headers_sha()
            want = e["dram_bytes_per_launch"] if same else None
            assert bench.recorded_traffic(kernel_file, workload) == want
            assert os.path.exists(os.path.join(bench.ROOT, "profiles", e["capture"]))
    assert bench.recorded_traffic("scan.cu", "no_such_workload") is None


def test_recorded_traffic_void_after_a_header_change(monkeypatch, tmp_path):
    # a table entry taken on the current sources, in a copy of the tree: valid until a shared
    # device header changes
    import shutil
    csrc = tmp_path / "recurrence_augmented_dilated_b200" / "csrc"
    csrc.mkdir(parents=True)
    src = os.path.join(bench.ROOT, "recurrence_augmented_dilated_b200", "csrc")
    for n in ("scan.cu",) + bench.KERNEL_HEADERS:
        shutil.copy(os.path.join(src, n), csrc / n)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    entry = {"dram_bytes_per_launch": 123, "source_sha": bench.file_sha(str(csrc / "scan.cu")),
             "capture": "x.md", "headers_sha": bench.headers_sha()}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"scan.cu": {"w": entry}}))
    assert bench.recorded_traffic("scan.cu", "w") == 123
    monkeypatch.setattr(bench, "headers_sha", lambda: "0000000000000000")
    assert bench.recorded_traffic("scan.cu", "w") is None
