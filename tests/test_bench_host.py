"""Host-side pieces of bench.py: the DRAM-traffic record lookup, the clock-log
parser and the algorithmic FLOP count (no GPU needed)."""
import hashlib
import json
import os

import bench
import workloads


def test_traffic_record_used_only_while_the_source_hash_matches(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel source\n")
    (tmp_path / "profiles").mkdir()
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    rec = {"attention:wan": {"workload": "wan", "source": "k.cu", "sha256": sha, "dram_bytes_per_launch": 123456},
           "attention:ropeslr": {"workload": "ropeslr", "source": "k.cu", "sha256": sha,
                                 "dram_bytes_per_launch": 654321}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("attention") == 123456
    assert bench.measured_traffic("attention", "ropeslr") == 654321
    assert bench.measured_traffic("attention", "lvsa") is None
    assert bench.measured_traffic("pool_means") is None
    src.write_text("kernel source, changed\n")
    assert bench.measured_traffic("attention") is None


def test_traffic_record_missing_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("attention") is None


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_log_parsing(tmp_path):
    path = tmp_path / "clocks.csv"
    lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 995.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    s = bench.ClockSampler(0)
    s.path = str(path)
    s.f = open(path, "w")
    s.f.write("\n".join(lines) + "\n")
    s.proc = _FakeProc()
    r = s.stop()
    assert r == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_sampler_without_nvidia_smi_reports_nothing():
    s = bench.ClockSampler(0)
    s.proc = None
    assert s.stop() is None


def test_critical_flops_of_the_32k_workload():
    # 4 * 64 * 64 * d FLOP per critical (query block, key block) pair, 26 of 512 key
    # blocks per row, 512 rows, 12 heads, d = 128: 0.335 TFLOP per call
    w = workloads.WAN
    crit, _ = bench.sla_flops(w, 26, 51)
    assert crit == 4 * 64 * 64 * 128 * 512 * 26 * 12
    assert abs(crit / 1e12 - 0.335) < 5e-4


def test_config_names_the_workload():
    c = bench.config_dict(workloads.WAN)
    assert c["seq_len"] == 32768 and c["heads"] == 12 and c["head_dim"] == 128 and c["global_batch"] == 1
    assert "32760 valid" in c["workload"] and "5% critical / 10% negligible" in c["workload"]


def test_tile3d_pair_count_of_the_rope_workload():
    # 2 x 16 x 16 tiles; clipped 3-neighbourhoods: 2*2 along frames, 2*2 + 14*3 = 46 along each
    # spatial axis -> 4 * 46 * 46 = 8464 local pairs per head, plus one far block per tile
    f, pairs = bench.tile3d_flops(workloads.ROPESLR)
    assert pairs == 8464
    assert f == 4 * 64 * 64 * 128 * (8464 + 512) * 16


def test_lvsa_flops_counts_attended_frame_blocks():
    from oracle import lvsa as olvsa
    w = workloads.LVSA
    sets = olvsa.attention_sets(w.frames, w.lvsa_C, w.lvsa_W, 0)
    # every frame attends C = 21 frames of 25 blocks: 121 * 25 * 21 * 25 block pairs
    assert bench.lvsa_flops(w, sets) == 4 * 64 * 64 * 128 * 121 * 25 * 21 * 25 * 12
    assert abs(bench.lvsa_flops(w, sets) / 1e12 - 39.97) < 0.01


def test_svoo_flops_and_config():
    # 103 kept key blocks (ceil(0.2 * 512)) per query block, 512 query blocks, 12 heads, d = 128
    w = workloads.SVOO
    f = bench.svoo_flops(w, 103)
    assert f == 4 * 64 * 64 * 128 * 512 * 103 * 12
    assert abs(f / 1e12 - 1.327) < 1e-3
    c = bench.config_dict(w)
    assert c["seq_len"] == 32768 and c["heads"] == 12
    assert "64 query + 64 key clusters" in c["workload"] and "top 20% key blocks" in c["workload"]
    assert "co-clustering + attention" in c["workload"]


def test_svoo_anchors_are_distinct_valid_tokens():
    w = workloads.SVOO
    for which, C in (("q", w.clusters[0]), ("k", w.clusters[1])):
        a = workloads.make_anchors(w, which, heads=3)
        assert a.shape == (1, 3, C)
        for h in range(3):
            row = a[0, h].tolist()
            assert len(set(row)) == C and min(row) >= 0 and max(row) < w.seg_len
    # the draw of a head does not depend on how many heads are drawn
    assert (workloads.make_anchors(w, "q", heads=2)[0, 1] == workloads.make_anchors(w, "q", heads=4)[0, 1]).all()
