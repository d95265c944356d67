"""Host-side facts bench.py relies on, checked against the oracle's layout.

The CUDA-graph measurement replays one captured frame-step per frame for
GRAPH_PERIOD frames, in order, again and again; that continues the rollout
exactly only if every slot a frame-step touches repeats with that period.
"""
import os
import sys

from oracle import SERVED

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _touched(L, t):
    """What frame-step t touches: the record's rows, the evicted frame's
    source and destination rows, and the filled prefix."""
    ev = L.evicted_frame(t)
    evict = None if ev is None else (L.raw_slot(ev), L.sum_slot(ev))
    return (tuple(L.record_rows(t)), evict, L.end(t))


def test_graph_period_is_the_served_slot_period():
    L = SERVED
    P = bench.GRAPH_PERIOD
    assert (bench.Y, bench.W, bench.X, bench.GH, bench.GW) == (L.Y, L.W, L.X, L.grid_h, L.grid_w)
    steady = range(bench.T_STEADY, bench.T_STEADY + 3 * P)
    for t in steady:
        assert _touched(L, t) == _touched(L, t + P), t
    # and it is the smallest such period
    for q in range(1, P):
        assert any(_touched(L, t) != _touched(L, t + q) for t in steady), q


def test_copy_byte_counts():
    L = SERVED
    row = bench.HEADS * bench.D * 2
    assert bench.EVICT_BYTES == 2 * 2 * L.X * row * bench.BLOCKS
    assert bench.WRITE_BYTES == 2 * 2 * L.R * row


NCU_CSV = '''==PROF== Connected to process 123
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","123","python3","127.0.0.1","void wmkv::(anonymous namespace)::evict_kernel(unsigned char *, long, long, long, long, long)","1","7","(256, 1, 1)","(12, 56, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","us","6.00"
"1","123","python3","127.0.0.1","void wmkv::(anonymous namespace)::attend_kernel<64>(wmkv::(anonymous namespace)::AttendParams)","1","7","(384, 1, 1)","(9, 16, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","usecond","50.00"
"1","123","python3","127.0.0.1","void wmkv::(anonymous namespace)::attend_kernel<64>(wmkv::(anonymous namespace)::AttendParams)","1","7","(384, 1, 1)","(9, 16, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","29.05"
"1","123","python3","127.0.0.1","void wmkv::(anonymous namespace)::attend_kernel<64>(wmkv::(anonymous namespace)::AttendParams)","1","7","(384, 1, 1)","(9, 16, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","Kbyte","8.00"
"2","123","python3","127.0.0.1","void wmkv::(anonymous namespace)::attend_kernel<64>(wmkv::(anonymous namespace)::AttendParams)","1","7","(384, 1, 1)","(9, 16, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","ns","54,000"
"2","123","python3","127.0.0.1","void wmkv::(anonymous namespace)::attend_kernel<64>(wmkv::(anonymous namespace)::AttendParams)","1","7","(384, 1, 1)","(9, 16, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","B","29,050,000"
"2","123","python3","127.0.0.1","void wmkv::(anonymous namespace)::attend_kernel<64>(wmkv::(anonymous namespace)::AttendParams)","1","7","(384, 1, 1)","(9, 16, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","8000"
'''


def test_ncu_summary_shares_units_and_digest(tmp_path):
    p = tmp_path / "cap.csv"
    p.write_text(NCU_CSV)
    s = bench.summarize_ncu_csv(str(p), "ncu ... python bench.py")
    assert s["captured_launches"] == 3 and s["source_sha256"] == bench.source_digest()
    k = {e["kernel"]: e for e in s["kernels"]}
    att, ev = k["attend_kernel<64>"], k["evict_kernel"]
    assert att["launches"] == 2 and ev["launches"] == 1
    assert abs(att["total_us"] - 104.0) < 1e-9 and abs(att["avg_us"] - 52.0) < 1e-9
    assert abs(att["share"] - 104.0 / 110.0) < 1e-4 and abs(ev["share"] - 6.0 / 110.0) < 1e-4
    assert att["dram_bytes_per_launch"] == 29058000
    assert s["kernels"][0]["kernel"] == "attend_kernel<64>"       # largest share first


def test_profile_entries_follow_the_source_digest(tmp_path, monkeypatch):
    p = tmp_path / "cap.csv"
    p.write_text(NCU_CSV)
    out = tmp_path / "s.json"
    import json
    json.dump(bench.summarize_ncu_csv(str(p), "cmd"), open(out, "w"))
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(out))
    assert bench.load_traffic() == 29058000
    j = json.load(open(out))
    j["sources"]["attend_sm100.cu"] = "0" * 16     # taken from another version: stale
    json.dump(j, open(out, "w"))
    assert bench.load_traffic() is None
    j["sources"]["attend_sm100.cu"] = bench.file_digests()["attend_sm100.cu"]
    j["sources"]["copy_kernels.cu"] = "0" * 16     # the copy kernels do not feed the attention entry
    json.dump(j, open(out, "w"))
    assert bench.load_traffic() == 29058000


def test_attention_launch_time_and_peak_choice():
    # 10 steps of 1.2 ms, 10 evictions of 8 us: 28 launches per step share the rest
    t = bench.attention_launch_time(12.0, 0.08, 10)
    assert abs(t - (12.0 - 0.08) / 280) < 1e-12
    assert bench.BLOCKS * t <= 12.0 / 10
    pk = {"sustained": 1368.6, "burst": 1654.5, "hbm": 6540.8, "source": "measured"}
    assert bench.choose_peak(pk, 0.25) == (1654.5, "bf16_tflops")
    assert bench.choose_peak(pk, bench.SUSTAINED_REGION_S) == (1368.6, "bf16_tflops_sustained")


def test_both_arms_describe_the_same_workload():
    assert bench.config_dict(1) == bench.config_dict(1)
    c = bench.config_dict(2)
    assert c["workload"] == bench.WORKLOAD and c["keys"] == bench.C == 6528 and c["queries"] == bench.R
    assert c["passes_per_frame"] == 1


def test_kernel_names_with_template_flags():
    """The attention kernel is instantiated per head dimension and per split
    mode; ncu prints both template arguments, and the bench's lookups match
    any instantiation of the head dimension."""
    import bench
    name = bench._kernel_short_name(
        "void wmkv::(anonymous namespace)::attend_kernel<64, false>(wmkv::(anonymous namespace)::AttendParams)")
    assert name == "attend_kernel<64, false>"
    assert name.startswith("attend_kernel<64")
    assert not bench._kernel_short_name("void x::attend_kernel<128, true>(x::P)").startswith("attend_kernel<64")
