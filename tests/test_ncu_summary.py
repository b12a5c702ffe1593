"""The ncu summary helpers that feed profiles/ and bench.py's roofline.traffic (host logic)."""

import json

from persistent_execution_b200 import ncu_summary as N

LONG = '''==PROF== Connected to process 1
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python3","h","gpuos_impl::gpuos_reset_kernel(KParams, unsigned long long, unsigned long long)","1","13","(256, 1, 1)","(64, 1, 1)","0","10.0","m","gpu__time_duration.sum","ns","3000"
"1","1","python3","h","gpuos_impl::gpuos_persistent_kernel(KParams)","1","13","(576, 1, 1)","(148, 1, 1)","0","10.0","m","gpu__time_duration.sum","ns","1000000"
"1","1","python3","h","gpuos_impl::gpuos_persistent_kernel(KParams)","1","13","(576, 1, 1)","(148, 1, 1)","0","10.0","m","dram__bytes_read.sum","Mbyte","1.5"
"1","1","python3","h","gpuos_impl::gpuos_persistent_kernel(KParams)","1","13","(576, 1, 1)","(148, 1, 1)","0","10.0","m","dram__bytes_write.sum","Kbyte","250"
"2","1","python3","h","gpuos_impl::gpuos_persistent_kernel(KParams)","1","13","(576, 1, 1)","(148, 1, 1)","0","10.0","m","gpu__time_duration.sum","ns","1000000"
'''

RAW = '''"ID","Kernel Name","FBSP.Triage.dram__bytes_read.sum","dram__bytes_write.sum","launch__grid_size"
"","","Gbyte","Mbyte",""
"0","gpuos_persistent_kernel(KParams)","1.25","500","148"
'''


def test_launch_table_shares(tmp_path):
    p = tmp_path / "launches.csv"
    p.write_text(LONG)
    t = N.launches(str(p))
    rows = [l for l in t.splitlines() if l.startswith("| `")]
    assert rows[0].startswith("| `gpuos_impl::gpuos_persistent_kernel` | 2 | 2.000 |")
    assert "99.85%" in rows[0] and "| 1 | 0.003 | 0.15% |" in rows[1]


def test_dram_bytes_long_and_raw_formats(tmp_path):
    a = tmp_path / "m.csv"
    a.write_text(LONG)
    assert N.dram_bytes(str(a)) == 1.5e6 + 250e3  # first launch only, units converted
    b = tmp_path / "raw.csv"
    b.write_text(RAW)
    assert N.dram_bytes(str(b)) == 1.25e9 + 500e6  # section-prefixed column found by suffix
    assert "| `launch__grid_size` | 148 |" in N.raw(str(b), ("launch__grid_size",))


def test_traffic_file_carries_the_source_hash(tmp_path):
    src = tmp_path / "m.csv"
    src.write_text(LONG)
    out = tmp_path / "t.json"
    N.main(["traffic", "7", str(src), str(out)])
    j = json.loads(out.read_text())
    assert j["config"] == 7 and j["dram_bytes_per_launch"] == 1.75e6
    assert j["kernel_source_hash"] == N.kernel_source_hash() and len(j["kernel_source_hash"]) == 16
