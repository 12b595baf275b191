"""Host logic of bench.py that needs no GPU: the DRAM-traffic record is reported only while
the kernel's code (comments aside, optionally a span of its file) is the captured one, and
the clock summary keeps only the nvidia-smi samples taken inside the timed windows."""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

SRC = """// kernel a
__global__ void a() { x = 1; }  // trailing
// ==== b
__global__ void b() { y = 2; }
"""


def write_tree(tmp_path, src, records):
    csrc = tmp_path / "rope_attention_fwd_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(src)
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(records))


def sha(text):
    return hashlib.sha256(bench.code_only(text).encode()).hexdigest()


def test_traffic_tracks_code_not_comments(tmp_path, monkeypatch):
    marker = "// ==== b"
    head, tail = SRC[:SRC.index(marker)], SRC[SRC.index(marker):]
    write_tree(tmp_path, SRC, {
        "a": {"bytes_per_launch": 10, "source": "k.cu", "span_end": marker,
              "source_sha256": sha(head)},
        "b": {"bytes_per_launch": 20, "source": "k.cu", "span_start": marker,
              "source_sha256": sha(tail)},
        "whole": {"bytes_per_launch": 30, "source": "k.cu", "source_sha256": sha(SRC)}})
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert (bench.traffic_for("a"), bench.traffic_for("b"), bench.traffic_for("whole")) == \
        (10, 20, 30)
    assert bench.traffic_for("missing") is None
    # a comment edit keeps every record; a code edit in b drops b and the whole-file record
    src = tmp_path / "rope_attention_fwd_b200" / "csrc" / "k.cu"
    src.write_text(SRC.replace("// kernel a", "// kernel a, reworded\n\n"))
    assert (bench.traffic_for("a"), bench.traffic_for("b"), bench.traffic_for("whole")) == \
        (10, 20, 30)
    src.write_text(SRC.replace("y = 2", "y = 3"))
    assert (bench.traffic_for("a"), bench.traffic_for("b"), bench.traffic_for("whole")) == \
        (10, None, None)


def test_clock_samples_inside_windows_only():
    import datetime
    rows = [
        "2026/12/03 10:39:12.900, 0, 1200 MHz, 1965 MHz, 90.0 W, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/03 10:39:13.100, 0, 1965 MHz, 1965 MHz, 700.0 W, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/03 10:39:13.150, 0, 1950 MHz, 1965 MHz, 710.0 W, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/03 10:39:14.000, 0, 1100 MHz, 1965 MHz, 500.0 W, 0x8, Active, Not Active, Not Active, Not Active",
        "2026/12/03 10:39:15.050, 0, 1965 MHz, 1965 MHz, 650.0 W, 0x0, Not Active, Not Active, Not Active, Not Active",
        "not a sample",
    ]
    t = lambda s, us: datetime.datetime(2026, 12, 3, 10, 39, s, us)
    windows = [(t(13, 0), t(13, 500000)), (t(15, 0), t(15, 100000))]
    got = bench.ClockSampler.parse(rows, windows)
    assert [r[0] for r in got] == [1965.0, 1950.0, 1965.0]
    assert [r[2][3] for r in got] == ["Active", "Active", "Not Active"]
    # the idle sample before and the slowed one between the windows are left out
    assert bench.ClockSampler.parse(rows, []) == []
