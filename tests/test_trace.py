"""CPU tests of the timeline decoder (persistent_task_runtime_b200/trace.py)
on a synthetic record array laid out as the kernel writes it."""

import json

import numpy as np

from persistent_task_runtime_b200 import trace as T


def _records():
    # three tasks: QKV on CTA 5 (layer 0), attention on CTA 7 (layer 0), one never traced
    base = 1_000_000_000
    raw = np.zeros((3, 8), dtype=np.uint64)
    raw[0, 0] = 5 | (2 << 32) | (0 << 40)
    raw[0, 1:] = base + np.array([0, 500, 1000, 2000, 2500, 5000, 7000])
    raw[1, 0] = 7 | (3 << 32) | (0 << 40)
    raw[1, 1:] = base + np.array([100, 600, 1500, 4000, 5000, 9000, 10000])
    return raw.reshape(-1)


def test_decode_fields_and_origin():
    d = T.decode(_records())
    assert list(d["cta"]) == [5, 7, 0]
    assert list(d["type"]) == [2, 3, 0]
    assert list(d["valid"]) == [True, True, False]
    assert d["t"][0, 0] == 0 and d["t"][1, 6] == 10000
    assert (d["t"][2] == -1).all()


def test_summary_means():
    s = T.summarize(_records())
    assert "tasks 3  traced 2  span 10.0 us" in s
    line = next(x for x in s.splitlines() if x.startswith("qkv"))
    # wait 1.0, stage 0.5, pages 2.5, store 2.0, loader slot latency 1.0 (us)
    assert line.split()[2:] == ["1.00", "0.50", "2.50", "2.00", "1.00"]


def test_chrome_trace(tmp_path):
    path = tmp_path / "t.json"
    doc = T.to_chrome_trace(_records(), str(path))
    assert json.loads(path.read_text()) == doc
    ev = doc["traceEvents"]
    assert len(ev) == 8          # 2 traced tasks x 4 phases
    q = {e["name"]: e for e in ev if e["tid"] == 5}
    assert q["qkv wait"]["ts"] == 1.0 and q["qkv wait"]["dur"] == 1.0
    assert q["qkv store"]["ts"] == 5.0 and q["qkv store"]["dur"] == 2.0
    assert {e["tid"] for e in ev} == {5, 7}
