"""Summaries of the per-task timeline a step records when given ``d_trace``.

The kernel writes, for every task, 8 unsigned 64-bit words:
  [0] CTA index | task type << 32 | layer << 40
  [1] loader: task handed to the compute warps
  [2] loader: last operand page issued
  [3] compute: task received
  [4] compute: input event satisfied
  [5] compute: activation staged (first page may be consumed)
  [6] compute: task done
  [7] storer: output released (event signalled)
Times are GPU global-timer nanoseconds.
"""

from __future__ import annotations

import json
from collections import defaultdict
from typing import Dict, Optional

import numpy as np

TYPE_NAMES = {1: "embed", 2: "qkv", 3: "attn", 4: "oproj", 5: "gateup", 6: "down", 7: "lmhead",
              8: "kvapp"}


def decode(raw: np.ndarray) -> Dict[str, np.ndarray]:
    raw = np.asarray(raw, dtype=np.uint64).reshape(-1, 8)
    w0 = raw[:, 0]
    out = {"cta": (w0 & 0xffffffff).astype(np.int64),
           "type": ((w0 >> 32) & 0xff).astype(np.int64),
           "layer": ((w0 >> 40) & 0xffff).astype(np.int64)}
    t = raw[:, 1:].astype(np.int64)
    valid = (t > 0).all(axis=1)
    t0 = t[valid].min() if valid.any() else 0
    out["t"] = np.where(t > 0, t - t0, -1)
    out["valid"] = valid
    return out


def summarize(raw: np.ndarray) -> str:
    d = decode(raw)
    t, ty, valid = d["t"], d["type"], d["valid"]
    lines = []
    span = t[valid].max() if valid.any() else 0
    lines.append(f"tasks {len(ty)}  traced {int(valid.sum())}  span {span / 1e3:.1f} us")
    lines.append(f"{'type':8s} {'n':>6s} {'wait_dep':>9s} {'stage':>8s} {'pages':>8s} "
                 f"{'store':>8s} {'slot_lat':>9s}  (mean us per task)")
    for code, name in TYPE_NAMES.items():
        m = valid & (ty == code)
        if not m.any():
            continue
        tt = t[m]
        wait = (tt[:, 3] - tt[:, 2]).mean() / 1e3
        stage = (tt[:, 4] - tt[:, 3]).mean() / 1e3
        pages = (tt[:, 5] - tt[:, 4]).mean() / 1e3
        store = (tt[:, 6] - tt[:, 5]).mean() / 1e3
        slot = (tt[:, 2] - tt[:, 0]).mean() / 1e3
        lines.append(f"{name:8s} {int(m.sum()):6d} {wait:9.2f} {stage:8.2f} {pages:8.2f} "
                     f"{store:8.2f} {slot:9.2f}")
    # per-layer op windows: first compute start .. last release
    win = defaultdict(list)
    for i in np.nonzero(valid)[0]:
        win[(int(d["layer"][i]), int(ty[i]))].append((t[i, 2], t[i, 6]))
    lines.append("layer op windows (us): first start, last release")
    for l in sorted({k[0] for k in win})[:4]:
        parts = []
        for code, name in TYPE_NAMES.items():
            if (l, code) in win:
                a = min(x[0] for x in win[(l, code)]) / 1e3
                b = max(x[1] for x in win[(l, code)]) / 1e3
                parts.append(f"{name} {a:.1f}-{b:.1f}")
        lines.append(f"  L{l}: " + ", ".join(parts))
    return "\n".join(lines)


PHASES = (("wait", 2, 3), ("stage", 3, 4), ("pages", 4, 5), ("store", 5, 6))


def to_chrome_trace(raw: np.ndarray, path: Optional[str] = None) -> dict:
    """Chrome trace-event JSON of a step's timeline (open in Perfetto or
    chrome://tracing): one track per CTA, one complete event per task phase
    (compute: input wait, staging, pages; storer: release), times in us from
    the first traced event.  Tasks with an unrecorded mark are left out.
    Written to `path` when given; returned either way."""
    d = decode(raw)
    t, ty, layer, cta, valid = d["t"], d["type"], d["layer"], d["cta"], d["valid"]
    events = []
    for i in np.nonzero(valid)[0]:
        name = TYPE_NAMES.get(int(ty[i]), f"type{int(ty[i])}")
        for phase, a, b in PHASES:
            dur = (t[i, b] - t[i, a]) / 1e3
            if dur <= 0:
                continue
            events.append({"name": f"{name} {phase}", "cat": name, "ph": "X",
                           "ts": t[i, a] / 1e3, "dur": dur, "pid": 0, "tid": int(cta[i]),
                           "args": {"task": int(i), "layer": int(layer[i])}})
    doc = {"traceEvents": events, "displayTimeUnit": "ns"}
    if path is not None:
        with open(path, "w") as f:
            json.dump(doc, f)
    return doc
