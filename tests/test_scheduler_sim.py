"""CPU simulation of the persistent kernel's scheduling over the plan's task
array (from mk_plan_describe): no deadlock, every task exactly once.

The model keeps what the kernel's progress depends on and nothing else:
  * one global queue, popped in ticket order by W workers (the SMs);
  * a worker holds the tasks it popped in a FIFO of at most `cap` entries
    (the loader's lookahead plus the slot ring) and its compute runs them in
    that order, each once its input event has reached the required count;
  * the pop gate: after taking a GEMV task whose input was incomplete, or an
    attention chunk, the worker pops nothing more until that input completes;
  * a finished task's output is released later, in order, by the worker's
    storer (red.release of its event; a split-K part bumps its row tile's
    counter and the part that completes the tile signals).
Which enabled action happens next is drawn at random (seeded), so each run
explores another interleaving.  Attention slots that the kernel leaves empty
(no tokens) skip their wait there; here every slot waits, which only adds
constraints.
"""

import random
from collections import deque

import numpy as np
import pytest

from persistent_task_runtime_b200 import build, mk
from tests.test_plan_layout import SHAPES, T_ATTN, T_DOWN, T_EMBED, T_GATEUP, T_OPROJ, T_QKV

GEMV = {2, 4, 5, 6, 7}


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def compile_tasks(cfg, info, t):
    """Per task: (type, input event or -1, required count, signalled event or -1,
    split-K row tile key or None, parts per tile)."""
    Hq, Hkv = cfg["n_q_heads"], cfg["n_kv_heads"]
    G = Hq // Hkv
    epl, spg = info["events_per_layer"], info["attn_slots_per_group"]
    out = []
    for r in t:
        ty, layer = int(r["type"]), int(r["layer"])
        wait, need = int(r["dep_event"]), int(r["dep_count"])
        if ty == T_ATTN:
            g = int(r["aux"]) // spg
            if info["prefill"]:
                wait = 1 + layer * epl + Hkv + info["o_parts"] + 2 + info["ffn_parts"] + g
                need = 1
            else:
                wait = 1 + layer * epl + g
                need = info["qkv_tasks_per_group"]
        elif wait == mk.NO_EVENT:
            wait, need = -1, 0
        if ty == T_QKV:
            head, mat = int(r["aux2"]), int(r["aux"])
            g = head // G if mat == 0 else (head - Hq if mat == 1 else head - Hq - Hkv)
            sig = 1 + layer * epl + g
        else:
            sig = int(r["out_event"])
            sig = -1 if sig == mk.NO_EVENT else sig
        split = ty in (T_QKV, T_OPROJ, T_GATEUP, T_DOWN) and int(r["nsplit"]) > 1
        key = (ty, layer, int(r["aux"]) if ty == T_QKV else 0, int(r["row0"]))
        out.append((ty, wait, need, sig, key if split else None, int(r["nsplit"])))
    return out


def simulate(tasks, n_events, workers, seed, lists=None):
    """``lists`` (a solidified schedule): worker w pops only the tasks of
    lists[w], in that order, instead of the next global ticket."""
    rng = random.Random(seed)
    n = len(tasks)
    ctr = [0] * n_events
    tile = {}
    nxt = 0
    pos = [0] * workers
    done = [0] * n
    held = [deque() for _ in range(workers)]
    store = [deque() for _ in range(workers)]
    cap = [rng.randint(1, 5) for _ in range(workers)]
    gate = [None] * workers
    finished = 0

    def satisfied(ev, need):
        return ev < 0 or ctr[ev] >= need

    while finished < n:
        enabled = []
        for w in range(workers):
            if gate[w] is not None and satisfied(*gate[w]):
                gate[w] = None
            more = pos[w] < len(lists[w]) if lists is not None else nxt < n
            if more and len(held[w]) < cap[w] and gate[w] is None:
                enabled.append((w, 0))
            if held[w]:
                _, wait, need, *_ = tasks[held[w][0]]
                if satisfied(wait, need):
                    enabled.append((w, 1))
            if store[w]:
                enabled.append((w, 2))
        assert enabled, f"deadlock: {finished} of {n} tasks finished, next ticket {nxt}"
        w, act = rng.choice(enabled)
        if act == 0:                          # pop the next ticket
            if lists is not None:
                i = lists[w][pos[w]]
                pos[w] += 1
            else:
                i = nxt
                nxt += 1
            held[w].append(i)
            ty, wait, need, *_ = tasks[i]
            if ty == T_ATTN or (ty in GEMV and not satisfied(wait, need)):
                gate[w] = (wait, need)
        elif act == 1:                        # compute finishes the head task
            i = held[w].popleft()
            done[i] += 1
            store[w].append(i)
        else:                                 # storer releases the oldest output
            i = store[w].popleft()
            finished += 1
            ty, _, _, sig, key, nsplit = tasks[i]
            if key is not None:
                tile[key] = tile.get(key, 0) + 1
                if tile[key] < nsplit:
                    continue
                tile[key] = 0
            if sig >= 0:
                ctr[sig] += 1
    assert done == [1] * n
    assert all(v == 0 for v in tile.values())
    return ctr


# (shape, max_batch, workers, GEMV path: 0 automatic, 2 tensor cores with
# split-K QKV / O / gate/up / down)
CASES = [("tiny", 1, 1, 0), ("tiny", 1, 5, 0), ("tiny", 3, 148, 0), ("tiny", 16, 37, 0),
         ("ragged", 1, 7, 0), ("ragged", 4, 148, 0), ("3groups", 2, 20, 0), ("d32", 1, 148, 0),
         ("1.5b", 1, 8, 0), ("8b", 1, 16, 0),
         ("3groups", 8, 20, 0), ("3groups", 1, 3, 2), ("3groups", 16, 148, 2), ("8b", 16, 16, 0)]


@pytest.mark.parametrize("name,batch,workers,path", CASES)
def test_no_deadlock_every_task_once(name, batch, workers, path):
    cfg = SHAPES[name]
    info, t = mk.describe(cfg, max_batch=batch, max_seq_len=600, gemv_path=path)
    if path == 2 or (batch >= 4 and cfg["head_dim"] == 128):
        assert info["gemv_path"] == 2
    tasks = compile_tasks(cfg, info, t)
    seeds = (1,) if name in ("1.5b", "8b") else (1, 2, 3)
    for seed in seeds:
        ctr = simulate(tasks, info["n_events"], workers, seed)
        # every waited-on event ends the step exactly at its required count
        for ty, wait, need, *_ in tasks:
            if wait >= 0:
                assert ctr[wait] == need


def test_simulator_detects_a_missing_signal():
    """The check itself: drop one QKV task's signal and the step must stall."""
    cfg = SHAPES["tiny"]
    info, t = mk.describe(cfg, max_batch=1, max_seq_len=64)
    tasks = compile_tasks(cfg, info, t)
    i = next(k for k, x in enumerate(tasks) if x[0] == T_QKV)
    ty, wait, need, sig, key, nsplit = tasks[i]
    tasks[i] = (ty, wait, need, -1, key, nsplit)
    with pytest.raises(AssertionError, match="deadlock"):
        simulate(tasks, info["n_events"], 4, seed=1)


def test_simulator_detects_a_consumer_before_its_producer():
    """Move the embedding task behind the first QKV task that waits on it:
    with one worker the queue order alone must stall."""
    cfg = SHAPES["tiny"]
    info, t = mk.describe(cfg, max_batch=1, max_seq_len=64)
    tasks = compile_tasks(cfg, info, t)
    assert tasks[0][0] == T_EMBED
    tasks = [tasks[1], tasks[0]] + tasks[2:]
    with pytest.raises(AssertionError, match="deadlock"):
        simulate(tasks, info["n_events"], 1, seed=1)


@pytest.mark.parametrize("name,batch,workers,path", [("tiny", 1, 5, 0), ("3groups", 2, 20, 0),
                                                     ("3groups", 16, 148, 2), ("1.5b", 1, 148, 0),
                                                     ("8b", 1, 148, 0)])
def test_solidified_schedule_no_deadlock(name, batch, workers, path):
    """Each CTA runs the plan's offline task list in order: every task is on
    exactly one list, lists ascend, and any interleaving finishes the step."""
    cfg = SHAPES[name]
    info, t = mk.describe(cfg, max_batch=batch, max_seq_len=600, gemv_path=path, schedule=1,
                          num_sms=workers)
    assert info["schedule"] == 1 and info["num_ctas"] == workers
    owner = mk.describe_schedule(cfg, info["n_tasks"], max_batch=batch, max_seq_len=600,
                                 gemv_path=path, num_sms=workers)
    assert owner.min() >= 0 and owner.max() < workers
    lists = [[int(i) for i in np.flatnonzero(owner == w)] for w in range(workers)]
    assert sum(len(x) for x in lists) == len(t)
    # the cost model spreads every operator's work over many CTAs
    used = len({int(owner[i]) for i in range(len(t)) if int(t["type"][i]) == 6})
    assert used >= min(workers, int((t["type"] == 6).sum())) // 2
    tasks = compile_tasks(cfg, info, t)
    ctr = simulate(tasks, info["n_events"], workers, seed=1, lists=lists)
    for ty, wait, need, *_ in tasks:
        if wait >= 0:
            assert ctr[wait] == need
    # the dynamic plan (its own task count: gate/up tasks of one row tile)
    # describes no schedule
    info2, _ = mk.describe(cfg, max_batch=batch, max_seq_len=600, gemv_path=path, schedule=2,
                           num_sms=workers)
    assert (mk.describe_schedule(cfg, info2["n_tasks"], max_batch=batch, max_seq_len=600,
                                 gemv_path=path, num_sms=workers, schedule=2) == -1).all()


@pytest.mark.parametrize("name,batch,workers,path", [("tiny", 16, 9, 0), ("3groups", 16, 148, 2),
                                                     ("8b", 16, 148, 0)])
def test_prefill_plan_no_deadlock(name, batch, workers, path):
    cfg = SHAPES[name]
    info, t = mk.describe(cfg, max_batch=batch, max_seq_len=600, gemv_path=path, prefill=True)
    tasks = compile_tasks(cfg, info, t)
    for seed in (1, 2):
        ctr = simulate(tasks, info["n_events"], workers, seed)
        for ty, wait, need, *_ in tasks:
            if wait >= 0:
                assert ctr[wait] == need


# (shape, max_batch, workers, describe options): the solidified lists of the
# plans the default options build at batch >= 4 (tensor-core tiles), with
# prompt chunks, 4-bit weights and tensor-memory staging
LIST_CASES = [("tiny", 16, 9, dict(prefill=True)),
              ("3groups", 16, 148, dict(prefill=True, gemv_path=2)),
              ("3groups", 4, 148, dict()),
              ("8b", 4, 148, dict()),
              ("8b", 1, 148, dict(weight_bits=4)),
              ("8b", 2, 148, dict(gemv_path=3))]


@pytest.mark.parametrize("name,batch,workers,opts", LIST_CASES)
def test_solidified_lists_of_other_plans(name, batch, workers, opts):
    cfg = SHAPES[name]
    info, t = mk.describe(cfg, max_batch=batch, max_seq_len=600, num_sms=workers, **opts)
    assert info["schedule"] == 1
    if batch >= 4 and cfg["head_dim"] == 128:
        assert info["gemv_path"] == 2
    owner = mk.describe_schedule(cfg, info["n_tasks"], max_batch=batch, max_seq_len=600,
                                 num_sms=workers, schedule=0, **opts)
    assert owner.min() >= 0 and owner.max() < workers
    lists = [[int(i) for i in np.flatnonzero(owner == w)] for w in range(workers)]
    tasks = compile_tasks(cfg, info, t)
    ctr = simulate(tasks, info["n_events"], workers, seed=2, lists=lists)
    for ty, wait, need, *_ in tasks:
        if wait >= 0:
            assert ctr[wait] == need
