"""CPU tests of the plan builder (mk_plan_describe): the task graph the
persistent kernel runs, checked without a GPU.

A step runs tasks in queue order on whichever SM asks first.  A task runs
once the event it names has been signalled `dep_count` times in the current
step.  The graph must therefore satisfy, for every shape and option:
  * every event receives, per step, exactly the completions its waiters
    require (else a wait never ends or ends early);
  * every producer of an event sits earlier in the queue than every task
    waiting on it (the in-order queue then cannot deadlock: the earliest
    unfinished task has all its inputs done);
  * the tasks of an operator cover its output rows (and split-K parts cover
    its columns) exactly once;
  * the shared-memory carve-up fits the device, and tasks stay within the
    row tiles the accumulators hold.
"""

from collections import Counter, defaultdict

import numpy as np
import pytest

from persistent_task_runtime_b200 import build, mk, synth

SHAPES = {
    "tiny": synth.CONFIGS["tiny"],
    "1.5b": synth.CONFIGS["1.5b"],
    "8b": synth.CONFIGS["8b"],
    # ragged rows, no QK-norm, G = 3
    "ragged": dict(n_layers=2, hidden=200, n_q_heads=3, n_kv_heads=1, head_dim=64, ffn=344,
                   vocab=1000, rms_eps=1e-6, rope_theta=1e4, qk_norm=False),
    # three KV groups of 4 x 128 (an O projection that can split into 2 + 1 groups)
    "3groups": dict(n_layers=2, hidden=1024, n_q_heads=12, n_kv_heads=3, head_dim=128,
                    ffn=2816, vocab=2048, rms_eps=1e-6, rope_theta=1e6, qk_norm=True),
    # head_dim 32, MHA
    "d32": dict(n_layers=1, hidden=128, n_q_heads=4, n_kv_heads=4, head_dim=32, ffn=256,
                vocab=512, rms_eps=1e-6, rope_theta=1e6, qk_norm=True),
}
SMEM = 232448
T_EMBED, T_QKV, T_ATTN, T_OPROJ, T_GATEUP, T_DOWN, T_LMHEAD, T_KVAPP = 1, 2, 3, 4, 5, 6, 7, 8


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def n_tiles_for(batch):
    return 1 if batch <= 4 else (2 if batch <= 8 else 4)


def check_plan(cfg, info, t, max_batch):
    H, Hq, Hkv, d = cfg["hidden"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    F, V, L = cfg["ffn"], cfg["vocab"], cfg["n_layers"]
    G = Hq // Hkv
    epl, spg = info["events_per_layer"], info["attn_slots_per_group"]
    o_parts, ffn_parts = info["o_parts"], info["ffn_parts"]
    n_events = info["n_events"]
    kvt = info["prefill"] == 1            # K/V appended by tasks of their own
    assert n_events == 1 + L * epl
    assert epl == Hkv + o_parts + 2 + ffn_parts + (Hkv if kvt else 0)

    def ev_kv_ready(l, g):
        return 1 + l * epl + Hkv + o_parts + 2 + ffn_parts + g

    def ev_attn_ready(l, g):
        return 1 + l * epl + g

    def ev_gateup(l, part):
        return 1 + l * epl + Hkv + o_parts + 1 + part

    # ---- resources -------------------------------------------------------------------
    assert info["smem_bytes"] <= SMEM
    assert info["n_pages"] >= 2
    assert info["n_pages"] * info["page_bytes"] < info["smem_bytes"]
    assert info["page_bytes"] % 1024 == 0     # swizzled TMA copies land on 1024-byte boundaries
    tc = info["gemv_path"] == 2
    tile = 128 if tc else 16                     # rows per row tile
    max_mt = 2 if tc else 8 // n_tiles_for(max_batch)

    # ---- who signals what, per step ----------------------------------------------------
    signals = Counter()
    producers = defaultdict(list)        # event -> task indices that signal it
    split_tiles = set()
    for i, r in enumerate(t):
        ty = int(r["type"])
        if ty == T_QKV:
            head, mat = int(r["aux2"]), int(r["aux"])
            g = head // G if mat == 0 else (head - Hq if mat == 1 else head - Hq - Hkv)
            assert 0 <= g < Hkv
            ev = ev_attn_ready(int(r["layer"]), g)
            if r["nsplit"] > 1:
                key = (ty, int(r["layer"]), mat, int(r["row0"]))
                if key in split_tiles:
                    producers[ev].append(i)
                    continue
                split_tiles.add(key)
        elif ty in (T_OPROJ, T_DOWN, T_GATEUP) and r["nsplit"] > 1:
            # the part that completes a row tile signals once for the tile
            key = (ty, int(r["layer"]), int(r["row0"]))
            if key in split_tiles:
                producers[int(r["out_event"])].append(i)
                continue
            split_tiles.add(key)
            ev = int(r["out_event"])
        else:
            ev = int(r["out_event"])
        if ev == mk.NO_EVENT:
            continue
        assert 0 <= ev < n_events
        signals[ev] += 1
        producers[ev].append(i)

    # ---- every wait is satisfied exactly, by earlier tasks ------------------------------
    for i, r in enumerate(t):
        ty = int(r["type"])
        if ty == T_ATTN:
            g = int(r["aux"]) // spg
            if kvt:
                ev, need = ev_kv_ready(int(r["layer"]), g), 1
            else:
                ev, need = ev_attn_ready(int(r["layer"]), g), info["qkv_tasks_per_group"]
        else:
            ev, need = int(r["dep_event"]), int(r["dep_count"])
            if ev == mk.NO_EVENT:
                assert ty == T_EMBED
                continue
        assert signals[ev] == need, (i, ty, ev, signals[ev], need)
        assert max(producers[ev]) < i, (i, ty, ev)

    # ---- coverage of output rows (and split-K columns) ----------------------------------
    for l in range(L):
        lay = t[t["layer"] == l]
        qkv = lay[lay["type"] == T_QKV]
        for mat, rows in ((0, Hq * d), (1, Hkv * d), (2, Hkv * d)):
            m = qkv[qkv["aux"] == mat]
            for ks in range(info["qkv_parts"]):
                cover = np.zeros(rows, dtype=int)
                for r in m[m["ksplit"] == ks]:
                    r0, n = int(r["row0"]), int(r["nrows"])
                    assert r0 // d == (r0 + n - 1) // d          # never straddles heads
                    assert int(r["nsplit"]) == max(info["qkv_parts"], 1) or info["qkv_parts"] == 1
                    cover[r0:r0 + n] += 1
                assert (cover == 1).all()
        for ty, rows, parts in ((T_OPROJ, H, max(o_parts, 1)), (T_DOWN, H, max(ffn_parts, 1))):
            m = lay[lay["type"] == ty]
            for ks in range(parts):
                cover = np.zeros(rows, dtype=int)
                for r in m[m["ksplit"] == ks]:
                    cover[int(r["row0"]):int(r["row0"]) + int(r["nrows"])] += 1
                assert (cover == 1).all(), (l, ty, ks)
        gu = lay[lay["type"] == T_GATEUP]
        cols = info["ffn_part_cols"]
        for ks in range(info["gateup_parts"]):
            cover = np.zeros(F, dtype=int)
            for r in gu[gu["ksplit"] == ks]:
                r0, n = int(r["row0"]), int(r["nrows"])
                cover[r0:r0 + n] += 1
                part = r0 // cols if ffn_parts > 1 else 0
                assert (r0 + n - 1) // cols == r0 // cols or ffn_parts == 1
                assert int(r["out_event"]) == ev_gateup(l, part)
                assert int(r["n_m"]) % 2 == 0 and tile * (int(r["n_m"]) // 2) >= n
            assert (cover == 1).all()
    assert ffn_parts * info["ffn_part_cols"] >= F > (ffn_parts - 1) * info["ffn_part_cols"]
    assert o_parts * info["o_part_cols"] >= Hq * d > (o_parts - 1) * info["o_part_cols"]
    lm = t[t["type"] == T_LMHEAD]
    cover = np.zeros(V, dtype=int)
    for r in lm:
        cover[int(r["row0"]):int(r["row0"]) + int(r["nrows"])] += 1
    assert (cover == 1).all()

    # ---- row tiles within the accumulators ------------------------------------------------
    gemv = t[np.isin(t["type"], [T_QKV, T_OPROJ, T_GATEUP, T_DOWN, T_LMHEAD])]
    assert int(gemv["n_m"].max()) <= max_mt
    ng = gemv[gemv["type"] != T_GATEUP]
    assert (tile * ng["n_m"].astype(int) >= ng["nrows"].astype(int)).all()
    if tc:
        # every tile names its tensor maps: wq/wk/wv 0-2, wo 3, gate 4 / up 5, down 6, LM head
        want = {T_OPROJ: 3, T_DOWN: 6}
        for r in gemv:
            ty, l = int(r["type"]), int(r["layer"])
            if ty == T_QKV:
                assert int(r["map0"]) == 7 * l + int(r["aux"])
            elif ty == T_GATEUP:
                assert (int(r["map0"]), int(r["map1"])) == (7 * l + 4, 7 * l + 5)
            elif ty == T_LMHEAD:
                assert int(r["map0"]) == 7 * L
            else:
                assert int(r["map0"]) == 7 * l + want[ty]
        # split-K parts are whole weight pages and about two tasks per CTA
        assert info["page_cols"] == [128] * 4
        for ty, parts in ((T_QKV, info["qkv_parts"]), (T_GATEUP, info["gateup_parts"]),
                          (T_OPROJ, o_parts), (T_DOWN, ffn_parts)):
            assert (t[t["type"] == ty]["nsplit"].astype(int) == (parts if parts > 1 else 0)).all() \
                or parts == 1

    # ---- attention slots: one block per KV group ------------------------------------------
    att = t[t["type"] == T_ATTN]
    assert len(att) == L * Hkv * spg == L * info["attn_slots"]
    kva = t[t["type"] == T_KVAPP]
    if kvt:
        # one K/V task per (layer, KV group), waiting for the group's QKV tiles
        assert len(kva) == L * Hkv
        for r in kva:
            l, g = int(r["layer"]), int(r["aux"])
            assert int(r["dep_event"]) == ev_attn_ready(l, g)
            assert int(r["dep_count"]) == info["qkv_tasks_per_group"]
            assert int(r["out_event"]) == ev_kv_ready(l, g)
    else:
        assert len(kva) == 0


CASES = [(name, b, split) for name in SHAPES for b in (1, 3, 4, 8, 16) for split in (False, True)]


@pytest.mark.parametrize("name,batch,o_split", CASES)
def test_task_graph_invariants(name, batch, o_split):
    cfg = SHAPES[name]
    info, t = mk.describe(cfg, max_batch=batch, max_seq_len=2048 if name == "8b" else 600,
                          o_split=o_split)
    check_plan(cfg, info, t, batch)


PREFILL_CASES = [(name, b, path) for name in ("tiny", "3groups", "8b", "ragged")
                 for b in (1, 4, 16) for path in (0, 1)]


@pytest.mark.parametrize("name,batch,path", PREFILL_CASES)
def test_prefill_plan_graph_invariants(name, batch, path):
    cfg = SHAPES[name]
    info, t = mk.describe(cfg, max_batch=batch, max_seq_len=2048 if name == "8b" else 600,
                          prefill=True, gemv_path=path)
    assert info["prefill"] == 1
    check_plan(cfg, info, t, batch)


@pytest.mark.parametrize("cols", [256, 1024, 2048])
def test_page_width_option(cols):
    cfg = SHAPES["8b"]
    info, t = mk.describe(cfg, max_batch=1, max_seq_len=1024, max_page_cols=cols)
    assert max(info["page_cols"]) <= cols
    check_plan(cfg, info, t, 1)


def test_batch1_8b_plan_facts():
    """The benchmark's plan: 3 ring pages of 16 x 2048 bf16, the down
    projection in 3 parts of 4096 columns, one O part."""
    info, _ = mk.describe(SHAPES["8b"], max_batch=1, max_seq_len=600)
    assert info["n_pages"] == 3 and info["page_cols"] == [2048, 2048, 2048, 2048]
    assert (info["ffn_parts"], info["ffn_part_cols"]) == (3, 4096)
    assert info["o_parts"] == 1


def test_attention_path_option():
    """CUDA-core attention by default at batch 1, the mma.sync attention
    from batch 2 up and on request, for head_dim 64 and 128 only; out-of-range values are argument errors.  The
    task graph does not depend on the attention path; the mma.sync path's
    scratch (the warps' partial outputs before their merge) may only add
    shared memory."""
    for name in ("tiny", "8b"):
        i0, t0 = mk.describe(SHAPES[name], max_batch=1, max_seq_len=256)
        i2, t2 = mk.describe(SHAPES[name], max_batch=1, max_seq_len=256, attn_path=2)
        assert i0["attn_path"] == 1 and i2["attn_path"] == 2
        assert mk.describe(SHAPES[name], max_batch=2, max_seq_len=256)[0]["attn_path"] == 2
        assert mk.describe(SHAPES[name], max_batch=16, max_seq_len=256,
                           attn_path=1)[0]["attn_path"] == 1
        assert (t0 == t2).all()
        assert i0["page_bytes"] == i2["page_bytes"] and i0["smem_bytes"] <= i2["smem_bytes"]
    d32 = dict(SHAPES["tiny"], head_dim=32)
    assert mk.describe(d32, attn_path=1)[0]["attn_path"] == 1
    with pytest.raises(mk.MkError) as e:
        mk.describe(d32, attn_path=2)
    assert e.value.code == mk.MK_ERR_UNSUPPORTED
    for bad in (-1, 3):
        with pytest.raises(mk.MkError) as e:
            mk.describe(SHAPES["tiny"], attn_path=bad)
        assert e.value.code == mk.MK_ERR_INVALID_ARG


@pytest.mark.parametrize("batch", [1, 2, 4])
def test_tensor_memory_gemv_plan(batch):
    """gemv_path 3 (mma.sync pages staged in tensor memory): the task graph
    of the plain mma.sync path, with every weight page a whole number of
    512-column boxes (the loader's TMA boxes, each four tcgen05.cp sources),
    and a valid graph by the same checks as every other plan."""
    cfg = SHAPES["8b"]
    i3, t3 = mk.describe(cfg, max_batch=batch, max_seq_len=1024, gemv_path=3)
    assert i3["gemv_path"] == 3
    assert all(c % 512 == 0 for c in i3["page_cols"])
    assert i3["ffn_part_cols"] % 512 == 0
    check_plan(cfg, i3, t3, batch)


def test_tensor_memory_gemv_rejections():
    for cfg in (SHAPES["tiny"], SHAPES["1.5b"]):   # ffn 688, 8960: not whole 512-column boxes
        with pytest.raises(mk.MkError) as e:
            mk.describe(cfg, gemv_path=3)
        assert e.value.code == mk.MK_ERR_UNSUPPORTED
    tiny = SHAPES["tiny"]
    with pytest.raises(mk.MkError) as e:
        mk.describe(tiny, gemv_path=3)
    assert e.value.code == mk.MK_ERR_UNSUPPORTED
    with pytest.raises(mk.MkError) as e:
        mk.describe(SHAPES["8b"], gemv_path=3, max_page_cols=1000)
    assert e.value.code == mk.MK_ERR_INVALID_ARG
    with pytest.raises(mk.MkError) as e:
        mk.describe(SHAPES["8b"], gemv_path=3, o_split=True)
    assert e.value.code == mk.MK_ERR_INVALID_ARG
    with pytest.raises(mk.MkError) as e:
        mk.describe(SHAPES["8b"], gemv_path=4)
    assert e.value.code == mk.MK_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["8b", "1.5b", "tiny"])
def test_schedule_default_and_task_sizes(name):
    """The solidified lists are the default (schedule 0 and 1), the dynamic
    queue on request (2); under the lists the mma.sync path's gate/up tasks
    take two row tiles, under the queue one (many small tasks for the queue's
    run-time balance).  Both graphs are valid."""
    cfg = SHAPES[name]
    i0, t0 = mk.describe(cfg, max_batch=1, max_seq_len=600)
    i1, _ = mk.describe(cfg, max_batch=1, max_seq_len=600, schedule=1)
    i2, t2 = mk.describe(cfg, max_batch=1, max_seq_len=600, schedule=2)
    assert i0["schedule"] == 1 and i1["schedule"] == 1 and i2["schedule"] == 0
    assert i0["rows_per_task"][2] == 32 and i2["rows_per_task"][2] == 16
    check_plan(cfg, i0, t0, 1)
    check_plan(cfg, i2, t2, 1)
    with pytest.raises(mk.MkError) as e:
        mk.describe(cfg, schedule=3)
    assert e.value.code == mk.MK_ERR_INVALID_ARG


def test_describe_rejects_what_create_rejects():
    cfg = dict(SHAPES["tiny"], head_dim=96)
    with pytest.raises(mk.MkError):
        mk.describe(cfg)
    with pytest.raises(mk.MkError):
        mk.describe(SHAPES["tiny"], max_page_cols=100)
    with pytest.raises(mk.MkError):
        mk.describe(SHAPES["tiny"], max_batch=17)


def test_describe_argument_errors_and_short_buffer():
    """NULL config or info and non-positive device sizes are host errors; a
    task buffer shorter than the plan is left untouched while info is filled."""
    import ctypes as C

    lib = mk.load_library()
    cfg = SHAPES["tiny"]
    c = mk._config(cfg, 64)
    opts = mk.mk_plan_options(1, 16, 0, 0, (C.c_int * 5)(0, 0, 0, 0, 0), 0, 0, 0)
    info = mk.mk_plan_info_t()
    assert lib.mk_plan_describe(None, C.byref(opts), 148, SMEM, C.byref(info), None, 0) == \
        mk.MK_ERR_INVALID_ARG
    assert lib.mk_plan_describe(C.byref(c), C.byref(opts), 148, SMEM, None, None, 0) == \
        mk.MK_ERR_INVALID_ARG
    assert lib.mk_plan_describe(C.byref(c), C.byref(opts), 0, SMEM, C.byref(info), None, 0) == \
        mk.MK_ERR_INVALID_ARG
    assert lib.mk_plan_describe(C.byref(c), C.byref(opts), 148, 0, C.byref(info), None, 0) == \
        mk.MK_ERR_INVALID_ARG
    # NULL options take the defaults
    assert lib.mk_plan_describe(C.byref(c), None, 148, SMEM, C.byref(info), None, 0) == mk.MK_OK
    n = info.n_tasks
    buf = np.full(n - 1, 0xAB, dtype=np.uint8).repeat(64)
    assert lib.mk_plan_describe(C.byref(c), C.byref(opts), 148, SMEM, C.byref(info),
                                buf.ctypes.data, n - 1) == mk.MK_OK
    assert info.n_tasks == n and (buf == 0xAB).all()
    # a smaller device gives fewer CTAs and still a valid graph
    info2, t2 = mk.describe(cfg, max_batch=2, num_sms=20, max_seq_len=64)
    assert info2["num_ctas"] == 20
    check_plan(cfg, info2, t2, 2)
