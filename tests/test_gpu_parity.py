"""GPU parity of the decode megakernel against the CPU oracle (small models).

Every test drives the CUDA path through the C ABI (mk.Plan -> libmk.so) and
the oracle on the same seeded inputs, step by step, with the tolerances in
tests/gpu_harness.py.  Sizes are chosen so the oracle finishes in seconds while
the kernels still see several tiles, ragged tails and page boundaries.
"""

import numpy as np
import pytest
import torch

import oracle
from persistent_task_runtime_b200 import mk, synth
from tests.gpu_harness import Pair, StepReport, assert_report

pytestmark = pytest.mark.gpu


def _weights(cfg, seed=0, gain="ones"):
    return synth.make_weights(cfg, seed=seed, device="cuda", gain=gain)


def test_tiny_prompt_then_greedy(cuda_device):
    """Tiny decoder: 16-token prompt (teacher-forced decode steps), then 32
    greedy steps, each step fed the oracle's token."""
    cfg = synth.CONFIGS["tiny"]
    pair = Pair(cfg, _weights(cfg), 1, [48])
    prompt = synth.make_ids(cfg["vocab"], (16,), seed=1).tolist()
    rep = StepReport()
    tok = None
    for t in range(16 + 32):
        o = pair.compare([prompt[t] if t < 16 else tok], [t], rep)
        tok = int(o["next_ids"][0])
    pair.close()
    assert_report(rep)
    assert rep.token_checked >= 10


SHAPES = {
    # ragged row tails (not multiples of 16), no QK-norm, G = 3
    "ragged_rows": dict(n_layers=2, hidden=200, n_q_heads=3, n_kv_heads=1, head_dim=64,
                        ffn=344, vocab=1000, rms_eps=1e-6, rope_theta=1e4, qk_norm=False),
    # head_dim 128, G = 8, several weight pages per row
    "d128_g8": dict(n_layers=2, hidden=1536, n_q_heads=8, n_kv_heads=1, head_dim=128,
                    ffn=2200, vocab=3000, rms_eps=1e-5, rope_theta=1e6, qk_norm=True),
    # head_dim 32, MHA (G = 1)
    "d32_mha": dict(n_layers=1, hidden=128, n_q_heads=4, n_kv_heads=4, head_dim=32,
                    ffn=256, vocab=512, rms_eps=1e-6, rope_theta=1e6, qk_norm=True),
    # 3 KV groups of 4 x 128: the O projection splits along K into parts of
    # whole groups (2 + 1), the down projection into 2 parts
    "o_split_3groups": dict(n_layers=2, hidden=1024, n_q_heads=12, n_kv_heads=3,
                            head_dim=128, ffn=2816, vocab=2048, rms_eps=1e-6,
                            rope_theta=1e6, qk_norm=True),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_odd_shapes(cuda_device, name):
    cfg = SHAPES[name]
    pair = Pair(cfg, _weights(cfg, seed=3, gain="random"), 1, [40],
                o_split=name.startswith("o_split"))
    ids = synth.make_ids(cfg["vocab"], (40,), seed=4).tolist()
    rep = StepReport()
    for t in range(40):
        pair.compare([ids[t]], [t], rep)
    pair.close()
    assert_report(rep)


@pytest.mark.parametrize("schedule", [0, 2])
def test_batch_ragged_history(cuda_device, schedule):
    """B = 5 sequences at ragged positions over a synthetic KV history whose
    lengths sit on and around page and chunk boundaries; under the default
    (solidified) schedule and the dynamic ticket queue."""
    cfg = synth.CONFIGS["tiny"]
    lengths = [0, 15, 16, 17, 300]
    steps = 6
    pair = Pair(cfg, _weights(cfg, seed=5), 5, [n + steps for n in lengths], schedule=schedule)
    assert pair.plan.info()["schedule"] == (0 if schedule == 2 else 1)
    hist = synth.make_kv_history(cfg, lengths, seed=6)
    pair.load_history(hist, lengths)
    ids = synth.make_ids(cfg["vocab"], (steps, 5), seed=7)
    rep = StepReport()
    for s in range(steps):
        pair.compare(ids[s].tolist(), [n + s for n in lengths], rep)
    pair.close()
    assert_report(rep)


def test_long_context_many_attention_chunks(cuda_device):
    """One sequence over a 1100-token history with 2 KV heads: each head's
    context splits into about 70 one-page chunks, so the split-attention
    merge runs over several register batches of chunk partials."""
    cfg = synth.CONFIGS["tiny"]
    n = 1100
    pair = Pair(cfg, _weights(cfg, seed=13), 1, [n + 3])
    pair.load_history(synth.make_kv_history(cfg, [n], seed=14), [n])
    ids = synth.make_ids(cfg["vocab"], (3, 1), seed=15)
    rep = StepReport()
    for s in range(3):
        pair.compare(ids[s].tolist(), [n + s], rep)
    pair.close()
    assert_report(rep)


@pytest.mark.parametrize("path,schedule", [(1, 0), (2, 0), (2, 2)])
def test_large_batch_chunked_activations(cuda_device, path, schedule):
    """B = 16 with activations too wide for one staging buffer: on the
    mma.sync path (four mma n-tiles) every projection stages its input in
    column chunks; on the tensor-core path chunks stream through two
    buffers."""
    cfg = dict(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=4096,
               vocab=8192, rms_eps=1e-6, rope_theta=1e6, qk_norm=True)
    B = 16
    lengths = [int(x) for x in np.linspace(1, 200, B)]
    pair = Pair(cfg, _weights(cfg, seed=8, gain="random"), B, [n + 8 for n in lengths],
                gemv_path=path, schedule=schedule)
    pair.load_history(synth.make_kv_history(cfg, lengths, seed=9), lengths)
    ids = synth.make_ids(cfg["vocab"], (3, B), seed=10)
    rep = StepReport()
    for s in range(3):
        pair.compare(ids[s].tolist(), [n + s for n in lengths], rep)
    # and a smaller batch on the same plan
    for s in range(2):
        pair.compare(ids[s, :3].tolist(), [lengths[b] + 3 + s for b in range(3)], rep,
                     check_kv=True)
    pair.close()
    assert_report(rep)


def test_megakernel_equals_per_operator_launches(cuda_device):
    """Same task code, three schedules: one persistent launch, one launch per
    operator, and the per-operator launches replayed from a CUDA graph (one
    recording, then replays with the step counter patched in).  Results must
    be bit-identical."""
    cfg = synth.CONFIGS["tiny"]
    w = _weights(cfg, seed=11)
    B, lengths, steps = 3, [5, 33, 64], 4
    outs = []
    stream = torch.cuda.Stream()   # graph capture needs a created stream
    with torch.cuda.stream(stream):
        for mode in (mk.MODE_MEGAKERNEL, mk.MODE_PER_OP, mk.MODE_PER_OP_GRAPH):
            pair = Pair(cfg, w, B, [n + steps for n in lengths])
            pair.load_history(synth.make_kv_history(cfg, lengths, seed=12), lengths)
            ids = synth.make_ids(cfg["vocab"], (steps, B), seed=13)
            rec = []
            for s in range(steps):
                rec.append(pair.gpu_step(ids[s].tolist(), [n + s for n in lengths], mode=mode))
            kvs = [t.clone() for t in pair.kv.k + pair.kv.v]
            outs.append((rec, kvs))
            pair.close()
    (ra, ka) = outs[0]
    for rb, kb in outs[1:]:
        for (ia, la, ha), (ib, lb, hb) in zip(ra, rb):
            assert np.array_equal(ia, ib)
            assert np.array_equal(la, lb)
            assert np.array_equal(ha, hb)
        for x, y in zip(ka, kb):
            assert torch.equal(x, y)


def test_lm_head_argmax_planted_ties_and_last_tile_maximum(cuda_device):
    """The argmax over the LM-head tiles picks the lowest index among equal
    logits, across tiles and inside one, and finds a maximum planted in the
    last row tile.  The plan reads the weights in place, so rows of the LM
    head are rewritten between steps.  Copies of a row give bit-equal logits;
    a row scaled by a power of 2 (exact in bf16) scales the logit exactly."""
    cfg = synth.CONFIGS["tiny"]
    V = cfg["vocab"]
    w = _weights(cfg, seed=21)
    pair = Pair(cfg, w, 2, [4, 4])
    ids, pos = [17, 3001], [0, 0]
    lm = w["lm_head"]
    orig = lm.clone()

    g_ids, g_logits, _ = pair.gpu_step(ids, pos)
    top = int(g_ids[0])
    assert g_logits[0, top] > 0
    # plant the winner at row 100: 4x the winning row
    win, nb = 100, 101          # rows 100 and 101 share a row tile and task
    lm[win] = orig[top] * 4
    g_ids, g_logits, _ = pair.gpu_step(ids, pos)
    assert int(g_ids[0]) == win
    assert g_logits[0, win] == 4 * g_logits[0, top]
    planted = lm[win].clone()

    # ties: copies of the winning row in the first row, its neighbour and the last row
    for r in (0, nb, V - 1):
        lm[r] = planted
    g_ids, g_logits, _ = pair.gpu_step(ids, pos)
    for b in range(2):
        assert int(g_ids[b]) == int(np.argmax(g_logits[b]))
        for r in (0, nb, V - 1):
            assert g_logits[b, r] == g_logits[b, win]
    assert int(g_ids[0]) == 0

    # a tie inside one tile only
    lm[0] = orig[0]
    lm[V - 1] = orig[V - 1]
    g_ids, g_logits, _ = pair.gpu_step(ids, pos)
    assert g_logits[0, nb] == g_logits[0, win]
    assert int(g_ids[0]) == win

    # a strict maximum in the last row tile
    lm[V - 1] = planted * 2
    g_ids, g_logits, _ = pair.gpu_step(ids, pos)
    assert g_logits[0, V - 1] == 2 * g_logits[0, win]
    assert int(g_ids[0]) == V - 1
    assert int(g_ids[1]) == int(np.argmax(g_logits[1]))
    pair.close()


def test_closed_loop_greedy_on_device(cuda_device):
    """out_ids and out_pos fed straight back as the next step's inputs (no host
    round trip); the token sequence must follow the oracle's greedy decode up
    to its first step with a top-2 margin below 0.1."""
    cfg = synth.CONFIGS["tiny"]
    w = _weights(cfg, seed=14)
    prompt = synth.make_ids(cfg["vocab"], (8,), seed=15).tolist()
    n = 24
    ref = oracle.greedy_decode(oracle.DecoderConfig(**{k: cfg[k] for k in (
        "n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
        "rms_eps", "rope_theta", "qk_norm")}), oracle.Weights(w), [prompt], n)
    pair = Pair(cfg, w, 1, [8 + n])
    for t in range(8):
        pair.gpu_step([prompt[t]], [t])
    ids = pair.d_out[:1].clone()
    pos = torch.tensor([8], dtype=torch.int32, device="cuda")
    trace = [ids.clone()]
    nxt_ids = torch.zeros_like(ids)
    nxt_pos = torch.zeros_like(pos)
    for s in range(1, n):
        pair.plan.step(ids, pos, pair.kv.view, nxt_ids, out_pos=nxt_pos)
        ids, nxt_ids = nxt_ids, ids
        pos, nxt_pos = nxt_pos, pos
        trace.append(ids.clone())
    assert pair.plan.status() == mk.MK_OK
    got = [int(t[0]) for t in trace]
    assert int(pos[0]) == 8 + n - 1
    for s in range(n):
        assert got[s] == int(ref["tokens"][s][0]), (s, got, ref["tokens"][:, 0])
        if ref["margins"][s][0] <= 0.1:
            break
    pair.close()


def test_host_buffer_entry_point(cuda_device):
    cfg = synth.CONFIGS["tiny"]
    pair = Pair(cfg, _weights(cfg, seed=16), 2, [20, 20])
    ids = torch.tensor([3, 7], dtype=torch.int32).pin_memory()
    pos = torch.tensor([0, 0], dtype=torch.int32).pin_memory()
    out = torch.zeros(2, dtype=torch.int32).pin_memory()
    logits = torch.zeros(2, cfg["vocab"], dtype=torch.float32).pin_memory()
    assert pair.plan.step_host(ids, pos, pair.kv.view, out, logits) == mk.MK_OK
    o = pair.oracle_step([3, 7], [0, 0])
    assert np.max(np.abs(logits.numpy() - o["logits"])) <= 5e-2
    assert out.tolist() == [int(np.argmax(r)) for r in logits.numpy()]
    pair.close()


def test_device_range_errors_then_reset(cuda_device):
    cfg = synth.CONFIGS["tiny"]
    pair = Pair(cfg, _weights(cfg, seed=17), 1, [32])
    V = cfg["vocab"]
    for ids, pos in (([V], [0]), ([-1], [0]), ([5], [32]), ([5], [-3])):
        pair.d_ids[:1] = torch.tensor(ids, dtype=torch.int32)
        pair.d_pos[:1] = torch.tensor(pos, dtype=torch.int32)
        pair.plan.step(pair.d_ids[:1], pair.d_pos[:1], pair.kv.view, pair.d_out[:1])
        assert pair.plan.status() == mk.MK_ERR_RANGE
        # sticky: a following valid step does nothing until reset
        pair.d_ids[:1] = 5
        pair.d_pos[:1] = 0
        pair.plan.step(pair.d_ids[:1], pair.d_pos[:1], pair.kv.view, pair.d_out[:1])
        assert pair.plan.status() == mk.MK_ERR_RANGE
        pair.plan.reset()
        assert pair.plan.status() == mk.MK_OK
    rep = StepReport()
    pair.compare([5], [0], rep)
    pair.close()
    assert_report(rep)


def test_wait_timeout_reports_status_and_recovers(cuda_device):
    """A plan whose first QKV task waits for a completion that never comes
    (host-built fault plan) must end the step with MK_ERR_TIMEOUT after the
    1 ms wait limit, leave the context usable, and a normal plan must then
    run correctly."""
    cfg = synth.CONFIGS["tiny"]
    w = _weights(cfg, seed=18)
    bad = Pair(cfg, w, 1, [16], wait_limit_ns=1_000_000, debug_unsatisfiable_dep=True)
    bad.plan.step(bad.d_ids[:1], bad.d_pos[:1], bad.kv.view, bad.d_out[:1])
    assert bad.plan.status() == mk.MK_ERR_TIMEOUT
    info = bad.plan.error_info()   # [task, event, value seen, -]
    assert 0 <= info[0] < bad.plan.info()["n_tasks"]
    bad.close()
    torch.cuda.synchronize()
    good = Pair(cfg, w, 1, [16])
    rep = StepReport()
    good.compare([9], [0], rep)
    good.close()
    assert_report(rep)


def test_host_argument_errors(cuda_device):
    cfg = synth.CONFIGS["tiny"]
    pair = Pair(cfg, _weights(cfg, seed=19), 2, [16, 16])
    with pytest.raises(mk.MkError) as e:
        pair.plan.step(pair.d_ids, pair.d_pos, pair.kv.view, pair.d_out, batch=3)
    assert e.value.code == mk.MK_ERR_INVALID_ARG
    # graph replay cannot record on the legacy default stream
    with pytest.raises(mk.MkError) as e:
        pair.plan.step(pair.d_ids, pair.d_pos, pair.kv.view, pair.d_out, batch=1,
                       mode=mk.MODE_PER_OP_GRAPH, stream=torch.cuda.default_stream())
    assert e.value.code == mk.MK_ERR_INVALID_ARG
    with pytest.raises(mk.MkError):
        mk.Plan(cfg, _weights(cfg), max_batch=17)
    with pytest.raises(mk.MkError) as e:
        mk.Plan(dict(cfg, head_dim=48), _weights(cfg))
    assert e.value.code in (mk.MK_ERR_UNSUPPORTED, mk.MK_ERR_INVALID_ARG)
    pair.close()
