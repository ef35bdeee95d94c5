"""GPU parity at the full model sizes the benchmark runs.

The model shapes are the 1.5B-shaped (28 layers) and 8B-shaped (36 layers)
decoders, with the plan options the benchmark uses.  The KV history is
synthetic: the GPU cache and the oracle's cache receive the same bf16 values,
so one decode step can be checked without replaying a long prompt.  At batch
16 with ragged contexts up to 8192 tokens, all 16 sequences run in one GPU
step and the oracle recomputes three of them (the shortest, the median and
the longest); the batch sweep at context 1024 (1, 2, 4, 8 and 16 sequences)
is checked the same way.  Decode treats sequences independently, so every sampled
output has a plain reference value.  Tolerances are those of
tests/gpu_harness.py.

Each test takes about a minute, mostly the oracle widening the bf16 weights
to float64 one layer at a time.
"""

import numpy as np
import pytest
import torch

import oracle
from persistent_task_runtime_b200 import mk, synth
from persistent_task_runtime_b200.kvcache import PagedKVCache
from tests.gpu_harness import (HIDDEN_RTOL, LOGITS_ATOL, MARGIN, Pair, StepReport,
                               assert_report, kv_rel, oracle_cfg, rel_l2)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,ctx,steps", [("1.5b", 256, 2), ("8b", 512, 1)])
def test_full_size_batch1(cuda_device, name, ctx, steps):
    cfg = synth.CONFIGS[name]
    w = synth.make_weights(cfg, seed=0, device="cuda")
    pair = Pair(cfg, w, 1, [ctx + steps + 1], max_seq_len=ctx + steps + 17, keep_f64=False)
    pair.load_history(synth.make_kv_history(cfg, [ctx], seed=3), [ctx])
    ids = synth.make_ids(cfg["vocab"], (steps, 1), seed=1)
    rep = StepReport()
    for s in range(steps):
        pair.compare(ids[s].tolist(), [ctx + s], rep)
    pair.close()
    assert_report(rep)


SAMPLED = {
    # the batch sweep at context 1024 (two sequences recomputed) and the
    # ragged batch of 16 (shortest, median, longest recomputed)
    "b1_ctx1024": (1, lambda: [1024]),
    "b2_ctx1024": (2, lambda: [1024] * 2),
    "b4_ctx1024": (4, lambda: [1024] * 4),
    "b8_ctx1024": (8, lambda: [1024] * 8),
    "b16_ctx1024": (16, lambda: [1024] * 16),
    "b16_ragged": (16, lambda: synth.ragged_lengths(16, 32, 8192, seed=2)),
}


@pytest.mark.parametrize("case", sorted(SAMPLED))
def test_full_size_8b_batched_sampled(cuda_device, case):
    cfg = synth.CONFIGS["8b"]
    B, make_lengths = SAMPLED[case]
    lengths = make_lengths()                                  # the benchmark's contexts
    order = np.argsort(lengths, kind="stable")
    pick = sorted({int(order[0]), int(order[B // 2]), int(order[-1])})
    w = synth.make_weights(cfg, seed=0, device="cuda")
    plan = mk.Plan(cfg, w, max_batch=B, page_size=16, max_seq_len=max(lengths) + 17)
    kv = PagedKVCache(cfg, B, [n + 2 for n in lengths], page=16,
                      page_order=synth.page_permutation(sum((n + 2 + 15) // 16 for n in lengths)))
    ocfg = oracle_cfg(cfg)
    ocache = oracle.KVCache(ocfg, len(pick), max(lengths[b] for b in pick) + 2)
    hist = synth.make_kv_history(cfg, lengths, seed=3, device="cuda")
    kv.load_history(hist, lengths)
    for l, hl in enumerate(hist):
        for j, b in enumerate(pick):
            n = lengths[b]
            ocache.load_history(l, j, hl["k"][b, :, :n].to(torch.float64).cpu().numpy(),
                                hl["v"][b, :, :n].to(torch.float64).cpu().numpy())
    del hist
    torch.cuda.empty_cache()

    ids = synth.make_ids(cfg["vocab"], (B,), seed=1)
    d_ids = ids.to(torch.int32).cuda()
    d_pos = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    d_out = torch.zeros(B, dtype=torch.int32, device="cuda")
    d_logits = torch.zeros(B, cfg["vocab"], dtype=torch.float32, device="cuda")
    d_hidden = torch.zeros(cfg["n_layers"], B, cfg["hidden"], dtype=torch.float32, device="cuda")
    plan.step(d_ids, d_pos, kv.view, d_out, out_logits=d_logits, hidden=d_hidden)
    st = plan.status()
    assert st == mk.MK_OK, f"device status {mk.ERROR_NAMES.get(st, st)} {plan.error_info()}"
    g_ids = d_out.cpu().numpy()
    g_logits = d_logits.cpu().numpy()
    g_hidden = d_hidden.cpu().numpy()

    o = oracle.decode_step(ocfg, oracle.Weights(w, keep_f64=False), ocache,
                           [int(ids[b]) for b in pick], [lengths[b] for b in pick])
    rep = StepReport(steps=1)
    for j, b in enumerate(pick):
        for l in range(cfg["n_layers"]):
            rep.max_hidden_rel = max(rep.max_hidden_rel, rel_l2(g_hidden[l, b], o["hidden"][l, j]))
            k, v = kv.token(l, b, lengths[b])
            e = max(kv_rel(k, o["k_new"][l, j]), kv_rel(v, o["v_new"][l, j]))
            rep.max_kv_rel = max(rep.max_kv_rel, e)
            rep.kv_ok = rep.kv_ok and e <= HIDDEN_RTOL
        rep.max_logit_err = max(rep.max_logit_err,
                                float(np.max(np.abs(g_logits[b] - o["logits"][j]))))
        if oracle.top2_margin(o["logits"][j]) > MARGIN:
            rep.token_checked += 1
            rep.token_mismatch += int(int(g_ids[b]) != int(o["next_ids"][j]))
    # every sequence's token is the argmax of its own logits
    assert np.array_equal(g_ids, np.argmax(g_logits, axis=-1))
    plan.close()
    assert_report(rep)
    assert rep.max_logit_err <= LOGITS_ATOL
