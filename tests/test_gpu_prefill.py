"""GPU parity of prompt chunks (mk_prefill_chunk) against the CPU oracle.

A prompt runs in launches of up to max_batch consecutive tokens of one
sequence: row j of a launch is the token at pos0 + j, every row's K/V is
appended by the layer's K/V tasks before the attention reads the cache, and
row j attends causally to positions 0 .. pos0 + j.  The oracle runs the
prompt as one whole-sequence pass (oracle.forward_full / oracle.prefill).

Checked with the tolerances of tests/gpu_harness.py: the K and V cached for
every prompt position of every layer, the residual stream after every layer
and the logits of every row of the last chunk, the greedy token where the
oracle's top-2 margin exceeds 0.1; then decode steps on the same plan and
cache against oracle.decode_step.
"""

import numpy as np
import pytest
import torch

import oracle
from persistent_task_runtime_b200 import mk, synth
from persistent_task_runtime_b200.kvcache import PagedKVCache
from tests.gpu_harness import (HIDDEN_RTOL, LOGITS_ATOL, MARGIN, StepReport, assert_report,
                               oracle_cfg, rel_l2)
from tests.test_gpu_configs import gpu_cache_rows, per_token_rel

pytestmark = pytest.mark.gpu

TC_CFG = dict(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=2240,
              vocab=5000, rms_eps=1e-6, rope_theta=1e6, qk_norm=True)


def run_prefill_case(cfg, w, n, max_batch, seq, n_seqs, decode_steps, **plan_kw):
    L, H, V = cfg["n_layers"], cfg["hidden"], cfg["vocab"]
    cap = n + decode_steps + 1
    plan = mk.Plan(cfg, w, max_batch=max_batch, page_size=16, max_seq_len=cap + 16,
                   prefill=True, **plan_kw)
    assert plan.info()["prefill"] == 1
    kv = PagedKVCache(cfg, max(max_batch, n_seqs), [cap] * n_seqs, page=16,
                      page_order=synth.page_permutation(n_seqs * ((cap + 15) // 16)))
    prompt = synth.make_ids(V, (n,), seed=71)
    d_prompt = prompt.to(torch.int32).cuda()
    # every chunk but the last without the LM head; the last with logits and
    # the per-layer residual stream of its rows
    T = max_batch
    last0 = ((n - 1) // T) * T
    m = n - last0
    out_ids = torch.zeros(T, dtype=torch.int32, device="cuda")
    logits = torch.zeros(m, V, dtype=torch.float32, device="cuda")
    hidden = torch.zeros(L, m, H, dtype=torch.float32, device="cuda")
    for p0 in range(0, last0, T):
        plan.prefill_chunk(d_prompt[p0:p0 + T], p0, seq, kv.view, with_lm_head=False)
    plan.prefill_chunk(d_prompt[last0:], last0, seq, kv.view, out_ids=out_ids[:m],
                       out_logits=logits, hidden=hidden)
    st = plan.status()
    assert st == mk.MK_OK, f"device status {mk.ERROR_NAMES.get(st, st)} {plan.error_info()}"

    ocfg = oracle_cfg(cfg)
    W = oracle.Weights(w, keep_f64=L <= 4)
    full = oracle.forward_full(ocfg, W, prompt.tolist())
    rep = StepReport()
    for l in range(L):
        gk, gv = gpu_cache_rows(kv, l, seq, n)
        e = max(per_token_rel(gk, full["k"][l]), per_token_rel(gv, full["v"][l]))
        rep.max_kv_rel = max(rep.max_kv_rel, e)
        rep.kv_ok = rep.kv_ok and e <= HIDDEN_RTOL
        for b in range(n_seqs):   # other sequences' pages are untouched
            if b != seq:
                ok, ov = gpu_cache_rows(kv, l, b, n)
                assert not ok.any() and not ov.any()
    g_logits, g_hidden, g_ids = logits.cpu().numpy(), hidden.cpu().numpy(), out_ids[:m].cpu().numpy()
    for j in range(m):
        t = last0 + j
        for l in range(L):
            rep.max_hidden_rel = max(rep.max_hidden_rel, rel_l2(g_hidden[l, j], full["hidden"][l, t]))
        rep.max_logit_err = max(rep.max_logit_err,
                                float(np.max(np.abs(g_logits[j] - full["logits"][t]))))
        assert int(g_ids[j]) == int(np.argmax(g_logits[j]))
        if oracle.top2_margin(full["logits"][t]) > MARGIN:
            rep.token_checked += 1
            rep.token_mismatch += int(int(g_ids[j]) != int(np.argmax(full["logits"][t])))
    rep.steps += 1

    # decode steps on the same plan and cache, from the oracle's prefilled cache
    ocache, _, _ = oracle.prefill(ocfg, W, [prompt.tolist()], cap)
    tok = int(g_ids[-1])
    d_ids = torch.zeros(n_seqs, dtype=torch.int32, device="cuda")
    d_pos = torch.zeros(n_seqs, dtype=torch.int32, device="cuda")
    d_out = torch.zeros(n_seqs, dtype=torch.int32, device="cuda")
    d_logits = torch.zeros(n_seqs, V, dtype=torch.float32, device="cuda")
    for s in range(decode_steps):
        if seq != 0:
            break
        d_ids[0] = tok
        d_pos[0] = n + s
        plan.step(d_ids[:1], d_pos[:1], kv.view, d_out[:1], out_logits=d_logits[:1])
        assert plan.status() == mk.MK_OK
        o = oracle.decode_step(ocfg, W, ocache, [tok], [n + s])
        gl = d_logits[0].cpu().numpy()
        rep.max_logit_err = max(rep.max_logit_err, float(np.max(np.abs(gl - o["logits"][0]))))
        if oracle.top2_margin(o["logits"][0]) > MARGIN:
            rep.token_checked += 1
            rep.token_mismatch += int(int(d_out[0]) != int(o["next_ids"][0]))
        k, v = kv.token(0, seq, n + s)
        rep.max_kv_rel = max(rep.max_kv_rel,
                             rel_l2(k.double().cpu().numpy(), o["k_new"][0, 0]),
                             rel_l2(v.double().cpu().numpy(), o["v_new"][0, 0]))
        tok = int(d_out[0])
        rep.steps += 1
    plan.close()
    assert_report(rep)
    assert rep.max_logit_err <= LOGITS_ATOL


@pytest.mark.parametrize("n,max_batch", [(37, 16), (16, 16), (9, 4), (1, 8)])
def test_prefill_tiny(cuda_device, n, max_batch):
    cfg = synth.CONFIGS["tiny"]
    w = synth.make_weights(cfg, seed=70, device="cuda", gain="random")
    run_prefill_case(cfg, w, n, max_batch, seq=0, n_seqs=1, decode_steps=4)


@pytest.mark.parametrize("path", [1, 2])
def test_prefill_tensor_core_shape(cuda_device, path):
    cfg = TC_CFG
    w = synth.make_weights(cfg, seed=72, device="cuda", gain="random")
    run_prefill_case(cfg, w, 45, 16, seq=0, n_seqs=1, decode_steps=3, gemv_path=path)


def test_prefill_other_sequence_row(cuda_device):
    """The chunk's sequence is a block-table row other than 0; rows of other
    sequences stay untouched."""
    cfg = synth.CONFIGS["tiny"]
    w = synth.make_weights(cfg, seed=73, device="cuda")
    run_prefill_case(cfg, w, 20, 8, seq=2, n_seqs=3, decode_steps=0)


def test_prefill_argument_errors(cuda_device):
    cfg = synth.CONFIGS["tiny"]
    w = synth.make_weights(cfg, seed=74, device="cuda")
    kv = PagedKVCache(cfg, 4, [32] * 4, page=16)
    ids = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = torch.zeros(4, dtype=torch.int32, device="cuda")
    decode_plan = mk.Plan(cfg, w, max_batch=4, page_size=16, max_seq_len=32)
    with pytest.raises(mk.MkError) as e:
        decode_plan.prefill_chunk(ids, 0, 0, kv.view, out_ids=out)
    assert e.value.code == mk.MK_ERR_INVALID_ARG
    decode_plan.close()
    plan = mk.Plan(cfg, w, max_batch=4, page_size=16, max_seq_len=32, prefill=True)
    for kwargs in (dict(pos0=-1, seq=0), dict(pos0=30, seq=0), dict(pos0=0, seq=4)):
        with pytest.raises(mk.MkError) as e:
            plan.prefill_chunk(ids, kwargs["pos0"], kwargs["seq"], kv.view, out_ids=out)
        assert e.value.code == mk.MK_ERR_INVALID_ARG
    with pytest.raises(mk.MkError):
        plan.prefill_chunk(torch.zeros(5, dtype=torch.int32, device="cuda"), 0, 0, kv.view,
                           out_ids=out)
    with pytest.raises(mk.MkError):   # the LM head needs an output
        plan.prefill_chunk(ids, 0, 0, kv.view, out_ids=None)
    plan.close()
