"""GPU parity on the decode workloads as they are specified, end to end.

The 1.5B-shaped decoder (28 layers) with a 256-token random prompt and the
8B-shaped decoder (36 layers) with a 512-token random prompt, batch 1, page
16: the GPU feeds the prompt through its own decode step (teacher-forced, one
token per launch), then runs greedy steps with the argmax fed back on the
device (out_ids -> ids, out_pos -> pos, no host round trip).  The oracle
(float64, CPU) runs the prompt as one whole-sequence pass (oracle.prefill),
then decode steps fed with the GPU's own tokens, so both stay on one path even
where a near-tie could flip a token.

Checked against the tolerances of tests/gpu_harness.py:
  * the K and V the GPU cached for every prompt position of every layer
    (relative L2 per token),
  * the residual stream after every layer and the logits at the last prompt
    position and at every greedy step,
  * the greedy token wherever the oracle's top-2 margin exceeds 0.1.
"""

import numpy as np
import pytest
import torch

import oracle
from persistent_task_runtime_b200 import mk, synth
from persistent_task_runtime_b200.kvcache import PagedKVCache
from tests.gpu_harness import (HIDDEN_RTOL, MARGIN, StepReport, assert_report, oracle_cfg,
                               rel_l2)

pytestmark = pytest.mark.gpu


def gpu_cache_rows(kv: PagedKVCache, l: int, b: int, n: int):
    """K and V the GPU holds for sequence b, positions 0..n-1 of layer l, as
    float64 arrays [Hkv, n, d]."""
    P = kv.page
    pos = torch.arange(n)
    phys = kv.block_table_cpu[b, pos // P].long().to(kv.device)
    slot = (pos % P).to(kv.device)
    k = kv.k[l][phys, :, slot].permute(1, 0, 2)
    v = kv.v[l][phys, :, slot].permute(1, 0, 2)
    return k.to(torch.float64).cpu().numpy(), v.to(torch.float64).cpu().numpy()


def per_token_rel(g: np.ndarray, r: np.ndarray) -> float:
    """Largest relative L2 error over positions of [Hkv, n, d] arrays."""
    num = np.linalg.norm((g - r).transpose(1, 0, 2).reshape(g.shape[1], -1), axis=1)
    den = np.linalg.norm(r.transpose(1, 0, 2).reshape(r.shape[1], -1), axis=1)
    return float(np.max(num / np.maximum(den, 1e-30)))


@pytest.mark.parametrize("name,prompt_len,steps", [("1.5b", 256, 12), ("8b", 512, 4)])
def test_specified_config_prompt_then_greedy(cuda_device, name, prompt_len, steps):
    cfg = synth.CONFIGS[name]
    L, H, V = cfg["n_layers"], cfg["hidden"], cfg["vocab"]
    w = synth.make_weights(cfg, seed=0, device="cuda")
    cap = prompt_len + steps + 1
    plan = mk.Plan(cfg, w, max_batch=1, page_size=16, max_seq_len=cap + 16)
    kv = PagedKVCache(cfg, 1, [cap], page=16,
                      page_order=synth.page_permutation((cap + 15) // 16))
    prompt = synth.make_ids(V, (prompt_len,), seed=1)

    # ---- GPU: teacher-forced prompt, then greedy steps fed back on device
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    nids, npos = torch.zeros_like(ids), torch.zeros_like(pos)
    logits = torch.zeros(steps, 1, V, dtype=torch.float32, device="cuda")
    hidden = torch.zeros(steps, L, 1, H, dtype=torch.float32, device="cuda")
    toks = torch.zeros(steps, dtype=torch.int32, device="cuda")
    d_prompt = prompt.to(torch.int32).cuda()
    for t in range(prompt_len - 1):
        ids.copy_(d_prompt[t:t + 1])
        pos.fill_(t)
        plan.step(ids, pos, kv.view, nids, out_pos=npos)
    ids.copy_(d_prompt[prompt_len - 1:])
    pos.fill_(prompt_len - 1)
    for s in range(steps):
        # step 0 is the last prompt token; its argmax is the first greedy token
        plan.step(ids, pos, kv.view, nids, out_pos=npos, out_logits=logits[s], hidden=hidden[s])
        toks[s:s + 1].copy_(nids)
        ids, nids = nids, ids
        pos, npos = npos, pos
    st = plan.status()
    assert st == mk.MK_OK, f"device status {mk.ERROR_NAMES.get(st, st)} {plan.error_info()}"
    g_logits = logits[:, 0].cpu().numpy()
    g_hidden = hidden[:, :, 0].cpu().numpy()
    g_toks = toks.cpu().numpy()
    assert int(pos[0]) == prompt_len - 1 + steps

    # ---- oracle: the prompt as one whole-sequence pass, then decode steps
    ocfg = oracle_cfg(cfg)
    W = oracle.Weights(w, keep_f64=False)
    ocache, last, outs = oracle.prefill(ocfg, W, [prompt.tolist()], cap)
    rep = StepReport()
    # every cached prompt position (the last one is written by step 0 below;
    # the oracle's prefill cache already holds it)
    for l in range(L):
        gk, gv = gpu_cache_rows(kv, l, 0, prompt_len)
        e = max(per_token_rel(gk, ocache.k[l][0][:, :prompt_len]),
                per_token_rel(gv, ocache.v[l][0][:, :prompt_len]))
        rep.max_kv_rel = max(rep.max_kv_rel, e)
        rep.kv_ok = rep.kv_ok and e <= HIDDEN_RTOL
    o_logits = [last[0]]
    o_hidden = [outs[0]["hidden"][:, -1]]
    for s in range(1, steps):
        o = oracle.decode_step(ocfg, W, ocache, [int(g_toks[s - 1])], [prompt_len - 1 + s])
        o_logits.append(o["logits"][0])
        o_hidden.append(o["hidden"][:, 0])
    for s in range(steps):
        for l in range(L):
            rep.max_hidden_rel = max(rep.max_hidden_rel, rel_l2(g_hidden[s, l], o_hidden[s][l]))
        rep.max_logit_err = max(rep.max_logit_err, float(np.max(np.abs(g_logits[s] - o_logits[s]))))
        assert int(g_toks[s]) == int(np.argmax(g_logits[s])), "out_ids != argmax(out_logits)"
        if oracle.top2_margin(o_logits[s]) > MARGIN:
            rep.token_checked += 1
            rep.token_mismatch += int(int(g_toks[s]) != int(np.argmax(o_logits[s])))
        rep.steps += 1
    plan.close()
    assert_report(rep)
