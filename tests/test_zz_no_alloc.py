"""The no-allocation entry point against the plan-based one (GPU).

mk_decode_step_noalloc serves callers that cannot call cudaMalloc: it keeps
all of its scratch in the library's static device array instead of a plan's
allocations.  This file is collected last so that a run stopping at the first
failure has already run every other test; it must pass alone in a fresh
process as well as after the other tests.
"""

import numpy as np
import pytest
import torch

from persistent_task_runtime_b200 import mk, synth
from persistent_task_runtime_b200.kvcache import PagedKVCache

pytestmark = pytest.mark.gpu

LOGITS_ATOL = 5e-2


def _cache(cfg, B, cap):
    return PagedKVCache(cfg, B, [cap] * B, page=16, device="cuda",
                        page_order=synth.page_permutation(B * ((cap + 15) // 16)))


@pytest.mark.parametrize("model,B", [("tiny", 2), ("mid", 3)])
def test_noalloc_matches_plan_entry_point_two_calls(cuda_device, model, B):
    cfg = synth.CONFIGS["tiny"] if model == "tiny" else dict(
        n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=2816,
        vocab=5000, rms_eps=1e-6, rope_theta=1e6, qk_norm=True)
    w = synth.make_weights(cfg, seed=21, device="cuda", gain="random")
    cap = 64
    plan = mk.Plan(cfg, w, max_batch=B, page_size=16, max_seq_len=cap)
    ref_kv, na_kv = _cache(cfg, B, cap), _cache(cfg, B, cap)
    hist_len = [5 + 7 * b for b in range(B)]
    hist = synth.make_kv_history(cfg, hist_len, seed=22, device="cuda")
    ref_kv.load_history(hist, hist_len)
    na_kv.load_history(hist, hist_len)
    model_ref = mk.ModelRef(cfg, w, max_seq_len=cap)
    ids = synth.make_ids(cfg["vocab"], (2, B), seed=23).cuda()
    for call in range(2):   # two calls in a row: the second reads the first's K/V
        pos = torch.tensor([n + call for n in hist_len], dtype=torch.int32, device="cuda")
        ref_ids = torch.zeros(B, dtype=torch.int32, device="cuda")
        ref_logits = torch.zeros(B, cfg["vocab"], dtype=torch.float32, device="cuda")
        plan.step(ids[call].contiguous(), pos, ref_kv.view, ref_ids, out_logits=ref_logits)
        assert plan.status() == mk.MK_OK
        na_ids = torch.zeros(B, dtype=torch.int32, device="cuda")
        na_logits = torch.zeros(B, cfg["vocab"], dtype=torch.float32, device="cuda")
        rc = mk.decode_step_noalloc(model_ref, ids[call].contiguous(), pos, na_kv.view, na_ids,
                                    na_logits)
        assert rc == mk.MK_OK
        a, b = ref_logits.cpu().numpy(), na_logits.cpu().numpy()
        assert np.max(np.abs(a - b)) <= LOGITS_ATOL
        part = np.partition(a, -2, axis=-1)
        confident = part[:, -1] - part[:, -2] > 0.1
        assert np.array_equal(ref_ids.cpu().numpy()[confident], na_ids.cpu().numpy()[confident])
    plan.close()


def test_noalloc_rejects_oversized_scratch(cuda_device):
    cfg = synth.CONFIGS["tiny"]
    w = synth.make_weights(cfg, seed=24, device="cuda")
    # a RoPE table alone larger than the static array
    too_long = mk.NOALLOC_SCRATCH_BYTES // (cfg["head_dim"] // 2 * 8) + 1
    model_ref = mk.ModelRef(cfg, w, max_seq_len=too_long)
    kv = _cache(cfg, 1, 32)
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(mk.MkError) as e:
        mk.decode_step_noalloc(model_ref, ids, pos, kv.view, out)
    assert e.value.code == mk.MK_ERR_UNSUPPORTED
    assert "MK_NOALLOC_SCRATCH_BYTES" in str(e.value)
