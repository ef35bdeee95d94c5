"""The no-allocation entry point against the plan-based one (GPU).

mk_decode_step_noalloc serves callers that cannot call cudaMalloc (a host
that routes every device allocation through its own pool, a memory-capped
sandbox, a callback that must not allocate): it keeps all of its scratch in
the library's static device array instead of a plan's allocations.  It runs
the same kernel on the same layout as a plan built with max_batch equal to
the step's batch, and every reduction in that kernel has a fixed order, so
its logits, token ids and the K/V it appends must be bit-identical to the
plan's.

This file is collected last so that a run stopping at the first failure has
already run every other test; it must pass alone in a fresh process as well
as after the other tests.
"""

import pytest
import torch

from persistent_task_runtime_b200 import mk, synth
from persistent_task_runtime_b200.kvcache import PagedKVCache

pytestmark = pytest.mark.gpu

MID = dict(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=2816,
           vocab=5000, rms_eps=1e-6, rope_theta=1e6, qk_norm=True)
CAP = 64


def _cache(cfg, B, cap=CAP):
    return PagedKVCache(cfg, B, [cap] * B, page=16, device="cuda",
                        page_order=synth.page_permutation(B * ((cap + 15) // 16)))


class Case:
    """One model at one batch size: a plan and the no-allocation path, each
    with its own copy of the same KV history."""

    def __init__(self, cfg, B, seed):
        self.cfg, self.B = cfg, B
        self.w = synth.make_weights(cfg, seed=seed, device="cuda", gain="random")
        self.plan = mk.Plan(cfg, self.w, max_batch=B, page_size=16, max_seq_len=CAP)
        self.ref_kv, self.na_kv = _cache(cfg, B), _cache(cfg, B)
        self.hist_len = [5 + 7 * b for b in range(B)]
        hist = synth.make_kv_history(cfg, self.hist_len, seed=seed + 1, device="cuda")
        self.ref_kv.load_history(hist, self.hist_len)
        self.na_kv.load_history(hist, self.hist_len)
        self.model = mk.ModelRef(cfg, self.w, max_seq_len=CAP)
        self.ids = synth.make_ids(cfg["vocab"], (4, B), seed=seed + 2).cuda()
        self.calls = 0

    def step_both(self):
        """One step through each entry point at the next position; asserts
        bit-identical logits, ids and appended K/V."""
        c, B, V = self.calls, self.B, self.cfg["vocab"]
        ids = self.ids[c].contiguous()
        pos = torch.tensor([n + c for n in self.hist_len], dtype=torch.int32, device="cuda")
        ref_ids = torch.full((B,), -1, dtype=torch.int32, device="cuda")
        ref_logits = torch.full((B, V), float("nan"), dtype=torch.float32, device="cuda")
        self.plan.step(ids, pos, self.ref_kv.view, ref_ids, out_logits=ref_logits)
        assert self.plan.status() == mk.MK_OK
        na_ids = torch.full((B,), -1, dtype=torch.int32, device="cuda")
        na_logits = torch.full((B, V), float("nan"), dtype=torch.float32, device="cuda")
        rc = mk.decode_step_noalloc(self.model, ids, pos, self.na_kv.view, na_ids, na_logits)
        assert rc == mk.MK_OK
        assert torch.equal(ref_logits, na_logits), \
            f"max |diff| {float((ref_logits - na_logits).abs().max())}"
        assert torch.equal(ref_ids, na_ids)
        assert torch.equal(na_ids.long(), torch.argmax(na_logits, dim=-1))
        for l in range(self.cfg["n_layers"]):
            for b in range(B):
                p = int(pos[b])
                rk, rv = self.ref_kv.token(l, b, p)
                nk, nv = self.na_kv.token(l, b, p)
                assert torch.equal(rk, nk) and torch.equal(rv, nv), (l, b, p)
        self.calls += 1

    def close(self):
        self.plan.close()


@pytest.mark.parametrize("model,B", [("tiny", 2), ("mid", 3)])
def test_noalloc_matches_plan_entry_point_two_calls(cuda_device, model, B):
    cfg = synth.CONFIGS["tiny"] if model == "tiny" else MID
    case = Case(cfg, B, seed=21)
    case.step_both()   # two calls in a row: the second reads the first's K/V
    case.step_both()
    case.close()


def test_noalloc_alternating_shapes_overwrite_the_array(cuda_device):
    # each call must replace what the previous call of another shape left in
    # the shared array: tiny B=2, mid B=3, tiny again, mid again
    a = Case(synth.CONFIGS["tiny"], 2, seed=41)
    b = Case(MID, 3, seed=51)
    for case in (a, b, a, b):
        case.step_both()
    a.close()
    b.close()


def test_plans_and_noalloc_of_other_batch_sizes_coexist(cuda_device):
    # the kernel's shared-memory limit is shared by every plan and by the
    # no-allocation path: creating or calling one shape must not break a
    # live one of another shape, in either order
    big = Case(MID, 3, seed=61)
    small = Case(MID, 1, seed=71)
    big.step_both()          # plan B=3, noalloc B=3
    small.step_both()        # plan B=1 created after, noalloc B=1
    big.step_both()          # the B=3 plan and B=3 noalloc still launch
    late = Case(MID, 3, seed=81)   # a new B=3 plan after the B=1 calls
    small.step_both()
    late.step_both()
    for c in (big, small, late):
        c.close()


def test_noalloc_rejects_trace_buffer(cuda_device):
    cfg = synth.CONFIGS["tiny"]
    w = synth.make_weights(cfg, seed=24, device="cuda")
    model_ref = mk.ModelRef(cfg, w, max_seq_len=32)
    kv = _cache(cfg, 1, 32)
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    trace = torch.zeros(1024, dtype=torch.int64, device="cuda")
    with pytest.raises(mk.MkError) as e:
        mk.decode_step_noalloc(model_ref, ids, pos, kv.view, out, trace=trace)
    assert e.value.code == mk.MK_ERR_INVALID_ARG


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
