"""GPU parity of 4-bit weights (W4A16) against the CPU oracle.

The seven projection matrices of every layer are 4-bit codes with one bf16
scale per row and 128 columns (synth.make_w4_weights), packed by mk_w4_pack
into the layout the kernel streams; the oracle dequantizes them by the
format's definition (oracle.dequantize_w4) and runs its float64 decoder.  The
embedding and the LM head stay bf16.  Tolerances are those of
tests/gpu_harness.py.
"""

import numpy as np
import pytest
import torch

import oracle
from persistent_task_runtime_b200 import mk, synth
from persistent_task_runtime_b200.kvcache import PagedKVCache
from tests.gpu_harness import (HIDDEN_RTOL, LOGITS_ATOL, MARGIN, Pair, StepReport, assert_report,
                               kv_rel, oracle_cfg, rel_l2)

pytestmark = pytest.mark.gpu

MID = dict(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=3072,
           vocab=5000, rms_eps=1e-6, rope_theta=1e6, qk_norm=True)


@pytest.mark.parametrize("B", [1, 3, 8])
def test_w4_decode_steps(cuda_device, B):
    w = synth.make_w4_weights(MID, seed=51, device="cuda", gain="random")
    lengths = [int(x) for x in np.linspace(0, 90, B)]
    steps = 3
    pair = Pair(MID, w, B, [n + steps + 1 for n in lengths])
    assert pair.plan.info()["weight_bits"] == 4
    pair.load_history(synth.make_kv_history(MID, lengths, seed=52), lengths)
    ids = synth.make_ids(MID["vocab"], (steps, B), seed=53)
    rep = StepReport()
    for s in range(steps):
        pair.compare(ids[s].tolist(), [n + s for n in lengths], rep)
    pair.close()
    assert_report(rep)


def test_w4_megakernel_equals_per_operator_launches(cuda_device):
    w = synth.make_w4_weights(MID, seed=54, device="cuda")
    B, lengths = 2, [10, 40]
    outs = []
    for mode in (mk.MODE_MEGAKERNEL, mk.MODE_PER_OP):
        pair = Pair(MID, w, B, [n + 2 for n in lengths])
        pair.load_history(synth.make_kv_history(MID, lengths, seed=55), lengths)
        ids = synth.make_ids(MID["vocab"], (B,), seed=56).tolist()
        outs.append(pair.gpu_step(ids, lengths, mode=mode))
        pair.close()
    for a, b in zip(outs[0], outs[1]):
        assert np.array_equal(a, b)


def test_w4_full_size_8b_batch1(cuda_device):
    """The 8B shape with 4-bit projections, one step over a 512-token history."""
    cfg = synth.CONFIGS["8b"]
    ctx = 512
    w = synth.make_w4_weights(cfg, seed=0, device="cuda")
    pair = Pair(cfg, w, 1, [ctx + 2], max_seq_len=ctx + 17, keep_f64=False)
    pair.load_history(synth.make_kv_history(cfg, [ctx], seed=3), [ctx])
    ids = synth.make_ids(cfg["vocab"], (1, 1), seed=1)
    rep = StepReport()
    pair.compare(ids[0].tolist(), [ctx], rep)
    pair.close()
    assert_report(rep)
