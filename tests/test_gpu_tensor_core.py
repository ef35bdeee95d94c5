"""GPU parity of the tensor-core GEMV path (tcgen05) against the CPU oracle.

Every projection of these plans runs on 128-row tiles: weights arrive by TMA
tensor copies in the 128-byte-swizzled layout the MMA reads, the activation
is staged as bf16 high/low halves, accumulators live in tensor memory, and the
QKV, O, gate/up and down projections are split along K with the parts summed
in a fixed order.  The shapes put ragged edges everywhere the path has them: a
last row tile of 64 rows (ffn 2240 and a 5000-row LM head, which TMA pads with
zeros), a down projection whose K ends in a half page, and batches that fill
the MMA's N partly (1, 5, 13) or exactly (8, 16).  Tolerances are those of
tests/gpu_harness.py.
"""

import numpy as np
import pytest
import torch

from persistent_task_runtime_b200 import mk, synth
from tests.gpu_harness import Pair, StepReport, assert_report

pytestmark = pytest.mark.gpu

TC_CFG = dict(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=2240,
              vocab=5000, rms_eps=1e-6, rope_theta=1e6, qk_norm=True)


@pytest.mark.parametrize("B", [1, 5, 8, 13, 16])
def test_tensor_core_path_batches(cuda_device, B):
    cfg = TC_CFG
    w = synth.make_weights(cfg, seed=31, device="cuda", gain="random")
    lengths = [int(x) for x in np.linspace(0, 150, B)]
    steps = 3
    pair = Pair(cfg, w, B, [n + steps + 2 for n in lengths], gemv_path=2)
    assert pair.plan.info()["gemv_path"] == 2
    pair.load_history(synth.make_kv_history(cfg, lengths, seed=32), lengths)
    ids = synth.make_ids(cfg["vocab"], (steps, B), seed=33)
    rep = StepReport()
    for s in range(steps):
        pair.compare(ids[s].tolist(), [n + s for n in lengths], rep)
    if B > 2:
        # a smaller batch on the same plan
        pair.compare(ids[0, :2].tolist(), [lengths[0] + steps, lengths[1] + steps], rep)
    pair.close()
    assert_report(rep)


def test_tensor_core_megakernel_equals_per_operator_launches(cuda_device):
    """The tensor-core plan under the three schedules (one persistent launch,
    one launch per operator, those launches replayed from a CUDA graph):
    bit-identical logits, ids, hidden states and cache."""
    cfg = TC_CFG
    w = synth.make_weights(cfg, seed=34, device="cuda")
    B, lengths, steps = 6, [3, 40, 64, 65, 100, 7], 3
    outs = []
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for mode in (mk.MODE_MEGAKERNEL, mk.MODE_PER_OP, mk.MODE_PER_OP_GRAPH):
            pair = Pair(cfg, w, B, [n + steps for n in lengths], gemv_path=2)
            pair.load_history(synth.make_kv_history(cfg, lengths, seed=35), lengths)
            ids = synth.make_ids(cfg["vocab"], (steps, B), seed=36)
            rec = [pair.gpu_step(ids[s].tolist(), [n + s for n in lengths], mode=mode)
                   for s in range(steps)]
            outs.append((rec, [t.clone() for t in pair.kv.k + pair.kv.v]))
            pair.close()
    (ra, ka) = outs[0]
    for rb, kb in outs[1:]:
        for (ia, la, ha), (ib, lb, hb) in zip(ra, rb):
            assert np.array_equal(ia, ib)
            assert np.array_equal(la, lb)
            assert np.array_equal(ha, hb)
        for x, y in zip(ka, kb):
            assert torch.equal(x, y)


def test_tensor_core_and_mma_paths_agree(cuda_device):
    """The two GEMV paths on one model and batch: both within the oracle's
    tolerances (checked above); here their logits agree to well inside the
    logits bar and their confident tokens are equal."""
    cfg = TC_CFG
    w = synth.make_weights(cfg, seed=37, device="cuda")
    B, lengths = 8, [50] * 8
    res = []
    for path in (1, 2):
        pair = Pair(cfg, w, B, [n + 2 for n in lengths], gemv_path=path)
        assert pair.plan.info()["gemv_path"] == path
        pair.load_history(synth.make_kv_history(cfg, lengths, seed=38), lengths)
        ids = synth.make_ids(cfg["vocab"], (B,), seed=39).tolist()
        res.append(pair.gpu_step(ids, lengths))
        pair.close()
    (ia, la, ha), (ib, lb, hb) = res
    assert np.max(np.abs(la - lb)) <= 2e-2
    part = np.partition(la, -2, axis=-1)
    confident = part[:, -1] - part[:, -2] > 0.1
    assert np.array_equal(ia[confident], ib[confident])
