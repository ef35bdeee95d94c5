"""GPU parity of the two attention paths against the CPU oracle.

attn_path 1 (the default) computes q.K and P.V with fp32 FMA over K/V pages
bulk-copied into shared memory; attn_path 2 copies the pages with TMA tensor
copies in the 128-byte-swizzled layout and runs q.K and P.V as mma.sync
m16n8k16 tiles fed by ldmatrix.  Both must meet the tolerances of
tests/gpu_harness.py on the same cases: a prompt followed by greedy steps,
ragged histories on and around page boundaries, a long context split into
many chunks, batch 16 on either projection path, head_dim 128 with G = 8,
and prompt chunks.
"""

import numpy as np
import pytest

from persistent_task_runtime_b200 import synth
from tests.gpu_harness import Pair, StepReport, assert_report
from tests.test_gpu_parity import SHAPES
from tests.test_gpu_prefill import TC_CFG, run_prefill_case

pytestmark = pytest.mark.gpu


def _weights(cfg, seed, gain="ones"):
    return synth.make_weights(cfg, seed=seed, device="cuda", gain=gain)


def test_attn_mma_prompt_then_greedy(cuda_device):
    cfg = synth.CONFIGS["tiny"]
    pair = Pair(cfg, _weights(cfg, 40), 1, [48], attn_path=2)
    assert pair.plan.info()["attn_path"] == 2
    prompt = synth.make_ids(cfg["vocab"], (16,), seed=41).tolist()
    rep = StepReport()
    tok = None
    for t in range(16 + 32):
        o = pair.compare([prompt[t] if t < 16 else tok], [t], rep)
        tok = int(o["next_ids"][0])
    pair.close()
    assert_report(rep)


@pytest.mark.parametrize("attn_path", [1, 2])
def test_attn_paths_ragged_history(cuda_device, attn_path):
    cfg = synth.CONFIGS["tiny"]
    lengths = [0, 15, 16, 17, 300, 1100]
    steps = 4
    B = len(lengths)
    pair = Pair(cfg, _weights(cfg, 42), B, [n + steps for n in lengths], attn_path=attn_path)
    assert pair.plan.info()["attn_path"] == attn_path
    pair.load_history(synth.make_kv_history(cfg, lengths, seed=43), lengths)
    ids = synth.make_ids(cfg["vocab"], (steps, B), seed=44)
    rep = StepReport()
    for s in range(steps):
        pair.compare(ids[s].tolist(), [n + s for n in lengths], rep)
    pair.close()
    assert_report(rep)


@pytest.mark.parametrize("gemv_path", [1, 2])
def test_attn_mma_batch16(cuda_device, gemv_path):
    cfg = dict(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=2048,
               vocab=4096, rms_eps=1e-6, rope_theta=1e6, qk_norm=True)
    B = 16
    lengths = [int(x) for x in np.linspace(1, 400, B)]
    pair = Pair(cfg, _weights(cfg, 45, gain="random"), B, [n + 4 for n in lengths],
                gemv_path=gemv_path, attn_path=2)
    pair.load_history(synth.make_kv_history(cfg, lengths, seed=46), lengths)
    ids = synth.make_ids(cfg["vocab"], (3, B), seed=47)
    rep = StepReport()
    for s in range(3):
        pair.compare(ids[s].tolist(), [n + s for n in lengths], rep)
    pair.close()
    assert_report(rep)


def test_attn_mma_d128_g8(cuda_device):
    cfg = SHAPES["d128_g8"]
    pair = Pair(cfg, _weights(cfg, 48, gain="random"), 1, [40], attn_path=2)
    ids = synth.make_ids(cfg["vocab"], (40,), seed=49).tolist()
    rep = StepReport()
    for t in range(40):
        pair.compare([ids[t]], [t], rep)
    pair.close()
    assert_report(rep)


def test_attn_mma_prefill(cuda_device):
    w = synth.make_weights(TC_CFG, seed=50, device="cuda", gain="random")
    run_prefill_case(TC_CFG, w, 45, 16, seq=0, n_seqs=1, decode_steps=2, attn_path=2)
