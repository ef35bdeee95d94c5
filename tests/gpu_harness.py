"""Shared helpers of the GPU parity tests: run the CUDA path (through the C ABI)
and the oracle on the same seeded inputs and compare them step by step.

Tolerances (per decode step):
  * residual stream after every layer: relative L2 error <= 1e-2,
  * logits: max |GPU - oracle| <= 5e-2,
  * greedy token identical wherever the oracle's top-2 logit margin > 0.1,
  * K/V written to the cache: relative L2 error per token <= 1e-2.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

import oracle
from persistent_task_runtime_b200 import mk, synth
from persistent_task_runtime_b200.kvcache import PagedKVCache

HIDDEN_RTOL = 1e-2
LOGITS_ATOL = 5e-2
MARGIN = 0.1


def oracle_cfg(cfg: dict) -> oracle.DecoderConfig:
    return oracle.DecoderConfig(**{k: cfg[k] for k in (
        "n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
        "rms_eps", "rope_theta", "qk_norm")})


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def bf16_diff(gpu: torch.Tensor, ref: np.ndarray):
    """(largest difference in bf16 ulps, fraction of elements that differ)."""
    g = gpu.to(torch.float64).cpu().numpy()
    r = np.asarray(ref, dtype=np.float64)
    ulp = np.ldexp(1.0, np.frexp(np.maximum(np.abs(r), np.abs(g)))[1] - 8)
    diff = np.abs(g - r)
    return float(np.max(diff / ulp)), float(np.mean(diff > 0))


def kv_rel(gpu: torch.Tensor, ref: np.ndarray) -> float:
    """Relative L2 error of one token's cached K (or V) over all KV heads.

    Per-element bf16 equality is not a usable bar: both sides round to bf16,
    but from values that differ by the upstream error (~1e-4 relative), so an
    element near zero can land many of its own ulps apart.  The cached vector
    is held to the same relative-L2 bar as the residual stream."""
    return rel_l2(gpu.to(torch.float64).cpu().numpy(), ref)


@dataclass
class StepReport:
    max_hidden_rel: float = 0.0
    max_logit_err: float = 0.0
    token_checked: int = 0
    token_mismatch: int = 0
    steps: int = 0
    kv_ok: bool = True
    max_kv_rel: float = 0.0
    worst: List[str] = field(default_factory=list)


class Pair:
    """The CUDA path and the oracle, fed identical inputs."""

    def __init__(self, cfg: dict, weights: dict, max_batch: int, capacity: List[int],
                 page: int = 16, max_seq_len: Optional[int] = None, keep_f64: bool = True,
                 **plan_kw):
        self.cfg = cfg
        self.B = max_batch
        self.ocfg = oracle_cfg(cfg)
        # (4-bit layers: the oracle dequantizes them by the format's definition)
        wcls = oracle.W4Weights if "w4" in weights["layers"][0] else oracle.Weights
        self.W = wcls(weights, keep_f64=keep_f64)
        msl = max_seq_len or max(capacity)
        self.plan = mk.Plan(cfg, weights, max_batch=max_batch, page_size=page,
                            max_seq_len=msl, **plan_kw)
        self.kv = PagedKVCache(cfg, max_batch, capacity, page=page,
                               page_order=synth.page_permutation(sum(
                                   (c + page - 1) // page for c in capacity)))
        self.ocache = oracle.KVCache(self.ocfg, max_batch, max(capacity))
        dev = "cuda"
        self.d_ids = torch.zeros(max_batch, dtype=torch.int32, device=dev)
        self.d_pos = torch.zeros(max_batch, dtype=torch.int32, device=dev)
        self.d_out = torch.zeros(max_batch, dtype=torch.int32, device=dev)
        self.d_logits = torch.zeros(max_batch, cfg["vocab"], dtype=torch.float32, device=dev)
        self.d_hidden = torch.zeros(cfg["n_layers"], max_batch, cfg["hidden"],
                                    dtype=torch.float32, device=dev)

    def load_history(self, hist, lengths):
        self.kv.load_history(hist, lengths)
        for l, hl in enumerate(hist):
            for b, n in enumerate(lengths):
                self.ocache.load_history(l, b, hl["k"][b, :, :n].to(torch.float64).numpy(),
                                         hl["v"][b, :, :n].to(torch.float64).numpy())

    def gpu_step(self, ids, pos, mode=mk.MODE_MEGAKERNEL):
        B = len(ids)
        self.d_ids[:B] = torch.tensor(ids, dtype=torch.int32)
        self.d_pos[:B] = torch.tensor(pos, dtype=torch.int32)
        # the hidden dump is packed as [n_layers, B, H] for the step's batch B
        self.plan.step(self.d_ids[:B], self.d_pos[:B], self.kv.view, self.d_out[:B],
                       out_logits=self.d_logits[:B], hidden=self.d_hidden, mode=mode, batch=B)
        st = self.plan.status()
        assert st == mk.MK_OK, f"device status {mk.ERROR_NAMES.get(st, st)} {self.plan.error_info()}"
        return (self.d_out[:B].cpu().numpy().copy(), self.d_logits[:B].cpu().numpy().copy(),
                self.d_hidden.view(-1)[: self.cfg["n_layers"] * B * self.cfg["hidden"]]
                .view(self.cfg["n_layers"], B, self.cfg["hidden"]).cpu().numpy().copy())

    def oracle_step(self, ids, pos):
        return oracle.decode_step(self.ocfg, self.W, self.ocache, ids, pos)

    def compare(self, ids, pos, rep: StepReport, check_kv=True, mode=mk.MODE_MEGAKERNEL):
        g_ids, g_logits, g_hidden = self.gpu_step(ids, pos, mode)
        o = self.oracle_step(ids, pos)
        B = len(ids)
        for l in range(self.cfg["n_layers"]):
            for b in range(B):
                e = rel_l2(g_hidden[l, b], o["hidden"][l, b])
                if e > rep.max_hidden_rel:
                    rep.max_hidden_rel = e
        err = float(np.max(np.abs(g_logits - o["logits"])))
        rep.max_logit_err = max(rep.max_logit_err, err)
        margins = oracle.top2_margin(o["logits"])
        for b in range(B):
            if margins[b] > MARGIN:
                rep.token_checked += 1
                if int(g_ids[b]) != int(o["next_ids"][b]):
                    rep.token_mismatch += 1
            # argmax of the GPU's own logits must be its returned token
            assert int(g_ids[b]) == int(np.argmax(g_logits[b])), "out_ids != argmax(out_logits)"
        if check_kv:
            for l in range(self.cfg["n_layers"]):
                for b in range(B):
                    k, v = self.kv.token(l, b, int(pos[b]))
                    e = max(kv_rel(k, o["k_new"][l, b]), kv_rel(v, o["v_new"][l, b]))
                    rep.max_kv_rel = max(rep.max_kv_rel, e)
                    if e > HIDDEN_RTOL:
                        rep.kv_ok = False
                        if len(rep.worst) < 8:
                            rep.worst.append(
                                f"step {rep.steps} layer {l} seq {b} pos {pos[b]}: kv rel {e:.3g} "
                                f"k ulps/frac {bf16_diff(k, o['k_new'][l, b])} "
                                f"v ulps/frac {bf16_diff(v, o['v_new'][l, b])}")
        rep.steps += 1
        return o

    def close(self):
        self.plan.close()


#: Every report checked in this process, with the test that produced it; the
#: session summary (tests/conftest.py) prints them, so the margins left under
#: the tolerances are visible in a passing run's log.
REPORTS: List[tuple] = []


def record(rep: StepReport):
    import os
    name = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    REPORTS.append((name, rep))


def assert_report(rep: StepReport):
    record(rep)
    assert rep.max_hidden_rel <= HIDDEN_RTOL, rep
    assert rep.max_logit_err <= LOGITS_ATOL, rep
    assert rep.token_mismatch == 0, rep
    assert rep.kv_ok, rep
