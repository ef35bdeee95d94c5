"""Seeded synthetic inputs: model configs, random-init weights, token ids,
ragged context lengths and KV-cache histories.

This module is the one place both the CUDA path and the CPU oracle draw their
inputs from.  It holds none of the decoder's arithmetic: it only draws random
numbers and lays them out.  Every draw is seeded (``torch.Generator``), so the
same (seed, device) gives the same tensors; CPU and CUDA generators produce
different streams, which is fine because both sides always receive the very
same tensors.

Workload shapes follow the decode workloads the pages measure on: a Qwen3-8B
sized decoder at batch 1-16 (MPK write-up, "6.1 单卡性能") and a 1.5B-class
low-latency decoder (Ada-MK summary, "Experimentelle Ergebnisse": Qwen3-1.7B /
Qwen2.5-1.5B), here with random weights and random token ids in place of the
real checkpoints and of the CSL / Human-eval datasets, which are not available.
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional

import torch

#: Model shapes.  ``tiny`` is a 2-layer decoder small enough for a pure-CPU
#: oracle run in seconds; ``1.5b`` and ``8b`` carry the layer shapes of the
#: 1.5B-class and 8B-class Qwen decoders.
CONFIGS: Dict[str, dict] = {
    "tiny": dict(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64,
                 ffn=688, vocab=4096, rms_eps=1e-6, rope_theta=1e6, qk_norm=True),
    "1.5b": dict(n_layers=28, hidden=1536, n_q_heads=12, n_kv_heads=2, head_dim=128,
                 ffn=8960, vocab=151936, rms_eps=1e-6, rope_theta=1e6, qk_norm=True),
    "8b": dict(n_layers=36, hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128,
               ffn=12288, vocab=151936, rms_eps=1e-6, rope_theta=1e6, qk_norm=True),
}

#: Decode workloads (batch, context, greedy steps, page size).
WORKLOADS: Dict[str, dict] = {
    "tiny_b1_p16": dict(model="tiny", batch=1, context=16, steps=32, page=16),
    "1.5b_b1_ctx256": dict(model="1.5b", batch=1, context=256, steps=64, page=16),
    "8b_b1_ctx512": dict(model="8b", batch=1, context=512, steps=128, page=16),
    "8b_sweep_ctx1024": dict(model="8b", batch=[1, 2, 4, 8, 16], context=1024, steps=64, page=16),
    "8b_b16_ragged": dict(model="8b", batch=16, context="loguniform(32,8192)", steps=64, page=16),
}

WEIGHT_STD = 0.02


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal_bf16(shape, std, g, device) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 and rounded (RNE) to bf16."""
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return (x * std).to(torch.bfloat16)


def make_weights(cfg: dict, seed: int = 0, device="cpu", gain: str = "ones",
                 layers: Optional[int] = None) -> dict:
    """Random-init bf16 weights in the nn.Linear [out, in] convention.

    Matrices are N(0, 0.02^2).  Norm gains are 1.0 (``gain="ones"``) or, for
    tests that must tell gain-dependent orderings apart, 1 + N(0, 0.1^2)
    (``gain="random"``).  ``layers`` overrides the layer count (for building a
    truncated stack of a large model).
    """
    H, F, V = cfg["hidden"], cfg["ffn"], cfg["vocab"]
    d, Hq, Hkv = cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"]
    L = cfg["n_layers"] if layers is None else layers
    g = _gen(seed, device)

    def norm(n):
        if gain == "ones":
            return torch.ones(n, device=device, dtype=torch.bfloat16)
        return (1.0 + 0.1 * torch.randn(n, generator=g, device=device)).to(torch.bfloat16)

    w = {"embed": _normal_bf16((V, H), WEIGHT_STD, g, device), "layers": []}
    for _ in range(L):
        w["layers"].append({
            "attn_norm": norm(H),
            "wq": _normal_bf16((Hq * d, H), WEIGHT_STD, g, device),
            "wk": _normal_bf16((Hkv * d, H), WEIGHT_STD, g, device),
            "wv": _normal_bf16((Hkv * d, H), WEIGHT_STD, g, device),
            "q_norm": norm(d),
            "k_norm": norm(d),
            "wo": _normal_bf16((H, Hq * d), WEIGHT_STD, g, device),
            "mlp_norm": norm(H),
            "w_gate": _normal_bf16((F, H), WEIGHT_STD, g, device),
            "w_up": _normal_bf16((F, H), WEIGHT_STD, g, device),
            "w_down": _normal_bf16((H, F), WEIGHT_STD, g, device),
        })
    w["final_norm"] = norm(H)
    w["lm_head"] = _normal_bf16((V, H), WEIGHT_STD, g, device)
    return w


W4_MATRIX_NAMES = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")
W4_GROUP = 128


def make_w4_weights(cfg: dict, seed: int = 0, device="cpu", gain: str = "ones",
                    layers: Optional[int] = None) -> dict:
    """Random-init 4-bit weights: the seven projection matrices of every layer
    as (codes, scales) pairs, everything else bf16 as in make_weights.

    codes: uint8 [out, in], uniform in 0..15; scales: bf16 [out, in / 128],
    uniform in [0.003, 0.006) (with codes centred on 8 that gives weights of
    about the 0.02 standard deviation of the bf16 initialisation).  Layer l
    holds ``w4[name] = (codes, scales)``.  Only random numbers are drawn here;
    what a code and a scale stand for is the decoder's business."""
    base = make_weights(cfg, seed=seed, device=device, gain=gain, layers=layers)
    g = _gen(seed + 1000, device)
    for lw in base["layers"]:
        q = {}
        for name in W4_MATRIX_NAMES:
            rows, cols = lw[name].shape
            codes = torch.randint(0, 16, (rows, cols), generator=g, device=device,
                                  dtype=torch.int64).to(torch.uint8)
            scales = (0.003 + 0.003 * torch.rand(rows, cols // W4_GROUP, generator=g,
                                                 device=device)).to(torch.bfloat16)
            q[name] = (codes, scales)
            del lw[name]
        lw["w4"] = q
    return base


def weights_to(w: dict, device) -> dict:
    """Copy a weight dict to another device (same values)."""
    out = {k: v.to(device) for k, v in w.items() if k != "layers"}
    out["layers"] = []
    for lw in w["layers"]:
        d = {k: v.to(device) for k, v in lw.items() if k != "w4"}
        if "w4" in lw:
            d["w4"] = {k: (c.to(device), sc.to(device)) for k, (c, sc) in lw["w4"].items()}
        out["layers"].append(d)
    return out


def make_ids(vocab: int, shape, seed: int = 1) -> torch.Tensor:
    """Token ids uniform in [0, vocab) (int32, CPU)."""
    g = _gen(seed, "cpu")
    return torch.randint(0, vocab, tuple(shape), generator=g, dtype=torch.int64).to(torch.int32)


def ragged_lengths(batch: int, lo: int = 32, hi: int = 8192, seed: int = 2) -> List[int]:
    """Context lengths floor(exp(U(ln lo, ln hi))), seeded (log-uniform)."""
    g = _gen(seed, "cpu")
    u = torch.rand(batch, generator=g, dtype=torch.float64)
    ln_lo, ln_hi = math.log(lo), math.log(hi)
    return [int(math.floor(math.exp(ln_lo + float(x) * (ln_hi - ln_lo)))) for x in u]


def make_kv_history(cfg: dict, lengths: List[int], seed: int = 3, device="cpu",
                    v_std: Optional[float] = None) -> List[Dict[str, torch.Tensor]]:
    """A synthetic KV-cache history for each layer: bf16 K, V [B, Hkv, T, d].

    Positions t < lengths[b] hold data; the rest is zero.  K entries are
    N(0, 1) (the scale of a key after a unit-gain per-head RMSNorm and a
    rotation); V entries are N(0, v_std^2) with v_std = 0.02 * sqrt(hidden)
    by default (the scale of W_v x for unit-RMS x and N(0, 0.02^2) weights).
    """
    B, Hkv, d = len(lengths), cfg["n_kv_heads"], cfg["head_dim"]
    T = max(lengths) if lengths else 0
    if v_std is None:
        v_std = WEIGHT_STD * math.sqrt(cfg["hidden"])
    g = _gen(seed, device)
    out = []
    for _ in range(cfg["n_layers"]):
        k = torch.randn(B, Hkv, T, d, generator=g, device=device).to(torch.bfloat16)
        v = (torch.randn(B, Hkv, T, d, generator=g, device=device) * v_std).to(torch.bfloat16)
        for b, n in enumerate(lengths):
            k[b, :, n:] = 0
            v[b, :, n:] = 0
        out.append({"k": k, "v": v})
    return out


def page_permutation(n_pages: int, seed: int = 4) -> torch.Tensor:
    """A seeded random order of physical page indices (to exercise paging)."""
    g = _gen(seed, "cpu")
    return torch.randperm(n_pages, generator=g)
