"""Reference decoder in float64: what one greedy decode step computes.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this file and this file imports nothing from the library.

Sources.  The pages this project follows describe *how* a persistent
megakernel runs a decoder (MPK write-up, "2.1 Mega-Kernel执行模型"; Ada-MK
summary, "Methodik", Phase I, which lowers "Transformer-Decoder und LM-Head"
into one kernel) and name the operators (MPK write-up, "1. GPU计算中的任务调度
挑战": Attention -> MLP per layer, attention cost growing with sequence length;
Ada-MK summary, "Experimentelle Ergebnisse": Qwen3 / Qwen2.5 models, decode at
batch 1-16).  None of them writes the arithmetic out.  The oracle therefore is
the plain, standard definition of a Qwen3-style decoder step; each point the
pages leave open is marked READING in the function that takes it:

  per layer:  x  = RMSNorm(h) * g_attn
              q, k, v = Wq x, Wk x, Wv x            (no biases)
              q, k = RMSNorm_d(q) * g_q, RMSNorm_d(k) * g_k   per head, then RoPE
              K/V cache[pos] = bf16(k), bf16(v)
              o  = softmax(q K^T / sqrt(d)) V      over positions 0..pos,
                   query head h reads KV head floor(h / G)
              h += Wo o
              x  = RMSNorm(h) * g_mlp
              h += Wd (silu(Wg x) * (Wu x))
  after the last layer:  logits = Wlm (RMSNorm(h) * g_final),  next = argmax

All arithmetic is float64.  Weights and cached K/V are bf16 values, widened
exactly.  Weights use the nn.Linear convention: a matrix is [out, in], y = W x.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np

try:  # torch is only used to widen bf16 tensors exactly; it is optional
    import torch
except Exception:  # pragma: no cover
    torch = None


# --------------------------------------------------------------------------
# configuration and weights
# --------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class DecoderConfig:
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float = 1e-6
    rope_theta: float = 1e6
    qk_norm: bool = True

    @property
    def group(self) -> int:
        """Query heads per KV head (grouped-query attention)."""
        assert self.n_q_heads % self.n_kv_heads == 0
        return self.n_q_heads // self.n_kv_heads


def as_f64(a) -> np.ndarray:
    """Widen an array of bf16 / fp32 / fp64 values to float64 exactly.

    torch bf16 tensors are widened by torch's own (exact) dtype conversion;
    numpy input is taken as values.  The conversion is exact because every
    bf16 and fp32 value is a float64 value.
    """
    if torch is not None and isinstance(a, torch.Tensor):
        return a.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


class Weights:
    """bf16 weights of one decoder, widened to float64 when first used.

    ``tensors`` uses the names below (torch tensors or numpy arrays):
      embed [V, H], final_norm [H], lm_head [V, H],
      layers[l]: attn_norm [H], wq [Hq*d, H], wk [Hkv*d, H], wv [Hkv*d, H],
                 q_norm [d], k_norm [d], wo [H, Hq*d], mlp_norm [H],
                 w_gate [F, H], w_up [F, H], w_down [H, F]
    ``keep_f64`` keeps the widened copies (fast for small models); with it
    off each layer is widened per use, which bounds host memory for large ones.
    """

    LAYER_KEYS = ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo",
                  "mlp_norm", "w_gate", "w_up", "w_down")

    def __init__(self, tensors: dict, keep_f64: bool = True):
        self.t = tensors
        self.keep = keep_f64
        self._cache: Dict[object, np.ndarray] = {}

    def _get(self, key, src):
        if self.keep:
            if key not in self._cache:
                self._cache[key] = as_f64(src)
            return self._cache[key]
        return as_f64(src)

    def layer(self, l: int) -> Dict[str, np.ndarray]:
        src = self.t["layers"][l]
        return {k: self._get((l, k), src[k]) for k in self.LAYER_KEYS}

    def embed_rows(self, ids: Sequence[int]) -> np.ndarray:
        ids = [int(i) for i in ids]
        e = self.t["embed"]
        if torch is not None and isinstance(e, torch.Tensor):
            return as_f64(e[torch.tensor(ids, dtype=torch.long, device=e.device)])
        return as_f64(np.asarray(e)[ids])

    def final_norm(self) -> np.ndarray:
        return self._get("final_norm", self.t["final_norm"])

    def lm_head(self) -> np.ndarray:
        return self._get("lm_head", self.t["lm_head"])


# --------------------------------------------------------------------------
# 4-bit weights (W4A16)
# --------------------------------------------------------------------------

W4_GROUP = 128     # columns that share one scale
W4_ZERO = 8        # the code that stands for 0
W4_MATRICES = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")


def dequantize_w4(codes, scales) -> np.ndarray:
    """The bf16 weight matrix a 4-bit matrix stands for.

    ``codes`` [rows, cols] hold integers 0..15, ``scales`` [rows, cols/128]
    bf16 values; element (r, c) is  bf16( scales[r, c // 128] * (codes[r, c] - 8) ).
    READING (the Ada-MK summary, "Quantisierungs-bewusste Optimierung", names
    GPTQ-style W4A16 without fixing its details): symmetric codes with zero
    point 8, one bf16 scale per row and group of 128 input columns, and the
    dequantized weight rounded once (to nearest, ties to even) to bf16, the
    precision the bf16 activations meet it in.  The product scale * (code - 8)
    is exact in float64; round_bf16 is the only rounding.
    """
    q = np.asarray(as_f64(codes), dtype=np.float64)
    s = as_f64(scales)
    rows, cols = q.shape
    assert s.shape == (rows, cols // W4_GROUP) and cols % W4_GROUP == 0
    return round_bf16(np.repeat(s, W4_GROUP, axis=1) * (q - W4_ZERO))


class W4Weights(Weights):
    """A decoder whose seven projection matrices per layer are 4-bit: layer
    ``l`` of ``tensors`` holds ``w4[name] = (codes, scales)`` for each name in
    W4_MATRICES (and the norms as bf16); embedding, final norm and LM head are
    bf16.  Each matrix is dequantized (dequantize_w4) when the layer is used."""

    def layer(self, l: int) -> Dict[str, np.ndarray]:
        src = self.t["layers"][l]
        out = {}
        for k in self.LAYER_KEYS:
            if k in W4_MATRICES:
                codes, scales = src["w4"][k]
                if self.keep:
                    key = (l, k, "w4")
                    if key not in self._cache:
                        self._cache[key] = dequantize_w4(codes, scales)
                    out[k] = self._cache[key]
                else:
                    out[k] = dequantize_w4(codes, scales)
            else:
                out[k] = self._get((l, k), src[k])
        return out


# --------------------------------------------------------------------------
# elementwise pieces
# --------------------------------------------------------------------------


def round_bf16(x) -> np.ndarray:
    """Round float64 values to bf16 (8 significant bits), ties to even.

    READING: the cache is bf16, so cached K and V are rounded once, straight
    from the exact value.  Valid for normal numbers (|x| >= 2**-126), which
    covers every cached value here.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                    # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.round(m * 256.0) / 256.0, e)   # np.round: half to even


def rms_norm(x: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x**2) + eps) * gain over the last axis (no mean removal)."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gain


def rope_angles(pos: int, d: int, theta: float) -> np.ndarray:
    """Angle of pair i at position pos: pos * theta**(-2i/d), i < d/2."""
    i = np.arange(d // 2, dtype=np.float64)
    return float(pos) * theta ** (-2.0 * i / d)


def apply_rope(x: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """Rotary position embedding of the last axis at position ``pos``.

    READING: the half-split ("rotate half") pairing used by Qwen-family
    models: element i pairs with element i + d/2, and the pair is rotated
    counter-clockwise by rope_angles(pos)[i]:
        (a, b) -> (a cos - b sin, b cos + a sin).
    """
    d = x.shape[-1]
    half = d // 2
    ang = rope_angles(pos, d, theta)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z))."""
    return z / (1.0 + np.exp(-z))


def softmax(s: np.ndarray) -> np.ndarray:
    """Softmax over the last axis, with the maximum subtracted first."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """One query against T cached positions: softmax(K q * scale) @ V.

    q [d], K [T, d], V [T, d] -> [d].  READING: scale 1/sqrt(d), no mask
    beyond the cache length, no sliding window, no logit soft-cap.
    """
    return softmax(K @ q * scale) @ V


def top2_margin(logits: np.ndarray) -> np.ndarray:
    """Largest minus second-largest logit of each row (>= 0)."""
    part = np.partition(logits, -2, axis=-1)
    return part[..., -1] - part[..., -2]


# --------------------------------------------------------------------------
# KV cache
# --------------------------------------------------------------------------


class KVCache:
    """Per layer, per sequence: K and V as float64 arrays [Hkv, capacity, d].

    Holds bf16 values (the caller rounds before writing).  ``length[b]`` is
    the number of valid positions 0..length-1 of sequence b.
    """

    def __init__(self, cfg: DecoderConfig, batch: int, capacity: int):
        self.cfg = cfg
        shape = (cfg.n_kv_heads, capacity, cfg.head_dim)
        self.k = [[np.zeros(shape) for _ in range(batch)] for _ in range(cfg.n_layers)]
        self.v = [[np.zeros(shape) for _ in range(batch)] for _ in range(cfg.n_layers)]
        self.length = [0] * batch

    def write(self, l: int, b: int, pos: int, k: np.ndarray, v: np.ndarray):
        self.k[l][b][:, pos, :] = k
        self.v[l][b][:, pos, :] = v

    def load_history(self, l: int, b: int, k: np.ndarray, v: np.ndarray):
        """Install positions 0..T-1 from arrays [Hkv, T, d] (bf16 values)."""
        T = k.shape[1]
        self.k[l][b][:, :T, :] = k
        self.v[l][b][:, :T, :] = v


# --------------------------------------------------------------------------
# the decoder
# --------------------------------------------------------------------------


def _qk_heads(cfg: DecoderConfig, w, q_row, k_row, v_row, pos):
    """Split one position's q/k/v rows into heads; QK-norm then RoPE.

    READING: QK-norm is an RMSNorm over head_dim with one gain vector [d]
    shared by all heads of q (resp. k), applied *before* RoPE; v is neither
    normed nor rotated.
    """
    d = cfg.head_dim
    qh = q_row.reshape(cfg.n_q_heads, d)
    kh = k_row.reshape(cfg.n_kv_heads, d)
    vh = v_row.reshape(cfg.n_kv_heads, d)
    if cfg.qk_norm:
        qh = rms_norm(qh, w["q_norm"], cfg.rms_eps)
        kh = rms_norm(kh, w["k_norm"], cfg.rms_eps)
    qh = apply_rope(qh, pos, cfg.rope_theta)
    kh = apply_rope(kh, pos, cfg.rope_theta)
    return qh, kh, vh


def decode_step(cfg: DecoderConfig, W: Weights, cache: KVCache,
                ids: Sequence[int], pos: Sequence[int],
                layers: Optional[int] = None) -> dict:
    """One decode step for B sequences, each feeding token ids[b] at pos[b].

    Appends K/V at pos[b] to ``cache`` (rounded to bf16) and attends over
    positions 0..pos[b].  Returns ``logits`` [B, V], ``next_ids`` [B] (argmax,
    lowest index on ties), ``hidden`` [L, B, H] (the residual stream after each
    layer), ``q`` [L, B, Hq, d] (query after QK-norm and RoPE) and ``k_new`` /
    ``v_new`` [L, B, Hkv, d] (what was written to the cache).

    ``layers`` < n_layers stops early (used to time a bounded sample); the
    logits are then those of the truncated stack.
    """
    L = cfg.n_layers if layers is None else layers
    B = len(ids)
    d, G = cfg.head_dim, cfg.group
    scale = 1.0 / math.sqrt(d)
    h = W.embed_rows(ids)                                     # [B, H]
    hidden, qs, ks, vs = [], [], [], []
    for l in range(L):
        w = W.layer(l)
        x = rms_norm(h, w["attn_norm"], cfg.rms_eps)
        q = x @ w["wq"].T
        k = x @ w["wk"].T
        v = x @ w["wv"].T
        o = np.zeros((B, cfg.n_q_heads * d))
        q_l = np.zeros((B, cfg.n_q_heads, d))
        k_l = np.zeros((B, cfg.n_kv_heads, d))
        v_l = np.zeros((B, cfg.n_kv_heads, d))
        for b in range(B):
            p = int(pos[b])
            qh, kh, vh = _qk_heads(cfg, w, q[b], k[b], v[b], p)
            kb, vb = round_bf16(kh), round_bf16(vh)
            cache.write(l, b, p, kb, vb)
            Kc = cache.k[l][b][:, : p + 1, :]
            Vc = cache.v[l][b][:, : p + 1, :]
            for hq in range(cfg.n_q_heads):
                g = hq // G
                o[b, hq * d:(hq + 1) * d] = attend(qh[hq], Kc[g], Vc[g], scale)
            q_l[b], k_l[b], v_l[b] = qh, kb, vb
        h = h + o @ w["wo"].T
        x = rms_norm(h, w["mlp_norm"], cfg.rms_eps)
        u = silu(x @ w["w_gate"].T) * (x @ w["w_up"].T)
        h = h + u @ w["w_down"].T
        hidden.append(h.copy())
        qs.append(q_l)
        ks.append(k_l)
        vs.append(v_l)
    for b in range(B):
        cache.length[b] = max(cache.length[b], int(pos[b]) + 1)
    x = rms_norm(h, W.final_norm(), cfg.rms_eps)
    logits = x @ W.lm_head().T
    def stack(xs, shape):
        return np.stack(xs) if xs else np.zeros((0,) + shape)

    return {
        "logits": logits,
        "next_ids": np.argmax(logits, axis=-1),
        "hidden": stack(hidden, (B, cfg.hidden)),
        "q": stack(qs, (B, cfg.n_q_heads, d)),
        "k_new": stack(ks, (B, cfg.n_kv_heads, d)),
        "v_new": stack(vs, (B, cfg.n_kv_heads, d)),
    }


def forward_full(cfg: DecoderConfig, W: Weights, ids: Sequence[int]) -> dict:
    """Whole-sequence forward of one sequence, positions 0..T-1, no cache.

    Causal attention in matrix form (scores masked above the diagonal).  K and
    V are rounded to bf16 before attention, as the cached decode path stores
    them, so the two paths compute the same function.  Returns ``logits``
    [T, V], ``hidden`` [L, T, H] and the rounded ``k`` / ``v`` [L, Hkv, T, d].
    """
    T = len(ids)
    d, G = cfg.head_dim, cfg.group
    scale = 1.0 / math.sqrt(d)
    h = W.embed_rows(ids)                                     # [T, H]
    causal = np.triu(np.full((T, T), -np.inf), k=1)
    hidden, k_all, v_all = [], [], []
    for l in range(cfg.n_layers):
        w = W.layer(l)
        x = rms_norm(h, w["attn_norm"], cfg.rms_eps)
        q = (x @ w["wq"].T).reshape(T, cfg.n_q_heads, d)
        k = (x @ w["wk"].T).reshape(T, cfg.n_kv_heads, d)
        v = (x @ w["wv"].T).reshape(T, cfg.n_kv_heads, d)
        if cfg.qk_norm:
            q = rms_norm(q, w["q_norm"], cfg.rms_eps)
            k = rms_norm(k, w["k_norm"], cfg.rms_eps)
        for t in range(T):
            q[t] = apply_rope(q[t], t, cfg.rope_theta)
            k[t] = apply_rope(k[t], t, cfg.rope_theta)
        k = round_bf16(k)
        v = round_bf16(v)
        o = np.zeros((T, cfg.n_q_heads, d))
        for hq in range(cfg.n_q_heads):
            g = hq // G
            S = q[:, hq, :] @ k[:, g, :].T * scale + causal   # [T, T]
            o[:, hq, :] = softmax(S) @ v[:, g, :]
        h = h + o.reshape(T, -1) @ w["wo"].T
        x = rms_norm(h, w["mlp_norm"], cfg.rms_eps)
        u = silu(x @ w["w_gate"].T) * (x @ w["w_up"].T)
        h = h + u @ w["w_down"].T
        hidden.append(h.copy())
        k_all.append(np.transpose(k, (1, 0, 2)))
        v_all.append(np.transpose(v, (1, 0, 2)))
    x = rms_norm(h, W.final_norm(), cfg.rms_eps)
    return {
        "logits": x @ W.lm_head().T,
        "hidden": np.stack(hidden),
        "k": np.stack(k_all),
        "v": np.stack(v_all),
    }


def prefill(cfg: DecoderConfig, W: Weights, prompts: List[Sequence[int]],
            capacity: int) -> tuple:
    """Run each prompt through ``forward_full`` and install its K/V in a cache.

    READING: a prompt is the same computation as feeding its tokens one by one
    as decode steps at positions 0..n-1 (the Ada-MK summary hands prefill to
    another engine; here it is teacher-forced decode).  The full-sequence form
    is only faster.  Returns (cache, last_logits [B, V], per-prompt outputs).
    """
    cache = KVCache(cfg, len(prompts), capacity)
    last, outs = [], []
    for b, ids in enumerate(prompts):
        out = forward_full(cfg, W, ids)
        for l in range(cfg.n_layers):
            cache.load_history(l, b, out["k"][l], out["v"][l])
        cache.length[b] = len(ids)
        last.append(out["logits"][-1])
        outs.append(out)
    return cache, np.stack(last), outs


def greedy_decode(cfg: DecoderConfig, W: Weights, prompts: List[Sequence[int]],
                  n_steps: int, force: Optional[np.ndarray] = None) -> dict:
    """Teacher-forced prompt, then ``n_steps`` greedy decode steps.

    The first generated token is the argmax after the last prompt token; each
    later step feeds the previous step's token at the next position.  All
    prompts must have the same length.  ``force`` [n_steps, B], if given,
    replaces the fed tokens (to keep two runs on one path).  Returns the
    per-step ``logits`` [n_steps, B, V], ``tokens`` [n_steps, B] (argmax of
    each step) and ``margins`` (top-2 logit gaps).
    """
    n = len(prompts[0])
    assert all(len(p) == n for p in prompts)
    cache, last_logits, _ = prefill(cfg, W, prompts, n + n_steps)
    logits = [last_logits]
    tok = np.argmax(last_logits, axis=-1)
    toks = [tok]
    for s in range(1, n_steps):
        feed = tok if force is None else force[s - 1]
        out = decode_step(cfg, W, cache, feed, [n + s - 1] * len(prompts))
        logits.append(out["logits"])
        tok = out["next_ids"]
        toks.append(tok)
    logits = np.stack(logits)
    return {"logits": logits, "tokens": np.stack(toks), "margins": top2_margin(logits)}
