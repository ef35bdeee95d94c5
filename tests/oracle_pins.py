"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes the oracle's decoder module ``O`` and raises
AssertionError (or any exception) if the oracle disagrees with:
  * closed forms (RMSNorm of a constant vector, RoPE at position 0, RoPE of a
    unit vector at a known angle, attention over one token, equal keys),
  * invariants (softmax rows sum to 1, RoPE preserves norms and depends only
    on relative position, causality, incremental decode == full recompute,
    GQA with one KV head per query head == MHA),
  * independent library routines (torch.nn.functional.rms_norm, silu,
    scaled_dot_product_attention with GQA, complex multiplication for RoPE,
    torch's fp32 -> bf16 conversion),
  * a brute-force scalar-loop decoder on a micro model,
  * a whole-decoder composition of torch library ops on the tiny model.
Taking the module as an argument lets ``test_oracle_pins.py`` also run every
pin against deliberately broken copies of the oracle (mutation test) and check
that each planted mistake is caught.
"""

from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

from persistent_task_runtime_b200 import synth

MICRO = dict(n_layers=2, hidden=8, n_q_heads=4, n_kv_heads=2, head_dim=4, ffn=12,
             vocab=16, rms_eps=1e-6, rope_theta=1e6, qk_norm=True)


def _cfg(O, d):
    return O.DecoderConfig(**d)


def _weights(O, d, seed=0, gain="random", keep=True):
    w = synth.make_weights(d, seed=seed, device="cpu", gain=gain)
    return w, O.Weights(w, keep_f64=keep)


# ---------------------------------------------------------------- pieces ---


def pin_round_bf16(O):
    # hand-worked values: 8 significant bits, ties to even
    x = np.array([1.0, 1 + 2**-8, 1 + 3 * 2**-8, 1 + 2**-8 + 2**-30, -(1 + 2**-7),
                  3.0, 2**-20 * (1 + 2**-9)])
    want = np.array([1.0, 1.0, 1 + 2**-6, 1 + 2**-7, -(1 + 2**-7), 3.0, 2**-20])
    np.testing.assert_array_equal(O.round_bf16(x), want)
    # fp32 inputs: torch's fp32 -> bf16 conversion (RNE) is a single rounding
    r = np.random.default_rng(0).standard_normal(20000).astype(np.float32)
    t = torch.from_numpy(r).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(r.astype(np.float64)), t)


def pin_rms_norm(O):
    # closed form: constant vector c*1 -> c / sqrt(c^2 + eps) * g
    for c in (0.5, -3.0, 1e-4):
        g = np.linspace(0.5, 1.5, 16)
        got = O.rms_norm(np.full(16, c), g, 1e-6)
        np.testing.assert_allclose(got, c / math.sqrt(c * c + 1e-6) * g, rtol=1e-15)
    # library routine: torch.nn.functional.rms_norm (fp64)
    rng = np.random.default_rng(1)
    x, g = rng.standard_normal((5, 64)), rng.standard_normal(64)
    ref = F.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(g), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(x, g, 1e-6), ref, rtol=1e-12, atol=1e-14)


def pin_rope(O):
    d, theta = 8, 1e6
    rng = np.random.default_rng(2)
    x = rng.standard_normal(d)
    # position 0 is the identity
    np.testing.assert_array_equal(O.apply_rope(x, 0, theta), x)
    # unit vector e_0 at pos 1: pair 0 turns by exactly 1 radian, into slot d/2
    e0 = np.zeros(d)
    e0[0] = 1.0
    want = np.zeros(d)
    want[0], want[d // 2] = math.cos(1.0), math.sin(1.0)
    np.testing.assert_allclose(O.apply_rope(e0, 1, theta), want, atol=1e-15)
    # pair i = d/4 turns by pos * theta**(-1/2): at theta 1e6, pos 1000 -> 1 rad
    e2 = np.zeros(d)
    e2[d // 4] = 1.0
    want = np.zeros(d)
    want[d // 4], want[d // 4 + d // 2] = math.cos(1.0), math.sin(1.0)
    np.testing.assert_allclose(O.apply_rope(e2, 1000, theta), want, atol=1e-12)
    # complex form: z_i = x_i + 1j x_{i+d/2} multiplied by exp(1j * angle_i)
    for pos in (1, 7, 513):
        z = x[: d // 2] + 1j * x[d // 2:]
        ang = torch.tensor([pos * theta ** (-2.0 * i / d) for i in range(d // 2)],
                           dtype=torch.float64)
        rot = torch.polar(torch.ones_like(ang), ang).numpy()
        zr = z * rot
        np.testing.assert_allclose(O.apply_rope(x, pos, theta),
                                   np.concatenate([zr.real, zr.imag]), atol=1e-13)
    # norm of every pair preserved; dot products depend only on m - n
    y = O.apply_rope(x, 37, theta)
    np.testing.assert_allclose(x[:4] ** 2 + x[4:] ** 2, y[:4] ** 2 + y[4:] ** 2, rtol=1e-13)
    k = rng.standard_normal(d)
    a = O.apply_rope(x, 50, theta) @ O.apply_rope(k, 20, theta)
    b = O.apply_rope(x, 30, theta) @ k
    assert abs(a - b) < 1e-12


def pin_silu_softmax(O):
    z = np.linspace(-20, 20, 101)
    np.testing.assert_allclose(O.silu(z), F.silu(torch.from_numpy(z)).numpy(), rtol=1e-13, atol=1e-300)
    assert O.silu(np.array([0.0]))[0] == 0.0
    s = np.random.default_rng(3).standard_normal((7, 33)) * 10
    p = O.softmax(s)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(p, torch.softmax(torch.from_numpy(s), -1).numpy(), rtol=1e-12)


def pin_attend(O):
    rng = np.random.default_rng(4)
    d = 16
    q, k, v = rng.standard_normal(d), rng.standard_normal((1, d)), rng.standard_normal((1, d))
    # one cached token -> its value exactly
    np.testing.assert_array_equal(O.attend(q, k, v, 0.25), v[0])
    # equal keys -> uniform weights -> mean of the values
    K = np.tile(rng.standard_normal(d), (9, 1))
    V = rng.standard_normal((9, d))
    np.testing.assert_allclose(O.attend(q, K, V, 0.25), V.mean(0), rtol=1e-13)
    # library routine: scaled_dot_product_attention (scale 1/sqrt(d))
    K, V = rng.standard_normal((40, d)), rng.standard_normal((40, d))
    ref = F.scaled_dot_product_attention(torch.from_numpy(q)[None, None, None],
                                         torch.from_numpy(K)[None, None],
                                         torch.from_numpy(V)[None, None])[0, 0, 0].numpy()
    np.testing.assert_allclose(O.attend(q, K, V, 1 / math.sqrt(d)), ref, rtol=1e-12)


def pin_top2_argmax(O):
    lg = np.array([[0.0, 3.0, 1.0, 3.0], [5.0, -1.0, 4.5, 2.0]])
    np.testing.assert_allclose(O.top2_margin(lg), [0.0, 0.5])
    # ties go to the lowest index (np.argmax semantics, used by decode_step)
    assert list(np.argmax(lg, -1)) == [1, 0]


# --------------------------------------------------------- whole decoder ---


def pin_incremental_equals_full(O):
    d = dict(synth.CONFIGS["tiny"])
    d["n_layers"] = 2
    cfg = _cfg(O, d)
    _, W = _weights(O, d, seed=5)
    ids = synth.make_ids(d["vocab"], (10,), seed=6).tolist()
    full = O.forward_full(cfg, W, ids)
    cache = O.KVCache(cfg, 1, 16)
    for t, tok in enumerate(ids):
        out = O.decode_step(cfg, W, cache, [tok], [t])
        np.testing.assert_allclose(out["logits"][0], full["logits"][t], rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(out["hidden"][:, 0], full["hidden"][:, t], rtol=1e-10, atol=1e-11)
    # the cache holds exactly the rounded K/V of the full pass
    for l in range(cfg.n_layers):
        np.testing.assert_allclose(cache.k[l][0][:, :10], full["k"][l], rtol=0, atol=1e-12)
        np.testing.assert_allclose(cache.v[l][0][:, :10], full["v"][l], rtol=0, atol=1e-12)


def pin_causality(O):
    d = dict(synth.CONFIGS["tiny"])
    cfg = _cfg(O, d)
    _, W = _weights(O, d, seed=7)
    ids = synth.make_ids(d["vocab"], (9,), seed=8).tolist()
    a = O.forward_full(cfg, W, ids)
    ids2 = ids[:5] + [(t + 17) % d["vocab"] for t in ids[5:]]
    b = O.forward_full(cfg, W, ids2)
    np.testing.assert_array_equal(a["logits"][:5], b["logits"][:5])
    assert np.abs(a["logits"][5:] - b["logits"][5:]).max() > 1e-3


def pin_batch_rows_independent(O):
    # a batch of sequences at different positions == each sequence alone
    d = dict(synth.CONFIGS["tiny"])
    cfg = _cfg(O, d)
    _, W = _weights(O, d, seed=9)
    p0 = synth.make_ids(d["vocab"], (6,), seed=10).tolist()
    p1 = synth.make_ids(d["vocab"], (3,), seed=11).tolist()
    both = O.KVCache(cfg, 2, 8)
    c0, c1 = O.KVCache(cfg, 1, 8), O.KVCache(cfg, 1, 8)
    for t in range(6):
        if t < 3:
            ob = O.decode_step(cfg, W, both, [p0[t], p1[t]], [t, t])
            o1 = O.decode_step(cfg, W, c1, [p1[t]], [t])
            np.testing.assert_allclose(ob["logits"][1], o1["logits"][0], rtol=1e-12, atol=1e-12)
        else:
            ob = O.decode_step(cfg, W, both, [p0[t], p1[2]], [t, 2])
        o0 = O.decode_step(cfg, W, c0, [p0[t]], [t])
        np.testing.assert_allclose(ob["logits"][0], o0["logits"][0], rtol=1e-12, atol=1e-12)


def pin_gqa_head_mapping(O):
    # one cached token per sequence: query head h must return v of KV head h // G
    d = dict(MICRO, n_layers=1, n_q_heads=6, n_kv_heads=2)
    cfg = _cfg(O, d)
    _, W = _weights(O, d, seed=12)
    cache = O.KVCache(cfg, 1, 4)
    out = O.decode_step(cfg, W, cache, [3], [0])
    vnew = out["v_new"][0, 0]                      # [Hkv, d]
    w = W.layer(0)
    h0 = W.embed_rows([3])
    # recover o from the layer: o = solve(Wo, delta) is not unique; instead
    # rebuild o directly from the rule and check the residual update matches
    o = np.concatenate([vnew[h // cfg.group] for h in range(cfg.n_q_heads)])
    h1 = h0 + o @ w["wo"].T
    x = O.rms_norm(h1, w["mlp_norm"], cfg.rms_eps)
    h2 = h1 + (O.silu(x @ w["w_gate"].T) * (x @ w["w_up"].T)) @ w["w_down"].T
    np.testing.assert_allclose(out["hidden"][0], h2, rtol=1e-12, atol=1e-12)


def pin_mha_equals_expanded_gqa(O):
    # GQA with G query heads per KV head == MHA with each KV head repeated G times
    d = dict(MICRO, n_layers=1, n_q_heads=4, n_kv_heads=2)
    cfg_g = _cfg(O, d)
    wg, Wg = _weights(O, d, seed=13)
    dm = dict(d, n_kv_heads=4)
    wm = {k: v for k, v in wg.items() if k != "layers"}
    lw = dict(wg["layers"][0])
    hd = d["head_dim"]
    lw["wk"] = wg["layers"][0]["wk"].reshape(2, hd, -1).repeat_interleave(2, 0).reshape(4 * hd, -1)
    lw["wv"] = wg["layers"][0]["wv"].reshape(2, hd, -1).repeat_interleave(2, 0).reshape(4 * hd, -1)
    wm["layers"] = [lw]
    cfg_m = _cfg(O, dm)
    ids = [1, 5, 9, 2]
    a = O.forward_full(cfg_g, Wg, ids)
    b = O.forward_full(cfg_m, O.Weights(wm), ids)
    np.testing.assert_allclose(a["logits"], b["logits"], rtol=1e-12, atol=1e-12)


# ------------------------------------------- brute-force scalar decoder ----


def _bf_decoder(w, d, tokens):
    """Scalar-loop decoder (lists and math only) on a micro model."""
    H, Hq, Hkv, hd, Fd, V = (d["hidden"], d["n_q_heads"], d["n_kv_heads"],
                             d["head_dim"], d["ffn"], d["vocab"])
    eps, theta, G = d["rms_eps"], d["rope_theta"], Hq // Hkv
    tl = lambda t: t.to(torch.float64).tolist()  # noqa: E731
    E, LM, FN = tl(w["embed"]), tl(w["lm_head"]), tl(w["final_norm"])
    layers = [{k: tl(v) for k, v in lw.items()} for lw in w["layers"]]

    def rms(vec, g):
        s = 0.0
        for a in vec:
            s += a * a
        r = 1.0 / math.sqrt(s / len(vec) + eps)
        return [vec[i] * r * g[i] for i in range(len(vec))]

    def mv(M, vec):
        out = []
        for row in M:
            acc = 0.0
            for j in range(len(vec)):
                acc += row[j] * vec[j]
            out.append(acc)
        return out

    def rope(vec, pos):
        half = len(vec) // 2
        out = list(vec)
        for i in range(half):
            ang = pos / (theta ** (2.0 * i / len(vec)))
            c, s = math.cos(ang), math.sin(ang)
            out[i] = vec[i] * c - vec[i + half] * s
            out[i + half] = vec[i + half] * c + vec[i] * s
        return out

    def bf16(a):
        if a == 0.0:
            return 0.0
        m, e = math.frexp(a)
        return math.ldexp(round(m * 256.0) / 256.0, e)   # round(): half to even

    cache = [[[[], []] for _ in range(Hkv)] for _ in layers]
    all_logits = []
    for pos, tok in enumerate(tokens):
        h = list(E[tok])
        for li, lw in enumerate(layers):
            x = rms(h, lw["attn_norm"])
            q, k, v = mv(lw["wq"], x), mv(lw["wk"], x), mv(lw["wv"], x)
            for kvh in range(Hkv):
                kk = k[kvh * hd:(kvh + 1) * hd]
                kk = rope(rms(kk, lw["k_norm"]), pos)
                cache[li][kvh][0].append([bf16(a) for a in kk])
                cache[li][kvh][1].append([bf16(a) for a in v[kvh * hd:(kvh + 1) * hd]])
            o = []
            for qh in range(Hq):
                qq = rope(rms(q[qh * hd:(qh + 1) * hd], lw["q_norm"]), pos)
                Ks, Vs = cache[li][qh // G]
                sc = [sum(qq[i] * kt[i] for i in range(hd)) / math.sqrt(hd) for kt in Ks]
                m = max(sc)
                ex = [math.exp(s - m) for s in sc]
                z = sum(ex)
                for i in range(hd):
                    o.append(sum(ex[t] / z * Vs[t][i] for t in range(len(Ks))))
            ao = mv(lw["wo"], o)
            h = [h[i] + ao[i] for i in range(H)]
            x = rms(h, lw["mlp_norm"])
            gt, up = mv(lw["w_gate"], x), mv(lw["w_up"], x)
            u = [gt[i] / (1.0 + math.exp(-gt[i])) * up[i] for i in range(Fd)]
            dn = mv(lw["w_down"], u)
            h = [h[i] + dn[i] for i in range(H)]
        all_logits.append(mv(LM, rms(h, FN)))
    return np.array(all_logits)


def pin_brute_force_micro(O):
    d = dict(MICRO)
    cfg = _cfg(O, d)
    w, W = _weights(O, d, seed=14)
    ids = [3, 11, 0, 15, 7, 7]
    ref = _bf_decoder(w, d, ids)
    full = O.forward_full(cfg, W, ids)
    np.testing.assert_allclose(full["logits"], ref, rtol=1e-10, atol=1e-12)
    cache = O.KVCache(cfg, 1, 8)
    for t, tok in enumerate(ids):
        out = O.decode_step(cfg, W, cache, [tok], [t])
        np.testing.assert_allclose(out["logits"][0], ref[t], rtol=1e-10, atol=1e-12)


def pin_greedy_decode_hand_loop(O):
    """greedy_decode against two things it must equal on tiny inputs:
    a hand-written loop over decode_step (teacher-forced prompt at positions
    0..n-1, first token = argmax after the last prompt token, token s-1 fed
    at position n+s-1), and the brute-force scalar decoder run over the
    prompt followed by the generated tokens (its logits at positions
    n-1 .. n+steps-2 are the greedy steps' logits)."""
    for base, seed in ((MICRO, 31), (synth.CONFIGS["tiny"], 32)):
        d = dict(base)
        cfg = _cfg(O, d)
        w, W = _weights(O, d, seed=seed)
        n, steps = 5, 4
        prompts = [synth.make_ids(d["vocab"], (n,), seed=seed + 1).tolist(),
                   synth.make_ids(d["vocab"], (n,), seed=seed + 2).tolist()]
        got = O.greedy_decode(cfg, W, prompts, steps)
        assert got["logits"].shape == (steps, 2, d["vocab"])
        # hand loop, one sequence at a time
        for b, prompt in enumerate(prompts):
            cache = O.KVCache(cfg, 1, n + steps)
            for t in range(n):
                out = O.decode_step(cfg, W, cache, [prompt[t]], [t])
            toks, logits = [], []
            for s in range(steps):
                logits.append(out["logits"][0])
                tok = int(np.argmax(out["logits"][0]))
                toks.append(tok)
                if s + 1 < steps:
                    out = O.decode_step(cfg, W, cache, [tok], [n + s])
            np.testing.assert_allclose(got["logits"][:, b], np.stack(logits), rtol=1e-10,
                                       atol=1e-11)
            assert got["tokens"][:, b].tolist() == toks
            np.testing.assert_allclose(got["margins"][:, b],
                                       [np.sort(x)[-1] - np.sort(x)[-2] for x in logits],
                                       rtol=0, atol=1e-12)
            if base is MICRO:
                # scalar-loop decoder over prompt + generated tokens
                ref = _bf_decoder(w, d, prompt + toks[:-1])
                np.testing.assert_allclose(got["logits"][:, b], ref[n - 1:], rtol=1e-10,
                                           atol=1e-12)
        # forced tokens replace the fed ones
        force = np.array([[1, 2], [3, 4], [5, 6]])
        fz = O.greedy_decode(cfg, W, prompts, steps, force=force)
        np.testing.assert_allclose(fz["logits"][0], got["logits"][0], rtol=0, atol=0)
        if base is MICRO:
            for b, prompt in enumerate(prompts):
                ref = _bf_decoder(w, d, prompt + force[:, b].tolist())
                np.testing.assert_allclose(fz["logits"][:, b], ref[n - 1:], rtol=1e-10,
                                           atol=1e-12)


def pin_prefill_equals_incremental(O):
    """prefill (whole-sequence pass installed into a cache) against feeding
    the prompt one decode step at a time: the same bf16 K/V at every cached
    position, the same last-position logits, and a later decode step from
    either cache gives the same result.  Two prompts of different lengths."""
    d = dict(synth.CONFIGS["tiny"])
    cfg = _cfg(O, d)
    _, W = _weights(O, d, seed=33)
    prompts = [synth.make_ids(d["vocab"], (7,), seed=34).tolist(),
               synth.make_ids(d["vocab"], (4,), seed=35).tolist()]
    cap = 12
    cache, last, outs = O.prefill(cfg, W, prompts, cap)
    assert last.shape == (2, d["vocab"]) and len(outs) == 2
    for b, prompt in enumerate(prompts):
        inc = O.KVCache(cfg, 1, cap)
        for t, tok in enumerate(prompt):
            out = O.decode_step(cfg, W, inc, [tok], [t])
        n = len(prompt)
        assert cache.length[b] == n
        np.testing.assert_allclose(last[b], out["logits"][0], rtol=1e-10, atol=1e-11)
        for l in range(cfg.n_layers):
            np.testing.assert_allclose(cache.k[l][b][:, :n], inc.k[l][0][:, :n], rtol=0, atol=1e-12)
            np.testing.assert_allclose(cache.v[l][b][:, :n], inc.v[l][0][:, :n], rtol=0, atol=1e-12)
            # nothing beyond the prompt is written
            assert not np.any(cache.k[l][b][:, n:]) and not np.any(cache.v[l][b][:, n:])
        nxt_a = O.decode_step(cfg, W, inc, [9], [n])
        one = O.KVCache(cfg, 1, cap)
        for l in range(cfg.n_layers):
            one.load_history(l, 0, cache.k[l][b][:, :n], cache.v[l][b][:, :n])
        nxt_b = O.decode_step(cfg, W, one, [9], [n])
        np.testing.assert_allclose(nxt_a["logits"], nxt_b["logits"], rtol=1e-10, atol=1e-11)


def pin_dequantize_w4(O):
    """4-bit weights: hand-worked codes and scales, the bf16 rounding of an
    inexact product, the group boundary at column 128, and torch's own
    float32 product and bf16 conversion (exact product, one rounding)."""
    codes = np.full((2, 256), 8, dtype=np.uint8)
    codes[0, :16] = np.arange(16)
    scales = np.array([[0.5, 2.0], [1.0078125, 0.25]])
    codes[1, 0] = 15            # 1.0078125 * 7 = 7.0546875 -> bf16 7.0625 (ties/nearest)
    codes[1, 127] = 0           # last column of group 0: scale 1.0078125
    codes[1, 128] = 0           # first column of group 1: scale 0.25
    got = O.dequantize_w4(codes, scales)
    np.testing.assert_array_equal(got[0, :16], 0.5 * (np.arange(16) - 8))
    assert got[0, 16] == 0.0 and got[0, 130] == 0.0
    assert got[1, 0] == 7.0625
    assert got[1, 127] == -8.0625         # 1.0078125 * -8 = -8.0625, exact in bf16
    assert got[1, 128] == -2.0
    # library: torch float32 product (exact: 8 + 4 significant bits) rounded to bf16
    rng = np.random.default_rng(17)
    c = torch.from_numpy(rng.integers(0, 16, (8, 384)).astype(np.uint8))
    sc = (0.003 + 0.003 * torch.rand(8, 3, generator=torch.Generator().manual_seed(5))).to(
        torch.bfloat16)
    ref = (sc.float().repeat_interleave(128, dim=1) * (c.float() - 8)).to(torch.bfloat16)
    np.testing.assert_array_equal(O.dequantize_w4(c, sc), ref.double().numpy())


def pin_w4_decoder_is_the_dequantized_decoder(O):
    """A 4-bit decoder computes what the bf16 decoder computes on its
    dequantized (torch-built) matrices."""
    d = dict(MICRO, hidden=128, ffn=256, n_q_heads=4, n_kv_heads=2, head_dim=32)
    cfg = _cfg(O, d)
    w4 = synth.make_w4_weights(d, seed=41, gain="random")
    wb = {k: v for k, v in w4.items() if k != "layers"}
    wb["layers"] = []
    for lw in w4["layers"]:
        e = {k: v for k, v in lw.items() if k != "w4"}
        for name, (c, sc) in lw["w4"].items():
            e[name] = (sc.float().repeat_interleave(128, dim=1) * (c.float() - 8)).to(torch.bfloat16)
        wb["layers"].append(e)
    ids = [1, 7, 3, 12]
    a = O.forward_full(cfg, O.W4Weights(w4), ids)["logits"]
    b = O.forward_full(cfg, O.Weights(wb), ids)["logits"]
    np.testing.assert_array_equal(a, b)


# ------------------------------------------ torch library composition ------


def torch_decoder(w, d, ids):
    """The tiny decoder written with torch.nn.functional ops (fp64, CPU).

    RoPE is complex multiplication; attention is scaled_dot_product_attention
    with is_causal and enable_gqa; K/V are rounded by torch's bf16 conversion.
    """
    f = lambda t: t.to(torch.float64)  # noqa: E731
    H, Hq, Hkv, hd = d["hidden"], d["n_q_heads"], d["n_kv_heads"], d["head_dim"]
    eps, theta = d["rms_eps"], d["rope_theta"]
    T = len(ids)
    idx = torch.tensor(ids)
    h = F.embedding(idx, f(w["embed"]))
    i = torch.arange(hd // 2, dtype=torch.float64)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * theta ** (-2.0 * i / hd)
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]      # [T, 1, hd/2]

    def rope(x):                                                   # x [T, nh, hd]
        z = torch.complex(x[..., : hd // 2], x[..., hd // 2:]) * rot
        return torch.cat([z.real, z.imag], -1)

    kv_rounded = []
    for lw in w["layers"]:
        x = F.rms_norm(h, (H,), f(lw["attn_norm"]), eps)
        q = F.linear(x, f(lw["wq"])).view(T, Hq, hd)
        k = F.linear(x, f(lw["wk"])).view(T, Hkv, hd)
        v = F.linear(x, f(lw["wv"])).view(T, Hkv, hd)
        q = rope(F.rms_norm(q, (hd,), f(lw["q_norm"]), eps))
        k = rope(F.rms_norm(k, (hd,), f(lw["k_norm"]), eps))
        kr = k.to(torch.bfloat16).to(torch.float64)
        vr = v.to(torch.bfloat16).to(torch.float64)
        kv_rounded.append((k, kr, v, vr))
        o = F.scaled_dot_product_attention(q.transpose(0, 1)[None], kr.transpose(0, 1)[None],
                                           vr.transpose(0, 1)[None], is_causal=True,
                                           enable_gqa=True)[0].transpose(0, 1).reshape(T, Hq * hd)
        h = h + F.linear(o, f(lw["wo"]))
        x = F.rms_norm(h, (H,), f(lw["mlp_norm"]), eps)
        h = h + F.linear(F.silu(F.linear(x, f(lw["w_gate"]))) * F.linear(x, f(lw["w_up"])),
                         f(lw["w_down"]))
    logits = F.linear(F.rms_norm(h, (H,), f(w["final_norm"]), eps), f(w["lm_head"]))
    return logits.numpy(), kv_rounded


def pin_torch_composition_tiny(O):
    d = dict(synth.CONFIGS["tiny"])
    cfg = _cfg(O, d)
    w, W = _weights(O, d, seed=15)
    ids = synth.make_ids(d["vocab"], (8,), seed=16).tolist()
    ref, kv = torch_decoder(w, d, ids)
    # precondition: torch's conversion (via fp32) and a single rounding agree
    # on this data, so both sides attend over the same bf16 K/V
    for k, kr, v, vr in kv:
        assert np.array_equal(O.round_bf16(k.numpy()), kr.numpy())
        assert np.array_equal(O.round_bf16(v.numpy()), vr.numpy())
    got = O.forward_full(cfg, W, ids)["logits"]
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-10)


ALL_PINS = [
    pin_round_bf16, pin_rms_norm, pin_rope, pin_silu_softmax, pin_attend, pin_top2_argmax,
    pin_incremental_equals_full, pin_causality, pin_batch_rows_independent,
    pin_gqa_head_mapping, pin_mha_equals_expanded_gqa, pin_brute_force_micro,
    pin_torch_composition_tiny, pin_greedy_decode_hand_loop, pin_prefill_equals_incremental,
    pin_dequantize_w4, pin_w4_decoder_is_the_dequantized_decoder,
]


def failing_pins(O):
    """Names of the pins that fail for oracle module ``O``."""
    bad = []
    for p in ALL_PINS:
        try:
            p(O)
        except Exception:
            bad.append(p.__name__)
    return bad
