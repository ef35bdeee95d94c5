"""CPU tests: the oracle against its pins, and planted mistakes against the pins.

The mutation test copies ``oracle/decoder.py``, plants one plausible mistake
(a dropped term, a wrong sign or index, a transposed operand, an off-by-one)
and checks that at least one pin fails.  Mistakes are planted only in the
oracle's source text, on the CPU.
"""

import importlib.util
import os
import sys
import types

import pytest

import oracle.decoder as O
from tests import oracle_pins as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(O)


MUTATIONS = {
    "rope_sign": ("a * c - b * s, b * c + a * s", "a * c + b * s, b * c - a * s"),
    "rope_freq": ("-2.0 * i / d", "-1.0 * i / d"),
    "gqa_index": ("g = hq // G", "g = hq % G"),
    "attn_scale": ("scale = 1.0 / math.sqrt(d)", "scale = 1.0 / d"),
    "rms_eps": ("np.sqrt(ms + eps)", "(np.sqrt(ms) + eps)"),
    "dropped_attn_residual": ('h = h + o @ w["wo"].T', 'h = o @ w["wo"].T'),
    "dropped_mlp_residual": ('h = h + u @ w["w_down"].T', 'h = u @ w["w_down"].T'),
    "transposed_wq": ('q = x @ w["wq"].T', 'q = x @ w["wq"]'),
    "gate_up_swapped": ('silu(x @ w["w_gate"].T) * (x @ w["w_up"].T)',
                        'silu(x @ w["w_up"].T) * (x @ w["w_gate"].T)'),
    "no_final_norm": ("x = rms_norm(h, W.final_norm(), cfg.rms_eps)", "x = h"),
    "decode_excludes_current": ("[:, : p + 1, :]", "[:, : max(p, 1), :]"),
    "causal_off_by_one": ("k=1)", "k=2)"),
    "bf16_truncates": ("np.round(m * 256.0)", "np.trunc(m * 256.0)"),
    "qk_norm_dropped": ("if cfg.qk_norm:", "if False:"),
    "silu_sign": ("z / (1.0 + np.exp(-z))", "z / (1.0 + np.exp(z))"),
    "softmax_no_norm": ("e / np.sum(e, axis=-1, keepdims=True)", "e"),
    "greedy_position_off_by_one": ("[n + s - 1] * len(prompts)", "[n + s] * len(prompts)"),
    "greedy_first_token_wrong_row": ('last.append(out["logits"][-1])',
                                     'last.append(out["logits"][-2])'),
    "w4_zero_point": ("(q - W4_ZERO)", "(q - W4_ZERO + 1)"),
    "w4_no_rounding": ("return round_bf16(np.repeat(s, W4_GROUP, axis=1) * (q - W4_ZERO))",
                       "return np.repeat(s, W4_GROUP, axis=1) * (q - W4_ZERO)"),
    "w4_scale_groups_transposed": ("np.repeat(s, W4_GROUP, axis=1)",
                                   "np.tile(s, (1, W4_GROUP))"),
    "prefill_drops_last_position": ("cache.load_history(l, b, out[\"k\"][l], out[\"v\"][l])",
                                    "cache.load_history(l, b, out[\"k\"][l][:, :-1], "
                                    "out[\"v\"][l][:, :-1])"),
}


def _mutant(name):
    src = open(os.path.join(ROOT, "oracle", "decoder.py")).read()
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    src = src.replace(old, new)
    mod = types.ModuleType(f"oracle_mutant_{name}")
    mod.__file__ = f"<mutant {name}>"
    sys.modules[mod.__name__] = mod
    exec(compile(src, mod.__file__, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    bad = P.failing_pins(_mutant(name))
    assert bad, f"planted mistake '{name}' passed every pin"
