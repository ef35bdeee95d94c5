"""Plain, slow CPU oracle for the decode megakernel.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its CPU-baseline leg and its ``--impl reference`` arm) may import
anything here.  The product path (``persistent_task_runtime_b200``) never does,
and this package imports nothing from it: the two share no kernels, helpers,
tables or constants.  The only thing both sides consume is the seeded input
generator in ``persistent_task_runtime_b200.synth``, which holds none of the
decoder's arithmetic.

Every function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
invariants, brute force on tiny inputs and independent library routines.
"""

from .decoder import (  # noqa: F401
    DecoderConfig,
    KVCache,
    W4Weights,
    Weights,
    apply_rope,
    dequantize_w4,
    attend,
    decode_step,
    forward_full,
    greedy_decode,
    prefill,
    rms_norm,
    round_bf16,
    silu,
    softmax,
    top2_margin,
)
