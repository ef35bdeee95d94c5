"""CPU tests of the 4-bit weight packing (mk_w4_pack) and of 4-bit plans.

The packed layout is the one include/mk.h describes for MK_W4_*: per row tile
of 16 rows and 1024 columns, 8 x 16 scales (group-major) then 32 sub-blocks of
32 columns holding, for mma lane (g, q), the codes of row g and then row g + 8
at columns 8 q .. 8 q + 7, with the codes of columns 2 k and 2 k + 1 in bits
4 k and 16 + 4 k of a 32-bit word.  `unpack` below reads that description
back; a round trip must give the codes and scales exactly.
"""

import numpy as np
import pytest
import torch

from persistent_task_runtime_b200 import build, mk, synth
from tests.test_plan_layout import check_plan

BLOCK = 8448


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def unpack(buf: np.ndarray, rows: int, cols: int):
    tiles, blocks = (rows + 15) // 16, cols // 1024
    codes = np.zeros((tiles * 16, cols), dtype=np.uint8)
    scales = np.zeros((tiles * 16, cols // 128), dtype=np.uint16)
    for t in range(tiles):
        for b in range(blocks):
            blk = buf[(t * blocks + b) * BLOCK:(t * blocks + b + 1) * BLOCK]
            sc = blk[:256].view(np.uint16).reshape(8, 16)          # [group][row]
            scales[16 * t:16 * t + 16, 8 * b:8 * b + 8] = sc.T
            words = blk[256:].view(np.uint32).reshape(32, 32, 2)   # [sub][lane][half]
            for s in range(32):
                for lane in range(32):
                    g, q = lane >> 2, lane & 3
                    for h in range(2):
                        w = int(words[s, lane, h])
                        for i in range(8):
                            shift = (i & 1) * 16 + (i >> 1) * 4
                            codes[16 * t + g + 8 * h, 1024 * b + 32 * s + 8 * q + i] = (w >> shift) & 15
    return codes[:rows], scales[:rows]


@pytest.mark.parametrize("rows,cols", [(16, 1024), (40, 2048), (3, 1024)])
def test_pack_round_trip(rows, cols):
    g = torch.Generator().manual_seed(rows * 7 + cols)
    codes = torch.randint(0, 16, (rows, cols), generator=g, dtype=torch.int64).to(torch.uint8)
    scales = (torch.rand(rows, cols // 128, generator=g) + 0.5).to(torch.bfloat16)
    packed = mk.w4_pack(codes, scales).numpy()
    assert packed.size == mk.load_library().mk_w4_packed_bytes(rows, cols) == \
        ((rows + 15) // 16) * (cols // 1024) * BLOCK
    c2, s2 = unpack(packed, rows, cols)
    assert np.array_equal(c2, codes.numpy())
    assert np.array_equal(s2, scales.view(torch.int16).numpy().view(np.uint16))
    # rows past the end of the matrix: code 8 (weight 0), scale 0
    if rows % 16:
        full_c, full_s = unpack(packed, ((rows + 15) // 16) * 16, cols)
        assert (full_c[rows:] == 8).all() and (full_s[rows:] == 0).all()


def test_pack_rejects_bad_input():
    lib = mk.load_library()
    assert lib.mk_w4_packed_bytes(16, 1000) == -1
    assert lib.mk_w4_packed_bytes(0, 1024) == -1
    codes = torch.full((16, 1024), 16, dtype=torch.uint8)
    scales = torch.ones(16, 8, dtype=torch.bfloat16)
    with pytest.raises(mk.MkError):
        mk.w4_pack(codes, scales)


W4_SHAPES = {
    "8b": synth.CONFIGS["8b"],
    "mid": dict(n_layers=2, hidden=1024, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=3072,
                vocab=5000, rms_eps=1e-6, rope_theta=1e6, qk_norm=True),
}


@pytest.mark.parametrize("name,batch", [("8b", 1), ("8b", 4), ("mid", 1), ("mid", 3), ("8b", 16)])
def test_w4_plan_graph(name, batch):
    cfg = W4_SHAPES[name]
    info, t = mk.describe(cfg, max_batch=batch, max_seq_len=600, weight_bits=4)
    assert info["weight_bits"] == 4 and info["gemv_path"] == 1
    nb = info["page_bytes"] // BLOCK               # packed blocks per page: 4, or fewer at large batch
    assert info["page_bytes"] == (nb * BLOCK + 1023) // 1024 * 1024 and nb in (1, 2, 4)
    assert nb == 4 or batch > 4
    # every page of the projections is whole packed blocks; the bf16 LM head's
    # 16-row pages fit the same size
    assert all(c % 1024 == 0 and c <= 1024 * nb for c in info["page_cols"][:3])
    lm_cols = info["page_cols"][3]
    assert 16 * ((lm_cols * 2 + 127) // 128 * 128 + 64) <= info["page_bytes"]
    assert info["ffn_part_cols"] % 1024 == 0
    check_plan(cfg, info, t, batch)
    # streamed bytes: packed projections (a quarter of bf16, plus scales) and the bf16 LM head
    bf16, _ = mk.describe(cfg, max_batch=batch, max_seq_len=600, gemv_path=1)
    lm = 2 * cfg["vocab"] * cfg["hidden"]
    ratio = (info["weight_bytes"] - lm) / (bf16["weight_bytes"] - lm)
    assert 0.25 < ratio < 0.27


def test_w4_plan_rejects_unsupported():
    with pytest.raises(mk.MkError) as e:
        mk.describe(synth.CONFIGS["tiny"], weight_bits=4)        # hidden 256
    assert e.value.code == mk.MK_ERR_UNSUPPORTED
    with pytest.raises(mk.MkError):
        mk.describe(W4_SHAPES["mid"], weight_bits=4, gemv_path=2)
    with pytest.raises(mk.MkError):
        mk.describe(W4_SHAPES["mid"], weight_bits=8)
