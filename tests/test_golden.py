"""Worked numbers from the pages and hand-derived mask counts
(tests/golden/worked_numbers.txt), checked against the oracle's index builder
and the workload mask recipes."""
import os

import numpy as np

import oracle
from block_sparse_attention_bsattn_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden", "worked_numbers.txt")


def _load():
    vals = {}
    for line in open(GOLD, encoding="utf-8"):
        line = line.split("#", 1)[0].strip()
        if line:
            key, val = (x.strip() for x in line.split("="))
            vals[key] = float(val)
    return vals


G = _load()


def test_page1_block_count_and_bitmap():
    nb = int(G["page1.N"]) // int(G["page1.block"])
    assert nb == G["page1.num_blocks"]
    # bitmap storage: one bit per block
    mask = np.ones((nb, nb), np.uint8)
    assert np.packbits(mask).nbytes == G["page1.bitmap_bytes"]


def test_page1_sparsity_example():
    nb = int(G["page1.num_blocks"])
    rng = np.random.default_rng(0)
    flat = np.zeros(nb * nb, np.uint8)
    flat[rng.permutation(nb * nb)[: int(G["page1.kept_blocks"])]] = 1
    _, _, nnz = oracle.build_index(flat.reshape(1, nb, nb), 64, 64, False)
    total = nb * nb
    assert total == G["page1.total_blocks"]
    assert 1 - nnz.sum() / total == G["page1.sparsity"]


def test_workload_mask_counts():
    for name, m in (("tiny", inputs.mask_tiny()), ("mmdit", inputs.mask_mmdit()),
                    ("videodit", inputs.mask_videodit())):
        _, _, nnz = oracle.build_index(m.numpy()[None], 128, 128, False)
        assert nnz.sum() == G[f"mask.{name}.nnz"], name
        assert m.numel() == G[f"mask.{name}.total"], name


def test_causal_dense_count():
    m = np.ones((1, 256, 256), np.uint8)
    _, _, nnz = oracle.build_index(m, 128, 128, True)
    assert nnz.sum() == G["mask.causal256.nnz"]


def test_video_mask_structure():
    m = inputs.mask_videodit().numpy()
    # block 40 is frame 1, spatial 8: local 36..44, spatial 8 in all frames, text 512..515
    row = set(np.nonzero(m[40])[0].tolist())
    expect = set(range(36, 45)) | {8 + 32 * f for f in range(16)} | {512, 513, 514, 515}
    assert row == expect
    # clipped window at a frame edge: block 32 (frame 1, spatial 0)
    row = set(np.nonzero(m[32])[0].tolist())
    assert set(range(32, 37)) <= row and 31 not in row
