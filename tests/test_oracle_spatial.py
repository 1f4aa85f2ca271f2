"""Pins for the oracle's spatial-similarity score (explainer §三: a score per
(t, l, h), a head is spatially repeated when it exceeds gamma = 0.87; §二
observation 4: the pixel rows of a frame attend alike).

The pages give no formula for s; the oracle reads it as the mean, over frames
and non-anchor pixel rows, of the cosine similarity between a pixel row's
block-energy profile and its nearest anchor row's. These tests pin that
statement to facts that do not repeat its code:
  - every profile sums to one (each query's softmax row does);
  - when B is a multiple of W, the mean of the profiles of a query block's
    pixel rows is that block's row of the (separately written) block energy;
  - queries that do not depend on the pixel row give s = 1, and so do
    uniform scores and a head whose every row is an anchor;
  - hand-computed scores of small profile tables, one of which fails if ties
    between two anchors went to the upper one or if anchor rows were counted.
"""
import math

import numpy as np
import pytest
import torch

from calibrated_block_sparse_b200 import synth


def _bits(t):
    return synth.bf16_bits(t)


def test_profiles_sum_to_one(oracle):
    F, H, W = 2, 5, 12  # n = 120, B = 32: key blocks of 32, 32, 32 and a ragged 24
    q, k, _ = synth.plain_qkv(2, F * H * W, seed=21, std=2.0)
    E = oracle.pixel_row_energy(_bits(q), _bits(k), F, H, W, B=32)
    assert E.shape == (2, F * H, 4)
    assert np.all(E >= 0)
    np.testing.assert_allclose(E.sum(-1), 1.0, rtol=0, atol=1e-12)


def test_profiles_average_to_the_block_energy(oracle):
    # W = 16 divides B = 128: query block r is pixel rows 8r .. 8r+7, and
    # (1/128) sum over the block = mean over its 8 rows of (1/16) sum over a row
    F, H, W, B = 2, 8, 16, 128
    q, k, _ = synth.plain_qkv(2, F * H * W, seed=22, std=1.5)
    Epx = oracle.pixel_row_energy(_bits(q), _bits(k), F, H, W, B=B)
    Eblk = oracle.block_energy(_bits(q), _bits(k), B=B)
    per = B // W
    for h in range(2):
        for r in range(Eblk.shape[1]):
            np.testing.assert_allclose(Epx[h, r * per:(r + 1) * per].mean(0), Eblk[h, r], rtol=0, atol=1e-13)


def test_row_independent_queries_score_one(oracle):
    # q_(f, r, c) depends on (f, c) only: every pixel row of a frame has the
    # same softmax rows, so every profile equals its anchor's
    F, H, W = 2, 7, 10
    base, k, _ = synth.plain_qkv(1, F * W, seed=23, std=2.0)
    q = base.view(1, F, 1, W, -1).expand(1, F, H, W, base.shape[-1]).reshape(1, F * H * W, -1).contiguous()
    k = torch.randn(1, F * H * W, base.shape[-1], generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    Epx = oracle.pixel_row_energy(_bits(q), _bits(k), F, H, W, B=32)
    assert oracle.spatial_score(Epx[0], F, H, k_anchor=3) == pytest.approx(1.0, abs=1e-12)


def test_uniform_scores_give_block_sizes(oracle):
    F, H, W = 1, 6, 20  # n = 120, B = 64: key blocks of 64 and 56
    _, k, _ = synth.plain_qkv(1, F * H * W, seed=24)
    q = torch.zeros_like(k)
    Epx = oracle.pixel_row_energy(_bits(q), _bits(k), F, H, W, B=64)
    np.testing.assert_allclose(Epx[0], np.tile([64 / 120, 56 / 120], (F * H, 1)), rtol=0, atol=1e-13)
    assert oracle.spatial_score(Epx[0], F, H, k_anchor=2) == pytest.approx(1.0, abs=1e-12)


def test_hand_computed_score():
    import oracle
    # H = 3, k = 1: the anchor is row 1; rows 0 and 2 copy it.
    # cos([0,1],[1,0]) = 0, cos([1,1],[1,0]) = 1/sqrt(2): s = 1/(2 sqrt(2))
    E = np.array([[0.0, 1.0], [1.0, 0.0], [1.0, 1.0]])
    assert oracle.spatial_score(E, 1, 3, k_anchor=1) == pytest.approx(0.5 / math.sqrt(2.0), abs=1e-15)


def test_hand_computed_score_tie_and_anchor_rows():
    import oracle
    # H = 5, k = 2: anchors 1 and 3; row 2 is equally near both and copies
    # the lower one (row 1). Non-anchor rows 0, 2, 4 compare with 1, 1, 3.
    e0, e1, e2 = [1.0, 0.0, 0.0], [0.0, 1.0, 0.0], [0.0, 0.0, 1.0]
    E = np.array([e0, e0, e2, e2, e2])
    # row 0 vs 1: 1; row 2 vs 1: 0 (it would be 1 against row 3); row 4 vs 3: 1
    assert oracle.spatial_score(E, 1, 5, k_anchor=2) == pytest.approx(2.0 / 3.0, abs=1e-15)
    # two frames: the second frame's rows only meet the second frame's anchors
    E2 = np.concatenate([E, np.array([e1, e0, e1, e1, e1])])
    # frame 2: row 0 vs 1: 0; row 2 vs 1: 0; row 4 vs 3: 1  -> (2 + 1) / 6
    assert oracle.spatial_score(E2, 2, 5, k_anchor=2) == pytest.approx(0.5, abs=1e-15)


def test_every_row_an_anchor_scores_one():
    import oracle
    E = np.eye(4)
    assert oracle.spatial_score(E, 1, 4, k_anchor=4) == 1.0


def test_repeat_flag_is_strict():
    import oracle
    assert oracle.repeat_flag(0.87) is False
    assert oracle.repeat_flag(np.nextafter(0.87, 1.0)) is True
    assert oracle.repeat_flag(0.5, gamma=0.4) is True
