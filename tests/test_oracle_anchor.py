"""Pins of the oracle's anchor-row block masks (repeated heads whose anchor
queries also follow a calibrated skip list; explainer §三 makes both
decisions per (t, l, h), §六 fixes the row-major frame order).

* anchor energies: every row sums to 1; with every row an anchor (k = H) the
  packed order is the token order and the energies are block_energy's, bit for
  bit; with W = 128 each packed block is one anchor pixel row, so the energies
  are pixel_row_energy's profiles of the anchor rows; uniform scores give the
  closed form |J_c| / n;
* masked repeated head: an all-ones anchor mask is repeat_attention, bit for
  bit; with k = H it is masked_attention with the same mask; rows of one band
  and column are copies of their anchor row; an anchor block with no kept
  block gives O = 0 and LSE = -inf to every row it feeds.
"""
import numpy as np
import pytest

from calibrated_block_sparse_b200 import synth


def _rand(h, n, d=128, seed=0, std=1.0):
    q, k, v = synth.plain_qkv(h, n, seed=seed, d=d, std=std)
    return synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v)


def test_anchor_energy_rows_sum_to_one(oracle):
    F, H, W = 3, 6, 20
    q, k, _ = _rand(2, F * H * W, seed=1, std=1.5)
    E = oracle.anchor_block_energy(q, k, F, H, W, k_anchor=3)
    assert E.shape == (2, oracle.anchor_blocks(F, H, W, 3), -(-F * H * W // 128))
    assert np.all(E >= 0)
    np.testing.assert_allclose(E.sum(-1), 1.0, atol=1e-12)


def test_every_row_an_anchor_is_block_energy(oracle):
    F, H, W = 2, 5, 40
    q, k, _ = _rand(2, F * H * W, seed=2, std=2.0)
    E = oracle.anchor_block_energy(q, k, F, H, W, k_anchor=H)
    np.testing.assert_array_equal(E, oracle.block_energy(q, k))


def test_whole_pixel_row_blocks_are_pixel_row_profiles(oracle):
    F, H, W, kk = 3, 8, 128, 3
    q, k, _ = _rand(1, F * H * W, seed=3, std=1.5)
    E = oracle.anchor_block_energy(q, k, F, H, W, k_anchor=kk)[0]
    P = oracle.pixel_row_energy(q, k, F, H, W)[0]
    anchors = oracle.anchor_rows(H, kk)
    for f in range(F):
        for j in range(kk):
            np.testing.assert_allclose(E[f * kk + j], P[f * H + anchors[j]], rtol=1e-12, atol=1e-15)


def test_uniform_scores_give_block_sizes(oracle):
    F, H, W = 2, 4, 50  # n = 400: blocks 128, 128, 128, 16
    q, k, _ = _rand(1, F * H * W, seed=4)
    q[:] = 0
    E = oracle.anchor_block_energy(q, k, F, H, W, k_anchor=2)
    sizes = np.array([128, 128, 128, 16], np.float64) / 400.0
    for r in range(E.shape[1]):
        np.testing.assert_allclose(E[0, r], sizes, rtol=1e-12)


def test_all_ones_anchor_mask_is_repeat_attention(oracle):
    F, H, W, kk = 3, 9, 24, 4
    q, k, v = _rand(2, F * H * W, seed=5, std=1.5)
    nbq, nb = oracle.anchor_blocks(F, H, W, kk), -(-F * H * W // 128)
    o, lse = oracle.repeat_attention_masked(q, k, v, F, H, W, np.ones((2, nbq, nb), np.uint8), k_anchor=kk)
    o_ref, lse_ref = oracle.repeat_attention(q, k, v, F, H, W, k_anchor=kk)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(lse, lse_ref)


def test_every_row_an_anchor_is_masked_attention(oracle):
    F, H, W = 2, 6, 30
    n = F * H * W
    q, k, v = _rand(1, n, seed=6, std=2.0)
    nb = -(-n // 128)
    mask = synth.random_mask(1, nb, 0.5, seed=6)
    o, lse = oracle.repeat_attention_masked(q, k, v, F, H, W, mask, k_anchor=H)
    o_ref, lse_ref = oracle.masked_attention(q, k, v, mask)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(lse, lse_ref)


def test_bands_copy_their_anchor_and_empty_blocks_give_zero(oracle):
    F, H, W, kk = 2, 10, 16, 3
    n = F * H * W
    q, k, v = _rand(1, n, seed=7)
    nbq, nb = oracle.anchor_blocks(F, H, W, kk), -(-n // 128)
    mask = synth.random_mask(1, max(nbq, nb), 0.6, seed=7)[:, :nbq, :nb].copy()
    mask[0, 0, :] = 0  # the first anchor block keeps nothing
    o, lse = oracle.repeat_attention_masked(q, k, v, F, H, W, mask, k_anchor=kk)
    anchors = oracle.anchor_rows(H, kk)
    owner = oracle.nearest_anchor(H, kk)
    o = o[0].reshape(F, H, W, 128)
    lse = lse[0].reshape(F, H, W)
    for f in range(F):
        for r in range(H):
            a = anchors[owner[r]]
            np.testing.assert_array_equal(o[f, r], o[f, a])
            np.testing.assert_array_equal(lse[f, r], lse[f, a])
            packed = f * kk * W + owner[r] * W + np.arange(W)
            empty = packed // 128 == 0
            assert np.all(o[f, r][empty] == 0) and np.all(np.isneginf(lse[f, r][empty]))
            assert np.all(np.isfinite(lse[f, r][~empty]))


def test_sampled_rows_equal_full_evaluation(oracle):
    F, H, W, kk = 2, 7, 40, 3
    n = F * H * W
    q, k, v = _rand(2, n, seed=8)
    nbq, nb = oracle.anchor_blocks(F, H, W, kk), -(-n // 128)
    mask = synth.random_mask(2, max(nbq, nb), 0.5, seed=8)[:, :nbq, :nb].copy()
    o, lse = oracle.repeat_attention_masked(q, k, v, F, H, W, mask, k_anchor=kk)
    rows = np.array([0, n - 1, n + 5, 2 * n - 1], np.int64)
    o2, lse2 = oracle.repeat_attention_masked(q, k, v, F, H, W, mask, k_anchor=kk, rows=rows)
    np.testing.assert_array_equal(o2, o.reshape(-1, 128)[rows])
    np.testing.assert_array_equal(lse2, lse.reshape(-1)[rows])
    br = np.array([0, 2 * nbq - 1], np.int64)
    E = oracle.anchor_block_energy(q, k, F, H, W, k_anchor=kk)
    np.testing.assert_array_equal(oracle.anchor_block_energy(q, k, F, H, W, k_anchor=kk, blockrows=br),
                                  E.reshape(-1, nb)[br])


def test_k_outside_range_is_refused(oracle):
    q, k, v = _rand(1, 2 * 3 * 8, seed=9)
    with pytest.raises(ValueError):
        oracle.anchor_block_energy(q, k, 2, 3, 8, k_anchor=4)


def test_row_skip_list_equals_the_square_one(oracle):
    mask = synth.random_mask(3, 11, 0.4, seed=10)
    rp, ci = oracle.mask_rows_to_csr(mask)
    rp2, ci2 = oracle.mask_to_csr(mask)
    np.testing.assert_array_equal(rp, rp2)
    np.testing.assert_array_equal(ci, ci2)
    rect = mask[:, :7, :].copy()  # 7 rows of 11 columns per head
    rp3, ci3 = oracle.mask_rows_to_csr(rect)
    assert rp3.size == 3 * 7 + 1 and rp3[-1] == rect.sum()
    for r in range(21):
        np.testing.assert_array_equal(ci3[rp3[r]:rp3[r + 1]], np.nonzero(rect.reshape(21, 11)[r])[0])
