"""Pins for the oracle's masked and repeated-head attention.

Each check is fixed by the mathematics of the method rather than by the
oracle's own formula: the all-ones mask must equal dense attention (an
invariant the method fixes), zero queries give a uniform average (closed form),
a hand-computable two-key case, and the anchor-row construction reduces to
plain attention when every row is an anchor.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from calibrated_block_sparse_b200 import synth


def _bits(t):
    return synth.bf16_bits(t)


def _f64(bits):
    return bits.astype(np.uint32).__lshift__(16).view(np.float32).astype(np.float64)


def _dense_numpy(q, k, v, scale):
    """Dense softmax(scale Q K^T) V by matrix ops (an independent route)."""
    qd, kd, vd = _f64(q), _f64(k), _f64(v)
    s = scale * np.einsum("hid,hjd->hij", qd, kd)
    m = s.max(-1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(-1, keepdims=True)
    return np.einsum("hij,hjd->hid", p / l, vd), (m + np.log(l))[..., 0]


def test_all_ones_mask_equals_dense(oracle):
    # ragged: n = 300 with B = 128 -> 3 blocks, last block 44 rows
    q, k, v = synth.plain_qkv(2, 300, seed=1)
    q, k, v = _bits(q), _bits(k), _bits(v)
    nb = 3
    o, lse = oracle.masked_attention(q, k, v, np.ones((2, nb, nb), np.uint8), B=128)
    o_ref, lse_ref = _dense_numpy(q, k, v, 1 / math.sqrt(128))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_zero_queries_average_kept_values(oracle):
    # q = 0: every kept key gets the same weight -> O_i = mean of kept v_j,
    # LSE_i = ln(number of kept keys). Asymmetric mask catches a transposed index.
    n, B = 200, 32
    nb = (n + B - 1) // B
    _, k, v = synth.plain_qkv(1, n, seed=2, d=16)
    q = torch.zeros_like(k)
    mask = synth.random_mask(1, nb, 0.4, seed=3)
    mask[0, 0, :] = 0
    mask[0, 0, nb - 1] = 1  # row 0 keeps only the ragged last block
    o, lse = oracle.masked_attention(_bits(q), _bits(k), _bits(v), mask, B=B)
    vd = _f64(_bits(v))[0]
    for i in range(n):
        r = i // B
        keys = [j for j in range(n) if mask[0, r, j // B]]
        np.testing.assert_allclose(o[0, i], vd[keys].mean(0), atol=1e-13)
        assert abs(lse[0, i] - math.log(len(keys))) < 1e-13


def test_two_key_hand_case(oracle):
    # B = 1, n = 2, d = 1, q = 1, k = (2, 0), v = (1, -1), scale = 0.5:
    # s = (1, 0) -> p = (e, 1)/(e + 1), O = (e - 1)/(e + 1) = tanh(1/2)
    bf = lambda a: _bits(torch.tensor(a, dtype=torch.float32).reshape(1, -1, 1).to(torch.bfloat16))
    o, lse = oracle.masked_attention(bf([1.0, 1.0]), bf([2.0, 0.0]), bf([1.0, -1.0]),
                                     np.ones((1, 2, 2), np.uint8), B=1, scale=0.5)
    assert abs(o[0, 0, 0] - math.tanh(0.5)) < 1e-15
    assert abs(lse[0, 0] - math.log(math.e + 1)) < 1e-15
    # keep only key block 1 for row 1: the single kept value is returned exactly
    mask = np.array([[[1, 1], [0, 1]]], np.uint8)
    o, lse = oracle.masked_attention(bf([1.0, 1.0]), bf([2.0, 0.0]), bf([1.0, -1.0]), mask, B=1, scale=0.5)
    assert o[0, 1, 0] == -1.0 and lse[0, 1] == 0.0


def test_single_block_equals_dense_over_that_block(oracle):
    n, B = 256, 64
    q, k, v = synth.plain_qkv(1, n, seed=4, d=32)
    q, k, v = _bits(q), _bits(k), _bits(v)
    nb = n // B
    mask = np.zeros((1, nb, nb), np.uint8)
    for r in range(nb):
        mask[0, r, (3 * r + 1) % nb] = 1
    o, lse = oracle.masked_attention(q, k, v, mask, B=B)
    for r in range(nb):
        c = (3 * r + 1) % nb
        sl = slice(c * B, (c + 1) * B)
        rows = slice(r * B, (r + 1) * B)
        o_ref, lse_ref = _dense_numpy(q[:, rows], k[:, sl], v[:, sl], 1 / math.sqrt(32))
        np.testing.assert_allclose(o[0, rows], o_ref[0], atol=1e-12)
        np.testing.assert_allclose(lse[0, rows], lse_ref[0], atol=1e-12)


def test_empty_row_is_zero_and_minus_inf(oracle):
    q, k, v = synth.plain_qkv(1, 64, seed=5, d=8)
    mask = np.ones((1, 2, 2), np.uint8)
    mask[0, 1] = 0
    o, lse = oracle.masked_attention(_bits(q), _bits(k), _bits(v), mask, B=32)
    assert np.all(o[0, 32:] == 0) and np.all(np.isneginf(lse[0, 32:]))
    assert np.all(np.isfinite(lse[0, :32]))


def test_sampled_rows_match_full(oracle):
    q, k, v = synth.plain_qkv(2, 130, seed=6, d=16)
    mask = synth.random_mask(2, 2, 0.5, seed=7)
    o, lse = oracle.masked_attention(_bits(q), _bits(k), _bits(v), mask, B=128)
    rows = np.array([0, 5, 129, 130, 259], np.int64)
    os_, ls_ = oracle.masked_attention(_bits(q), _bits(k), _bits(v), mask, B=128, rows=rows)
    np.testing.assert_array_equal(os_, o.reshape(-1, 16)[rows])
    np.testing.assert_array_equal(ls_, lse.reshape(-1)[rows])


def test_anchor_rows_closed_form(oracle):
    # centres of k equal bands: floor((2j+1) H / (2k))
    assert list(oracle.anchor_rows(45, 5)) == [4, 13, 22, 31, 40]
    assert list(oracle.anchor_rows(30, 5)) == [3, 9, 15, 21, 27]
    assert list(oracle.anchor_rows(8, 5)) == [0, 2, 4, 5, 7]
    assert list(oracle.anchor_rows(7, 7)) == list(range(7))
    assert list(oracle.anchor_rows(9, 1)) == [4]


@pytest.mark.parametrize("H,kk", [(45, 5), (30, 5), (8, 5), (7, 3), (10, 10), (5, 1)])
def test_nearest_anchor_is_brute_force_argmin(oracle, H, kk):
    a = oracle.anchor_rows(H, kk)
    owner = oracle.nearest_anchor(H, kk)
    for r in range(H):
        d = [abs(r - int(x)) for x in a]
        assert owner[r] == d.index(min(d))  # first minimum = lower j on ties
    # bands are contiguous and every anchor owns itself
    assert all(owner[int(a[j])] == j for j in range(kk))
    assert all(owner[r] <= owner[r + 1] for r in range(H - 1))


def test_repeat_with_k_equal_H_is_plain_attention(oracle):
    F, H, W = 2, 4, 8
    n = F * H * W
    q, k, v = synth.plain_qkv(1, n, seed=8, d=32)
    q, k, v = _bits(q), _bits(k), _bits(v)
    o, lse = oracle.repeat_attention(q, k, v, F, H, W, k_anchor=H)
    o_ref, lse_ref = _dense_numpy(q, k, v, 1 / math.sqrt(32))
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


def test_repeat_rows_copy_their_anchor(oracle):
    F, H, W, kk = 3, 8, 5, 3
    n = F * H * W
    q, k, v = synth.plain_qkv(2, n, seed=9, d=16)
    q, k, v = _bits(q), _bits(k), _bits(v)
    o, lse = oracle.repeat_attention(q, k, v, F, H, W, k_anchor=kk)
    o_ref, lse_ref = _dense_numpy(q, k, v, 1 / math.sqrt(16))
    a = oracle.anchor_rows(H, kk)
    owner = oracle.nearest_anchor(H, kk)
    for f, r, c in itertools.product(range(F), range(H), range(W)):
        t = f * H * W + r * W + c
        src = f * H * W + int(a[owner[r]]) * W + c
        # anchor rows are plain attention rows; others are exact copies
        np.testing.assert_allclose(o[:, t], o_ref[:, src], atol=1e-12)
        np.testing.assert_array_equal(o[:, t], o[:, src])
        np.testing.assert_array_equal(lse[:, t], lse[:, src])


def test_repeat_rejects_bad_k(oracle):
    q, k, v = synth.plain_qkv(1, 16, seed=1, d=8)
    with pytest.raises(ValueError):
        oracle.repeat_attention(_bits(q), _bits(k), _bits(v), 1, 4, 4, k_anchor=5)
