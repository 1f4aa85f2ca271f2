"""Pins for the oracle's calibration steps: block energy, greedy eps
selection, rho aggregation, the skip-list (CSR) form and the eps(t) schedule.

They check the oracle against what the method fixes: every energy row sums to
one; uniform scores give |J_c| / n exactly; eps = 1 keeps every nonzero block;
brute-force minimal subsets on tiny rows agree with the greedy count; n = 1
aggregation reproduces its input; the schedule's closed-form values.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from calibrated_block_sparse_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(t):
    return synth.bf16_bits(t)


# ---------------------------------------------------------------- energy

def test_energy_rows_sum_to_one_and_nonnegative(oracle):
    # ragged: n = 300, B = 128 -> last block-row has 44 rows
    q, k, _ = synth.plain_qkv(2, 300, seed=11, std=2.0)
    E = oracle.block_energy(_bits(q), _bits(k), B=128)
    assert E.shape == (2, 3, 3)
    assert np.all(E >= 0)
    np.testing.assert_allclose(E.sum(-1), 1.0, rtol=0, atol=1e-12)


def test_energy_uniform_scores_closed_form(oracle):
    # q = 0 -> P_ij = 1/n for every j -> E[r, c] = |J_c| / n on every row
    n, B = 300, 128
    _, k, _ = synth.plain_qkv(1, n, seed=12)
    q = torch.zeros_like(k)
    E = oracle.block_energy(_bits(q), _bits(k), B=B)
    expect = np.array([128, 128, 44]) / n
    for r in range(3):
        np.testing.assert_allclose(E[0, r], expect, rtol=0, atol=1e-12)  # 16k fp64 additions


def test_energy_one_dominant_key(oracle):
    # one key aligned with every query and far larger than the rest: P -> one-hot
    n, B, d = 256, 64, 16
    q = torch.zeros(1, n, d)
    q[..., 0] = 1.0
    k = torch.zeros(1, n, d)
    k[0, 150, 0] = 200.0  # key 150 lives in block 2
    E = oracle.block_energy(_bits(q.to(torch.bfloat16)), _bits(k.to(torch.bfloat16)), B=B, scale=1.0)
    np.testing.assert_allclose(E[0][:, 2], 1.0, atol=1e-12)
    np.testing.assert_allclose(np.delete(E[0], 2, axis=1), 0.0, atol=1e-12)


def test_energy_lse_matches_attention_lse(oracle):
    q, k, v = synth.plain_qkv(1, 200, seed=13)
    E, lse = oracle.block_energy(_bits(q), _bits(k), B=128, want_lse=True)
    _, lse_att = oracle.masked_attention(_bits(q), _bits(k), _bits(v), np.ones((1, 2, 2), np.uint8), B=128)
    np.testing.assert_allclose(lse[0, 0], lse_att[0, :128], atol=1e-12)
    np.testing.assert_allclose(lse[0, 1, :72], lse_att[0, 128:], atol=1e-12)


def test_energy_sampled_blockrows_match_full(oracle):
    q, k, _ = synth.plain_qkv(2, 260, seed=14)
    E = oracle.block_energy(_bits(q), _bits(k), B=128)
    br = np.array([5, 0, 3], np.int64)
    Es = oracle.block_energy(_bits(q), _bits(k), B=128, blockrows=br)
    np.testing.assert_array_equal(Es, E.reshape(-1, 3)[br])


# ---------------------------------------------------------------- selection

def _brute_min_count(e, eps):
    """Smallest cardinality of any subset whose sum reaches eps (exhaustive)."""
    nb = len(e)
    for m in range(1, nb + 1):
        if any(sum(e[list(s)]) >= eps for s in itertools.combinations(range(nb), m)):
            return m
    return None


@pytest.mark.parametrize("seed", range(6))
def test_greedy_count_equals_brute_force_minimum(oracle, seed):
    rng = np.random.default_rng(seed)
    for trial in range(40):
        nb = int(rng.integers(1, 11))
        e = rng.dirichlet(np.full(nb, 0.5))
        eps = float(rng.uniform(0.05, 0.98))
        mask, kept = oracle.select(e[None], eps)
        m = _brute_min_count(e, eps)
        assert m is not None and kept[0] == m
        # with distinct energies the minimal set is the unique top-m set
        top = set(np.argsort(-e, kind="stable")[:m].tolist())
        assert set(np.nonzero(mask[0])[0].tolist()) == top
        assert e[mask[0] == 1].sum() >= eps


def test_eps_one_keeps_every_nonzero_block(oracle):
    rng = np.random.default_rng(21)
    E = rng.dirichlet(np.ones(12), size=50)
    E[:, ::3] = 0.0
    E /= E.sum(1, keepdims=True)
    mask, kept = oracle.select(E, 1.0)
    np.testing.assert_array_equal(mask, (E > 0).astype(np.uint8))


def test_one_hot_rows_keep_one(oracle):
    E = np.eye(7)
    mask, kept = oracle.select(E, 0.9)
    np.testing.assert_array_equal(mask, np.eye(7, dtype=np.uint8))
    assert np.all(kept == 1)


def test_equal_energies_prefer_lower_column(oracle):
    E = np.array([[0.25, 0.25, 0.25, 0.25]])
    mask, kept = oracle.select(E, 0.5)
    assert mask.tolist() == [[1, 1, 0, 0]] and kept[0] == 2
    mask, kept = oracle.select(np.array([[0.1, 0.3, 0.3, 0.3]]), 0.55)
    assert mask.tolist() == [[0, 1, 1, 0]]


def test_nonpositive_eps_keeps_the_top_block(oracle):
    mask, kept = oracle.select(np.array([[0.1, 0.6, 0.3]]), 0.0)
    assert mask.tolist() == [[0, 1, 0]] and kept[0] == 1


def test_cut_description(oracle):
    E = np.array([[0.5, 0.3, 0.2]])
    mask, kept, (before, at, e_last, e_next) = oracle.select(E, 0.7, with_cut=True)
    assert kept[0] == 2 and before[0] == 0.5 and at[0] == 0.8
    assert e_last[0] == 0.3 and e_next[0] == 0.2


# ---------------------------------------------------------------- aggregation

def test_aggregate_single_input_is_identity(oracle):
    rng = np.random.default_rng(31)
    m = (rng.random((1, 3, 9, 9)) < 0.4).astype(np.uint8)
    out, counts = oracle.aggregate(m, 0.5)
    np.testing.assert_array_equal(out, m[0])
    np.testing.assert_array_equal(counts, m[0])


def test_aggregate_counts_threshold_and_ties(oracle):
    rng = np.random.default_rng(32)
    n = 8
    m = (rng.random((n, 2, 7, 7)) < 0.5).astype(np.uint8)
    out, counts = oracle.aggregate(m, 0.5)
    np.testing.assert_array_equal(counts, m.astype(np.int32).sum(0))
    # rho = 0.5 keeps exactly the cells with 2*count >= n (ties kept)
    np.testing.assert_array_equal(out, (2 * counts >= n).astype(np.uint8))
    assert np.any(2 * counts == n)
    np.testing.assert_array_equal(oracle.binarize_counts(counts, n, 0.5), out)


def test_aggregate_monotone_in_rho(oracle):
    rng = np.random.default_rng(33)
    m = (rng.random((10, 40)) < 0.5).astype(np.uint8)
    prev = None
    for rho in np.linspace(0.0, 1.0, 11):
        out, _ = oracle.aggregate(m, float(rho))
        if prev is not None:
            assert np.all(out <= prev)
        prev = out
    assert np.all(oracle.aggregate(m, 0.0)[0] == 1)


def test_csr_round_trip(oracle):
    rng = np.random.default_rng(34)
    mask = (rng.random((3, 11, 11)) < 0.3).astype(np.uint8)
    mask[1, 4] = 0  # an empty row
    row_ptr, col_idx = oracle.mask_to_csr(mask)
    assert row_ptr[0] == 0 and row_ptr[-1] == mask.sum()
    dense = np.zeros_like(mask).reshape(-1, 11)
    for row in range(33):
        cols = col_idx[row_ptr[row]:row_ptr[row + 1]]
        assert np.all(np.diff(cols) > 0)
        dense[row, cols] = 1
    np.testing.assert_array_equal(dense.reshape(mask.shape), mask)


# ---------------------------------------------------------------- schedule

def _golden():
    vals = {}
    with open(os.path.join(GOLDEN, "paper_constants.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, value = line.split()[:2]
                vals[name] = float(value)
    return vals


def test_eps_schedule_closed_form(oracle):
    g = _golden()
    A, C = g["eps_late"], g["eps_early"]
    assert oracle.eps_schedule(A, C, 5, 0, 1000) == C
    assert abs(oracle.eps_schedule(A, C, 5, 500, 1000) - 0.852312749793585) < 1e-15
    assert abs(oracle.eps_schedule(A, C, 5, 1000, 1000) - (0.84 + 0.15 * math.exp(-5))) < 1e-15
    ts = [oracle.eps_schedule(A, C, 5, t, 50) for t in range(51)]
    assert all(a > b for a, b in zip(ts, ts[1:]))
    assert oracle.eps_schedule(A, C, 5, 1e9, 1.0) == A


# ---------------------------------------------------------------- keep-rate histogram

def test_keep_histogram_counts_every_block(oracle):
    rng = np.random.default_rng(31)
    masks = (rng.random((16, 3, 9, 9)) < 0.3).astype(np.uint8)
    _, counts = oracle.aggregate(masks, 0.5)
    hist = oracle.keep_histogram(counts, 16)
    assert hist.shape == (3, 17)
    np.testing.assert_array_equal(hist.sum(-1), 81)
    # the histogram's first moment is the total number of kept (input, block) pairs
    np.testing.assert_array_equal((hist * np.arange(17)).sum(-1), masks.sum(axis=(0, 2, 3)))


def test_keep_histogram_small_cases(oracle):
    # one input: the histogram is (#skipped, #kept) of the mask itself
    mask = np.array([[[1, 0, 0], [1, 1, 0], [0, 0, 0]]], np.uint8)
    np.testing.assert_array_equal(oracle.keep_histogram(mask, 1), [[6, 3]])
    # hand-made counts over 4 inputs
    counts = np.array([[[0, 4, 4], [2, 0, 4]]])
    np.testing.assert_array_equal(oracle.keep_histogram(counts, 4), [[2, 0, 1, 0, 3]])
    with pytest.raises(ValueError):
        oracle.keep_histogram(np.array([[5]]), 4)
