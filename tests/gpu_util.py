"""Helpers shared by the GPU parity tests (comparison rules, tie accounting)."""
import numpy as np
import pytest
import torch


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from calibrated_block_sparse_b200 import binding
    binding.load()  # fails loudly when the library is missing
    return binding


def attn_tolerance_ok(o_gpu, o_ref):
    """max|O - O_ref| <= 1e-2 * max|O_ref| + 1e-3 (bf16 inputs, fp32 accumulation)."""
    err = float(np.max(np.abs(o_gpu.astype(np.float64) - o_ref)))
    bound = 1e-2 * float(np.max(np.abs(o_ref))) + 1e-3
    return err <= bound, err, bound


def bf16_to_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def tie_affected(cut, eps, delta):
    """Rows whose greedy cut lies within delta of eps, or whose energies on the
    two sides of the cut are within delta (oracle.select's cut description)."""
    before, at, e_last, e_next = cut
    return (np.abs(at - eps) < delta) | (np.abs(before - eps) < delta) | \
        ((e_next >= 0) & (np.abs(e_last - e_next) < delta))


def compare_masks(mask_gpu, mask_ref, affected):
    """Bit-exact per row except tie-affected rows; returns (n_diff_rows, n_tie_rows, n_unexplained)."""
    mg = mask_gpu.reshape(-1, mask_gpu.shape[-1])
    mr = mask_ref.reshape(-1, mask_ref.shape[-1])
    diff = np.any(mg != mr, axis=1)
    aff = affected.reshape(-1)
    return int(diff.sum()), int(aff.sum()), int((diff & ~aff).sum())


# ---------------------------------------------------------------- energy tolerance and tie windows
#
# Energies computed on the GPU (fp32 scores from the tensor core, an fp32
# log-sum-exp, ex2.approx, fp32 tile sums) are accepted against the fp64
# oracle at |E - E_ref| <= ENERGY_REL * E_ref + ENERGY_ABS * max_c E_ref[r, c]
# per entry: the relative tolerance of 1e-5 on row entries that the parity
# contract fixes (the rounding of the scores, the log-sum-exp, ex2.approx and
# the tile sums adds up to a few 1e-6 relative; measured worst 1.9e-6), plus a
# floor for the probabilities below 2^-126 that ex2.approx.ftz flushes to zero.
ENERGY_REL = 1e-5
ENERGY_ABS = 1e-12
SAME_ENERGY_TIE = 1e-6  # the tie window when both sides select from the same energies


def energy_bound(E_ref):
    return ENERGY_REL * E_ref + ENERGY_ABS * E_ref.max(-1, keepdims=True)


def energy_ok(E, E_ref):
    """(all entries within the bound, worst |E - E_ref| / bound, worst relative error)."""
    b = energy_bound(E_ref)
    d = np.abs(E - E_ref)
    rel = d / np.maximum(E_ref, 1e-300)
    return bool(np.all(d <= b)), float(np.max(d / np.maximum(b, 1e-300))), float(np.max(np.where(E_ref > 0, rel, 0)))


def independent_tie_window(E_ref):
    """Per-row window for comparing a selection made from GPU energies with one
    made from the oracle's energies of the same input. Within the accepted
    energy bound every running sum of the greedy order moves by at most the sum
    of the per-entry bounds, and two energies can swap order only when they are
    closer than their two bounds: so a row whose cut lies within
    sum_c bound_c (plus the 1e-6 spec window) of eps, or whose energies
    at the cut are that close, may legitimately differ. Shape: rows."""
    return energy_bound(E_ref).sum(-1) + SAME_ENERGY_TIE


def cells_explained(agg_gpu, agg_ref, affected_rows):
    """Per-cell attribution of aggregated-mask differences.

    agg_gpu, agg_ref: [heads][nb][nb] aggregated masks; affected_rows:
    [n_inputs][heads][nb] booleans, the (input, head, block-row) selections
    that are tie-affected. A cell (h, r, c) may differ only if at least one
    input's selection of row (h, r) is tie-affected; returns (n_diff_cells,
    n_unexplained_cells)."""
    diff = agg_gpu != agg_ref
    row_aff = np.any(affected_rows, axis=0)  # [heads][nb]
    unexplained = diff & ~row_aff[..., None]
    return int(diff.sum()), int(unexplained.sum())
