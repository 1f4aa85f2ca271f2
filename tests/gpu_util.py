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
