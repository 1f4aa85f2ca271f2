"""The allocation-free skip-list build (calibatt_aggregate_masks_noalloc),
for callers that cannot allocate device memory themselves: it must give the
same mask, row_ptr, col_idx and nnz as calibatt_aggregate_masks with a
caller-supplied workspace and as the oracle's binarisation and skip list
(integer work: bit-exact), on two calls in a row that share its static
scratch array.

Named so that pytest collects it last; it passes alone in a fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _outputs(heads, nb, dev):
    return (torch.full((heads, nb, nb), 9, dtype=torch.uint8, device=dev),
            torch.full((heads * nb + 1,), -1, dtype=torch.int32, device=dev),
            torch.full((heads * nb * nb,), -1, dtype=torch.int32, device=dev),
            torch.full((1,), -1, dtype=torch.int64, device=dev))


@pytest.mark.parametrize("heads,nb,n_inputs,rho", [(40, 591, 16, 0.5), (3, 37, 8, 0.3)])
def test_noalloc_matches_workspace_variant_twice(oracle, heads, nb, n_inputs, rho):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from calibrated_block_sparse_b200 import binding
    lib = binding.load()
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream()
    rng = np.random.default_rng(heads * 1000 + nb)
    for call in range(2):
        # a different input each call: the second call must not see the first's scratch
        keep = rng.random((heads, 1, 1)) * (0.3 + 0.6 * call)
        counts_h = rng.binomial(n_inputs, np.broadcast_to(keep, (heads, nb, nb))).astype(np.int16)
        counts = torch.from_numpy(counts_h).to(dev).view(torch.uint16)
        ref = binding.aggregate_masks(counts, n_inputs, rho, trim=False)
        mask, row_ptr, col_idx, nnz = _outputs(heads, nb, dev)
        rc = lib.calibatt_aggregate_masks_noalloc(
            ctypes.c_void_p(counts.data_ptr()), n_inputs, heads, nb, ctypes.c_double(rho),
            ctypes.c_void_p(mask.data_ptr()), ctypes.c_void_p(row_ptr.data_ptr()),
            ctypes.c_void_p(col_idx.data_ptr()), col_idx.numel(), ctypes.c_void_p(nnz.data_ptr()),
            ctypes.c_void_p(stream.cuda_stream))
        assert rc == 0
        assert binding.get_status() == 0
        total = int(ref[3].item())
        assert int(nnz.item()) == total
        assert torch.equal(mask, ref[0])
        assert torch.equal(row_ptr, ref[1])
        assert torch.equal(col_idx[:total], ref[2][:total])
        # and the oracle's rule written out: keep where count / n >= rho
        m_ref = oracle.binarize_counts(counts_h.astype(np.int32), n_inputs, rho)
        rp_ref, ci_ref = oracle.mask_to_csr(m_ref)
        np.testing.assert_array_equal(mask.cpu().numpy(), m_ref)
        np.testing.assert_array_equal(row_ptr.cpu().numpy(), rp_ref)
        np.testing.assert_array_equal(col_idx[:total].cpu().numpy(), ci_ref)
        assert total == ci_ref.size


def test_noalloc_rejects_oversize():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from calibrated_block_sparse_b200 import binding
    lib = binding.load()
    P = ctypes.c_void_p
    fake = P(0x100000)
    # heads * nb above the static array's 2^18 rows: rejected before any launch
    assert lib.calibatt_aggregate_masks_noalloc(fake, 4, 1024, 257, ctypes.c_double(0.5), fake, fake, fake, 16,
                                                fake, None) == -1
