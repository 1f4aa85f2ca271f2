"""GPU parity: block energy, greedy eps selection (standalone and fused),
mask accumulation and rho aggregation into the CSR skip list.

Rules:
* energies: |E - E_ref| <= 1e-5 * E_ref + 1e-12 * max_c E_ref[r, :] per row
  (gpu_util.energy_bound; derived in the design notes from fp32 score
  accumulation, the fp32 log-sum-exp and ex2.approx);
* selection given the same fp32 energies: bit-exact, except rows whose cut lies
  within 1e-6 of eps (counted, reported); the GPU's own tie flags at 1e-6
  equal the oracle's cut description;
* selection from independently computed energies: a row may differ only if
  its cut lies within the per-row window that the energy bound propagates to
  (gpu_util.independent_tie_window);
* aggregation and CSR: bit-exact (integer work); an aggregated cell may differ
  from the oracle's only when a tie-affected selection of its row is behind it.
"""
import numpy as np
import pytest
import torch

from calibrated_block_sparse_b200 import synth
from gpu_util import (SAME_ENERGY_TIE, cells_explained, compare_masks, energy_ok, independent_tie_window,
                      require_gpu, tie_affected)

pytestmark = pytest.mark.gpu


def _energy_ok(E, E_ref):
    ok, worst, rel = energy_ok(E, E_ref)
    print(f"energy: worst error / bound {worst:.3f}, worst relative error {rel:.2e}")
    return ok, worst


@pytest.mark.parametrize("heads,n,std,seed", [(1, 2048, 1.0, 1), (2, 1000, 2.0, 2), (1, 300, 3.0, 3)])
def test_block_energy_matches_oracle(oracle, heads, n, std, seed):
    binding = require_gpu()
    q, k, _ = synth.plain_qkv(heads, n, seed=seed, std=std)
    dev = torch.device("cuda")
    E, _, _, _ = binding.block_energy(q.to(dev), k.to(dev))
    assert binding.get_status() == 0
    E = E.cpu().numpy().astype(np.float64)
    E_ref = oracle.block_energy(synth.bf16_bits(q), synth.bf16_bits(k))
    ok, worst = _energy_ok(E, E_ref)
    assert ok, worst
    np.testing.assert_allclose(E.sum(-1), 1.0, atol=1e-4)


def test_positional_workload_energy_and_fused_selection(oracle):
    binding = require_gpu()
    wl = synth.WORKLOADS["tiny"]
    q, k, _ = synth.qkv(wl, 0, with_v=False)
    dev = torch.device("cuda")
    eps = 0.9
    E, mask, kept, _ = binding.block_energy(q.to(dev), k.to(dev), eps=eps)
    assert binding.get_status() == 0
    E = E.cpu().numpy().astype(np.float64)
    mask = mask.cpu().numpy()
    E_ref = oracle.block_energy(synth.bf16_bits(q), synth.bf16_bits(k))
    assert _energy_ok(E, E_ref)[0]
    # the fused selection equals the oracle's selection of the same fp32 energies
    m_same, kept_same, cut_same = oracle.select(E, eps, with_cut=True)
    n_diff, n_tie, bad = compare_masks(mask, m_same, tie_affected(cut_same, eps, 1e-6))
    assert bad == 0, (n_diff, n_tie)
    np.testing.assert_array_equal(kept.cpu().numpy(), mask.reshape(-1, mask.shape[-1]).sum(-1).reshape(kept.shape))
    # and the oracle's own energies, up to ties within the propagated energy bound
    m_ref, _, cut_ref = oracle.select(E_ref, eps, with_cut=True)
    n_diff, n_tie, bad = compare_masks(mask, m_ref, tie_affected(cut_ref, eps, independent_tie_window(E_ref)))
    print(f"fused selection vs oracle: {n_diff} rows differ, {n_tie} tie-affected rows")
    assert bad == 0


@pytest.mark.parametrize("nb,eps,seed", [(16, 0.9, 1), (591, 0.84, 2), (256, 0.99, 3), (348, 1.0, 4), (5, 0.0, 5),
                                         (1024, 0.95, 6), (1, 0.5, 7)])
def test_select_mask_is_bit_exact_on_same_energies(oracle, nb, eps, seed):
    binding = require_gpu()
    rng = np.random.default_rng(seed)
    heads = 3
    E = rng.dirichlet(np.full(nb, 0.3), size=(heads, nb)).astype(np.float32)
    E[0, :, ::7] = 0.0                       # exact zeros
    E[1, 0, :] = np.float32(1.0 / nb)         # a row of equal energies
    dev = torch.device("cuda")
    counts = torch.zeros((heads, nb, nb), dtype=torch.uint16, device=dev)
    mask, kept, counts = binding.select_mask(torch.from_numpy(E).to(dev), eps, counts=counts)
    assert binding.get_status() == 0
    mask = mask.cpu().numpy()
    m_ref, kept_ref, cut = oracle.select(E.astype(np.float64), eps, with_cut=True)
    n_diff, n_tie, bad = compare_masks(mask, m_ref, tie_affected(cut, eps, 1e-6))
    assert bad == 0, (n_diff, n_tie)
    if n_diff == 0:
        np.testing.assert_array_equal(kept.cpu().numpy(), kept_ref)
    np.testing.assert_array_equal(counts.cpu().numpy().astype(np.int64), mask.astype(np.int64))


def test_select_handles_nan_negative_and_large():
    binding = require_gpu()
    E = np.array([[[np.nan, -1.0, 0.5, 0.25], [0.0, 0.0, 0.0, 0.0], [9.0, 0.1, 0.1, 0.1], [0.3, 0.3, 0.3, 0.1]]],
                 np.float32)
    dev = torch.device("cuda")
    mask, kept, _ = binding.select_mask(torch.from_numpy(E).to(dev), 0.7)
    mask = mask.cpu().numpy()[0]
    assert mask[0].tolist() == [0, 0, 1, 1]   # NaN and negatives count as zero energy
    assert mask[1].tolist() == [1, 0, 0, 0]   # nothing to keep: the top block (lowest column)
    assert mask[2].tolist() == [1, 0, 0, 0]   # energies clamp at 4
    assert mask[3].tolist() == [1, 1, 1, 0]


def test_accumulate_and_aggregate_match_oracle(oracle):
    binding = require_gpu()
    rng = np.random.default_rng(11)
    heads, nb, n_in = 3, 37, 16
    masks = (rng.random((n_in, heads, nb, nb)) < rng.random((1, heads, nb, 1))).astype(np.uint8)
    dev = torch.device("cuda")
    counts = torch.zeros((heads, nb, nb), dtype=torch.uint16, device=dev)
    for p in range(n_in):
        binding.accumulate_masks(torch.from_numpy(masks[p]).to(dev), counts)
    for rho in (0.5, 0.3, 0.7, 0.0, 1.0):
        mask, row_ptr, col_idx, nnz = binding.aggregate_masks(counts, n_in, rho)
        assert binding.get_status() == 0
        m_ref, c_ref = oracle.aggregate(masks, rho)
        np.testing.assert_array_equal(counts.cpu().numpy().astype(np.int32), c_ref)
        np.testing.assert_array_equal(mask.cpu().numpy(), m_ref)
        rp_ref, ci_ref = oracle.mask_to_csr(m_ref)
        np.testing.assert_array_equal(row_ptr.cpu().numpy(), rp_ref)
        np.testing.assert_array_equal(col_idx.cpu().numpy(), ci_ref)
        assert int(nnz.item()) == int(m_ref.sum())


@pytest.mark.parametrize("rows,cols", [(1, 1), (45, 591), (3, 20000), (2000, 37)])
def test_aggregate_spans_ragged_tails_and_alignment(oracle, rows, cols):
    """The aggregation walks the flat mask in spans of whole 4096-cell rounds
    (at least one row each), with 16-byte vector accesses when counts and mask
    are 16-byte aligned and byte accesses otherwise. Several spans, a ragged
    last span, rows wider than the default span, and both access forms give
    the oracle's mask and skip list bit for bit."""
    binding = require_gpu()
    lib = binding.load()
    rng = np.random.default_rng(rows * 7 + cols)
    n_in = 5
    masks = (rng.random((n_in, rows, cols)) < rng.random((1, rows, 1))).astype(np.uint8)
    m_ref, c_ref = oracle.aggregate(masks, 0.5)
    rp_ref, ci_ref = oracle.mask_rows_to_csr(m_ref[None])
    dev = torch.device("cuda")
    cells = rows * cols
    for c_off, m_off in ((0, 0), (1, 3)):  # element / byte offsets into the buffers
        cbuf = torch.zeros(cells + 8, dtype=torch.uint16, device=dev)
        cbuf[c_off:c_off + cells] = torch.from_numpy(c_ref.astype(np.uint16).reshape(-1)).to(dev)
        mbuf = torch.full((cells + 16,), 7, dtype=torch.uint8, device=dev)
        row_ptr = torch.full((rows + 1,), -1, dtype=torch.int32, device=dev)
        col_idx = torch.full((cells,), -1, dtype=torch.int32, device=dev)
        nnz = torch.zeros(1, dtype=torch.int64, device=dev)
        ws = torch.empty(lib.calibatt_aggregate_rows_workspace_size(rows), dtype=torch.uint8, device=dev)
        rc = lib.calibatt_aggregate_mask_rows(cbuf.data_ptr() + 2 * c_off, n_in, rows, cols, 0.5,
                                              mbuf.data_ptr() + m_off, binding._ptr(row_ptr),
                                              binding._ptr(col_idx), cells, binding._ptr(nnz), binding._ptr(ws),
                                              ws.numel(), binding._stream(None))
        assert rc == 0
        torch.cuda.synchronize()
        assert binding.get_status() == 0
        mb = mbuf.cpu().numpy()
        np.testing.assert_array_equal(mb[m_off:m_off + cells].reshape(rows, cols), m_ref)
        assert np.all(mb[:m_off] == 7) and np.all(mb[m_off + cells:] == 7)  # nothing written outside
        total = int(nnz.item())
        assert total == int(m_ref.sum())
        np.testing.assert_array_equal(row_ptr.cpu().numpy(), rp_ref)
        ci = col_idx.cpu().numpy()
        np.testing.assert_array_equal(ci[:total], ci_ref)
        assert np.all(ci[total:] == -1)


def test_aggregate_scanned_span_prefixes(oracle):
    """Above 4096 spans the span totals are scanned into prefixes by a third
    launch before the compaction; 68 000 rows of 1003 columns (4163 spans)
    take that path. Mask and skip list bit for bit against the oracle, with
    16-byte aligned and misaligned buffers."""
    binding = require_gpu()
    lib = binding.load()
    rows, cols, n_in = 68000, 1003, 8
    rng = np.random.default_rng(68)
    c_ref = rng.integers(0, n_in + 1, (rows, cols), dtype=np.int16)
    m_ref = oracle.binarize_counts(c_ref, n_in, 0.5)
    rp_ref, ci_ref = oracle.mask_rows_to_csr(m_ref[None])
    dev = torch.device("cuda")
    cells = rows * cols
    for c_off, m_off in ((0, 0), (3, 5)):
        cbuf = torch.zeros(cells + 8, dtype=torch.int16, device=dev)
        cbuf[c_off:c_off + cells] = torch.from_numpy(c_ref.reshape(-1)).to(dev)
        mbuf = torch.empty(cells + 16, dtype=torch.uint8, device=dev)
        row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=dev)
        col_idx = torch.empty(cells, dtype=torch.int32, device=dev)
        nnz = torch.zeros(1, dtype=torch.int64, device=dev)
        ws = torch.empty(lib.calibatt_aggregate_rows_workspace_size(rows), dtype=torch.uint8, device=dev)
        rc = lib.calibatt_aggregate_mask_rows(cbuf.data_ptr() + 2 * c_off, n_in, rows, cols, 0.5,
                                              mbuf.data_ptr() + m_off, binding._ptr(row_ptr),
                                              binding._ptr(col_idx), cells, binding._ptr(nnz), binding._ptr(ws),
                                              ws.numel(), binding._stream(None))
        assert rc == 0
        torch.cuda.synchronize()
        assert binding.get_status() == 0
        np.testing.assert_array_equal(mbuf[m_off:m_off + cells].cpu().numpy().reshape(rows, cols), m_ref)
        np.testing.assert_array_equal(row_ptr.cpu().numpy(), rp_ref)
        total = int(nnz.item())
        assert total == rp_ref[-1]
        np.testing.assert_array_equal(col_idx[:total].cpu().numpy(), ci_ref)


def test_aggregate_capacity_is_reported():
    binding = require_gpu()
    dev = torch.device("cuda")
    counts = torch.ones((1, 8, 8), dtype=torch.uint16, device=dev)
    mask, row_ptr, col_idx, nnz = binding.aggregate_masks(counts, 1, 0.5, nnz_cap=10, trim=False)
    assert binding.get_status() == -7  # CALIBATT_ERR_CAPACITY
    assert int(nnz.item()) == 64
    assert col_idx.cpu().numpy().tolist() == [0, 1, 2, 3, 4, 5, 6, 7, 0, 1]


def test_tiny_calibration_pipeline(oracle):
    """The tiny workload end to end: calibrate over 8 inputs at eps = 0.9,
    aggregate at rho = 0.5, then sparse attention on a 9th input. Every
    per-input selection row and every aggregated cell is attributed: a
    difference from the oracle needs a tie-affected selection behind it."""
    binding = require_gpu()
    from gpu_util import attn_tolerance_ok, bf16_to_f64
    wl = synth.WORKLOADS["tiny"]
    dev = torch.device("cuda")
    nb = wl.nb
    eps, rho, n_in = 0.9, 0.5, 8
    counts = torch.zeros((wl.heads, nb, nb), dtype=torch.uint16, device=dev)
    ref_masks, gpu_masks, affected, gpu_ties = [], [], [], 0
    for p in range(n_in):
        q, k, _ = synth.qkv(wl, p, with_v=False)
        m_p = torch.empty((wl.heads, nb, nb), dtype=torch.uint8, device=dev)
        _, _, _, _, tie = binding.block_energy(q.to(dev), k.to(dev), eps=eps, energy=False, mask=m_p, counts=counts,
                                               tie=True)
        E_ref = oracle.block_energy(synth.bf16_bits(q), synth.bf16_bits(k))
        m_ref, _, cut = oracle.select(E_ref, eps, with_cut=True)
        aff = tie_affected(cut, eps, independent_tie_window(E_ref))
        n_diff, n_tie, bad = compare_masks(m_p.cpu().numpy(), m_ref, aff)
        assert bad == 0, (p, n_diff, n_tie)
        ref_masks.append(m_ref)
        gpu_masks.append(m_p.cpu().numpy())
        affected.append(aff)
        gpu_ties += int(tie.sum().item())
    assert binding.get_status() == 0
    mask, row_ptr, col_idx, _ = binding.aggregate_masks(counts, n_in, rho)
    # the GPU's aggregation of its own per-input masks is exact
    m_gpu_agg, c_gpu = oracle.aggregate(np.stack(gpu_masks), rho)
    np.testing.assert_array_equal(counts.cpu().numpy().astype(np.int32), c_gpu)
    np.testing.assert_array_equal(mask.cpu().numpy(), m_gpu_agg)
    # against the oracle's whole pipeline, cell by cell
    m_ref, c_ref = oracle.aggregate(np.stack(ref_masks), rho)
    diff_cells, unexplained = cells_explained(mask.cpu().numpy(), m_ref, np.stack(affected))
    print(f"tiny pipeline: sparsity {1 - m_ref.mean():.3f}, {diff_cells} aggregated cells differ, "
          f"{int(np.stack(affected).sum())} tie-affected selections (oracle energies), "
          f"{gpu_ties} rows tie-affected at 1e-6 (GPU flags)")
    assert unexplained == 0
    # attention on a 9th input with the GPU's own skip list
    q, k, v = synth.qkv(wl, n_in)
    work = binding.build_plan(row_ptr.cpu().numpy(), wl.heads, nb)
    o, _ = binding.sparse_attn_fwd(q.to(dev), k.to(dev), v.to(dev), row_ptr, col_idx,
                                   torch.from_numpy(work).to(dev))
    o_ref, _ = oracle.masked_attention(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v),
                                       mask.cpu().numpy())
    assert attn_tolerance_ok(bf16_to_f64(o), o_ref)[0]


def test_calibrate_sharded_single_rank_matches_oracle(oracle):
    """The multi-GPU calibration entry on one rank (no process group)."""
    binding = require_gpu()
    from calibrated_block_sparse_b200 import multi
    wl = synth.WORKLOADS["tiny"]
    dev = torch.device("cuda")
    inputs = {p: synth.qkv(wl, p, with_v=False) for p in range(4)}
    mask, row_ptr, col_idx, _ = multi.calibrate_sharded(
        lambda p: (inputs[p][0].to(dev), inputs[p][1].to(dev)), wl.heads, wl.nb, 4, 0.9, 0.5, device=dev)
    ref, affected = [], []
    for p in range(4):
        E_ref = oracle.block_energy(synth.bf16_bits(inputs[p][0]), synth.bf16_bits(inputs[p][1]))
        m, _, cut = oracle.select(E_ref, 0.9, with_cut=True)
        ref.append(m)
        affected.append(tie_affected(cut, 0.9, independent_tie_window(E_ref)))
    m_ref, _ = oracle.aggregate(np.stack(ref), 0.5)
    assert cells_explained(mask.cpu().numpy(), m_ref, np.stack(affected))[1] == 0


@pytest.mark.parametrize("nb", [7, 64, 591, 1024])
def test_select_with_many_equal_energies_is_exact(oracle, nb):
    """Energies from a coarse grid (multiples of 1/64) make long runs of equal
    values at the cut; eps sits between grid points, so no row is tie-affected
    and the GPU's cut (largest tau, then lowest columns) must equal the
    oracle's stable greedy order exactly."""
    binding = require_gpu()
    rng = np.random.default_rng(nb)
    heads = 2
    E = (rng.integers(0, 5, size=(heads, nb, nb)) / 64.0).astype(np.float32)
    dev = torch.device("cuda")
    for eps in (0.3 + 1 / 128, 0.7 + 1 / 128, 2.0 + 1 / 256):
        mask, kept, _ = binding.select_mask(torch.from_numpy(E).to(dev), eps)
        m_ref, kept_ref = oracle.select(E.astype(np.float64), eps)
        np.testing.assert_array_equal(mask.cpu().numpy(), m_ref)
        np.testing.assert_array_equal(kept.cpu().numpy(), kept_ref)



# ---------------------------------------------------------------- single-pass energy

@pytest.mark.parametrize("heads,n,std,seed", [(1, 2048, 1.0, 1), (2, 1000, 2.0, 2), (1, 300, 3.0, 3),
                                              (3, 128 * 40 + 7, 1.5, 4)])
def test_single_pass_energy_matches_oracle(oracle, heads, n, std, seed):
    binding = require_gpu()
    q, k, _ = synth.plain_qkv(heads, n, seed=seed, std=std)
    dev = torch.device("cuda")
    qd, kd = q.to(dev), k.to(dev)
    E1, _, _, _, _ = binding.block_energy_1pass(qd, kd)
    assert binding.get_status() == 0
    E1 = E1.cpu().numpy().astype(np.float64)
    E_ref = oracle.block_energy(synth.bf16_bits(q), synth.bf16_bits(k))
    ok, worst = _energy_ok(E1, E_ref)
    assert ok, worst
    np.testing.assert_allclose(E1.sum(-1), 1.0, atol=1e-4)


def test_single_pass_fused_selection_and_profiles(oracle):
    binding = require_gpu()
    wl = synth.WORKLOADS["tiny"]
    q, k, _ = synth.qkv(wl, 3, with_v=False)
    dev = torch.device("cuda")
    eps = 0.9
    E, mask, kept, _, pix = binding.block_energy_1pass(q.to(dev), k.to(dev), eps=eps, pix_W=wl.W)
    assert binding.get_status() == 0
    E = E.cpu().numpy().astype(np.float64)
    mask = mask.cpu().numpy()
    E_ref = oracle.block_energy(synth.bf16_bits(q), synth.bf16_bits(k))
    assert _energy_ok(E, E_ref)[0]
    # the fused selection equals the oracle's selection of the same fp32 energies
    m_same, _, cut_same = oracle.select(E, eps, with_cut=True)
    n_diff, n_tie, bad = compare_masks(mask, m_same, tie_affected(cut_same, eps, 1e-6))
    assert bad == 0, (n_diff, n_tie)
    np.testing.assert_array_equal(kept.cpu().numpy(), mask.reshape(-1, mask.shape[-1]).sum(-1).reshape(kept.shape))
    # pixel-row profiles from the same pass
    P_ref = oracle.pixel_row_energy(synth.bf16_bits(q), synth.bf16_bits(k), wl.F, wl.H, wl.W)
    assert _energy_ok(pix.cpu().numpy().astype(np.float64), P_ref)[0]


def test_single_pass_counts_equal_two_pass_counts_away_from_ties(oracle):
    """Calibrating 4 inputs with either energy kernel gives the same counts,
    except blocks whose selection is tie-affected at the energy error bound."""
    binding = require_gpu()
    wl = synth.WORKLOADS["tiny"]
    dev = torch.device("cuda")
    nb = wl.nb
    c1 = torch.zeros((wl.heads, nb, nb), dtype=torch.uint16, device=dev)
    c2 = torch.zeros_like(c1)
    aff = np.zeros((wl.heads, nb), bool)
    for p in range(4):
        q, k, _ = synth.qkv(wl, 10 + p, with_v=False, device=dev)
        E1, _, _, _, _ = binding.block_energy_1pass(q, k, eps=0.9, counts=c1)
        binding.block_energy(q, k, eps=0.9, energy=False, counts=c2)
        _, _, cut = oracle.select(E1.cpu().numpy().astype(np.float64), 0.9, with_cut=True)
        aff |= tie_affected(cut, 0.9, 1e-4)
    assert binding.get_status() == 0
    d = (c1 != c2).cpu().numpy().any(-1)
    assert not np.any(d & ~aff), int((d & ~aff).sum())


# ---------------------------------------------------------------- radix selection and tie flags

def _hard_rows(rng, nb, rows):
    """Energy rows that stress the exact radix search: heavy tails over many
    binades, long runs of equal values, exact zeros, values below 2^-50 (zero
    in fixed point), and more than 32 blocks sharing the cut's leading bits."""
    out = []
    for i in range(rows):
        kind = i % 6
        if kind == 0:
            e = np.exp(rng.normal(-12.0, 6.0, nb))
        elif kind == 1:
            e = rng.integers(0, 4, nb) / 32.0
        elif kind == 2:
            e = rng.dirichlet(np.full(nb, 0.05))
            e[::3] = 0.0
        elif kind == 3:
            e = np.full(nb, 1.0) + (rng.random(nb) < 0.2) * 2.0 ** -20  # one binade, near-equal
        elif kind == 4:
            e = rng.dirichlet(np.full(nb, 1.0))
            e[rng.random(nb) < 0.3] = 2.0 ** -60  # below the fixed point's resolution
        else:
            e = rng.dirichlet(np.full(nb, 0.3))
        out.append(e / e.sum())
    return np.stack(out).astype(np.float32)


@pytest.mark.parametrize("nb", [1, 3, 32, 33, 100, 256, 591, 1024])
def test_radix_select_is_exact_on_hard_rows(oracle, nb):
    binding = require_gpu()
    rng = np.random.default_rng(100 + nb)
    E = _hard_rows(rng, nb, 2 * nb if nb < 64 else nb)
    heads = E.shape[0] // nb
    E = E[: heads * nb].reshape(heads, nb, nb)
    dev = torch.device("cuda")
    Ed = torch.from_numpy(E).to(dev)
    for eps in (0.0, 0.3 + 1 / 128, 0.84, 0.9, 0.99, 1.0, 1.5):
        mask, kept, _, tie = binding.select_mask(Ed, eps, tie=True)
        m_ref, kept_ref, cut = oracle.select(E.astype(np.float64), eps, with_cut=True)
        aff = tie_affected(cut, eps, SAME_ENERGY_TIE)
        n_diff, n_tie, bad = compare_masks(mask.cpu().numpy(), m_ref, aff)
        assert bad == 0, (eps, n_diff, n_tie)
        rows_ok = ~aff.reshape(-1)
        np.testing.assert_array_equal(kept.cpu().numpy().reshape(-1)[rows_ok], kept_ref.reshape(-1)[rows_ok])


def _margin_ok(cut, eps, delta, margin):
    """Rows whose tie decision is not within `margin` of the window's edge."""
    before, at, e_last, e_next = cut
    dist = np.minimum(np.abs(np.abs(at - eps) - delta), np.abs(np.abs(before - eps) - delta))
    dist = np.where(e_next >= 0, np.minimum(dist, np.abs(np.abs(e_last - e_next) - delta)), dist)
    return dist > margin


@pytest.mark.parametrize("nb", [16, 591])
def test_tie_flags_match_the_oracle_cut(oracle, nb):
    """The selection's own tie flags at 1e-6 equal the oracle's description of
    the cut (running sums before and at the last kept block, the energies on
    both sides) on the same fp32 energies. Rows are built so that many cuts
    land within the window: the energies are rescaled so that a prefix sums to
    eps +- 5e-7."""
    binding = require_gpu()
    rng = np.random.default_rng(7 + nb)
    heads = 4
    E = rng.dirichlet(np.full(nb, 0.4), size=(heads, nb))
    eps = 0.9
    for h in range(heads):
        for r in range(0, nb, 2):
            order = np.argsort(-E[h, r], kind="stable")
            cs = np.cumsum(E[h, r, order])
            m = int(np.searchsorted(cs, eps))
            m = min(m, nb - 1)
            E[h, r] *= (eps + rng.uniform(-5e-7, 5e-7)) / cs[m]
    E = E.astype(np.float32)
    dev = torch.device("cuda")
    mask, _, _, tie = binding.select_mask(torch.from_numpy(E).to(dev), eps, tie=True, tie_window=SAME_ENERGY_TIE)
    _, _, cut = oracle.select(E.astype(np.float64), eps, with_cut=True)
    aff = tie_affected(cut, eps, SAME_ENERGY_TIE)
    sure = _margin_ok(cut, eps, SAME_ENERGY_TIE, 1e-12)
    got = tie.cpu().numpy().astype(bool)
    assert aff.sum() > nb // 4  # the construction produced ties
    np.testing.assert_array_equal(got[sure], aff[sure])
    # the fused selection of the energy kernels flags the same rows
    q, k, _ = synth.plain_qkv(2, 128 * 24 + 5, seed=nb)
    E2, _, _, _, t2 = binding.block_energy(q.to(dev), k.to(dev), eps=eps, tie=True)
    _, _, cut2 = oracle.select(E2.cpu().numpy().astype(np.float64), eps, with_cut=True)
    sure2 = _margin_ok(cut2, eps, SAME_ENERGY_TIE, 1e-12)
    np.testing.assert_array_equal(t2.cpu().numpy().astype(bool)[sure2],
                                  tie_affected(cut2, eps, SAME_ENERGY_TIE)[sure2])
