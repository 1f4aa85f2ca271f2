"""GPU parity: block masks on the repeated heads' anchor rows.

* calibatt_anchor_block_energy against oracle.anchor_block_energy (energies
  within the energy bound), its fused selection against the oracle's selection
  of the same fp32 energies (ties at 1e-6) and its tie flags;
* calibatt_mixed_masked_attn_fwd against oracle.repeat_attention_masked for
  the repeated heads and oracle.masked_attention for the block-sparse heads
  (max|O - O_ref| <= 1e-2 max|O_ref| + 1e-3), empty anchor blocks included; an
  all-ones anchor mask gives calibatt_mixed_attn_fwd's output bit for bit;
* the pipeline: anchor masks calibrated over several inputs, aggregated with
  calibatt_aggregate_mask_rows (bit-exact against the oracle's aggregation of
  the GPU's per-input masks), then the masked launch;
* the Wan-720p shape (8 repeated heads of 45 rows, k = 5) on sampled rows.
"""
import numpy as np
import pytest
import torch

from calibrated_block_sparse_b200 import synth
from gpu_util import (SAME_ENERGY_TIE, attn_tolerance_ok, compare_masks, energy_ok, independent_tie_window,
                      require_gpu, tie_affected)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits(t):
    return synth.bf16_bits(t)


def _csr(mask):
    rows = mask.reshape(-1, mask.shape[-1])
    rp = np.zeros(rows.shape[0] + 1, np.int32)
    rp[1:] = np.cumsum(rows.sum(-1))
    ci = np.nonzero(rows)[1].astype(np.int32)
    return rp, ci


@pytest.mark.parametrize("F,H,W,heads,rep,kk,std,seed", [(4, 8, 40, 3, (0, 2), 3, 1.5, 1), (16, 8, 16, 2, (1,), 5, 1.0, 2),
                                                          (3, 10, 53, 2, (0, 1), 4, 2.0, 3)])
def test_anchor_energy_and_selection_match_oracle(oracle, F, H, W, heads, rep, kk, std, seed):
    binding = require_gpu()
    n = F * H * W
    q, k, _ = synth.plain_qkv(heads, n, seed=seed, std=std)
    dev = torch.device(DEV)
    rep_t = torch.tensor(rep, dtype=torch.int32, device=dev)
    eps = 0.9
    E, mask, kept, _, tie = binding.anchor_block_energy(q.to(dev), k.to(dev), F, H, W, rep_t, k_anchor=kk, eps=eps,
                                                        tie=True)
    assert binding.get_status() == 0
    E = E.cpu().numpy().astype(np.float64)
    hs = list(rep)
    E_ref = oracle.anchor_block_energy(_bits(q[hs]), _bits(k[hs]), F, H, W, k_anchor=kk)
    ok, worst, rel = energy_ok(E, E_ref)
    assert ok, (worst, rel)
    np.testing.assert_allclose(E.sum(-1), 1.0, atol=1e-4)
    m_same, kept_same, cut = oracle.select(E, eps, with_cut=True)
    aff = tie_affected(cut, eps, SAME_ENERGY_TIE)
    assert compare_masks(mask.cpu().numpy(), m_same, aff)[2] == 0
    np.testing.assert_array_equal(kept.cpu().numpy()[~aff], kept_same[~aff])
    np.testing.assert_array_equal(tie.cpu().numpy().astype(bool), aff)
    m_ref, _, cut_ref = oracle.select(E_ref, eps, with_cut=True)
    assert compare_masks(mask.cpu().numpy(), m_ref, tie_affected(cut_ref, eps, independent_tie_window(E_ref)))[2] == 0


def _masked_case(binding, F, H, W, heads, rep, kk, keep, seed, dev):
    n = F * H * W
    nb = -(-n // 128)
    nbq = binding.anchor_blocks(F, W, kk)
    q, k, v = synth.plain_qkv(heads, n, seed=seed, std=1.5)
    mask = synth.random_mask(heads, nb, keep, seed=seed)
    mask_b = synth.random_mask(len(rep), max(nbq, nb), keep, seed=seed + 50)[:, :nbq, :nb].copy()
    mask_b[0, 0, :] = 0  # an anchor block that keeps nothing
    rp, ci = _csr(mask)
    rpb, cib = _csr(mask_b)
    work = binding.build_mixed_plan(rp, heads, nb, list(rep), F, H, W, kk)
    work = binding.balance_mixed_plan(work, rp, heads, nb, rpb, len(rep), F, W, kk)
    t = lambda a: torch.from_numpy(a).to(dev)
    return (q, k, v), mask, mask_b, t(rp), t(ci), t(rpb), t(cib), t(work)


@pytest.mark.parametrize("F,H,W,heads,rep,kk,keep,seed", [(4, 8, 40, 3, (0, 2), 3, 0.5, 4), (16, 8, 16, 2, (1,), 5, 0.4, 5),
                                                          (3, 10, 53, 3, (1,), 4, 0.6, 6)])
def test_masked_mixed_launch_matches_oracle(oracle, F, H, W, heads, rep, kk, keep, seed):
    binding = require_gpu()
    dev = torch.device(DEV)
    (q, k, v), mask, mask_b, rp, ci, rpb, cib, work = _masked_case(binding, F, H, W, heads, rep, kk, keep, seed, dev)
    rep_t = torch.tensor(rep, dtype=torch.int32, device=dev)
    o, lse = binding.mixed_masked_attn_fwd(q.to(dev), k.to(dev), v.to(dev), F, H, W, rp, ci, rep_t, rpb, cib, work,
                                           k_anchor=kk)
    assert binding.get_status() == 0
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    for h in range(heads):
        qb, kb, vb = (_bits(t[h:h + 1]) for t in (q, k, v))
        if h in rep:
            i = rep.index(h)
            o_ref, lse_ref = oracle.repeat_attention_masked(qb, kb, vb, F, H, W, mask_b[i:i + 1], k_anchor=kk)
        else:
            o_ref, lse_ref = oracle.masked_attention(qb, kb, vb, mask[h:h + 1])
        ok, err, bound = attn_tolerance_ok(o[h], o_ref[0])
        assert ok, (h, err, bound)
        fin = np.isfinite(lse_ref[0])
        np.testing.assert_array_equal(np.isfinite(lse[h]), fin)
        np.testing.assert_allclose(lse[h][fin], lse_ref[0][fin], atol=2e-3)


def test_all_ones_anchor_mask_is_the_unmasked_launch():
    binding = require_gpu()
    dev = torch.device(DEV)
    F, H, W, heads, rep, kk = 6, 9, 24, 3, [0, 2], 3
    n = F * H * W
    nb = -(-n // 128)
    nbq = binding.anchor_blocks(F, W, kk)
    q, k, v = (t.to(dev) for t in synth.plain_qkv(heads, n, seed=7))
    mask = synth.random_mask(heads, nb, 0.5, seed=7)
    rp, ci = _csr(mask)
    rpb, cib = _csr(np.ones((len(rep), nbq, nb), np.uint8))
    work = torch.from_numpy(binding.build_mixed_plan(rp, heads, nb, rep, F, H, W, kk)).to(dev)
    t = lambda a: torch.from_numpy(a).to(dev)
    rep_t = torch.tensor(rep, dtype=torch.int32, device=dev)
    o1, l1 = binding.mixed_attn_fwd(q, k, v, F, H, W, t(rp), t(ci), rep_t, work, k_anchor=kk)
    o2, l2 = binding.mixed_masked_attn_fwd(q, k, v, F, H, W, t(rp), t(ci), rep_t, t(rpb), t(cib), work, k_anchor=kk)
    assert binding.get_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_calibrated_anchor_masks_pipeline(oracle):
    """Anchor masks of the tiny positional workload's head (k = 5 of 8 rows)
    calibrated over 4 inputs at eps = 0.9, aggregated at rho = 0.5, then the
    masked launch on a fifth input."""
    binding = require_gpu()
    dev = torch.device(DEV)
    wl = synth.WORKLOADS["tiny"]
    F, H, W, kk = wl.F, wl.H, wl.W, wl.k_anchor
    nbq = binding.anchor_blocks(F, W, kk)
    eps, n_in = 0.9, 4
    rep_t = torch.zeros(1, dtype=torch.int32, device=dev)
    counts = torch.zeros((1, nbq, wl.nb), dtype=torch.uint16, device=dev)
    per_input, affected = [], []
    for p in range(n_in):
        q, k, _ = synth.qkv(wl, p, with_v=False)
        m_p = torch.empty((1, nbq, wl.nb), dtype=torch.uint8, device=dev)
        binding.anchor_block_energy(q.to(dev), k.to(dev), F, H, W, rep_t, k_anchor=kk, eps=eps, energy=False,
                                    mask=m_p, counts=counts)
        E_ref = oracle.anchor_block_energy(_bits(q), _bits(k), F, H, W, k_anchor=kk)
        m_ref, _, cut = oracle.select(E_ref, eps, with_cut=True)
        aff = tie_affected(cut, eps, independent_tie_window(E_ref))
        assert compare_masks(m_p.cpu().numpy(), m_ref, aff)[2] == 0
        per_input.append(m_p.cpu().numpy())
    assert binding.get_status() == 0
    mask_b, rpb, cib, nnz = binding.aggregate_mask_rows(counts, n_in, 0.5)
    m_agg, c_agg = oracle.aggregate(np.stack(per_input), 0.5)
    np.testing.assert_array_equal(counts.cpu().numpy().astype(np.int32), c_agg)
    np.testing.assert_array_equal(mask_b.cpu().numpy(), m_agg)
    rp_ref, ci_ref = oracle.mask_rows_to_csr(m_agg)
    np.testing.assert_array_equal(rpb.cpu().numpy(), rp_ref)
    np.testing.assert_array_equal(cib.cpu().numpy(), ci_ref)
    # attention of one repeated head (and nothing else) on a fifth input
    q, k, v = synth.qkv(wl, n_in)
    rp0 = np.zeros(wl.nb + 1, np.int32)
    work = torch.from_numpy(binding.build_mixed_plan(rp0, 1, wl.nb, [0], F, H, W, kk)).to(dev)
    o, _ = binding.mixed_masked_attn_fwd(q.to(dev), k.to(dev), v.to(dev), F, H, W, torch.from_numpy(rp0).to(dev),
                                         torch.zeros(0, dtype=torch.int32, device=dev), rep_t, rpb, cib, work,
                                         k_anchor=kk)
    assert binding.get_status() == 0
    o_ref, _ = oracle.repeat_attention_masked(_bits(q), _bits(k), _bits(v), F, H, W, m_agg, k_anchor=kk)
    ok, err, bound = attn_tolerance_ok(o.float().cpu().numpy().astype(np.float64), o_ref)
    assert ok, (err, bound)
    print(f"tiny anchor masks: {1 - m_agg.mean():.3f} of anchor blocks skipped")


def test_wan720_anchor_masks_sampled(oracle):
    """The Wan-720p step with anchor-row masks on its 8 repeated heads
    (calibrated on 2 inputs at eps = 0.95): sampled anchor energies against the
    oracle, then the masked launch with the block-sparse heads' random masks,
    sampled rows of repeated and block-sparse heads against the oracle."""
    import os
    binding = require_gpu()
    dev = torch.device(DEV)
    wl = synth.WORKLOADS["wan720"]
    F, H, W, kk = wl.F, wl.H, wl.W, wl.k_anchor
    nbq = binding.anchor_blocks(F, W, kk)
    rep = list(wl.repeat_heads)
    rep_t = torch.tensor(rep, dtype=torch.int32, device=dev)
    counts = torch.zeros((len(rep), nbq, wl.nb), dtype=torch.uint16, device=dev)
    threads = min(32, os.cpu_count() or 1)
    rng = np.random.default_rng(30)
    for p in range(2):
        q, k, _ = synth.qkv(wl, p, with_v=False, device=dev)
        E, _, _, _ = binding.anchor_block_energy(q, k, F, H, W, rep_t, k_anchor=kk, eps=0.95, counts=counts)
        if p == 0:
            i = int(rng.integers(len(rep)))
            brs = np.array([nbq - 1, int(rng.integers(nbq - 1))], np.int64)
            E_ref = oracle.anchor_block_energy(_bits(q[rep[i]:rep[i] + 1]), _bits(k[rep[i]:rep[i] + 1]), F, H, W,
                                               k_anchor=kk, blockrows=brs, threads=threads)
            ok, worst, rel = energy_ok(E.cpu().numpy().astype(np.float64)[i][brs], E_ref)
            assert ok, (worst, rel)
        del q, k
    mask_b, rpb, cib, _ = binding.aggregate_mask_rows(counts, 2, 0.5)
    masks = synth.random_block_masks(wl)
    rp, ci = _csr(masks)
    work = binding.balance_mixed_plan(binding.build_mixed_plan(rp, wl.heads, wl.nb, rep, F, H, W, kk), rp, wl.heads,
                                      wl.nb, rpb.cpu().numpy(), len(rep), F, W, kk)
    q, k, v = synth.qkv(wl, 11, device=dev)
    t = lambda a: torch.from_numpy(a).to(dev)
    o, _ = binding.mixed_masked_attn_fwd(q, k, v, F, H, W, t(rp), t(ci), rep_t, rpb, cib, t(work), k_anchor=kk)
    assert binding.get_status() == 0
    mb = mask_b.cpu().numpy()
    print(f"wan720 anchor masks: {1 - mb.mean():.3f} of anchor blocks skipped")
    for h in (rep[0], rep[-1], 0):
        rows = rng.choice(wl.n, size=16, replace=False).astype(np.int64)
        rows[0] = wl.n - 1
        qb, kb, vb = (_bits(x[h:h + 1]) for x in (q, k, v))
        if h in rep:
            i = rep.index(h)
            o_ref, _ = oracle.repeat_attention_masked(qb, kb, vb, F, H, W, mb[i:i + 1], k_anchor=kk, rows=rows,
                                                      threads=threads)
        else:
            o_ref, _ = oracle.masked_attention(qb, kb, vb, masks[h:h + 1], rows=rows, threads=threads)
        ok, err, bound = attn_tolerance_ok(o[h].float().cpu().numpy().astype(np.float64)[rows], o_ref)
        assert ok, (h, err, bound)
