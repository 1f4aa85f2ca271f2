"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times, on sampled outputs the fp64 oracle computes one by one.

* Wan 2.1 14B 720p: 40 heads x N = 75600 (last block 80 rows); 32 block-sparse
  heads over random Beta(2,3) masks at 62.5 % sparsity, 8 repeated heads with
  k = 5 anchor rows of 45; sampled query rows of both kinds.
* Wan 2.1 14B 480p: calibration energies and fused eps(T/2) selection on
  sampled block-rows of all 40 heads (N = 32760, last block 120 rows); the
  whole pipeline (16 inputs, aggregation at rho = 0.5, attention over the
  calibrated skip lists in the benchmark's launch) on sampled rows.
* The single-pass energy kernel at the Wan-720p, Wan-480p and Mochi lengths
  (nb = 591, 256, 348) on sampled block-rows, the ragged last row included:
  energies, the fused selection, its tie flags and the counts.
* Mochi 1 480p: masks calibrated on the GPU over 16 inputs at eps = 0.84,
  aggregated at rho = 0.5, then attention of 20 block-sparse + 4 repeated
  heads (k = 5 of 30 rows) on sampled rows.
* Calibration sweep at the Wan-720p shape: eps in {0.84, 0.9, 0.95, 0.99} on
  sampled block-rows; aggregation of 16 inputs against the oracle aggregator;
  and the workload at its own scale (40 heads, 64 inputs, all four eps):
  counts, masks and skip lists bit-exact against the oracle's aggregation of
  the GPU's per-input masks, sampled energy rows against the oracle.
* Spatial repetition at the Wan-720p and Mochi shapes: pixel-row profiles and
  scores of every head; the heads flagged at gamma = 0.87 are the workloads'
  repeated heads.

Inputs come from the seeded generator (synth), drawn on the device; the
sampled heads are copied to the host for the oracle.
"""
import os

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


def _energy_ok(E, E_ref):
    ok, worst, rel = energy_ok(E, E_ref)
    print(f"energy: worst error / bound {worst:.3f}, worst relative error {rel:.2e}")
    return ok


def _oracle_threads():
    return min(32, os.cpu_count() or 1)


def _skiplist(binding, masks, dev):
    counts = torch.from_numpy(masks.astype(np.int16)).to(dev).view(torch.uint16)
    _, row_ptr, col_idx, _ = binding.aggregate_masks(counts, 1, 0.5)
    return row_ptr, col_idx


def _sample_rows(rng, heads, n, per_head):
    rows = []
    for h in heads:
        r = rng.choice(n, size=per_head, replace=False)
        r[0], r[1] = n - 1, 0  # the ragged tail and the first row
        rows.extend(int(h) * n + r)
    return np.array(rows, np.int64)


def test_wan720_attention_sampled_rows(oracle):
    binding = require_gpu()
    wl = synth.WORKLOADS["wan720"]
    dev = torch.device(DEV)
    q, k, v = synth.qkv(wl, 7, device=dev)
    masks = synth.random_block_masks(wl)
    rep = list(wl.repeat_heads)
    sparse = [h for h in range(wl.heads) if h not in rep]
    row_ptr, col_idx = _skiplist(binding, masks, dev)
    work = torch.from_numpy(binding.build_plan(row_ptr.cpu().numpy(), wl.heads, wl.nb,
                                               np.array([h not in rep for h in range(wl.heads)], np.uint8))).to(dev)
    o = torch.zeros_like(q)
    lse = torch.zeros((wl.heads, wl.n), dtype=torch.float32, device=dev)
    binding.sparse_attn_fwd(q, k, v, row_ptr, col_idx, work, o=o, lse=lse)
    binding.repeat_attn_fwd(q, k, v, wl.F, wl.H, wl.W, torch.tensor(rep, dtype=torch.int32, device=dev),
                            wl.k_anchor, o=o, lse=lse)
    assert binding.get_status() == 0
    rng = np.random.default_rng(1)
    for kind, heads in (("sparse", sparse[::8]), ("repeat", rep[::4])):
        for h in heads:
            rows = _sample_rows(rng, [0], wl.n, 24)
            qh, kh, vh = (_bits(t[h:h + 1]) for t in (q, k, v))
            if kind == "sparse":
                o_ref, lse_ref = oracle.masked_attention(qh, kh, vh, masks[h:h + 1], rows=rows)
            else:
                o_ref, lse_ref = oracle.repeat_attention(qh, kh, vh, wl.F, wl.H, wl.W, wl.k_anchor, rows=rows)
            og = o[h].float().cpu().numpy().astype(np.float64)[rows]
            ok, err, bound = attn_tolerance_ok(og, o_ref)
            assert ok, (kind, h, err, bound)
            np.testing.assert_allclose(lse[h].cpu().numpy()[rows], lse_ref, atol=2e-3)


def test_wan480_energy_and_selection_sampled_blockrows(oracle):
    binding = require_gpu()
    wl = synth.WORKLOADS["wan480"]
    dev = torch.device(DEV)
    q, k, _ = synth.qkv(wl, 3, with_v=False, device=dev)
    eps = binding.eps_schedule(0.84, 0.99, 5, 0.5, 1.0)
    E, mask, kept, _ = binding.block_energy(q, k, eps=eps)
    assert binding.get_status() == 0
    E = E.cpu().numpy().astype(np.float64)
    mask = mask.cpu().numpy()
    rng = np.random.default_rng(2)
    for h in rng.choice(wl.heads, size=3, replace=False):
        brs = np.array([wl.nb - 1, 0] + list(rng.choice(wl.nb, size=4, replace=False)), np.int64)
        E_ref = oracle.block_energy(_bits(q[h:h + 1]), _bits(k[h:h + 1]), blockrows=brs)
        assert _energy_ok(E[h][brs], E_ref), h
        # fused selection == oracle selection of the same fp32 energies
        m_same, _, cut = oracle.select(E[h][brs], eps, with_cut=True)
        assert compare_masks(mask[h][brs], m_same, tie_affected(cut, eps, 1e-6))[2] == 0
        m_ref, _, cut_ref = oracle.select(E_ref, eps, with_cut=True)
        assert compare_masks(mask[h][brs], m_ref, tie_affected(cut_ref, eps, independent_tie_window(E_ref)))[2] == 0


def test_calib720_eps_sweep_and_aggregation(oracle):
    binding = require_gpu()
    wl = synth.WORKLOADS["calib720"]
    heads = [0, 17]  # a subset of heads at the full sequence length
    dev = torch.device(DEV)
    rng = np.random.default_rng(3)
    brs = np.array([wl.nb - 1, 0] + list(rng.choice(wl.nb, size=2, replace=False)), np.int64)
    n_in, rho = 16, 0.5
    counts = torch.zeros((len(heads), wl.nb, wl.nb), dtype=torch.uint16, device=dev)
    per_input = []
    for p in range(n_in):
        q, k, _ = synth.qkv(wl, p, heads=heads, with_v=False, device=dev)
        if p == 0:
            E, _, _, _ = binding.block_energy(q, k)
            E = E.cpu().numpy().astype(np.float64)
            E_ref = oracle.block_energy(_bits(q[:1]), _bits(k[:1]), blockrows=brs)
            assert _energy_ok(E[0][brs], E_ref)
            for eps in (0.84, 0.9, 0.95, 0.99):
                _, m, _, _ = binding.block_energy(q, k, eps=eps, energy=False)
                m = m.cpu().numpy()[0][brs]
                m_same, _, cut = oracle.select(E[0][brs], eps, with_cut=True)
                assert compare_masks(m, m_same, tie_affected(cut, eps, 1e-6))[2] == 0
                m_ref, _, cut_ref = oracle.select(E_ref, eps, with_cut=True)
                assert compare_masks(m, m_ref, tie_affected(cut_ref, eps, independent_tie_window(E_ref)))[2] == 0
        m_p = torch.zeros((len(heads), wl.nb, wl.nb), dtype=torch.uint8, device=dev)
        binding.block_energy(q, k, eps=0.9, energy=False, mask=m_p, counts=counts)
        per_input.append(m_p.cpu().numpy())
    assert binding.get_status() == 0
    mask, row_ptr, col_idx, nnz = binding.aggregate_masks(counts, n_in, rho)
    m_ref, c_ref = oracle.aggregate(np.stack(per_input), rho)
    np.testing.assert_array_equal(counts.cpu().numpy().astype(np.int32), c_ref)
    np.testing.assert_array_equal(mask.cpu().numpy(), m_ref)
    rp_ref, ci_ref = oracle.mask_to_csr(m_ref)
    np.testing.assert_array_equal(row_ptr.cpu().numpy(), rp_ref)
    np.testing.assert_array_equal(col_idx.cpu().numpy(), ci_ref)


def test_mochi_calibrated_attention_sampled_rows(oracle):
    binding = require_gpu()
    wl = synth.WORKLOADS["mochi480"]
    dev = torch.device(DEV)
    n_in, eps, rho = 16, 0.84, 0.5
    counts = torch.zeros((wl.heads, wl.nb, wl.nb), dtype=torch.uint16, device=dev)
    for p in range(n_in):
        q, k, _ = synth.qkv(wl, p, with_v=False, device=dev)
        binding.block_energy(q, k, eps=eps, energy=False, counts=counts)
    mask, row_ptr, col_idx, _ = binding.aggregate_masks(counts, n_in, rho)
    assert binding.get_status() == 0
    m = mask.cpu().numpy()
    rep = list(wl.repeat_heads)
    sparse = [h for h in range(wl.heads) if h not in rep]
    sparsity = 1.0 - float(np.mean([m[h].mean() for h in sparse]))
    print(f"mochi calibrated sparsity {sparsity:.3f}")
    work = torch.from_numpy(binding.build_plan(row_ptr.cpu().numpy(), wl.heads, wl.nb,
                                               np.array([h not in rep for h in range(wl.heads)], np.uint8))).to(dev)
    q, k, v = synth.qkv(wl, n_in, device=dev)
    o = torch.zeros_like(q)
    binding.sparse_attn_fwd(q, k, v, row_ptr, col_idx, work, o=o)
    binding.repeat_attn_fwd(q, k, v, wl.F, wl.H, wl.W, torch.tensor(rep, dtype=torch.int32, device=dev),
                            wl.k_anchor, o=o)
    assert binding.get_status() == 0
    rng = np.random.default_rng(4)
    for h in (sparse[0], sparse[11], rep[0], rep[-1]):
        rows = _sample_rows(rng, [0], wl.n, 24)
        qh, kh, vh = (_bits(t[h:h + 1]) for t in (q, k, v))
        if h in rep:
            o_ref, _ = oracle.repeat_attention(qh, kh, vh, wl.F, wl.H, wl.W, wl.k_anchor, rows=rows)
        else:
            o_ref, _ = oracle.masked_attention(qh, kh, vh, m[h:h + 1], rows=rows)
        og = o[h].float().cpu().numpy().astype(np.float64)[rows]
        ok, err, bound = attn_tolerance_ok(og, o_ref)
        assert ok, (h, err, bound)


@pytest.mark.parametrize("name", ["wan720", "mochi480"])
def test_spatial_classification_full_size(oracle, name):
    """Pixel-row profiles and spatial scores of every head: the flagged heads
    (score > 0.87) are exactly the workload's repeated heads; sampled profile
    rows against the oracle; every score against the oracle's score of the
    same profiles."""
    binding = require_gpu()
    wl = synth.WORKLOADS[name]
    dev = torch.device(DEV)
    q, k, _ = synth.qkv(wl, 0, device=dev, with_v=False)
    pix, _ = binding.pixel_row_energy(q, k, wl.F, wl.H, wl.W)
    s, flag = binding.spatial_score(pix, wl.F, wl.H, wl.k_anchor, gamma=0.87)
    assert binding.get_status() == 0
    assert np.nonzero(flag.cpu().numpy())[0].tolist() == list(wl.repeat_heads)
    got = pix.cpu().numpy().astype(np.float64)
    s = s.cpu().numpy()
    for h in range(wl.heads):
        assert abs(s[h] - oracle.spatial_score(got[h], wl.F, wl.H, wl.k_anchor)) <= 1e-5
    rows_per_head = wl.F * wl.H
    heads = [0, wl.repeat_heads[0]]
    sample = np.array([h * rows_per_head + r for h in heads for r in (0, rows_per_head - 1)], np.int64)
    hs = sorted(set(heads))
    ref = oracle.pixel_row_energy(_bits(q[hs].cpu()), _bits(k[hs].cpu()), wl.F, wl.H, wl.W,
                                  prows=np.array([hs.index(int(g // rows_per_head)) * rows_per_head +
                                                  int(g % rows_per_head) for g in sample], np.int64),
                                  threads=min(16, os.cpu_count() or 1))
    assert _energy_ok(got.reshape(-1, got.shape[-1])[sample], ref)


def test_wan720_mixed_launch_equals_separate_calls():
    """The benchmark's step (one launch for the 32 block-sparse and 8 repeated
    heads) gives bit for bit the outputs of the separate calls, whose rows the
    test above checks against the oracle."""
    binding = require_gpu()
    wl = synth.WORKLOADS["wan720"]
    dev = torch.device(DEV)
    q, k, v = synth.qkv(wl, 8, device=dev)
    masks = synth.random_block_masks(wl)
    row_ptr, col_idx = _skiplist(binding, masks, dev)
    rp_h = row_ptr.cpu().numpy()
    rep = list(wl.repeat_heads)
    rep_d = torch.tensor(rep, dtype=torch.int32, device=dev)
    # work lists laid out for this device, as the benchmark's are
    work = torch.from_numpy(binding.balance_plan(
        binding.build_mixed_plan(rp_h, wl.heads, wl.nb, rep, wl.F, wl.H, wl.W), rp_h, wl.heads, wl.nb)).to(dev)
    o, lse = binding.mixed_attn_fwd(q, k, v, wl.F, wl.H, wl.W, row_ptr, col_idx, rep_d, work)
    ha = np.array([h not in rep for h in range(wl.heads)], np.uint8)
    work_s = torch.from_numpy(binding.balance_plan(binding.build_plan(rp_h, wl.heads, wl.nb, ha), rp_h, wl.heads,
                                                   wl.nb)).to(dev)
    o2, lse2 = binding.sparse_attn_fwd(q, k, v, row_ptr, col_idx, work_s)
    binding.repeat_attn_fwd(q, k, v, wl.F, wl.H, wl.W, rep_d, o=o2, lse=lse2)
    assert binding.get_status() == 0
    assert torch.equal(o, o2)
    assert torch.equal(lse, lse2)


def test_wan720_host_buffer_call_equals_device_call():
    """The benchmark's end-to-end call (pinned host q, k, v in, o and lse out,
    pipelined over chunks of 2 heads on two compute streams) returns bit for
    bit the device call's o and lse at the full Wan-720p size."""
    binding = require_gpu()
    wl = synth.WORKLOADS["wan720"]
    dev = torch.device(DEV)
    q, k, v = synth.qkv(wl, 9, device=dev)
    masks = synth.random_block_masks(wl)
    row_ptr, col_idx = _skiplist(binding, masks, dev)
    rp_h = row_ptr.cpu().numpy()
    rep = list(wl.repeat_heads)
    rep_d = torch.tensor(rep, dtype=torch.int32, device=dev)
    work = torch.from_numpy(binding.build_mixed_plan(rp_h, wl.heads, wl.nb, rep, wl.F, wl.H, wl.W)).to(dev)
    o_ref, lse_ref = binding.mixed_attn_fwd(q, k, v, wl.F, wl.H, wl.W, row_ptr, col_idx, rep_d, work)
    o_ref, lse_ref = o_ref.cpu(), lse_ref.cpu()
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((wl.heads, wl.n), dtype=torch.float32).pin_memory()
    bufs = [torch.empty_like(q) for _ in range(4)]
    ld = torch.empty((wl.heads, wl.n), dtype=torch.float32, device=dev)
    binding.mixed_attn_fwd_host(qh, kh, vh, oh, wl.F, wl.H, wl.W, rp_h, row_ptr, col_idx, rep, *bufs, lse_host=lh,
                                lse_dev=ld, heads_per_chunk=2, k_anchor=wl.k_anchor)
    torch.cuda.synchronize()
    assert binding.get_status() == 0
    assert torch.equal(oh, o_ref)
    assert torch.equal(lh, lse_ref)


# ---------------------------------------------------------------- single-pass energy at full size

@pytest.mark.parametrize("name", ["wan720", "wan480", "mochi480"])
def test_single_pass_energy_full_size(oracle, name):
    """calibatt_block_energy_1pass over every head of the workload (the launch
    the benchmark and multi.calibrate_sharded use), checked on sampled
    block-rows of three heads, the ragged last block-row included: energies
    within the bound, the fused selection bit-exact against the oracle's
    selection of the same fp32 energies (ties at 1e-6), against the oracle's
    own energies within the propagated window, the tie flags against the
    oracle's cut description, and counts == mask."""
    binding = require_gpu()
    wl = synth.WORKLOADS[name]
    dev = torch.device(DEV)
    eps = synth.CALIBRATION.get(name, (16, 0.9))[1]
    q, k, _ = synth.qkv(wl, 5, with_v=False, device=dev)
    counts = torch.zeros((wl.heads, wl.nb, wl.nb), dtype=torch.uint16, device=dev)
    mask = torch.empty((wl.heads, wl.nb, wl.nb), dtype=torch.uint8, device=dev)
    E, _, kept, _, _, tie = binding.block_energy_1pass(q, k, eps=eps, mask=mask, kept=torch.empty(
        (wl.heads, wl.nb), dtype=torch.int32, device=dev), counts=counts, tie=True)
    assert binding.get_status() == 0
    np.testing.assert_array_equal(counts.cpu().numpy(), mask.cpu().numpy().astype(np.uint16))
    np.testing.assert_array_equal(kept.cpu().numpy(), mask.cpu().numpy().sum(-1))
    E = E.cpu().numpy().astype(np.float64)
    mask = mask.cpu().numpy()
    tie = tie.cpu().numpy().astype(bool)
    rng = np.random.default_rng(20)
    heads = [0, wl.heads // 2, wl.heads - 1]
    brs = np.array([wl.nb - 1, 0] + list(rng.choice(np.arange(1, wl.nb - 1), size=2, replace=False)), np.int64)
    hs = np.array(heads)
    E_ref = oracle.block_energy(_bits(q[hs]), _bits(k[hs]),
                                blockrows=np.array([i * wl.nb + r for i in range(len(heads)) for r in brs]),
                                threads=_oracle_threads()).reshape(len(heads), len(brs), wl.nb)
    for i, h in enumerate(heads):
        assert _energy_ok(E[h][brs], E_ref[i]), (name, h)
        np.testing.assert_allclose(E[h][brs].sum(-1), 1.0, atol=1e-4)
        m_same, _, cut = oracle.select(E[h][brs], eps, with_cut=True)
        assert compare_masks(mask[h][brs], m_same, tie_affected(cut, eps, SAME_ENERGY_TIE))[2] == 0
        np.testing.assert_array_equal(tie[h][brs], tie_affected(cut, eps, SAME_ENERGY_TIE))
        m_ref, _, cut_ref = oracle.select(E_ref[i], eps, with_cut=True)
        assert compare_masks(mask[h][brs], m_ref, tie_affected(cut_ref, eps, independent_tie_window(E_ref[i])))[2] == 0
    print(f"{name}: {int(tie.sum())} of {tie.size} block-rows tie-affected at 1e-6")


# ---------------------------------------------------------------- Wan-480p end to end

def test_wan480_calibrated_pipeline_end_to_end(oracle):
    """Wan 2.1 14B 480p as the benchmark runs it: 16 calibration inputs at
    eps(T/2) through the single-pass energy kernel with fused selection, the
    per-input masks aggregated at rho = 0.5 into the skip list, then one
    attention call (every head block-sparse) over that skip list in the
    benchmark's launch (mixed plan, balanced). Checked: sampled energy rows of
    two inputs against the oracle; the aggregation (counts, mask, skip list)
    bit-exact against the oracle's aggregation of the GPU's per-input masks;
    sampled output rows of the attention against the oracle's masked attention
    with the calibrated mask."""
    binding = require_gpu()
    wl = synth.WORKLOADS["wan480"]
    dev = torch.device(DEV)
    n_in, eps = synth.CALIBRATION["wan480"]
    rho = 0.5
    counts = torch.zeros((wl.heads, wl.nb, wl.nb), dtype=torch.uint16, device=dev)
    ws = torch.empty(binding.energy_workspace_size(wl.heads, wl.n), dtype=torch.uint8, device=dev)
    per_input, ties = [], 0
    rng = np.random.default_rng(21)
    for p in range(n_in):
        q, k, _ = synth.qkv(wl, p, with_v=False, device=dev)
        m_p = torch.empty((wl.heads, wl.nb, wl.nb), dtype=torch.uint8, device=dev)
        E, _, _, _, _, tie = binding.block_energy_1pass(q, k, eps=eps, energy=p in (0, n_in - 1), mask=m_p,
                                                        counts=counts, ws=ws, tie=True)
        per_input.append(m_p.cpu().numpy())
        ties += int(tie.sum().item())
        if p in (0, n_in - 1):
            h = int(rng.integers(wl.heads))
            brs = np.array([wl.nb - 1, int(rng.integers(wl.nb - 1))], np.int64)
            E_ref = oracle.block_energy(_bits(q[h:h + 1]), _bits(k[h:h + 1]), blockrows=brs,
                                        threads=_oracle_threads())
            Eg = E.cpu().numpy().astype(np.float64)[h][brs]
            assert _energy_ok(Eg, E_ref)
            m_ref, _, cut_ref = oracle.select(E_ref, eps, with_cut=True)
            assert compare_masks(per_input[-1][h][brs], m_ref,
                                 tie_affected(cut_ref, eps, independent_tie_window(E_ref)))[2] == 0
    assert binding.get_status() == 0
    mask, row_ptr, col_idx, nnz = binding.aggregate_masks(counts, n_in, rho)
    m_agg, c_agg = oracle.aggregate(np.stack(per_input), rho)
    np.testing.assert_array_equal(counts.cpu().numpy().astype(np.int32), c_agg)
    np.testing.assert_array_equal(mask.cpu().numpy(), m_agg)
    rp_ref, ci_ref = oracle.mask_to_csr(m_agg)
    np.testing.assert_array_equal(row_ptr.cpu().numpy(), rp_ref)
    np.testing.assert_array_equal(col_idx.cpu().numpy(), ci_ref)
    sparsity = 1.0 - float(m_agg.mean())
    print(f"wan480: calibrated block sparsity {sparsity:.4f}, {ties} tie-affected selections at 1e-6")
    assert 0.5 < sparsity < 0.9
    # attention on a held-out input through the benchmark's launch
    q, k, v = synth.qkv(wl, 1000, device=dev)
    rp_h = row_ptr.cpu().numpy()
    work = torch.from_numpy(binding.balance_plan(
        binding.build_mixed_plan(rp_h, wl.heads, wl.nb, [], wl.F, wl.H, wl.W), rp_h, wl.heads, wl.nb)).to(dev)
    o, lse = binding.mixed_attn_fwd(q, k, v, wl.F, wl.H, wl.W, row_ptr, col_idx,
                                    torch.empty(0, dtype=torch.int32, device=dev), work)
    assert binding.get_status() == 0
    for h in (0, 13, wl.heads - 1):
        rows = _sample_rows(rng, [0], wl.n, 24)
        o_ref, lse_ref = oracle.masked_attention(_bits(q[h:h + 1]), _bits(k[h:h + 1]), _bits(v[h:h + 1]),
                                                 m_agg[h:h + 1], rows=rows, threads=_oracle_threads())
        og = o[h].float().cpu().numpy().astype(np.float64)[rows]
        ok, err, bound = attn_tolerance_ok(og, o_ref)
        assert ok, (h, err, bound)
        np.testing.assert_allclose(lse[h].cpu().numpy()[rows], lse_ref, atol=2e-3)


# ---------------------------------------------------------------- calibration sweep at its own scale

def test_calib720_sweep_40_heads_64_inputs(oracle):
    """The calibration sweep workload at its stated scale: 40 heads of the
    Wan-720p shape, 64 inputs, eps in {0.84, 0.9, 0.95, 0.99}, rho = 0.5. Each
    input's energies come from the single-pass kernel (kept on the device);
    the standalone selection then runs at every eps and folds each mask into
    that eps's counts. Checked per eps: the GPU's counts, aggregated mask and
    skip list bit-exact against the oracle's aggregation of the GPU's
    per-input masks, and the fused selection of the energy kernel equal to the
    standalone one; sampled energy rows of the first and last inputs against
    the oracle, with their selections."""
    binding = require_gpu()
    wl = synth.WORKLOADS["calib720"]
    dev = torch.device(DEV)
    n_in, rho = 64, 0.5
    eps_list = (0.84, 0.9, 0.95, 0.99)
    ws = torch.empty(binding.energy_workspace_size(wl.heads, wl.n), dtype=torch.uint8, device=dev)
    energies = []
    rng = np.random.default_rng(22)
    for p in range(n_in):
        q, k, _ = synth.qkv(wl, p, with_v=False, device=dev)
        m_f = torch.empty((wl.heads, wl.nb, wl.nb), dtype=torch.uint8, device=dev) if p == 1 else None
        E, _, _, _, _ = binding.block_energy_1pass(q, k, eps=0.9 if p == 1 else None, mask=m_f, ws=ws)
        energies.append(E)
        if p == 1:
            m_s, _, _ = binding.select_mask(E, 0.9, kept=False)
            assert torch.equal(m_s, m_f)
        if p in (0, n_in - 1):
            hs = [int(rng.integers(wl.heads)), int(rng.integers(wl.heads))]
            brs = np.array([wl.nb - 1, int(rng.integers(wl.nb - 1))], np.int64)
            E_ref = oracle.block_energy(_bits(q[hs]), _bits(k[hs]),
                                        blockrows=np.array([i * wl.nb + r for i in range(2) for r in brs]),
                                        threads=_oracle_threads())
            Eg = E.cpu().numpy().astype(np.float64)[hs][:, brs].reshape(-1, wl.nb)
            assert _energy_ok(Eg, E_ref)
            for eps in eps_list:
                m_same, _, cut = oracle.select(Eg, eps, with_cut=True)
                m_g, _, _ = binding.select_mask(E, eps, kept=False)
                mg = m_g.cpu().numpy()[hs][:, brs].reshape(-1, wl.nb)
                assert compare_masks(mg, m_same, tie_affected(cut, eps, SAME_ENERGY_TIE))[2] == 0
                m_ref, _, cut_ref = oracle.select(E_ref, eps, with_cut=True)
                assert compare_masks(mg, m_ref, tie_affected(cut_ref, eps, independent_tie_window(E_ref)))[2] == 0
    assert binding.get_status() == 0
    for eps in eps_list:
        counts = torch.zeros((wl.heads, wl.nb, wl.nb), dtype=torch.uint16, device=dev)
        masks = np.empty((n_in, wl.heads, wl.nb, wl.nb), np.uint8)
        ties = 0
        for p in range(n_in):
            m_g, _, _, tie = binding.select_mask(energies[p], eps, kept=False, counts=counts, tie=True)
            masks[p] = m_g.cpu().numpy()
            ties += int(tie.sum().item())
        mask, row_ptr, col_idx, nnz = binding.aggregate_masks(counts, n_in, rho)
        assert binding.get_status() == 0
        m_agg, c_agg = oracle.aggregate(masks, rho)
        np.testing.assert_array_equal(counts.cpu().numpy().astype(np.int32), c_agg)
        np.testing.assert_array_equal(mask.cpu().numpy(), m_agg)
        rp_ref, ci_ref = oracle.mask_to_csr(m_agg)
        np.testing.assert_array_equal(row_ptr.cpu().numpy(), rp_ref)
        np.testing.assert_array_equal(col_idx.cpu().numpy(), ci_ref)
        assert int(nnz.item()) == ci_ref.size
        print(f"calib720 eps={eps}: block sparsity {1 - m_agg.mean():.4f}, {ties} tie-affected selections "
              f"at 1e-6 of {n_in * wl.heads * wl.nb}")
        del masks


def test_aggregate_rows_near_the_cell_limit(oracle):
    """The aggregation's flat indices and ranks are 32-bit (cells <= INT_MAX).
    At 2^21 rows of 1023 columns (2 145 386 496 cells, within 2.1 M of the
    limit; 4.3 GB of counts) every row's kept count is checked against the
    oracle's binarisation, chunk by chunk on the host, and sampled rows (the
    first, last and ones spread between) column by column; the mask is
    compared in full."""
    binding = require_gpu()
    dev = torch.device("cuda")
    rows, cols, n_in = 1 << 21, 1023, 100
    assert rows * cols <= 2**31 - 1
    gen = torch.Generator(device=dev)
    gen.manual_seed(2024)
    # counts in [0, 50]: about 2 % of the cells reach the threshold of 50
    counts = torch.randint(0, 51, (rows, cols), device=dev, dtype=torch.int16, generator=gen).view(torch.uint16)
    cap = 64 << 20
    mask, row_ptr, col_idx, nnz = binding.aggregate_mask_rows(counts, n_in, 0.5, nnz_cap=cap, trim=False)
    torch.cuda.synchronize()
    assert binding.get_status() == 0
    rp = row_ptr.cpu().numpy().astype(np.int64)
    total = int(nnz.item())
    assert rp[0] == 0 and rp[-1] == total and total < cap
    chunk = 1 << 16
    for r0 in range(0, rows, chunk):
        c = counts[r0:r0 + chunk].view(torch.int16).cpu().numpy()
        ref = oracle.binarize_counts(c, n_in, 0.5)
        np.testing.assert_array_equal(mask[r0:r0 + chunk].cpu().numpy(), ref, err_msg=f"rows {r0}+")
        np.testing.assert_array_equal(np.diff(rp[r0:r0 + chunk + 1]), ref.sum(1, dtype=np.int64), err_msg=f"rows {r0}+")
    del c, ref
    rng = np.random.default_rng(7)
    sample = np.unique(np.concatenate([[0, 1, rows // 2, rows - 2, rows - 1], rng.integers(0, rows, 27)]))
    ci = col_idx[:total]
    for r in sample.tolist():
        c = counts[r].view(torch.int16).cpu().numpy()
        ref = oracle.binarize_counts(c[None], n_in, 0.5)[0]
        np.testing.assert_array_equal(mask[r].cpu().numpy(), ref, err_msg=f"row {r}")
        np.testing.assert_array_equal(ci[rp[r]:rp[r + 1]].cpu().numpy(), np.nonzero(ref)[0], err_msg=f"row {r}")
