"""GPU parity: pixel-row energy profiles and the spatial-similarity score
(explainer §三: a head whose score exceeds gamma = 0.87 is spatially
repeated; §二 observation 4).

Rules:
* profiles: per pixel row |E - E_ref| <= 1e-5 * E_ref + 1e-12 * max_c E_ref,
  the block-energy bound (the same fp32 terms, summed over W rows instead of
  128, in an atomic order);
* block energies written by the same pass: identical to calibatt_block_energy;
* scores: |s - s_ref| <= 1e-4 (cosines of profiles within the bound above);
  flags equal wherever |s_ref - gamma| > 1e-4;
* score of given profiles: within 1e-6 of the fp64 oracle on the same values.
"""
import math

import numpy as np
import pytest
import torch

from calibrated_block_sparse_b200 import synth
from gpu_util import energy_ok, require_gpu

pytestmark = pytest.mark.gpu

GAMMA = 0.87


def _profiles_ok(E, E_ref):
    ok, worst, rel = energy_ok(E, E_ref)
    print(f"profiles: worst error / bound {worst:.3f}, worst relative error {rel:.2e}")
    return ok, worst


def _check_scores(binding, oracle, pix, ref, F, H, k_anchor):
    s, flag = binding.spatial_score(pix, F, H, k_anchor=k_anchor, gamma=GAMMA)
    assert binding.get_status() == 0
    s = s.cpu().numpy().astype(np.float64)
    flag = flag.cpu().numpy()
    s_ref = np.array([oracle.spatial_score(ref[h], F, H, k_anchor) for h in range(ref.shape[0])])
    assert np.all(np.abs(s - s_ref) <= 1e-4), (s, s_ref)
    clear = np.abs(s_ref - GAMMA) > 1e-4
    np.testing.assert_array_equal(flag[clear], (s_ref[clear] > GAMMA).astype(np.uint8))
    return s_ref


# (frames, H, W): W a multiple of 16, W below a warp (many pixel rows per
# warp), W = 1, a Mochi-like odd W, a W wider than a warp; ragged key blocks
@pytest.mark.parametrize("F,H,W,heads,std,seed", [(16, 8, 16, 1, 1.0, 1), (3, 10, 12, 2, 2.0, 2), (2, 6, 53, 1, 1.5, 3),
                                                  (4, 40, 1, 1, 1.0, 4), (2, 5, 80, 2, 2.0, 5)])
def test_pixel_row_energy_and_score_match_oracle(oracle, F, H, W, heads, std, seed):
    binding = require_gpu()
    q, k, _ = synth.plain_qkv(heads, F * H * W, seed=seed, std=std)
    dev = torch.device("cuda")
    qd, kd = q.to(dev), k.to(dev)
    pix, E = binding.pixel_row_energy(qd, kd, F, H, W, energy=True)
    assert binding.get_status() == 0
    ref = oracle.pixel_row_energy(synth.bf16_bits(q), synth.bf16_bits(k), F, H, W)
    got = pix.cpu().numpy().astype(np.float64)
    ok, worst = _profiles_ok(got, ref)
    assert ok, worst
    np.testing.assert_allclose(got.sum(-1), 1.0, atol=1e-4)
    # the block energies of the same pass are those of calibatt_block_energy
    E2, _, _, _ = binding.block_energy(qd, kd)
    assert torch.equal(E, E2)
    _check_scores(binding, oracle, pix, ref, F, H, min(5, H))


def test_positional_workload_profiles_and_score(oracle):
    binding = require_gpu()
    wl = synth.WORKLOADS["tiny"]
    q, k, _ = synth.qkv(wl, 2, with_v=False)
    dev = torch.device("cuda")
    pix, _ = binding.pixel_row_energy(q.to(dev), k.to(dev), wl.F, wl.H, wl.W)
    assert binding.get_status() == 0
    ref = oracle.pixel_row_energy(synth.bf16_bits(q), synth.bf16_bits(k), wl.F, wl.H, wl.W)
    assert _profiles_ok(pix.cpu().numpy().astype(np.float64), ref)[0]
    _check_scores(binding, oracle, pix, ref, wl.F, wl.H, wl.k_anchor)


def test_score_of_given_profiles(oracle):
    binding = require_gpu()
    dev = torch.device("cuda")
    rng = np.random.default_rng(9)
    F, H, nb = 3, 45, 591
    E = rng.dirichlet(np.full(nb, 0.5), size=(2, F * H)).astype(np.float32)
    E[1, 7] = 0.0  # an all-zero profile: its cosine counts as 0
    s, _ = binding.spatial_score(torch.from_numpy(E).to(dev), F, H, k_anchor=5)
    s = s.cpu().numpy()
    for h in range(2):
        assert abs(s[h] - oracle.spatial_score(E[h].astype(np.float64), F, H, 5)) <= 1e-6


def test_score_hand_values_and_threshold():
    binding = require_gpu()
    dev = torch.device("cuda")
    # anchor row 1; cos 0 and 1/sqrt(2): s = 1/(2 sqrt(2))
    E = torch.tensor([[[0.0, 1.0], [1.0, 0.0], [1.0, 1.0]]], device=dev)
    s, flag = binding.spatial_score(E, 1, 3, k_anchor=1, gamma=0.87)
    assert abs(float(s[0]) - 0.5 / math.sqrt(2.0)) <= 1e-6 and int(flag[0]) == 0
    s, flag = binding.spatial_score(E, 1, 3, k_anchor=1, gamma=0.3)
    assert int(flag[0]) == 1
    # every row an anchor: s = 1
    s, _ = binding.spatial_score(E, 1, 3, k_anchor=3)
    assert float(s[0]) == 1.0


def test_repeated_head_is_flagged_mid_workload(oracle):
    # frames of 16 x 64 tokens (8 key blocks each); head 1 is a spatially
    # repeated head of the synthetic recipe (features independent of the row)
    binding = require_gpu()
    wl = synth.Workload("mid", 4, 16, 64, 2, (1,), 5, 6, (1.0, 3.0))
    q, k, _ = synth.qkv(wl, 0, with_v=False)
    dev = torch.device("cuda")
    pix, _ = binding.pixel_row_energy(q.to(dev), k.to(dev), wl.F, wl.H, wl.W)
    assert binding.get_status() == 0
    ref = oracle.pixel_row_energy(synth.bf16_bits(q), synth.bf16_bits(k), wl.F, wl.H, wl.W)
    assert _profiles_ok(pix.cpu().numpy().astype(np.float64), ref)[0]
    s_ref = _check_scores(binding, oracle, pix, ref, wl.F, wl.H, wl.k_anchor)
    assert s_ref[0] < GAMMA < s_ref[1], s_ref
