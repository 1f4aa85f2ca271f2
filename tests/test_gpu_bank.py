"""GPU: the whole calibration flow over (t, l) entries into the mask bank,
then online inference by lookup (explainer §三: calibrate once per
(t, l, h) at eps(t), aggregate at rho, mark spatially repeated heads; online,
look up and run with no decision at run time).

Checks:
* the keep-rate histogram of every entry equals the oracle's histogram of the
  same counts (integer work: exact), and its first moment is the kept total;
* the bank hands back exactly the stored skip list, repeated heads and eps;
* the spatial score marks the workload's repeated head in every entry;
* the attention of each entry, run through the bank, matches the oracle on
  sampled rows of every head with that entry's mask (tolerance of the
  attention parity rule).
"""
import dataclasses

import numpy as np
import pytest
import torch

from calibrated_block_sparse_b200 import synth
from gpu_util import attn_tolerance_ok, bf16_to_f64, require_gpu

pytestmark = pytest.mark.gpu

T, L, N_IN = 3, 2, 4
BASE = synth.Workload("bank", 4, 16, 64, 3, (1,), 5, 20, (1.0, 3.0))  # n = 4096, nb = 32; head 1 repeated


def test_calibrate_into_bank_then_infer_by_lookup(oracle):
    binding = require_gpu()
    dev = torch.device("cuda")
    F, H, W, heads, kk = BASE.F, BASE.H, BASE.W, BASE.heads, BASE.k_anchor
    nb = BASE.nb
    bank = binding.MaskBank(T, L, heads, F, H, W, kk)
    stored = {}
    for t in range(T):
        eps_t = binding.eps_schedule(0.84, 0.99, 5.0, t, T)
        for l in range(L):
            wl = dataclasses.replace(BASE, config_id=BASE.config_id + t * L + l)
            counts = torch.zeros((heads, nb, nb), dtype=torch.uint16, device=dev)
            scores = []
            for p in range(N_IN):
                q, k, _ = synth.qkv(wl, p, with_v=False, device=dev)
                binding.block_energy(q, k, eps=eps_t, energy=False, counts=counts)
                pix, _ = binding.pixel_row_energy(q, k, F, H, W)
                s, _ = binding.spatial_score(pix, F, H, kk, flag=False)
                scores.append(s.cpu().numpy())
            rep = np.nonzero(np.mean(scores, axis=0) > 0.87)[0].tolist()
            assert rep == list(BASE.repeat_heads), (t, l, np.mean(scores, axis=0))
            hist = binding.keep_histogram(counts, N_IN).cpu().numpy()
            c_host = counts.view(torch.int16).cpu().numpy().astype(np.int64) & 0xFFFF
            np.testing.assert_array_equal(hist, oracle.keep_histogram(c_host, N_IN))
            np.testing.assert_array_equal((hist * np.arange(N_IN + 1)).sum(-1), c_host.sum(axis=(1, 2)))
            mask, row_ptr, col_idx, _ = binding.aggregate_masks(counts, N_IN, 0.5)
            bank.put(t, l, eps_t, row_ptr, col_idx, rep)
            stored[(t, l)] = (wl, eps_t, mask.cpu().numpy(), row_ptr.cpu().numpy(), col_idx.cpu().numpy(), rep)
    assert binding.get_status() == 0

    rng = np.random.default_rng(3)
    for (t, l), (wl, eps_t, mask, rp, ci, rep) in stored.items():
        e = bank.get(t, l)
        assert e["eps"] == eps_t
        np.testing.assert_array_equal(e["row_ptr"].cpu().numpy(), rp)
        np.testing.assert_array_equal(e["col_idx"].cpu().numpy(), ci)
        assert e["rep_heads"].cpu().numpy().tolist() == rep
        q, k, v = synth.qkv(wl, 99)
        o, lse = bank.attention(q.to(dev), k.to(dev), v.to(dev), t, l)
        assert binding.get_status() == 0
        og = bf16_to_f64(o)
        n = wl.n
        sparse = [h for h in range(heads) if h not in rep]
        rows = np.concatenate([h * n + rng.choice(n, 48, replace=False) for h in sparse])
        hs = sorted(sparse)
        sub_rows = np.array([hs.index(int(g // n)) * n + int(g % n) for g in rows], np.int64)
        o_ref, _ = oracle.masked_attention(synth.bf16_bits(q[hs]), synth.bf16_bits(k[hs]), synth.bf16_bits(v[hs]),
                                           mask[hs], rows=sub_rows)
        got = og.reshape(-1, og.shape[-1])[rows]
        assert attn_tolerance_ok(got, o_ref)[0], (t, l)
        rrows = np.concatenate([i * n + rng.choice(n, 48, replace=False) for i in range(len(rep))])
        o_rep, _ = oracle.repeat_attention(synth.bf16_bits(q[rep]), synth.bf16_bits(k[rep]),
                                           synth.bf16_bits(v[rep]), F, H, W, k_anchor=kk, rows=rrows)
        got_rep = og[rep].reshape(-1, og.shape[-1])[rrows]
        assert attn_tolerance_ok(got_rep, o_rep)[0], (t, l)
    bank.close()


def test_keep_histogram_matches_oracle_and_reports_bad_counts(oracle):
    binding = require_gpu()
    dev = torch.device("cuda")
    rng = np.random.default_rng(4)
    n_in = 64
    c = rng.integers(0, n_in + 1, size=(5, 591 * 591)).astype(np.int64)
    c[:, :1000] = 0
    c[:, 1000:2000] = n_in
    counts = torch.from_numpy(c.astype(np.int16)).to(dev).view(torch.uint16)
    hist = binding.keep_histogram(counts, n_in).cpu().numpy()
    np.testing.assert_array_equal(hist, oracle.keep_histogram(c, n_in))
    assert binding.get_status() == 0
    bad = counts.clone()
    bad[0, 0] = n_in + 3
    hist = binding.keep_histogram(bad, n_in).cpu().numpy()
    assert binding.get_status() == -1   # reported ...
    assert hist[0].sum() == 591 * 591   # ... and counted in the last bin


def test_bank_lookup_of_a_missing_entry_raises():
    binding = require_gpu()
    bank = binding.MaskBank(2, 2, 1, 2, 8, 16, 5)
    with pytest.raises(binding.CalibattError):
        bank.get(1, 1)
    bank.close()
