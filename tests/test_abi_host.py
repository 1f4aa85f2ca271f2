"""Host-side tests of libcalibatt (no GPU work is launched): the library
loads, exports every entry point the header declares, its host helpers agree
with the oracle, and argument errors are caught before anything is enqueued."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "calibatt.h")


@pytest.fixture(scope="module")
def binding():
    from calibrated_block_sparse_b200 import binding as b, build
    build.build()
    b.load()
    return b


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(calibatt_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = _declared()
    for n in ("calibatt_block_energy", "calibatt_select_mask", "calibatt_aggregate_masks",
              "calibatt_sparse_attn_fwd", "calibatt_repeat_attn_fwd"):
        assert n in names


def test_every_declared_symbol_is_exported(binding):
    lib = ctypes.CDLL(binding.library_path())
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_strerror_and_version(binding):
    lib = binding.load()
    assert lib.calibatt_version() >= 100
    for code in range(0, -8, -1):
        assert binding.strerror(code)
    assert binding.strerror(-99) == "unknown status"


def test_eps_schedule_matches_oracle(binding, oracle):
    for t in (0, 10, 25, 49, 50):
        assert binding.eps_schedule(0.84, 0.99, 5, t, 50) == pytest.approx(oracle.eps_schedule(0.84, 0.99, 5, t, 50),
                                                                           abs=1e-15)
    assert abs(binding.eps_schedule(0.84, 0.99, 5, 0.5, 1.0) - 0.852312749793585) < 1e-15


@pytest.mark.parametrize("H,k", [(45, 5), (30, 5), (8, 5), (16, 16), (7, 1), (100, 64)])
def test_anchor_rows_match_oracle(binding, oracle, H, k):
    np.testing.assert_array_equal(binding.anchor_rows(H, k), oracle.anchor_rows(H, k))


def test_rho_threshold_matches_oracle_decisions(binding, oracle):
    for n in (1, 2, 3, 8, 10, 16, 64):
        for rho in (0.0, 0.1, 0.3, 0.5, 0.7, 1 / 3, 0.9999, 1.0, 1.5):
            thr = binding.rho_threshold(n, rho)
            counts = np.arange(n + 1, dtype=np.int32)
            ref = oracle.binarize_counts(counts, n, rho)
            np.testing.assert_array_equal((counts >= thr).astype(np.uint8), ref)


def test_validate_csr(binding, oracle):
    rng = np.random.default_rng(1)
    mask = (rng.random((2, 9, 9)) < 0.4).astype(np.uint8)
    rp, ci = oracle.mask_to_csr(mask)
    assert binding.validate_csr(rp, ci, 2, 9) == 0
    bad = ci.copy()
    bad[0] = 9
    assert binding.validate_csr(rp, bad, 2, 9) == -2
    if ci.size > 1 and rp[1] - rp[0] > 1:
        dup = ci.copy()
        dup[1] = dup[0]
        assert binding.validate_csr(rp, dup, 2, 9) == -2
    rp2 = rp.copy()
    rp2[3] = rp2[4] + 1
    assert binding.validate_csr(rp2, ci, 2, 9) == -2


def test_build_plan_is_head_by_head_longest_first(binding, oracle):
    rng = np.random.default_rng(2)
    mask = (rng.random((3, 7, 7)) < rng.random((3, 1, 1))).astype(np.uint8)
    rp, _ = oracle.mask_to_csr(mask)
    work = binding.build_plan(rp, 3, 7)
    nnz = np.diff(rp)
    assert sorted(work.tolist()) == list(range(21))
    heads = work // 7
    assert heads.tolist() == sorted(heads.tolist())  # head by head, in index order
    for h in range(3):
        w = work[heads == h]
        assert np.all(np.diff(nnz[w]) <= 0)  # longest first inside a head
        for a, b in zip(w, w[1:]):
            if nnz[a] == nnz[b]:
                assert a < b  # ties keep block order
    work = binding.build_plan(rp, 3, 7, head_active=np.array([0, 1, 0], np.uint8))
    assert sorted(work.tolist()) == list(range(7, 14))


def test_argument_errors_are_caught_on_the_host(binding):
    lib = binding.load()
    P = ctypes.c_void_p
    fake = P(0x100000)       # aligned, never dereferenced: calls must fail first
    odd = P(0x100008)        # 8-byte aligned only
    # head dim other than 128
    assert lib.calibatt_sparse_attn_fwd(fake, fake, fake, 1, 256, 64, 0.1, fake, fake, 4, fake, 2, fake, None,
                                        None) == -4
    # misaligned q
    assert lib.calibatt_sparse_attn_fwd(odd, fake, fake, 1, 256, 128, 0.1, fake, fake, 4, fake, 2, fake, None,
                                        None) == -3
    # non-positive scale, missing row_ptr, bad sizes
    assert lib.calibatt_sparse_attn_fwd(fake, fake, fake, 1, 256, 128, 0.0, fake, fake, 4, fake, 2, fake, None,
                                        None) == -1
    assert lib.calibatt_sparse_attn_fwd(fake, fake, fake, 1, 256, 128, 0.1, None, fake, 4, fake, 2, fake, None,
                                        None) == -1
    assert lib.calibatt_sparse_attn_fwd(fake, fake, fake, 0, 256, 128, 0.1, fake, fake, 4, fake, 2, fake, None,
                                        None) == -1
    assert lib.calibatt_sparse_attn_fwd(fake, fake, fake, 1, 256, 128, 0.1, fake, fake, 4, fake, 3, fake, None,
                                        None) == -1
    # repeat: k larger than H, workspace too small, too many anchors
    assert lib.calibatt_repeat_attn_fwd(fake, fake, fake, 2, 2, 4, 8, 128, 5, 0.1, fake, 1, fake, None, fake,
                                        1 << 30, None) == -1
    assert lib.calibatt_repeat_attn_fwd(fake, fake, fake, 2, 2, 8, 8, 128, 5, 0.1, fake, 1, fake, None, fake,
                                        16, None) == -1
    assert lib.calibatt_repeat_attn_fwd(fake, fake, fake, 2, 2, 80, 8, 128, 70, 0.1, fake, 1, fake, None, fake,
                                        1 << 30, None) == -4
    # calibration beyond 1024 blocks per row
    assert lib.calibatt_block_energy(fake, fake, 1, 1025 * 128, 128, 0.1, fake, None, 0, 0.0, None, None, None,
                                     None, 0.0, None) == -4
    assert lib.calibatt_block_energy(fake, fake, 1, 1024, 128, 0.1, fake, None, 1, 0.9, None, None, None,
                                     None, 0.0, None) == -1  # fused selection with no output
    assert lib.calibatt_block_energy(fake, fake, 1, 1024, 128, 0.1, fake, None, 1, 0.9, None, None, None,
                                     fake, float("nan"), None) == -1
    assert lib.calibatt_select_mask(fake, 1, 2000, 0.9, fake, None, None, None, 0.0, None) == -4
    assert lib.calibatt_select_mask(fake, 1, 16, 0.9, None, None, None, None, 0.0, None) == -1
    assert lib.calibatt_select_mask(fake, 1, 16, float("nan"), fake, None, None, None, 0.0, None) == -1
    assert lib.calibatt_select_mask(fake, 1, 16, 0.9, None, None, None, fake, float("nan"), None) == -1
    # the wait limit: NaN and more than a minute are refused before any device call
    assert lib.calibatt_set_wait_limit(float("nan")) == -1
    assert lib.calibatt_set_wait_limit(61.0) == -1
    # aggregation: short workspace, zero inputs
    assert lib.calibatt_aggregate_masks(fake, 4, 1, 16, 0.5, fake, fake, fake, 256, fake, fake, 4, None) == -1
    assert lib.calibatt_aggregate_masks(fake, 0, 1, 16, 0.5, fake, fake, fake, 256, fake, fake, 1024, None) == -1
    assert lib.calibatt_accumulate_masks(None, 10, fake, None) == -1
    # pixel-row profiles and the spatial score
    odd2 = P(0x100002)       # 2-byte aligned only
    assert lib.calibatt_pixel_row_energy(fake, fake, 1, 0, 8, 16, 128, 0.1, fake, None, fake, None) == -1
    assert lib.calibatt_pixel_row_energy(fake, fake, 1, 2, 8, 16, 64, 0.1, fake, None, fake, None) == -4
    assert lib.calibatt_pixel_row_energy(fake, fake, 1, 1025, 8, 16, 128, 0.1, fake, None, fake, None) == -4
    assert lib.calibatt_pixel_row_energy(fake, fake, 1, 2, 8, 16, 128, 0.1, fake, None, None, None) == -1
    assert lib.calibatt_pixel_row_energy(fake, fake, 1, 2, 8, 16, 128, 0.1, fake, None, odd2, None) == -3
    assert lib.calibatt_spatial_score(fake, 1, 2, 600, 16, 5, 0.87, fake, None, None) == -4
    assert lib.calibatt_spatial_score(fake, 1, 2, 4, 16, 5, 0.87, fake, None, None) == -1
    assert lib.calibatt_spatial_score(fake, 1, 2, 8, 16, 5, float("nan"), fake, None, None) == -1
    assert lib.calibatt_spatial_score(fake, 1, 2, 8, 16, 5, 0.87, None, None, None) == -1
    assert lib.calibatt_spatial_score(odd2, 1, 2, 8, 16, 5, 0.87, fake, None, None) == -3
    # mixed launch: too many units, k above H, missing workspace
    assert lib.calibatt_mixed_attn_fwd(fake, fake, fake, 2, 2, 8, 16, 128, 5, 0.1, fake, fake, 4, fake, 1, fake,
                                       100, fake, None, fake, 1 << 30, None) == -1
    assert lib.calibatt_mixed_attn_fwd(fake, fake, fake, 2, 2, 4, 16, 128, 5, 0.1, fake, fake, 4, fake, 1, fake,
                                       2, fake, None, fake, 1 << 30, None) == -1
    assert lib.calibatt_mixed_attn_fwd(fake, fake, fake, 2, 2, 8, 16, 128, 5, 0.1, fake, fake, 4, fake, 1, fake,
                                       2, fake, None, None, 0, None) == -1


def test_mixed_plan_orders_both_kinds_of_units(binding):
    # 3 heads, nb = 4; head 1 repeated; F*k*W = 2*5*30 = 300 anchor queries -> 3 anchor blocks
    heads, nb, F, H, W, kk = 3, 4, 2, 10, 30, 5
    counts = np.array([[4, 0, 2, 1], [9, 9, 9, 9], [3, 4, 1, 4]], np.int32)
    row_ptr = np.concatenate([[0], np.cumsum(counts.reshape(-1))]).astype(np.int32)
    work = binding.build_mixed_plan(row_ptr, heads, nb, [1], F, H, W, kk)
    # head 1's anchor units, then head 0 and head 2 longest first (ties in block order)
    assert work.tolist() == [12, 13, 14, 0, 2, 3, 1, 9, 11, 8, 10]
    # no repeated heads: the plain plan
    plain = binding.build_mixed_plan(row_ptr, heads, nb, [], F, H, W, kk)
    np.testing.assert_array_equal(plain, binding.build_plan(row_ptr, heads, nb))


def test_bank_index_on_the_host(binding):
    lib = binding.load()
    P = ctypes.c_void_p
    assert not lib.calibatt_bank_create(0, 2, 4, 2, 8, 16, 5)
    assert not lib.calibatt_bank_create(2, 2, 4, 2, 4, 16, 5)  # k above H
    b = lib.calibatt_bank_create(3, 2, 2, 2, 8, 16, 5)  # n = 256: nb = 2
    assert b
    try:
        # [row_ptr 5 ints | col_idx 3 | work 4 + 2 anchor units | rep 1], each on 256 B
        assert lib.calibatt_bank_entry_bytes(b, 3, 1) == 256 * 4
        assert lib.calibatt_bank_entry_bytes(b, 3, 5) == 0
        e = binding.BankEntry()
        assert lib.calibatt_bank_get(b, 0, 0, ctypes.byref(e)) == -1  # never stored
        assert lib.calibatt_bank_get(b, 3, 0, ctypes.byref(e)) == -1  # out of range
        fake = P(0x100000)
        rp = np.array([0, 1, 2, 2, 3], np.int32)
        put = lambda rp_, dst, nbytes, t=0: lib.calibatt_bank_put(b, t, 0, 0.9, binding._ptr(rp_), fake, 3, None, 0,
                                                                  dst, nbytes, None)
        assert put(np.array([0, 1, 2, 2, 4], np.int32), fake, 4096) == -2  # row_ptr does not end at nnz
        assert put(rp, P(0x100010), 4096) == -3                            # dst not 256-byte aligned
        assert put(rp, fake, 16) == -1                                     # dst too small
        assert put(rp, fake, 4096, t=3) == -1                              # t out of range
    finally:
        lib.calibatt_bank_destroy(b)
    # single-pass energy: short workspace, pixel rows that do not divide n
    assert lib.calibatt_block_energy_1pass(P(0x100000), P(0x100000), 1, 4096, 128, 0.1, P(0x100000), 16, None, 0,
                                           0.0, None, None, None, None, 0.0, None, 0, None) == -1
    assert lib.calibatt_block_energy_1pass(P(0x100000), P(0x100000), 1, 4096, 128, 0.1, P(0x100000), 1 << 40,
                                           None, 0, 0.0, None, None, None, None, 0.0, P(0x100000), 100, None) == -1
    # host-buffer pipeline: short workspace, missing host buffer
    assert lib.calibatt_mixed_attn_fwd_host(fake, fake, fake, fake, None, 2, 2, 8, 16, 128, 5, 0.1, fake, fake, fake,
                                            4, None, 0, 8, fake, fake, fake, fake, None, fake, 4, None) == -1
    assert lib.calibatt_mixed_attn_fwd_host(None, fake, fake, fake, None, 2, 2, 8, 16, 128, 5, 0.1, fake, fake, fake,
                                            4, None, 0, 8, fake, fake, fake, fake, None, fake, 1 << 30, None) == -1
    # anchor-row masks: missing anchor skip list, bad sizes, short workspace
    assert lib.calibatt_mixed_masked_attn_fwd(fake, fake, fake, 2, 2, 8, 16, 128, 5, 0.1, fake, fake, 4, fake, 1,
                                              None, None, 0, fake, 2, fake, None, fake, 1 << 30, None) == -1
    assert lib.calibatt_anchor_energy_workspace_size(2, 3, 2, 8, 16, 5) == 0      # more repeated heads than heads
    assert lib.calibatt_anchor_energy_workspace_size(2, 1, 2, 8, 16, 9) == 0      # k above H
    assert lib.calibatt_anchor_block_energy(fake, fake, 2, 2, 8, 16, 128, 5, 0.1, fake, 1, fake, 16, None, 1, 0.9,
                                            fake, None, None, None, 0.0, None) == -1
    assert lib.calibatt_anchor_block_energy(fake, fake, 2, 2, 8, 16, 128, 5, 0.1, None, 1, fake, 1 << 30, None, 0,
                                            0.9, None, None, None, None, 0.0, None) == -1
    assert lib.calibatt_aggregate_rows_workspace_size(0) == 0
    assert lib.calibatt_aggregate_mask_rows(fake, 4, 10, 16, 0.5, fake, fake, fake, 160, fake, fake, 4, None) == -1
    assert lib.calibatt_aggregate_mask_rows(fake, 4, 0, 16, 0.5, fake, fake, fake, 160, fake, fake, 4096, None) == -1
    # keep-rate histogram arguments
    assert lib.calibatt_keep_histogram(P(0x100000), 1, 16, 0, P(0x100000), None) == -1
    assert lib.calibatt_keep_histogram(P(0x100000), 1, 16, 8, P(0x100004), None) == -3


def test_head_sharding_balances_and_partitions(binding, oracle):
    from calibrated_block_sparse_b200 import synth
    wl = synth.WORKLOADS["wan720"]
    masks = synth.random_block_masks(wl)
    row_ptr, _ = oracle.mask_to_csr(masks)
    rep = list(wl.repeat_heads)
    full = binding.build_mixed_plan(row_ptr, wl.heads, wl.nb, rep, wl.F, wl.H, wl.W)
    cost = [int(row_ptr[(h + 1) * wl.nb] - row_ptr[h * wl.nb]) for h in range(wl.heads)]
    for h in rep:
        cost[h] = -(-wl.F * 5 * wl.W // 128) * wl.nb
    for n_ranks in (1, 2, 4, 8):
        owner, load = binding.shard_heads(row_ptr, wl.heads, wl.nb, rep, wl.F, wl.W, 5, n_ranks)
        assert owner.min() >= 0 and owner.max() < n_ranks
        np.testing.assert_array_equal(load, [sum(c for h, c in enumerate(cost) if owner[h] == r) for r in range(n_ranks)])
        assert load.max() <= sum(cost) / n_ranks + max(cost)  # greedy longest-first bound
        # the ranks' work lists partition the units of the whole call
        units = []
        for r in range(n_ranks):
            w, rep_r = binding.build_rank_plan(row_ptr, wl.heads, wl.nb, rep, owner, r, wl.F, wl.H, wl.W)
            assert all(owner[h] == r for h in rep_r)
            nbq_b = -(-wl.F * 5 * wl.W // 128)
            base = wl.heads * wl.nb
            # anchor codes are local to the rank's repeated-head list: map them back
            units += [int(u) if u < base else base + rep.index(rep_r[(u - base) // nbq_b]) * nbq_b + (u - base) % nbq_b
                      for u in w]
        assert sorted(units) == sorted(full.tolist())


def test_workspace_sizes(binding):
    lib = binding.load()
    assert binding.repeat_workspace_size(8, 21, 45, 80, 5) == 8 * 21 * 5 * 80 * 256
    assert lib.calibatt_aggregate_workspace_size(40, 591) >= 40 * 591 * 4
    assert lib.calibatt_aggregate_workspace_size(0, 5) == 0
    # host-buffer call: two anchor buffers (consecutive chunks may run at once)
    # of min(heads per chunk, repeated heads) heads each, then every chunk's lists
    nb = (21 * 45 * 80 + 127) // 128
    anchors = binding.repeat_workspace_size(2, 21, 45, 80, 5)
    lists = (40 * nb + 8 * (-(-21 * 5 * 80 // 128)) + 8) * 4
    assert lib.calibatt_mixed_host_workspace_size(40, 21, 45, 80, 5, 8, 2) == 2 * anchors + (-(-lists // 256)) * 256
    assert lib.calibatt_mixed_host_workspace_size(40, 21, 45, 80, 5, 8, 0) == \
        lib.calibatt_mixed_host_workspace_size(40, 21, 45, 80, 5, 8, 2)
    assert lib.calibatt_mixed_host_workspace_size(40, 21, 45, 80, 6, 8, 2) > 0
    assert lib.calibatt_mixed_host_workspace_size(40, 21, 45, 80, 46, 8, 2) == 0  # k above H


def test_no_cpu_fallback_when_library_missing(monkeypatch, tmp_path):
    from calibrated_block_sparse_b200 import binding as b
    monkeypatch.setattr(b, "_lib", None)
    monkeypatch.setattr(b, "library_path", lambda: str(tmp_path / "absent.so"))
    with pytest.raises(ImportError):
        b.load()


def _slot_loads(work, cost, n_slots):
    """Per-slot work under the kernels' static schedule: G = 2*min(n_slots/2,
    ceil(n/2)) slots; slot g takes entry t*G + g in even rounds t and
    t*G + G-1-g in odd ones."""
    n = len(work)
    G = 2 * min(n_slots // 2, (n + 1) // 2)
    load = np.zeros(G, np.int64)
    for i, code in enumerate(work):
        t, q = divmod(i, G)
        g = q if t % 2 == 0 else G - 1 - q
        load[g] += cost[code]
    return load, G


@pytest.mark.parametrize("n_slots,seed", [(296, 1), (16, 2), (6, 3), (296, 4)])
def test_balance_plan_permutes_within_rounds_and_evens_slot_loads(binding, n_slots, seed):
    rng = np.random.default_rng(seed)
    heads, nb = 7, 61
    # heads of very different density, as calibrated masks give
    kept = np.concatenate([rng.binomial(nb, p, nb) for p in rng.uniform(0.02, 0.9, heads)]).astype(np.int32)
    row_ptr = np.concatenate([[0], np.cumsum(kept)]).astype(np.int32)
    n_rep_units = 9  # anchor-query unit codes after the block-sparse ones
    work = binding.build_plan(row_ptr, heads, nb)
    work = np.concatenate([heads * nb + np.arange(n_rep_units, dtype=np.int32), work])
    cost = np.concatenate([kept + 2, np.full(n_rep_units, nb + 2)])
    out = binding.balance_plan(work, row_ptr, heads, nb, n_slots)
    assert sorted(out.tolist()) == sorted(work.tolist())
    load0, G = _slot_loads(work, cost, n_slots)
    load1, _ = _slot_loads(out, cost, n_slots)
    for r in range(0, len(work), G):  # every round keeps its own entries
        assert sorted(out[r:r + G].tolist()) == sorted(work[r:r + G].tolist())
    # matching the costliest unit of a round to the least-loaded slot keeps
    # the spread within one unit's cost over the full rounds, two with the
    # last, partial round
    assert load1.max() - load1.min() <= 2 * cost.max()
    assert load1.max() <= load0.max()
    assert load1.sum() == load0.sum()


def test_balance_plan_edge_cases(binding):
    rp = np.array([0, 3, 3, 4], np.int32)
    assert binding.balance_plan(np.zeros(0, np.int32), rp, 1, 3, 8).size == 0
    w = np.array([2, 0, 1], np.int32)
    assert sorted(binding.balance_plan(w, rp, 1, 3, 2).tolist()) == [0, 1, 2]  # one CTA: two slots
    lib = binding.load()
    assert lib.calibatt_balance_plan(binding._ptr(w), 3, binding._ptr(rp), 1, 3, 1) == -1  # fewer than 2 slots
    assert lib.calibatt_balance_plan(None, 3, binding._ptr(rp), 1, 3, 8) == -1


def test_balance_mixed_plan_costs_anchor_units_by_their_skip_list(binding):
    """Anchor units with few kept blocks weigh less: the balanced list is a
    permutation within rounds, and with two slots the heavy anchor unit and
    the light ones are spread so that both slots carry similar work."""
    heads, nb, F, W, kk = 2, 4, 1, 256, 1   # one repeated head: 2 anchor blocks
    rp = np.array([0, 4, 8, 12, 16, 20, 24, 28, 32], np.int32)  # every block kept
    rpb = np.array([0, 4, 5], np.int32)   # anchor block 0 keeps 4 blocks, block 1 keeps 1
    work = binding.build_mixed_plan(rp, heads, nb, [1], F, 4, W, kk)
    assert sorted(work.tolist()) == sorted(list(range(0, 4)) + [heads * nb, heads * nb + 1])
    bal = binding.balance_mixed_plan(work, rp, heads, nb, rpb, 1, F, W, kk, n_slots=2)
    assert sorted(bal.tolist()) == sorted(work.tolist())
    with pytest.raises(binding.CalibattError):
        binding.balance_mixed_plan(work, rp, heads, nb, None, 1, F, W, kk, n_slots=2)
