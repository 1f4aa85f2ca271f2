"""GPU parity: block-sparse and repeated-head attention through the C ABI,
element by element against the fp64 oracle on the same bf16 inputs.

Tolerance (stated by the method's parity rule for bf16 inputs with fp32
accumulation): max|O - O_ref| <= 1e-2 * max|O_ref| + 1e-3.
"""
import math

import numpy as np
import pytest
import torch

from calibrated_block_sparse_b200 import synth
from gpu_util import attn_tolerance_ok, bf16_to_f64, require_gpu

pytestmark = pytest.mark.gpu


def _run_sparse(binding, q, k, v, mask):
    import oracle
    heads, nb, _ = mask.shape
    row_ptr, col_idx = oracle.mask_to_csr(mask)  # the reference skip list
    assert binding.validate_csr(row_ptr, col_idx, heads, nb) == 0
    work = binding.build_plan(row_ptr, heads, nb)
    dev = torch.device("cuda")
    o, lse = binding.sparse_attn_fwd(q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(row_ptr).to(dev),
                                     torch.from_numpy(col_idx).to(dev), torch.from_numpy(work).to(dev))
    assert binding.get_status() == 0
    return bf16_to_f64(o), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("heads,n,keep,seed", [
    (1, 2048, 0.4, 1),     # the tiny workload's shape: 16 blocks
    (2, 300, 0.6, 2),      # ragged: last block 44 rows
    (3, 1000, 0.3, 3),     # ragged: last block 104 rows, several tiles per CTA slot
    (2, 128, 1.0, 4),      # a single block
    (1, 4096 + 80, 0.25, 5),  # 33 blocks, last 80 rows (Wan-720p's tail)
])
def test_sparse_attention_matches_oracle(oracle, heads, n, keep, seed):
    binding = require_gpu()
    q, k, v = synth.plain_qkv(heads, n, seed=seed, std=1.5)
    nb = (n + 127) // 128
    mask = synth.random_mask(heads, nb, keep, seed=seed)
    o, lse = _run_sparse(binding, q, k, v, mask)
    o_ref, lse_ref = oracle.masked_attention(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), mask)
    ok, err, bound = attn_tolerance_ok(o, o_ref)
    assert ok, (err, bound)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=2e-3)


def test_all_ones_mask_is_dense_attention(oracle):
    binding = require_gpu()
    q, k, v = synth.plain_qkv(2, 700, seed=7)
    nb = 6
    o, lse = _run_sparse(binding, q, k, v, np.ones((2, nb, nb), np.uint8))
    o_ref, _ = oracle.masked_attention(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v),
                                       np.ones((2, nb, nb), np.uint8))
    assert attn_tolerance_ok(o, o_ref)[0]


def test_empty_rows_and_large_scores(oracle):
    binding = require_gpu()
    # large-magnitude scores exercise the running-max rescale; an empty row
    # must come out as O = 0, lse = -inf
    q, k, v = synth.plain_qkv(1, 640, seed=8, std=4.0)
    mask = synth.random_mask(1, 5, 0.5, seed=8)
    mask[0, 2] = 0
    o, lse = _run_sparse(binding, q, k, v, mask)
    o_ref, lse_ref = oracle.masked_attention(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), mask)
    assert attn_tolerance_ok(o, o_ref)[0]
    assert np.all(o[0, 256:384] == 0) and np.all(np.isneginf(lse[0, 256:384]))


def test_rows_of_other_heads_untouched():
    binding = require_gpu()
    import oracle
    q, k, v = synth.plain_qkv(3, 256, seed=9)
    mask = np.ones((3, 2, 2), np.uint8)
    row_ptr, col_idx = oracle.mask_to_csr(mask)
    work = binding.build_plan(row_ptr, 3, 2, head_active=np.array([1, 0, 1], np.uint8))
    assert len(work) == 4
    dev = torch.device("cuda")
    o = torch.full((3, 256, 128), 7.0, dtype=torch.bfloat16, device=dev)
    binding.sparse_attn_fwd(q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(row_ptr).to(dev),
                            torch.from_numpy(col_idx).to(dev), torch.from_numpy(work).to(dev), o=o)
    assert binding.get_status() == 0
    assert torch.all(o[1] == 7.0)
    assert not torch.any(o[0] == 7.0)


@pytest.mark.parametrize("F,H,W,kk", [(3, 8, 16, 5), (2, 6, 20, 6), (2, 30, 5, 5), (4, 5, 9, 2)])
def test_repeat_attention_matches_oracle(oracle, F, H, W, kk):
    binding = require_gpu()
    heads = 3
    n = F * H * W
    q, k, v = synth.plain_qkv(heads, n, seed=10 + H)
    rep = [0, 2]
    dev = torch.device("cuda")
    o = torch.zeros((heads, n, 128), dtype=torch.bfloat16, device=dev)
    o, lse = binding.repeat_attn_fwd(q.to(dev), k.to(dev), v.to(dev), F, H, W,
                                     torch.tensor(rep, dtype=torch.int32, device=dev), k_anchor=kk, o=o)
    assert binding.get_status() == 0
    o_ref, lse_ref = oracle.repeat_attention(synth.bf16_bits(q[rep]), synth.bf16_bits(k[rep]),
                                             synth.bf16_bits(v[rep]), F, H, W, k_anchor=kk)
    og = bf16_to_f64(o)
    ok, err, bound = attn_tolerance_ok(og[rep], o_ref)
    assert ok, (err, bound)
    np.testing.assert_allclose(lse.cpu().numpy()[rep], lse_ref, rtol=0, atol=2e-3)
    assert np.all(og[1] == 0)  # not a repeat head: untouched
    # rows of one band are exact copies of their anchor row
    a = binding.anchor_rows(H, kk)
    for f in range(F):
        for r in range(H):
            j = int(np.argmin(np.abs(r - a)))
            src = f * H * W + int(a[j]) * W
            dst = f * H * W + r * W
            assert np.array_equal(og[rep, dst:dst + W], og[rep, src:src + W])


def test_repeat_with_every_row_an_anchor_is_plain_attention(oracle):
    binding = require_gpu()
    F, H, W = 2, 8, 24
    n = F * H * W
    q, k, v = synth.plain_qkv(1, n, seed=12)
    dev = torch.device("cuda")
    o, _ = binding.repeat_attn_fwd(q.to(dev), k.to(dev), v.to(dev), F, H, W,
                                   torch.zeros(1, dtype=torch.int32, device=dev), k_anchor=H)
    nb = (n + 127) // 128
    o_ref, _ = oracle.masked_attention(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v),
                                       np.ones((1, nb, nb), np.uint8))
    assert attn_tolerance_ok(bf16_to_f64(o), o_ref)[0]


def test_malformed_skip_list_is_reported_not_faulted():
    binding = require_gpu()
    import oracle
    q, k, v = synth.plain_qkv(1, 256, seed=13)
    mask = np.ones((1, 2, 2), np.uint8)
    row_ptr, col_idx = oracle.mask_to_csr(mask)
    bad = col_idx.copy()
    bad[1] = 57  # column out of range
    assert binding.validate_csr(row_ptr, bad, 1, 2) != 0
    dev = torch.device("cuda")
    binding.get_status()
    binding.sparse_attn_fwd(q.to(dev), k.to(dev), v.to(dev), torch.from_numpy(row_ptr).to(dev),
                            torch.from_numpy(bad).to(dev), torch.tensor([0, 1], dtype=torch.int32, device=dev))
    assert binding.get_status() == -2  # CALIBATT_ERR_CSR
    assert binding.get_status() == 0   # cleared


@pytest.mark.parametrize("F,H,W,kk,keep,seed", [(3, 8, 16, 5, 0.4, 1), (2, 30, 5, 5, 0.5, 2), (4, 5, 9, 2, 0.3, 3),
                                                (2, 45, 8, 5, 0.35, 4)])
def test_mixed_launch_matches_oracle_and_separate_calls(oracle, F, H, W, kk, keep, seed):
    """Block-sparse and repeated heads in one persistent launch: each head
    against the oracle, and bit for bit the outputs of the two separate calls
    (a unit's arithmetic does not depend on which slot runs it)."""
    binding = require_gpu()
    heads = 4
    n = F * H * W
    nb = (n + 127) // 128
    q, k, v = synth.plain_qkv(heads, n, seed=40 + seed)
    rng = np.random.default_rng(seed)
    mask = (rng.random((heads, nb, nb)) < keep).astype(np.uint8)
    mask[:, np.arange(nb), np.arange(nb)] = 1
    rep = [1, 3]
    sparse = [0, 2]
    row_ptr, col_idx = oracle.mask_to_csr(mask)
    work = binding.build_mixed_plan(row_ptr, heads, nb, rep, F, H, W, kk)
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    rp_d, ci_d = torch.from_numpy(row_ptr).to(dev), torch.from_numpy(col_idx).to(dev)
    rep_d = torch.tensor(rep, dtype=torch.int32, device=dev)
    o, lse = binding.mixed_attn_fwd(qd, kd, vd, F, H, W, rp_d, ci_d, rep_d, torch.from_numpy(work).to(dev),
                                    k_anchor=kk)
    assert binding.get_status() == 0
    # against the oracle
    og = bf16_to_f64(o)
    o_ref, lse_ref = oracle.masked_attention(synth.bf16_bits(q[sparse]), synth.bf16_bits(k[sparse]),
                                             synth.bf16_bits(v[sparse]), mask[sparse])
    assert attn_tolerance_ok(og[sparse], o_ref)[0]
    o_rep, lse_rep = oracle.repeat_attention(synth.bf16_bits(q[rep]), synth.bf16_bits(k[rep]),
                                             synth.bf16_bits(v[rep]), F, H, W, k_anchor=kk)
    assert attn_tolerance_ok(og[rep], o_rep)[0]
    np.testing.assert_allclose(lse.cpu().numpy()[rep], lse_rep, rtol=0, atol=2e-3)
    # against the two separate calls, bit for bit
    ha = np.ones(heads, np.uint8)
    ha[rep] = 0
    work_s = torch.from_numpy(binding.build_plan(row_ptr, heads, nb, head_active=ha)).to(dev)
    o2 = torch.zeros_like(qd)
    lse2 = torch.zeros((heads, n), dtype=torch.float32, device=dev)
    binding.sparse_attn_fwd(qd, kd, vd, rp_d, ci_d, work_s, o=o2, lse=lse2)
    binding.repeat_attn_fwd(qd, kd, vd, F, H, W, rep_d, k_anchor=kk, o=o2, lse=lse2)
    assert binding.get_status() == 0
    assert torch.equal(o, o2)
    assert torch.equal(lse, lse2)


def test_mixed_launch_without_repeated_heads_is_the_sparse_call(oracle):
    binding = require_gpu()
    F, H, W, heads = 2, 8, 16, 2
    n = F * H * W
    nb = (n + 127) // 128
    q, k, v = synth.plain_qkv(heads, n, seed=60)
    mask = np.ones((heads, nb, nb), np.uint8)
    mask[0, 0, 1] = 0
    row_ptr, col_idx = oracle.mask_to_csr(mask)
    dev = torch.device("cuda")
    args = [t.to(dev) for t in (q, k, v)]
    rp_d, ci_d = torch.from_numpy(row_ptr).to(dev), torch.from_numpy(col_idx).to(dev)
    work = torch.from_numpy(binding.build_mixed_plan(row_ptr, heads, nb, [], F, H, W)).to(dev)
    o, lse = binding.mixed_attn_fwd(*args, F, H, W, rp_d, ci_d, torch.zeros(0, dtype=torch.int32, device=dev), work)
    o2, lse2 = binding.sparse_attn_fwd(*args, rp_d, ci_d, torch.from_numpy(binding.build_plan(row_ptr, heads, nb)).to(dev))
    assert binding.get_status() == 0
    assert torch.equal(o, o2) and torch.equal(lse, lse2)



@pytest.mark.parametrize("chunk", [1, 2, 8])
def test_host_buffer_pipeline_equals_device_call(oracle, chunk):
    """calibatt_mixed_attn_fwd_host (copies in, compute, copies out, pipelined
    over chunks of heads) returns bit for bit the device call's o and lse; of
    a repeated head's q it copies the anchor pixel rows only and leaves the
    other rows of the device buffer as they were."""
    binding = require_gpu()
    F, H, W, heads, kk = 3, 8, 16, 5, 5
    n = F * H * W
    nb = (n + 127) // 128
    q, k, v = synth.plain_qkv(heads, n, seed=70 + chunk)
    rng = np.random.default_rng(chunk)
    mask = (rng.random((heads, nb, nb)) < 0.5).astype(np.uint8)
    mask[:, np.arange(nb), np.arange(nb)] = 1
    rep = [1, 4]
    row_ptr, col_idx = oracle.mask_to_csr(mask)
    dev = torch.device("cuda")
    rp_d, ci_d = torch.from_numpy(row_ptr).to(dev), torch.from_numpy(col_idx).to(dev)
    rep_d = torch.tensor(rep, dtype=torch.int32, device=dev)
    work = torch.from_numpy(binding.build_mixed_plan(row_ptr, heads, nb, rep, F, H, W, kk)).to(dev)
    o_ref, lse_ref = binding.mixed_attn_fwd(q.to(dev), k.to(dev), v.to(dev), F, H, W, rp_d, ci_d, rep_d, work,
                                            k_anchor=kk)
    qh, kh, vh = (t.contiguous().pin_memory() for t in (q, k, v))
    oh = torch.empty_like(q).pin_memory()
    lh = torch.empty((heads, n), dtype=torch.float32).pin_memory()
    qd, kd, vd, od = (torch.empty_like(q, device=dev) for _ in range(4))
    qd.fill_(float("nan"))
    ld = torch.empty((heads, n), dtype=torch.float32, device=dev)
    binding.mixed_attn_fwd_host(qh, kh, vh, oh, F, H, W, row_ptr, rp_d, ci_d, rep, qd, kd, vd, od, lse_host=lh,
                                lse_dev=ld, heads_per_chunk=chunk, k_anchor=kk)
    torch.cuda.synchronize()
    assert binding.get_status() == 0
    assert torch.equal(oh, o_ref.cpu())
    assert torch.equal(lh, lse_ref.cpu())
    anchors = oracle.anchor_rows(H, kk)
    rows = (np.arange(n) // W) % H
    copied = np.isin(rows, anchors)
    qd_h = qd.cpu()
    for h in range(heads):
        if h in rep:
            assert torch.equal(qd_h[h, torch.from_numpy(copied)], q[h, torch.from_numpy(copied)])
            assert bool(torch.isnan(qd_h[h, torch.from_numpy(~copied)].float()).all())
        else:
            assert torch.equal(qd_h[h], q[h])


@pytest.mark.parametrize("n_ranks", [2, 3])
def test_head_shards_together_equal_the_whole_call(oracle, n_ranks):
    """The ranks' shares of one call (calibatt_shard_heads), run one after
    another here, write bit for bit the output of the whole call."""
    binding = require_gpu()
    F, H, W, heads, kk = 3, 8, 16, 6, 5
    n = F * H * W
    nb = (n + 127) // 128
    q, k, v = synth.plain_qkv(heads, n, seed=90 + n_ranks)
    rng = np.random.default_rng(n_ranks)
    mask = (rng.random((heads, nb, nb)) < rng.random((heads, 1, 1))).astype(np.uint8)
    mask[:, np.arange(nb), np.arange(nb)] = 1
    rep = [2, 5]
    row_ptr, col_idx = oracle.mask_to_csr(mask)
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    rp_d, ci_d = torch.from_numpy(row_ptr).to(dev), torch.from_numpy(col_idx).to(dev)
    work = torch.from_numpy(binding.build_mixed_plan(row_ptr, heads, nb, rep, F, H, W, kk)).to(dev)
    o_all, lse_all = binding.mixed_attn_fwd(qd, kd, vd, F, H, W, rp_d, ci_d, torch.tensor(rep, dtype=torch.int32,
                                                                                         device=dev), work, k_anchor=kk)
    owner, _ = binding.shard_heads(row_ptr, heads, nb, rep, F, W, kk, n_ranks)
    o = torch.zeros_like(qd)
    lse = torch.zeros((heads, n), dtype=torch.float32, device=dev)
    for r in range(n_ranks):
        w, rep_r = binding.build_rank_plan(row_ptr, heads, nb, rep, owner, r, F, H, W, kk)
        binding.mixed_attn_fwd(qd, kd, vd, F, H, W, rp_d, ci_d, torch.tensor(rep_r, dtype=torch.int32, device=dev),
                               torch.from_numpy(w).to(dev), k_anchor=kk, o=o, lse=lse)
    assert binding.get_status() == 0
    assert torch.equal(o, o_all) and torch.equal(lse, lse_all)


def test_mixed_launch_edge_cases(oracle):
    """Every head repeated (no block-sparse unit); an empty work list (nothing
    written); a host-buffer chunk larger than the head count."""
    binding = require_gpu()
    F, H, W, heads, kk = 2, 8, 16, 3, 5
    n = F * H * W
    nb = (n + 127) // 128
    q, k, v = synth.plain_qkv(heads, n, seed=77)
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    mask = np.ones((heads, nb, nb), np.uint8)
    row_ptr, col_idx = oracle.mask_to_csr(mask)
    rp_d, ci_d = torch.from_numpy(row_ptr).to(dev), torch.from_numpy(col_idx).to(dev)
    rep = [0, 1, 2]
    rep_d = torch.tensor(rep, dtype=torch.int32, device=dev)
    work = binding.build_mixed_plan(row_ptr, heads, nb, rep, F, H, W, kk)
    assert work.min() >= heads * nb  # anchor-query units only
    o, _ = binding.mixed_attn_fwd(qd, kd, vd, F, H, W, rp_d, ci_d, rep_d, torch.from_numpy(work).to(dev), k_anchor=kk)
    o_ref, _ = oracle.repeat_attention(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), F, H, W,
                                       k_anchor=kk)
    assert attn_tolerance_ok(bf16_to_f64(o), o_ref)[0]
    # an empty work list writes nothing
    o2 = torch.full_like(qd, 3.0)
    binding.mixed_attn_fwd(qd, kd, vd, F, H, W, rp_d, ci_d, torch.zeros(0, dtype=torch.int32, device=dev),
                           torch.zeros(0, dtype=torch.int32, device=dev), k_anchor=kk, o=o2)
    assert binding.get_status() == 0
    assert bool((o2 == 3.0).all())
    # host buffers with one chunk holding every head
    qh, kh, vh = (t.contiguous().pin_memory() for t in (q, k, v))
    oh = torch.empty_like(q).pin_memory()
    bufs = [torch.empty_like(qd) for _ in range(4)]
    binding.mixed_attn_fwd_host(qh, kh, vh, oh, F, H, W, row_ptr, rp_d, ci_d, rep, *bufs, heads_per_chunk=16,
                                k_anchor=kk)
    torch.cuda.synchronize()
    assert binding.get_status() == 0
    assert torch.equal(oh, o.cpu())


def test_balanced_plan_gives_the_same_output():
    """calibatt_balance_plan only reorders the work list: the mixed launch
    writes bit for bit the same o and lse with the balanced list, laid out
    for this device or for another slot count."""
    binding = require_gpu()
    F, H, W, heads, kk = 4, 8, 40, 6, 5
    n = F * H * W
    nb = (n + 127) // 128
    q, k, v = synth.plain_qkv(heads, n, seed=123)
    rng = np.random.default_rng(5)
    mask = (rng.random((heads, nb, nb)) < rng.uniform(0.05, 0.95, (heads, 1, 1))).astype(np.uint8)
    rp = np.concatenate([[0], np.cumsum(mask.reshape(-1, nb).sum(1))]).astype(np.int32)
    ci = np.concatenate([np.nonzero(row)[0] for row in mask.reshape(-1, nb)]).astype(np.int32)
    rep = [3]
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    rp_d, ci_d = torch.from_numpy(rp).to(dev), torch.from_numpy(ci).to(dev)
    rep_d = torch.tensor(rep, dtype=torch.int32, device=dev)
    w0 = binding.build_mixed_plan(rp, heads, nb, rep, F, H, W, kk)
    outs = []
    for w in (w0, binding.balance_plan(w0, rp, heads, nb), binding.balance_plan(w0, rp, heads, nb, 6)):
        assert sorted(w.tolist()) == sorted(w0.tolist())
        o, lse = binding.mixed_attn_fwd(qd, kd, vd, F, H, W, rp_d, ci_d, rep_d, torch.from_numpy(w).to(dev),
                                        k_anchor=kk)
        outs.append((o.cpu(), lse.cpu()))
    assert binding.get_status() == 0
    for o, lse in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(lse, outs[0][1])
