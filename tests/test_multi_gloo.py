"""World-size-2 tests of the multi-process path on CPU (gloo): calibration
inputs sharded over ranks, one integer all-reduce of the mask counts, and the
slowest-rank timing reduction. The per-input masks come from the oracle
(these processes have no GPU); the reduction and binarisation must equal the
single-process oracle aggregation over all inputs."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, masks, rho, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from calibrated_block_sparse_b200 import multi
        n_in = masks.shape[0]
        lo, hi = multi.shard_range(n_in, rank, world)
        local = masks[lo:hi].astype(np.int64).sum(0) if hi > lo else np.zeros(masks.shape[1:], np.int64)
        counts = torch.from_numpy(local.astype(np.int16)).view(torch.uint16)
        multi.allreduce_counts(counts)
        total = counts.view(torch.int16).to(torch.int32).numpy() & 0xFFFF
        mask = oracle.binarize_counts(total.astype(np.int32), n_in, rho)
        slowest = multi.max_over_ranks(float(rank + 1))
        out_q.put((rank, total, mask, slowest))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_in,world", [(16, 2), (7, 2), (1, 2)])
def test_sharded_counts_equal_single_process(oracle, n_in, world):
    rng = np.random.default_rng(n_in)
    masks = (rng.random((n_in, 3, 9, 9)) < 0.5).astype(np.uint8)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, masks, 0.5, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref_mask, ref_counts = oracle.aggregate(masks, 0.5)
    for rank, total, mask, slowest in results:
        np.testing.assert_array_equal(total, ref_counts)
        np.testing.assert_array_equal(mask, ref_mask)
        assert slowest == float(world)


def test_shard_range_partitions():
    from calibrated_block_sparse_b200 import multi
    for n in (0, 1, 7, 16, 64):
        for w in (1, 2, 3, 8):
            parts = [multi.shard_range(n, r, w) for r in range(w)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
            sizes = [hi - lo for lo, hi in parts]
            assert max(sizes) - min(sizes) <= 1


def _plan_worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from calibrated_block_sparse_b200 import binding, synth
        wl = synth.WORKLOADS["mochi480"]
        row_ptr, _ = oracle.mask_to_csr(synth.random_block_masks(wl))
        rep = list(wl.repeat_heads)
        owner, load = binding.shard_heads(row_ptr, wl.heads, wl.nb, rep, wl.F, wl.W, wl.k_anchor, world)
        work, rep_r = binding.build_rank_plan(row_ptr, wl.heads, wl.nb, rep, owner, rank, wl.F, wl.H, wl.W)
        # every rank derives the same owners on its own
        owners = [torch.zeros(wl.heads, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(owners, torch.from_numpy(owner))
        # the slowest rank's share of kept tiles
        heaviest = torch.tensor([int(load[rank])], dtype=torch.int64)
        dist.all_reduce(heaviest, op=dist.ReduceOp.MAX)
        out_q.put((rank, [o.numpy() for o in owners], work, rep_r, int(heaviest.item()), load))
    finally:
        dist.destroy_process_group()


def test_head_sharding_over_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_plan_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted([q.get(timeout=120) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, owners, _, _, heaviest, load in results:
        np.testing.assert_array_equal(owners[0], owners[1])
        assert heaviest == max(load)
    owner = results[0][1][0]
    for rank, _, work, rep_r, _, _ in results:
        assert all(owner[h] == rank for h in rep_r)
    # the two ranks' block-sparse units are disjoint and cover the sparse heads
    from calibrated_block_sparse_b200 import synth
    wl = synth.WORKLOADS["mochi480"]
    base = wl.heads * wl.nb
    sp = [set(int(u) for u in r[2] if u < base) for r in results]
    assert not (sp[0] & sp[1])
    assert sorted(sp[0] | sp[1]) == [h * wl.nb + r for h in range(wl.heads) if h not in wl.repeat_heads
                                     for r in range(wl.nb)]
