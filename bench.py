#!/usr/bin/env python
"""Benchmark of the CalibAtt hot path on B200 (one JSON line on rank 0).

One step = one attention call of the Wan 2.1 14B 720p shape (40 heads,
N = 75600 = 21 x 45 x 80 tokens, d = 128, bf16): block-sparse attention of the
32 non-repeated heads over their skip lists (random per-head masks, 62.5 %
mean block sparsity) followed by the anchor-row attention of the 8 repeated
heads (k = 5 anchor rows of 45). The metric is kept-tile attention TFLOPS
(algorithmic: 4 * d * valid query rows * valid key columns per kept tile),
reported against the BF16 tensor roofline and next to the same kernel run at
0 % sparsity. The calibration kernels (block energy with fused selection,
standalone selection, aggregation) are timed in the same run on the same
shape and reported under "calibration".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun), every rank runs its own copy of the workload on its own
inputs (weak scaling, no data-path collective); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from calibrated_block_sparse_b200 import synth  # noqa: E402

D = 128
METRIC = "kept-tile attention TFLOPS"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- work accounting

def valid_sizes(n, nb):
    v = np.full(nb, 128, np.int64)
    v[-1] = n - (nb - 1) * 128
    return v


def sparse_flops(mask, heads, n):
    """Algorithmic flops of the block-sparse heads: 4 d |valid q| |valid k| per kept tile."""
    nb = mask.shape[-1]
    v = valid_sizes(n, nb)
    pair = np.outer(v, v)
    return float(4 * D * sum(int((mask[h].astype(np.int64) * pair).sum()) for h in heads))


def repeat_flops(wl, n_rep):
    return float(4 * D * wl.F * wl.k_anchor * wl.W * wl.n * n_rep)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- distributed plumbing

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif args.impl == "ours":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- CPU baseline (oracle)

def cpu_oracle_sample(wl, q_cpu, k_cpu, v_cpu, heads, masks, budget_s, rng, repeat=False):
    """Time the fp64 oracle on randomly sampled query rows of the given heads.

    Returns (seconds, algorithmic flops, rows, threads)."""
    import oracle
    threads = os.cpu_count() or 1
    nb = wl.nb
    v_sz = valid_sizes(wl.n, nb)
    spent, flops, rows_done, batch = 0.0, 0.0, 0, max(threads, 8)
    while spent < budget_s:
        hi = int(rng.integers(len(heads)))
        rows = rng.integers(0, wl.n, size=batch).astype(np.int64)
        qb, kb, vb = (synth.bf16_bits(t[hi:hi + 1]) for t in (q_cpu, k_cpu, v_cpu))
        t0 = time.perf_counter()
        if repeat:
            oracle.repeat_attention(qb, kb, vb, wl.F, wl.H, wl.W, wl.k_anchor, rows=rows, threads=threads)
            flops += 4.0 * D * wl.n * batch
        else:
            oracle.masked_attention(qb, kb, vb, masks[heads[hi]][None], rows=rows, threads=threads)
            kept = masks[heads[hi]][rows // 128].astype(np.int64) @ v_sz
            flops += 4.0 * D * float(kept.sum())
        spent += time.perf_counter() - t0
        rows_done += batch
    return spent, flops, rows_done, threads


def arm_config(wl, heads, kept_frac, world, shard=False):
    """The workload description both arms print."""
    sparse = [h for h in range(heads) if h not in wl.repeat_heads]
    return {"workload": f"{wl.name}: {heads} heads x N={wl.n} (F={wl.F},H={wl.H},W={wl.W}), d={D}, "
                        f"{len(sparse)} block-sparse + {heads - len(sparse)} repeated (k={wl.k_anchor})",
            "kept_block_fraction": kept_frac, "block_sparsity": 1 - kept_frac,
            "l2": "inputs (3 x %.2f GB) larger than L2; no flush" % (heads * wl.n * D * 2 / 1e9),
            "parallelism": f"heads sharded over {world} GPUs" if shard else f"replica per GPU x{world}"}


def run_reference(args, world, rank):
    """Reference arm: the oracle as it stands, on the host cores, same metric."""
    if rank != 0:
        return
    wl = synth.WORKLOADS[args.workload]
    masks = synth.random_block_masks(wl) if wl.repeat_heads or args.workload == "wan720" else \
        np.ones((wl.heads, wl.nb, wl.nb), np.uint8)
    sparse_heads = [h for h in range(wl.heads) if h not in wl.repeat_heads]
    rng = np.random.default_rng(1234)
    hs = [sparse_heads[0]]
    q, k, v = synth.qkv(wl, 0, heads=hs)
    qm = np.stack([masks[h] for h in hs])
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, q, k, v, [0], qm, 0.2, rng)
    tot_s, tot_f, rows, threads = 0.0, 0.0, 0, 1
    for _ in range(args.steps):
        s, f, r, threads = cpu_oracle_sample(wl, q, k, v, [0], qm, per_step, rng)
        tot_s += s
        tot_f += f
        rows += r
    value = tot_f / tot_s / 1e12
    sample = (f"{rows} query rows of one block-sparse head of {wl.name}, fp64 oracle "
              f"(plain C, {threads} threads), throughput in kept-tile flops")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(wl, wl.heads, float(np.mean([masks[h].mean() for h in sparse_heads])), world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm

def cuda_time(fn, reps, stream):
    """Average device ms of fn() over reps, CUDA events on `stream`."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(reps):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / reps


def graph_time(fn, reps, stream):
    """Average device ms of fn() for kernels too short to time one by one: the
    reps calls are captured in a CUDA graph and replayed, so host launch
    overhead does not open gaps between them."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    g.replay()
    end.record(stream)
    end.synchronize()
    ms = start.elapsed_time(end) / reps
    del g
    return ms


TRAFFIC_PER_TILE = 565.24e6 / 514058  # dram bytes per kept tile, measured (see the roofline block)


def run_ours(args, world, rank, local):
    from calibrated_block_sparse_b200 import binding
    binding.load()
    wl = synth.WORKLOADS[args.workload]
    if args.heads:
        # a smaller case of the same kernels: the first `heads` heads only
        import dataclasses
        wl = dataclasses.replace(wl, heads=args.heads, repeat_heads=tuple(h for h in wl.repeat_heads if h < args.heads))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    n, nb, heads = wl.n, wl.nb, wl.heads
    rep_heads = list(wl.repeat_heads)
    sparse_heads = [h for h in range(heads) if h not in rep_heads]

    # inputs: resident in HBM before the timed region
    if args.workload == "wan720":
        # random per-head masks at 62.5 % sparsity; skip lists built on the GPU
        # by the aggregation kernel (one input, rho 0.5)
        masks = synth.random_block_masks(synth.WORKLOADS["wan720"])[:heads]
        counts = torch.from_numpy(masks.astype(np.int16)).to(dev).view(torch.uint16)
        mask_d, row_ptr, col_idx, _ = binding.aggregate_masks(counts, 1, 0.5)
    else:
        # masks calibrated on the GPU over the workload's seeded inputs
        n_cal, eps_cal = synth.CALIBRATION[args.workload]
        counts = torch.zeros((heads, nb, nb), dtype=torch.uint16, device=dev)
        cws = torch.empty(binding.energy_workspace_size(heads, n), dtype=torch.uint8, device=dev)
        for pi in range(n_cal):
            qc, kc, _ = synth.qkv(wl, pi, with_v=False, device=dev)
            binding.block_energy_1pass(qc, kc, eps=eps_cal, energy=False, counts=counts, ws=cws)
            del qc, kc
        del cws
        mask_d, row_ptr, col_idx, _ = binding.aggregate_masks(counts, n_cal, 0.5)
        masks = mask_d.cpu().numpy()
    binding.check_status(what="skip lists")
    q, k, v = synth.qkv(wl, 1000 + rank, device=dev)
    row_ptr_h = row_ptr.cpu().numpy()
    head_active = np.array([h not in rep_heads for h in range(heads)], np.uint8)
    # every work list is laid out for the device's worker slots (balanced
    # static schedule; any order gives the same output)
    work = torch.from_numpy(binding.balance_plan(binding.build_plan(row_ptr_h, heads, nb, head_active), row_ptr_h,
                                                 heads, nb)).to(dev)
    rep_t = torch.tensor(rep_heads, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((heads, n), dtype=torch.float32, device=dev)
    ws = torch.empty(max(binding.repeat_workspace_size(max(len(rep_heads), 1), wl.F, wl.H, wl.W, wl.k_anchor), 256),
                     dtype=torch.uint8, device=dev)

    f_sparse = sparse_flops(masks, sparse_heads, n)
    f_rep = repeat_flops(wl, len(rep_heads))
    f_step = f_sparse + f_rep
    kept_frac = float(np.mean([masks[h].mean() for h in sparse_heads]))

    def sparse_call():
        binding.sparse_attn_fwd(q, k, v, row_ptr, col_idx, work, o=o, lse=lse, stream=stream)

    def repeat_call():
        if rep_heads:
            binding.repeat_attn_fwd(q, k, v, wl.F, wl.H, wl.W, rep_t, wl.k_anchor, o=o, lse=lse, ws=ws,
                                    stream=stream)

    # the step: block-sparse and repeated heads in one persistent launch
    # (after the anchor gather). --shard heads: one call split over the ranks
    # by heads (balanced by kept tiles, no exchange), strong scaling
    shard = args.shard == "heads" and world > 1
    if shard:
        owner, _ = binding.shard_heads(row_ptr_h, heads, nb, rep_heads, wl.F, wl.W, wl.k_anchor, world)
        work_np, my_rep = binding.build_rank_plan(row_ptr_h, heads, nb, rep_heads, owner, rank, wl.F, wl.H, wl.W,
                                                  wl.k_anchor)
        f_rank = sparse_flops(masks, [h for h in sparse_heads if owner[h] == rank], n) + repeat_flops(wl, len(my_rep))
    else:
        work_np = binding.build_mixed_plan(row_ptr_h, heads, nb, rep_heads, wl.F, wl.H, wl.W, wl.k_anchor)
        my_rep, f_rank = rep_heads, f_step
    work_mixed = torch.from_numpy(binding.balance_plan(work_np, row_ptr_h, heads, nb)).to(dev)
    my_rep_t = torch.tensor(my_rep, dtype=torch.int32, device=dev)

    def step():
        binding.mixed_attn_fwd(q, k, v, wl.F, wl.H, wl.W, row_ptr, col_idx, my_rep_t, work_mixed, wl.k_anchor, o=o,
                               lse=lse, ws=ws, stream=stream)

    launches_per_step = 1 + (1 if my_rep else 0)
    for _ in range(args.warmup):
        step()
    binding.check_status(what="warmup")

    # ---- timed region: K steps, events around each step's launches
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        t_start.record(stream)
        for e0, e1 in evs:
            e0.record(stream)
            step()
            e1.record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = t_start.elapsed_time(t_end)
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    binding.check_status(what="timed steps")
    attn_ms = sum(e0.elapsed_time(e1) for e0, e1 in evs) / args.steps
    ms_step = elapsed_ms / args.steps

    # the same work as two separate calls (block-sparse, then repeated heads)
    sparse_ms = repeat_ms = None
    if not shard:
        sparse_ms = cuda_time(sparse_call, max(2, min(5, args.steps)), stream)
        repeat_ms = cuda_time(repeat_call, max(2, min(5, args.steps)), stream) if rep_heads else 0.0
        binding.check_status(what="separate calls")
    # weak scaling: every rank runs the whole call (replicas); strong: the
    # ranks share one call
    value = (1 if shard else world) * f_step / (ms_step * 1e-3) / 1e12

    # ---- 0 %-sparse run: the same kernel with every block kept, all 40 heads
    full = torch.ones((heads, nb, nb), dtype=torch.int16, device=dev).view(torch.uint16)
    _, rp_full, ci_full, _ = binding.aggregate_masks(full, 1, 0.5)
    rp_full_h = rp_full.cpu().numpy()
    work_full = torch.from_numpy(binding.balance_plan(binding.build_plan(rp_full_h, heads, nb), rp_full_h, heads,
                                                      nb)).to(dev)

    def dense_call():
        binding.sparse_attn_fwd(q, k, v, rp_full, ci_full, work_full, o=o, lse=lse, stream=stream)

    dense_call()
    dense_ms = cuda_time(dense_call, max(2, min(5, args.steps)), stream)
    binding.check_status(what="dense")
    f_dense = float(4 * D * n * n * heads)
    del rp_full, ci_full, work_full, full

    # ---- context, not this library's path: the same dense attention by the
    # cuDNN backend of torch's scaled_dot_product_attention, timed the same way
    library_dense = None
    try:
        import torch.nn.functional as F
        from torch.nn.attention import SDPBackend, sdpa_kernel

        def library_call():
            with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
                return F.scaled_dot_product_attention(q[None], k[None], v[None])

        with torch.cuda.stream(stream):
            library_call()
            lib_ms = cuda_time(library_call, max(2, min(5, args.steps)), stream)
        library_dense = {"kernel": "torch scaled_dot_product_attention, cuDNN backend, all blocks kept",
                         "ms": lib_ms, "tflops": f_dense / (lib_ms * 1e-3) / 1e12,
                         "step_speedup": lib_ms / ms_step}
    except Exception as exc:  # the backend may be missing: report why
        library_dense = {"unavailable": str(exc)[:200]}

    # ---- end to end through the C ABI with host buffers: H2D q,k,v, call, D2H o
    e2e = None
    if not args.no_e2e and not shard:
        qh = q.cpu().pin_memory()
        kh = k.cpu().pin_memory()
        vh = v.cpu().pin_memory()
        oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()

        ws_host = torch.empty(binding.load().calibatt_mixed_host_workspace_size(
            heads, wl.F, wl.H, wl.W, wl.k_anchor, len(rep_heads), args.e2e_chunk), dtype=torch.uint8, device=dev)

        def e2e_step():
            # the host-buffer call: q, k, v in, o out, pipelined over chunks of heads
            binding.mixed_attn_fwd_host(qh, kh, vh, oh, wl.F, wl.H, wl.W, row_ptr_h, row_ptr, col_idx, rep_heads,
                                        q, k, v, o, ws=ws_host, heads_per_chunk=args.e2e_chunk, k_anchor=wl.k_anchor,
                                        stream=stream)

        e2e_step()
        reps = max(2, min(5, args.steps))
        barrier(world)
        e2e_ms = max_over_ranks(cuda_time(e2e_step, reps, stream), world)
        binding.check_status(what="e2e")

        # the host link on its own: the same pinned q, k, v copied in whole
        # with plain copies, no compute (the bound of the call above)
        def link_step():
            with torch.cuda.stream(stream):
                q.copy_(qh, non_blocking=True)
                k.copy_(kh, non_blocking=True)
                v.copy_(vh, non_blocking=True)

        link_step()
        link_ms = cuda_time(link_step, reps, stream)
        link_gbs = 3 * q.numel() * q.element_size() / (link_ms * 1e-3) / 1e9
        e2e = {"value": world * f_step / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               # q of a repeated head: its anchor pixel rows only
               "h2d_bytes_per_step": int(3 * q.numel() * q.element_size()
                                         - len(rep_heads) * wl.F * (wl.H - wl.k_anchor) * wl.W * D * 2),
               "d2h_bytes_per_step": int(o.numel() * o.element_size()), "ms_per_step": e2e_ms,
               "h2d_link_gbs": link_gbs,
               "call": f"calibatt_mixed_attn_fwd_host, pinned host buffers, {args.e2e_chunk} heads per chunk"}
        # share of the link's copy-in rate that the call sustains
        e2e["h2d_link_frac"] = e2e["h2d_bytes_per_step"] / (e2e_ms * 1e-3) / 1e9 / link_gbs
        del qh, kh, vh, oh, ws_host

    # ---- calibration kernels on the same shape (8 heads of it)
    calib = None
    if not args.no_calib:
        ch = min(8, heads)
        qc, kc = q[:ch].contiguous(), k[:ch].contiguous()
        lse_ws = torch.empty((ch, nb * 128), dtype=torch.float32, device=dev)
        energy = torch.empty((ch, nb, nb), dtype=torch.float32, device=dev)
        cmask = torch.empty((ch, nb, nb), dtype=torch.uint8, device=dev)
        ccounts = torch.zeros((ch, nb, nb), dtype=torch.uint16, device=dev)

        def energy_call():
            binding.block_energy(qc, kc, eps=0.9, energy=energy, mask=cmask, counts=ccounts, lse_ws=lse_ws,
                                 stream=stream)

        energy_call()
        e_ms = cuda_time(energy_call, 2, stream)
        ews = torch.empty(binding.energy_workspace_size(ch, n), dtype=torch.uint8, device=dev)

        def energy1_call():
            binding.block_energy_1pass(qc, kc, eps=0.9, energy=energy, mask=cmask, counts=ccounts, ws=ews,
                                       stream=stream)

        energy1_call()
        e1_ms = cuda_time(energy1_call, 2, stream)
        del ews
        f_energy_alg = float(2 * D * n * n * ch)  # one S = Q K^T per input
        f_energy_issued = 2 * f_energy_alg        # two passes recompute S

        gstream = torch.cuda.Stream()

        def select_call():
            binding.select_mask(energy, 0.9, mask=cmask, kept=False, stream=torch.cuda.current_stream())

        with torch.cuda.stream(gstream):
            s_ms = graph_time(select_call, 20, gstream)
        sel_bytes = ch * nb * nb * (4 + 1)
        agg_ws = torch.empty(binding.load().calibatt_aggregate_workspace_size(ch, nb), dtype=torch.uint8, device=dev)
        am = torch.empty((ch, nb, nb), dtype=torch.uint8, device=dev)
        arp = torch.empty(ch * nb + 1, dtype=torch.int32, device=dev)
        aci = torch.empty(ch * nb * nb, dtype=torch.int32, device=dev)
        annz = torch.zeros(1, dtype=torch.int64, device=dev)
        lib = binding.load()

        def agg_call():
            lib.calibatt_aggregate_masks(binding._ptr(ccounts), 64, ch, nb, 0.5, binding._ptr(am),
                                         binding._ptr(arp), binding._ptr(aci), aci.numel(), binding._ptr(annz),
                                         binding._ptr(agg_ws), agg_ws.numel(),
                                         binding._stream(torch.cuda.current_stream()))

        with torch.cuda.stream(gstream):
            a_ms = graph_time(agg_call, 20, gstream)
        # spatial repetition: pixel-row profiles (same two passes, plus the
        # profile atomics) and the per-head score
        pix = torch.empty((ch, wl.F * wl.H, nb), dtype=torch.float32, device=dev)

        def pix_call():
            binding.pixel_row_energy(qc, kc, wl.F, wl.H, wl.W, pix=pix, lse_ws=lse_ws, stream=stream)

        pix_call()
        p_ms = cuda_time(pix_call, 2, stream)
        sscore = torch.empty(ch, dtype=torch.float32, device=dev)
        sflag = torch.empty(ch, dtype=torch.uint8, device=dev)

        def score_call():
            binding.spatial_score(pix, wl.F, wl.H, wl.k_anchor, score=sscore, flag=sflag,
                                  stream=torch.cuda.current_stream())

        with torch.cuda.stream(gstream):
            sc_ms = graph_time(score_call, 20, gstream)
        binding.check_status(what="calibration")
        kept_agg = int(annz.item())
        agg_bytes = ch * nb * nb * (2 + 1 + 1) + kept_agg * 4 + (ch * nb + 1) * 4 * 3
        calib = {
            "shape": f"{ch} heads x N={n}",
            "energy_ms": e_ms, "energy_tflops_algorithmic": f_energy_alg / (e_ms * 1e-3) / 1e12,
            "energy_tflops_issued": f_energy_issued / (e_ms * 1e-3) / 1e12,
            "energy_1pass_ms": e1_ms, "energy_1pass_tflops": f_energy_alg / (e1_ms * 1e-3) / 1e12,
            "select_ms": s_ms, "select_gbs": sel_bytes / (s_ms * 1e-3) / 1e9,
            "aggregate_ms": a_ms, "aggregate_gbs": agg_bytes / (a_ms * 1e-3) / 1e9,
            "eps": 0.9, "kept_fraction_at_eps": float(cmask.float().mean().item()),
            "pixel_row_energy_ms": p_ms, "pixel_row_energy_tflops_issued": f_energy_issued / (p_ms * 1e-3) / 1e12,
            "spatial_score_ms": sc_ms,
            "spatial_score_gbs": ch * wl.F * (wl.H - wl.k_anchor) * nb * 8 / (sc_ms * 1e-3) / 1e9,
            "spatial_flagged_heads": np.nonzero(sflag.cpu().numpy())[0].tolist(),
        }
        del qc, kc, lse_ws, energy, cmask, ccounts, pix

    # ---- roofline of the dominant kernel: the attention kernel of the step
    # (block-sparse and repeated heads in one launch; its event window also
    # holds the short anchor-gather launch before it)
    pk, pk_src = peaks()
    long_run = elapsed_ms > 1000.0
    peak = pk.get("bf16_tflops_sustained" if long_run else "bf16_tflops")
    achieved = f_rank / (attn_ms * 1e-3) / 1e12
    kname = ("attn_kernel<attention> (%d block-sparse + %d repeated heads, one launch; window includes the "
             "anchor gather)" % (len(sparse_heads), len(rep_heads)))
    if shard:
        kname += "; rank 0 share of the heads"
    # DRAM traffic per launch: the given figure, else the bytes per kept tile
    # of the one ncu capture (profiles/attn_kernel_wan720_5heads_ncu_full.md:
    # 565.2 MB over 514 058 kept tiles) times the tiles of this launch
    mine = [h for h in sparse_heads if not shard or owner[h] == rank]
    tiles = int(sum(int(masks[h].sum()) for h in mine)) + len(my_rep) * -(-wl.F * wl.k_anchor * wl.W // 128) * nb
    traffic = args.traffic_bytes if args.traffic_bytes else TRAFFIC_PER_TILE * tiles
    roofline = {"bound": "tensor", "kernel": kname,
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": f"{pk_src} {'sustained' if long_run else 'burst'} bf16",
                "traffic": traffic,
                "traffic_source": "given" if args.traffic_bytes else
                "ncu dram bytes of a 5-head capture, scaled by kept tiles (%d in this launch)" % tiles,
                "algorithmic_bytes": 4.0 * heads * n * D * 2}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        hs = [sparse_heads[0]]
        qc, kc, vc = (t[hs].cpu() for t in (q, k, v))
        s, f, rows, threads = cpu_oracle_sample(wl, qc, kc, vc, [0], np.stack([masks[h] for h in hs]),
                                                args.cpu_seconds, np.random.default_rng(5))
        cpu = {"value": f / s / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{rows} query rows of one block-sparse head, fp64 plain-C oracle, {s:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if shard else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": arm_config(wl, heads, kept_frac, world, shard),
            "gpu_launches": launches_per_step * args.steps,
            "attn_ms": attn_ms,
            "separate_calls": None if shard else {"sparse_ms": sparse_ms, "repeat_ms": repeat_ms,
                                                  "sparse_tflops": f_sparse / (sparse_ms * 1e-3) / 1e12},
            "dense_ms": dense_ms, "dense_tflops": f_dense / (dense_ms * 1e-3) / 1e12,
            "speedup_vs_dense": dense_ms / ms_step,
            "library_dense": library_dense,
            "roofline": roofline, "e2e": e2e, "cpu_baseline": cpu, "calibration": calib,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["wan720", "wan480", "mochi480"], default="wan720")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--heads", type=int, default=0, help="run only the first HEADS heads (profiling case)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunk", type=int, default=2, help="heads per chunk of the host-buffer pipeline")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N>1: a replica of the call per rank (weak scaling) or one call split by heads (strong)")
    ap.add_argument("--no-calib", action="store_true")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="dram bytes per launch of the sparse kernel from an ncu capture")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
