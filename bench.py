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


# DRAM bytes per kept tile of the attention kernel: one ncu capture of the
# 5-head Wan-720p launch (heads 0-3 block-sparse, head 4 repeated), 538.9 MB
# read + 89.5 MB written (dram__bytes_read.sum + dram__bytes_write.sum) over
# its 514 058 kept tiles; the roofline's traffic scales it by the tiles of
# the timed launch.
TRAFFIC_PER_TILE = 628.43e6 / 514058


def frac_of(achieved, pk, key):
    return achieved / pk[key] if pk.get(key) else None


def calibrate(binding, wl, n_in, eps, dev, stream, first_input=0):
    """Calibration of one (t, l) on the device: every input through the
    single-pass energy kernel with fused eps selection, masks folded into
    counts; the tie-affected selections (1e-6) are counted. Returns (counts,
    info)."""
    heads, nb, n = wl.heads, wl.nb, wl.n
    counts = torch.zeros((heads, nb, nb), dtype=torch.uint16, device=dev)
    tie = torch.empty((heads, nb), dtype=torch.uint8, device=dev)
    ws = torch.empty(binding.energy_workspace_size(heads, n), dtype=torch.uint8, device=dev)
    ms, ties = 0.0, 0
    for p in range(first_input, first_input + n_in):
        q, k, _ = synth.qkv(wl, p, with_v=False, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        binding.block_energy_1pass(q, k, eps=eps, energy=False, counts=counts, ws=ws, tie=tie, stream=stream)
        e1.record(stream)
        e1.synchronize()
        ms += e0.elapsed_time(e1)
        ties += int(tie.sum().item())
    binding.check_status(what=f"calibration of {wl.name}")
    f_alg = 2.0 * D * n * n * heads  # one S = Q K^T per input
    info = {"inputs": n_in, "eps": eps, "rho": 0.5,
            "energy_ms_per_input": ms / n_in, "energy_tflops": f_alg / (ms / n_in * 1e-3) / 1e12,
            "tie_affected_selections": ties, "selections": n_in * heads * nb, "tie_window": binding.TIE_WINDOW,
            "kernel": "calibatt_block_energy_1pass (fused eps selection, counts and tie flags)"}
    return counts, info


def skip_lists(binding, wl, dev, stream):
    """Masks and skip lists of a workload: random block masks (Wan-720p) or
    calibration on the GPU over the workload's seeded inputs."""
    if wl.name == "wan720":
        masks = synth.random_block_masks(synth.WORKLOADS["wan720"])[:wl.heads]
        counts = torch.from_numpy(masks.astype(np.int16)).to(dev).view(torch.uint16)
        _, row_ptr, col_idx, _ = binding.aggregate_masks(counts, 1, 0.5)
        calib = {"source": "random per-head block masks (Beta(2,3) keep rates, diagonal and first frame kept)"}
    else:
        n_cal, eps_cal = synth.CALIBRATION[wl.name]
        counts, calib = calibrate(binding, wl, n_cal, eps_cal, dev, stream)
        mask_d, row_ptr, col_idx, _ = binding.aggregate_masks(counts, n_cal, 0.5)
        masks = mask_d.cpu().numpy()
        calib["source"] = "calibrated on the GPU"
    binding.check_status(what="skip lists")
    return masks, row_ptr, col_idx, calib


def dense_run(binding, q, k, v, o, lse, heads, nb, dev, stream, reps):
    """The same kernel with every block kept on every head (0 % sparsity)."""
    full = torch.ones((heads, nb, nb), dtype=torch.int16, device=dev).view(torch.uint16)
    _, rp_full, ci_full, _ = binding.aggregate_masks(full, 1, 0.5)
    rp_full_h = rp_full.cpu().numpy()
    work_full = torch.from_numpy(binding.balance_plan(binding.build_plan(rp_full_h, heads, nb), rp_full_h, heads,
                                                      nb)).to(dev)

    def dense_call():
        binding.sparse_attn_fwd(q, k, v, rp_full, ci_full, work_full, o=o, lse=lse, stream=stream)

    dense_call()
    ms = cuda_time(dense_call, reps, stream)
    binding.check_status(what="dense")
    return ms


def library_dense(q, k, v, stream, reps, f_dense):
    """Context, not this library's path: the same dense attention by the cuDNN
    backend of torch's scaled_dot_product_attention, timed the same way."""
    try:
        import torch.nn.functional as F
        from torch.nn.attention import SDPBackend, sdpa_kernel

        def library_call():
            with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
                return F.scaled_dot_product_attention(q[None], k[None], v[None])

        with torch.cuda.stream(stream):
            library_call()
            lib_ms = cuda_time(library_call, reps, stream)
        return {"kernel": "torch scaled_dot_product_attention, cuDNN backend, all blocks kept",
                "ms": lib_ms, "tflops": f_dense / (lib_ms * 1e-3) / 1e12}
    except Exception as exc:  # the backend may be missing: report why
        return {"unavailable": str(exc)[:200]}


class Step:
    """One attention call of a workload through calibatt_mixed_attn_fwd:
    block-sparse heads over their skip lists and repeated heads' anchor rows
    in one persistent launch (after the anchor gather)."""

    def __init__(self, binding, wl, masks, row_ptr, col_idx, dev, stream, input_idx=1000, rep_heads=None):
        self.b, self.wl, self.stream = binding, wl, stream
        heads, nb, n = wl.heads, wl.nb, wl.n
        self.rep = list(wl.repeat_heads) if rep_heads is None else list(rep_heads)
        self.sparse_heads = [h for h in range(heads) if h not in self.rep]
        self.masks, self.row_ptr, self.col_idx = masks, row_ptr, col_idx
        self.row_ptr_h = row_ptr.cpu().numpy()
        self.q, self.k, self.v = synth.qkv(wl, input_idx, device=dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((heads, n), dtype=torch.float32, device=dev)
        self.ws = torch.empty(max(binding.repeat_workspace_size(max(len(self.rep), 1), wl.F, wl.H, wl.W,
                                                                wl.k_anchor), 256), dtype=torch.uint8, device=dev)
        self.rep_t = torch.tensor(self.rep, dtype=torch.int32, device=dev)
        work = binding.build_mixed_plan(self.row_ptr_h, heads, nb, self.rep, wl.F, wl.H, wl.W, wl.k_anchor)
        self.work = torch.from_numpy(binding.balance_plan(work, self.row_ptr_h, heads, nb)).to(dev)
        self.f_sparse = sparse_flops(masks, self.sparse_heads, n)
        self.f_rep = repeat_flops(wl, len(self.rep))
        self.flops = self.f_sparse + self.f_rep
        self.kept_frac = float(np.mean([masks[h].mean() for h in self.sparse_heads])) if self.sparse_heads else 1.0
        self.tiles = int(sum(int(masks[h].sum()) for h in self.sparse_heads)) + \
            len(self.rep) * -(-wl.F * wl.k_anchor * wl.W // 128) * nb
        self.launches = 1 + (1 if self.rep else 0)

    def __call__(self):
        wl = self.wl
        self.b.mixed_attn_fwd(self.q, self.k, self.v, wl.F, wl.H, wl.W, self.row_ptr, self.col_idx, self.rep_t,
                              self.work, wl.k_anchor, o=self.o, lse=self.lse, ws=self.ws, stream=self.stream)

    def summary(self, ms, dense_ms, pk, library=None):
        wl = self.wl
        tflops = self.flops / (ms * 1e-3) / 1e12
        out = {"shape": f"{wl.heads} heads x N={wl.n} (F={wl.F},H={wl.H},W={wl.W}), d={D}, "
                        f"{len(self.sparse_heads)} block-sparse + {len(self.rep)} repeated (k={wl.k_anchor})",
               "ms_per_call": ms, "kept_tile_tflops": tflops,
               "frac_of_bf16_burst": frac_of(tflops, pk, "bf16_tflops"),
               "frac_of_bf16_sustained": frac_of(tflops, pk, "bf16_tflops_sustained"),
               "kept_tile_flops": self.flops, "kept_tiles": self.tiles,
               "block_sparsity": 1.0 - self.kept_frac, "kept_block_fraction": self.kept_frac}
        if dense_ms is not None:
            f_dense = float(4 * D * wl.n * wl.n * wl.heads)
            out.update({"dense_ms": dense_ms, "dense_tflops": f_dense / (dense_ms * 1e-3) / 1e12,
                        "speedup_vs_dense": dense_ms / ms})
        if library is not None:
            out["library_dense"] = library
        return out


def anchor_masked_step(binding, step, dev, stream, pk, reps, n_in, eps):
    """The step with block masks on the repeated heads' anchor rows: the anchor
    queries calibrated over n_in seeded inputs at eps (single-pass energy with
    fused selection), aggregated at rho = 0.5, then the masked mixed launch on
    the step's inputs. Kept-tile flops count each kept anchor tile by its valid
    anchor rows and key columns."""
    wl = step.wl
    rep = step.rep
    if not rep:
        return None
    heads, nb, n = wl.heads, wl.nb, wl.n
    nbq = binding.anchor_blocks(wl.F, wl.W, wl.k_anchor)
    rep_t = step.rep_t
    counts = torch.zeros((len(rep), nbq, nb), dtype=torch.uint16, device=dev)
    ws = torch.empty(binding.load().calibatt_anchor_energy_workspace_size(heads, len(rep), wl.F, wl.H, wl.W,
                                                                          wl.k_anchor), dtype=torch.uint8, device=dev)
    ms_cal = 0.0
    for p in range(n_in):
        q, k, _ = synth.qkv(wl, p, with_v=False, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        binding.anchor_block_energy(q, k, wl.F, wl.H, wl.W, rep_t, k_anchor=wl.k_anchor, eps=eps, energy=False,
                                    counts=counts, ws=ws, stream=stream)
        e1.record(stream)
        e1.synchronize()
        ms_cal += e0.elapsed_time(e1)
        del q, k
    del ws
    mask_b, rpb, cib, _ = binding.aggregate_mask_rows(counts, n_in, 0.5, stream=stream)
    mb = mask_b.cpu().numpy()
    rpb_h = rpb.cpu().numpy()
    work = binding.build_mixed_plan(step.row_ptr_h, heads, nb, rep, wl.F, wl.H, wl.W, wl.k_anchor)
    work = torch.from_numpy(binding.balance_mixed_plan(work, step.row_ptr_h, heads, nb, rpb_h, len(rep), wl.F, wl.W,
                                                       wl.k_anchor)).to(dev)

    def call():
        binding.mixed_masked_attn_fwd(step.q, step.k, step.v, wl.F, wl.H, wl.W, step.row_ptr, step.col_idx, rep_t,
                                      rpb, cib, work, wl.k_anchor, o=step.o, lse=step.lse, ws=step.ws, stream=stream)

    for _ in range(3):
        call()
    ms = cuda_time(call, reps, stream)
    binding.check_status(what="anchor-masked step")
    step()  # restore the unmasked call's output in the shared buffers
    vq = valid_sizes(wl.F * wl.k_anchor * wl.W, nbq)
    vk = valid_sizes(n, nb)
    f_anchor = float(4 * D * sum(int((mb[i].astype(np.int64) * np.outer(vq, vk)).sum()) for i in range(len(rep))))
    flops = step.f_sparse + f_anchor
    tflops = flops / (ms * 1e-3) / 1e12
    f_alg = 2.0 * D * (wl.F * wl.k_anchor * wl.W) * n * len(rep)
    return {"calibration": {"inputs": n_in, "eps": eps, "rho": 0.5, "kernel": "calibatt_anchor_block_energy",
                            "ms_per_input": ms_cal / n_in, "energy_tflops": f_alg / (ms_cal / n_in * 1e-3) / 1e12},
            "anchor_block_sparsity": 1.0 - float(mb.mean()), "ms_per_call": ms, "kept_tile_tflops": tflops,
            "frac_of_bf16_burst": frac_of(tflops, pk, "bf16_tflops"), "kept_tile_flops": flops,
            "speedup_vs_unmasked_step": None}


def attention_config(binding, name, dev, pk, reps, with_library):
    """Skip lists (calibrated or random), then one attention call timed, and
    the same kernel at 0 % sparsity, on a stream of its own (CUDA graphs time
    the launch-bound small workloads; they cannot capture the legacy stream)."""
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        out, step = _attention_config(binding, name, dev, stream, pk, reps, with_library)
    torch.cuda.synchronize()
    return out, step


def _attention_config(binding, name, dev, stream, pk, reps, with_library):
    wl = synth.WORKLOADS[name]
    masks, row_ptr, col_idx, calib = skip_lists(binding, wl, dev, stream)
    step = Step(binding, wl, masks, row_ptr, col_idx, dev, stream)
    for _ in range(3):
        step()
    timer = graph_time if wl.n * wl.heads < 1_000_000 else cuda_time
    ms = timer(step, reps, stream)
    binding.check_status(what=name)
    dense_ms = dense_run(binding, step.q, step.k, step.v, step.o, step.lse, wl.heads, wl.nb, dev, stream,
                         max(2, reps // 3)) if wl.n * wl.heads >= 1_000_000 else None
    if dense_ms is None:
        # launch-bound sizes: the dense run through a graph as well
        full = torch.ones((wl.heads, wl.nb, wl.nb), dtype=torch.int16, device=dev).view(torch.uint16)
        _, rpf, cif, _ = binding.aggregate_masks(full, 1, 0.5)
        rpf_h = rpf.cpu().numpy()
        wf = torch.from_numpy(binding.build_plan(rpf_h, wl.heads, wl.nb)).to(dev)
        dense_ms = graph_time(lambda: binding.sparse_attn_fwd(step.q, step.k, step.v, rpf, cif, wf, o=step.o,
                                                              lse=step.lse, stream=stream), reps, stream)
    lib = library_dense(step.q, step.k, step.v, stream, max(2, reps // 3),
                        float(4 * D * wl.n * wl.n * wl.heads)) if with_library else None
    step()  # the dense run wrote the same output buffers: restore the call's result
    out = step.summary(ms, dense_ms, pk, lib)
    out["skip_lists"] = calib
    if step.rep:
        n_cal, eps_cal = synth.CALIBRATION[name]
        am = anchor_masked_step(binding, step, dev, stream, pk, reps, n_cal, eps_cal)
        am["speedup_vs_unmasked_step"] = ms / am["ms_per_call"]
        out["anchor_masked"] = am
    return out, step


def calibration_kernels(binding, wl, q, k, dev, stream, pk):
    """The calibration kernels on one input of the full Wan-720p shape (all
    heads): both energy kernels with fused selection, standalone selection,
    aggregation into the skip list, pixel-row profiles and the spatial score.
    The bandwidth-bound ones are timed through CUDA graphs and reported
    against the measured HBM copy bandwidth."""
    heads, nb, n = wl.heads, wl.nb, wl.n
    hbm = pk.get("hbm_gbs")
    lse_ws = torch.empty((heads, nb * 128), dtype=torch.float32, device=dev)
    energy = torch.empty((heads, nb, nb), dtype=torch.float32, device=dev)
    cmask = torch.empty((heads, nb, nb), dtype=torch.uint8, device=dev)
    ccounts = torch.zeros((heads, nb, nb), dtype=torch.uint16, device=dev)

    def energy_call():
        binding.block_energy(q, k, eps=0.9, energy=energy, mask=cmask, counts=ccounts, lse_ws=lse_ws, stream=stream)

    energy_call()
    e_ms = cuda_time(energy_call, 2, stream)
    ews = torch.empty(binding.energy_workspace_size(heads, n), dtype=torch.uint8, device=dev)

    def energy1_call():
        binding.block_energy_1pass(q, k, eps=0.9, energy=energy, mask=cmask, counts=ccounts, ws=ews, stream=stream)

    energy1_call()
    e1_ms = cuda_time(energy1_call, 2, stream)
    del ews
    f_alg = float(2 * D * n * n * heads)  # one S = Q K^T per input
    gstream = torch.cuda.Stream()
    tie = torch.empty((heads, nb), dtype=torch.uint8, device=dev)

    def select_call():
        binding.select_mask(energy, 0.9, mask=cmask, kept=False, tie=tie, stream=torch.cuda.current_stream())

    with torch.cuda.stream(gstream):
        s_ms = graph_time(select_call, 20, gstream)
    sel_bytes = heads * nb * nb * (4 + 1) + heads * nb
    agg_ws = torch.empty(binding.load().calibatt_aggregate_workspace_size(heads, nb), dtype=torch.uint8, device=dev)
    am = torch.empty((heads, nb, nb), dtype=torch.uint8, device=dev)
    arp = torch.empty(heads * nb + 1, dtype=torch.int32, device=dev)
    aci = torch.empty(heads * nb * nb, dtype=torch.int32, device=dev)
    annz = torch.zeros(1, dtype=torch.int64, device=dev)
    lib = binding.load()

    # the aggregation's input: this input's eps = 0.9 selection as the counts
    # of one input (kept where the mask is), so the skip list has ~19 % of the
    # blocks
    acounts = cmask.to(torch.int16).view(torch.uint16)

    def agg_call():
        lib.calibatt_aggregate_masks(binding._ptr(acounts), 1, heads, nb, 0.5, binding._ptr(am),
                                     binding._ptr(arp), binding._ptr(aci), aci.numel(), binding._ptr(annz),
                                     binding._ptr(agg_ws), agg_ws.numel(),
                                     binding._stream(torch.cuda.current_stream()))

    with torch.cuda.stream(gstream):
        a_ms = graph_time(agg_call, 20, gstream)
    pix = torch.empty((heads, wl.F * wl.H, nb), dtype=torch.float32, device=dev)

    def pix_call():
        binding.pixel_row_energy(q, k, wl.F, wl.H, wl.W, pix=pix, lse_ws=lse_ws, stream=stream)

    pix_call()
    p_ms = cuda_time(pix_call, 2, stream)
    sscore = torch.empty(heads, dtype=torch.float32, device=dev)
    sflag = torch.empty(heads, dtype=torch.uint8, device=dev)

    def score_call():
        binding.spatial_score(pix, wl.F, wl.H, wl.k_anchor, score=sscore, flag=sflag,
                              stream=torch.cuda.current_stream())

    with torch.cuda.stream(gstream):
        sc_ms = graph_time(score_call, 20, gstream)
    binding.check_status(what="calibration kernels")
    kept_agg = int(annz.item())
    agg_bytes = heads * nb * nb * (2 + 1) + kept_agg * 4 + (heads * nb + 1) * 4
    score_bytes = heads * wl.F * wl.H * nb * 4  # every profile row read once
    out = {
        "shape": f"{heads} heads x N={n}",
        "energy_2pass_ms": e_ms, "energy_2pass_tflops_algorithmic": f_alg / (e_ms * 1e-3) / 1e12,
        "energy_2pass_tflops_issued": 2 * f_alg / (e_ms * 1e-3) / 1e12,
        "energy_1pass_ms": e1_ms, "energy_1pass_tflops": f_alg / (e1_ms * 1e-3) / 1e12,
        "select_ms": s_ms, "select_gbs": sel_bytes / (s_ms * 1e-3) / 1e9,
        "select_bytes": sel_bytes,
        "aggregate_ms": a_ms, "aggregate_gbs": agg_bytes / (a_ms * 1e-3) / 1e9, "aggregate_bytes": agg_bytes,
        "aggregate_kept_blocks": kept_agg,
        "eps": 0.9, "kept_fraction_at_eps": float(cmask.float().mean().item()),
        "tie_affected_rows_at_eps": int(tie.sum().item()),
        "pixel_row_energy_ms": p_ms, "pixel_row_energy_tflops_issued": 2 * f_alg / (p_ms * 1e-3) / 1e12,
        "spatial_score_ms": sc_ms, "spatial_score_gbs": score_bytes / (sc_ms * 1e-3) / 1e9,
        "spatial_flagged_heads": np.nonzero(sflag.cpu().numpy())[0].tolist(),
    }
    if hbm:
        for key in ("select", "aggregate", "spatial_score"):
            out[key + "_frac_of_hbm"] = out[key + "_gbs"] / hbm
    return out


def calib_sweep(binding, dev, stream, pk, n_in):
    """The calibration sweep workload: 40 heads of the Wan-720p shape, n_in
    inputs (64), eps in {0.84, 0.9, 0.95, 0.99}, rho = 0.5. Each input's
    energies come from the single-pass kernel (the full P never reaches HBM)
    and stay on the device; the standalone selection then runs at every eps,
    folding each mask into that eps's counts, and the counts are aggregated
    into the skip list."""
    wl = synth.WORKLOADS["calib720"]
    heads, nb, n = wl.heads, wl.nb, wl.n
    hbm = pk.get("hbm_gbs")
    ws = torch.empty(binding.energy_workspace_size(heads, n), dtype=torch.uint8, device=dev)
    energies, e_ms = [], 0.0
    fused_ms = None
    for p in range(n_in):
        q, k, _ = synth.qkv(wl, p, with_v=False, device=dev)
        E = torch.empty((heads, nb, nb), dtype=torch.float32, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        binding.block_energy_1pass(q, k, energy=E, ws=ws, stream=stream)
        e1.record(stream)
        if p == 0:
            # the same pass with the selection fused (eps = 0.9), for its cost
            fm = torch.empty((heads, nb, nb), dtype=torch.uint8, device=dev)
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            binding.block_energy_1pass(q, k, eps=0.9, energy=False, mask=fm, ws=ws, stream=stream)
            f1.record(stream)
            f1.synchronize()
            fused_ms = f0.elapsed_time(f1)
            del fm
        e1.synchronize()
        e_ms += e0.elapsed_time(e1)
        energies.append(E)
        del q, k
    del ws
    f_alg = float(2 * D * n * n * heads)
    out = {"shape": f"{heads} heads x N={n} (F={wl.F},H={wl.H},W={wl.W}), d={D}", "inputs": n_in, "rho": 0.5,
           "energy_kernel": "calibatt_block_energy_1pass",
           "energy_ms_per_input": e_ms / n_in, "energy_tflops": f_alg / (e_ms / n_in * 1e-3) / 1e12,
           "energy_fused_select_ms": fused_ms,
           "energy_fused_select_tflops": f_alg / (fused_ms * 1e-3) / 1e12 if fused_ms else None, "eps": {}}
    agg_ws = torch.empty(binding.load().calibatt_aggregate_workspace_size(heads, nb), dtype=torch.uint8, device=dev)
    tie = torch.empty((heads, nb), dtype=torch.uint8, device=dev)
    cells = heads * nb * nb
    for eps in (0.84, 0.9, 0.95, 0.99):
        counts = torch.zeros((heads, nb, nb), dtype=torch.uint16, device=dev)
        ties = 0
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tie_sum = torch.zeros((), dtype=torch.int64, device=dev)
        torch.cuda.synchronize()
        s0.record(stream)
        for E in energies:
            binding.select_mask(E, eps, mask=False, kept=False, counts=counts, tie=tie, stream=stream)
            with torch.cuda.stream(stream):
                tie_sum += tie.sum()
        s1.record(stream)
        s1.synchronize()
        sel_ms = s0.elapsed_time(s1) / n_in
        ties = int(tie_sum.item())
        kept_cells = int((counts.view(torch.int16).to(torch.int32) & 0xFFFF).sum().item())
        mask, row_ptr, col_idx, nnz = binding.aggregate_masks(counts, n_in, 0.5, ws=agg_ws, stream=stream)
        nnz_v = int(nnz.item())

        def agg_call():
            binding.aggregate_masks(counts, n_in, 0.5, ws=agg_ws, stream=torch.cuda.current_stream(), trim=False)

        gstream = torch.cuda.Stream()
        with torch.cuda.stream(gstream):
            a_ms = graph_time(agg_call, 10, gstream)
        binding.check_status(what=f"sweep eps {eps}")
        # selection: the energies read, plus each kept block's count read and written
        sel_bytes = cells * 4 + (kept_cells / n_in) * 4 + heads * nb
        agg_bytes = cells * (2 + 1) + nnz_v * 4 + (heads * nb + 1) * 4
        e = {"block_sparsity": 1.0 - nnz_v / cells, "kept_blocks": nnz_v,
             "mean_kept_fraction_per_input": kept_cells / n_in / cells,
             "tie_affected_selections": ties, "selections": n_in * heads * nb, "tie_window": binding.TIE_WINDOW,
             "select_ms_per_input": sel_ms, "select_gbs": sel_bytes / (sel_ms * 1e-3) / 1e9,
             "aggregate_ms": a_ms, "aggregate_gbs": agg_bytes / (a_ms * 1e-3) / 1e9}
        if hbm:
            e["select_frac_of_hbm"] = e["select_gbs"] / hbm
            e["aggregate_frac_of_hbm"] = e["aggregate_gbs"] / hbm
        out["eps"][str(eps)] = e
        del counts, mask, row_ptr, col_idx
    del energies
    return out


def fp8_probe(binding, name, n_in, dev, stream):
    """Calibration with q and k rounded to FP8 e4m3 (the operands an FP8
    Q K^T would see; products are exact in fp32 either way) against the same
    calibration in bf16: energy error, selections that change, aggregated
    cells that change."""
    wl = synth.WORKLOADS[name]
    heads, nb, n = wl.heads, wl.nb, wl.n
    eps = synth.CALIBRATION[name][1]
    ws = torch.empty(binding.energy_workspace_size(heads, n), dtype=torch.uint8, device=dev)
    c16 = torch.zeros((heads, nb, nb), dtype=torch.uint16, device=dev)
    c8 = torch.zeros_like(c16)
    t16 = torch.empty((heads, nb), dtype=torch.uint8, device=dev)
    max_rel, max_abs_rowmax, rows_diff, rows_diff_untied, rows = 0.0, 0.0, 0, 0, 0
    for p in range(n_in):
        q, k, _ = synth.qkv(wl, p, with_v=False, device=dev)
        E16, m16, _, _, _, _ = binding.block_energy_1pass(q, k, eps=eps, mask=torch.empty(
            (heads, nb, nb), dtype=torch.uint8, device=dev), counts=c16, ws=ws, tie=t16, stream=stream)
        q8 = q.to(torch.float8_e4m3fn).to(torch.bfloat16)
        k8 = k.to(torch.float8_e4m3fn).to(torch.bfloat16)
        E8, m8, _, _, _ = binding.block_energy_1pass(q8, k8, eps=eps, mask=torch.empty(
            (heads, nb, nb), dtype=torch.uint8, device=dev), counts=c8, ws=ws, stream=stream)
        rowmax = E16.amax(-1, keepdim=True)
        sig = E16 >= 1e-3 * rowmax
        max_rel = max(max_rel, float(((E8 - E16).abs() / E16.clamp_min(1e-30))[sig].max().item()))
        max_abs_rowmax = max(max_abs_rowmax, float(((E8 - E16).abs() / rowmax).max().item()))
        d = (m16 != m8).any(-1)
        rows_diff += int(d.sum().item())
        rows_diff_untied += int((d & (t16 == 0)).sum().item())
        rows += heads * nb
    a16, _, _, _ = binding.aggregate_masks(c16, n_in, 0.5, stream=stream)
    a8, _, _, _ = binding.aggregate_masks(c8, n_in, 0.5, stream=stream)
    binding.check_status(what="fp8 probe")
    return {"inputs": n_in, "eps": eps, "rounding": "q and k to float8_e4m3fn (no scaling), energies otherwise bf16",
            "max_rel_energy_error_on_entries_above_1e-3_rowmax": max_rel,
            "max_abs_energy_error_over_rowmax": max_abs_rowmax,
            "selection_rows_changed": rows_diff, "selection_rows_changed_not_tie_affected_at_1e-6": rows_diff_untied,
            "selection_rows": rows, "aggregated_cells_changed": int((a16 != a8).sum().item()),
            "aggregated_cells": heads * nb * nb}


def run_calib_only(args):
    """Only the calibration kernels (energy, selection, aggregation, profiles,
    spatial score) on the first --heads heads of the Wan-720p shape: the small
    case that ncu captures of those kernels run."""
    from calibrated_block_sparse_b200 import binding
    binding.load()
    import dataclasses
    wl = synth.WORKLOADS["calib720"]
    wl = dataclasses.replace(wl, heads=args.heads or wl.heads)
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    pk, _ = peaks()
    q, k, _ = synth.qkv(wl, 0, with_v=False, device=dev)
    out = calibration_kernels(binding, wl, q, k, dev, stream, pk)
    print(json.dumps({"calibration_kernels": out}), flush=True)


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
    pk, pk_src = peaks()
    n, nb, heads = wl.n, wl.nb, wl.heads
    rep_heads = list(wl.repeat_heads)
    sparse_heads = [h for h in range(heads) if h not in rep_heads]

    # inputs and skip lists: resident in HBM before the timed region
    masks, row_ptr, col_idx, calib_info = skip_lists(binding, wl, dev, stream)
    row_ptr_h = row_ptr.cpu().numpy()
    # --shard heads: one call split over the ranks by heads (balanced by kept
    # tiles, no exchange), strong scaling; else a replica of the call per rank
    shard = args.shard == "heads" and world > 1
    owner = None
    if shard:
        owner, _ = binding.shard_heads(row_ptr_h, heads, nb, rep_heads, wl.F, wl.W, wl.k_anchor, world)
        my_rep = [h for h in rep_heads if owner[h] == rank]
    else:
        my_rep = rep_heads
    step = Step(binding, wl, masks, row_ptr, col_idx, dev, stream, input_idx=1000 + rank, rep_heads=my_rep)
    if shard:
        work_np, _ = binding.build_rank_plan(row_ptr_h, heads, nb, rep_heads, owner, rank, wl.F, wl.H, wl.W,
                                             wl.k_anchor)
        step.work = torch.from_numpy(binding.balance_plan(work_np, row_ptr_h, heads, nb)).to(dev)
        mine = [h for h in sparse_heads if owner[h] == rank]
        step.flops = sparse_flops(masks, mine, n) + repeat_flops(wl, len(my_rep))
        step.tiles = int(sum(int(masks[h].sum()) for h in mine)) + \
            len(my_rep) * -(-wl.F * wl.k_anchor * wl.W // 128) * nb
    f_step = sparse_flops(masks, sparse_heads, n) + repeat_flops(wl, len(rep_heads))  # the whole call
    q, k, v, o, lse = step.q, step.k, step.v, step.o, step.lse

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
    # weak scaling: every rank runs the whole call (replicas); strong: the
    # ranks share one call
    value = (1 if shard else world) * f_step / (ms_step * 1e-3) / 1e12
    reps = max(2, min(5, args.steps))

    # the same work as two separate calls (block-sparse, then repeated heads)
    separate = None
    if not shard:
        head_active = np.array([h not in rep_heads for h in range(heads)], np.uint8)
        work_s = torch.from_numpy(binding.balance_plan(binding.build_plan(row_ptr_h, heads, nb, head_active),
                                                       row_ptr_h, heads, nb)).to(dev)

        def sparse_call():
            binding.sparse_attn_fwd(q, k, v, row_ptr, col_idx, work_s, o=o, lse=lse, stream=stream)

        def repeat_call():
            if rep_heads:
                binding.repeat_attn_fwd(q, k, v, wl.F, wl.H, wl.W, step.rep_t, wl.k_anchor, o=o, lse=lse, ws=step.ws,
                                        stream=stream)

        sparse_ms = cuda_time(sparse_call, reps, stream)
        repeat_ms = cuda_time(repeat_call, reps, stream) if rep_heads else 0.0
        binding.check_status(what="separate calls")
        separate = {"sparse_ms": sparse_ms, "repeat_ms": repeat_ms,
                    "sparse_tflops": step.f_sparse / (sparse_ms * 1e-3) / 1e12}

    # ---- 0 %-sparse run: the same kernel with every block kept, all heads
    dense_ms = dense_run(binding, q, k, v, o, lse, heads, nb, dev, stream, reps)
    f_dense = float(4 * D * n * n * heads)
    lib_dense = library_dense(q, k, v, stream, reps, f_dense)
    if "ms" in lib_dense:
        lib_dense["step_speedup"] = lib_dense["ms"] / ms_step

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

    # ---- roofline of the dominant kernel: the attention kernel of the step
    # (block-sparse and repeated heads in one launch; its event window also
    # holds the short anchor-gather launch before it)
    long_run = elapsed_ms > 1000.0
    peak = pk.get("bf16_tflops_sustained" if long_run else "bf16_tflops")
    achieved = step.flops / (attn_ms * 1e-3) / 1e12
    kname = ("attn_kernel<attention> (%d block-sparse + %d repeated heads, one launch; window includes the "
             "anchor gather)" % (len(sparse_heads), len(rep_heads)))
    if shard:
        kname += "; rank 0 share of the heads"
    traffic = args.traffic_bytes if args.traffic_bytes else TRAFFIC_PER_TILE * step.tiles
    roofline = {"bound": "tensor", "kernel": kname,
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": f"{pk_src} {'sustained' if long_run else 'burst'} bf16",
                "traffic": traffic,
                "traffic_source": "given" if args.traffic_bytes else
                "ncu dram bytes per kept tile of a 5-head capture, scaled by the %d kept tiles of this launch"
                % step.tiles,
                "algorithmic_bytes": 4.0 * heads * n * D * 2}

    # ---- the other workloads, the calibration kernels and the sweep (rank 0
    # of a one-GPU run; each is timed on its own after the timed region)
    configs = {args.workload: step.summary(ms_step, dense_ms, pk, lib_dense)}
    configs[args.workload]["skip_lists"] = calib_info
    if world == 1 and not args.heads and step.rep and args.workload == "wan720":
        # anchor-row masks of the repeated heads, calibrated at eps(T/2)
        am = anchor_masked_step(binding, step, dev, stream, pk, reps, 4, synth.CALIBRATION["wan480"][1])
        am["speedup_vs_unmasked_step"] = ms_step / am["ms_per_call"]
        configs[args.workload]["anchor_masked"] = am
    calib = sweep = fp8 = tiny_step = None
    if world == 1 and not args.heads:
        for name in (args.configs or []):
            if name in configs:
                continue
            if name == "calib720":
                sweep = calib_sweep(binding, dev, stream, pk, args.sweep_inputs)
                configs[name] = sweep
            else:
                res, st = attention_config(binding, name, dev, pk, reps=max(6, args.steps // 2),
                                           with_library=name != "tiny")
                configs[name] = res
                if name == "tiny":
                    tiny_step = st
                del st
            torch.cuda.empty_cache()
        if not args.no_calib:
            calib = calibration_kernels(binding, wl, q, k, dev, stream, pk)
        if args.fp8_probe:
            fp8 = {name: fp8_probe(binding, name, n_in, dev, stream) for name, n_in in (("tiny", 8), ("wan480", 4))}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        hs = [sparse_heads[0]]
        qc, kc, vc = (t[hs].cpu() for t in (q, k, v))
        s, f, rows, threads = cpu_oracle_sample(wl, qc, kc, vc, [0], np.stack([masks[h] for h in hs]),
                                                args.cpu_seconds, np.random.default_rng(5))
        cpu = {"value": f / s / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{rows} query rows of one block-sparse head, fp64 plain-C oracle, {s:.1f} s"}
        if tiny_step is not None:
            cpu["tiny_full"] = tiny_oracle_full(tiny_step, configs["tiny"])

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if shard else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": arm_config(wl, heads, step.kept_frac, world, shard),
            "gpu_launches": step.launches * args.steps,
            "attn_ms": attn_ms,
            "separate_calls": separate,
            "dense_ms": dense_ms, "dense_tflops": f_dense / (dense_ms * 1e-3) / 1e12,
            "speedup_vs_dense": dense_ms / ms_step,
            "library_dense": lib_dense,
            "roofline": roofline, "e2e": e2e, "cpu_baseline": cpu,
            "configs": configs, "calibration": calib, "fp8_probe": fp8,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)


def tiny_oracle_full(step, gpu_summary):
    """The oracle's whole tiny pipeline, timed on the host cores: calibration
    energies of the 8 inputs, greedy selection, aggregation, skip list, and the
    masked attention of the held-out input. Reported beside it: the aggregated
    cells where the oracle's mask and the GPU's differ (a selection whose cut
    lies within the energy error of eps can go either way), and the largest
    error of the GPU's output against the oracle's attention over the GPU's
    own calibrated mask (the parity rule for the attention)."""
    import oracle
    wl = step.wl
    threads = os.cpu_count() or 1
    n_cal, eps = synth.CALIBRATION["tiny"]
    t0 = time.perf_counter()
    masks = []
    for p in range(n_cal):
        qc, kc, _ = synth.qkv(wl, p, with_v=False)
        E = oracle.block_energy(synth.bf16_bits(qc), synth.bf16_bits(kc), threads=threads)
        m, _ = oracle.select(E, eps)
        masks.append(m)
    agg, _ = oracle.aggregate(np.stack(masks), 0.5)
    oracle.mask_to_csr(agg)
    qb, kb, vb = (synth.bf16_bits(t) for t in (step.q, step.k, step.v))
    oracle.masked_attention(qb, kb, vb, agg, threads=threads)
    secs = time.perf_counter() - t0
    o_ref, _ = oracle.masked_attention(qb, kb, vb, step.masks, threads=threads)
    o_gpu = step.o.float().cpu().numpy().astype(np.float64)
    err = float(np.max(np.abs(o_gpu - o_ref)))
    return {"seconds": secs, "cores": threads, "what": "calibration of 8 inputs + selection + aggregation + "
            "attention of the held-out input, fp64 plain C",
            "max_abs_output_error_gpu_vs_oracle": err, "tolerance": 1e-2 * float(np.max(np.abs(o_ref))) + 1e-3,
            "mask_cells_differing_from_gpu": int(np.sum(agg != step.masks))}


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
    ap.add_argument("--configs", default="tiny,wan480,mochi480,calib720",
                    help="other workloads reported under 'configs' (comma-separated; 'none' for none)")
    ap.add_argument("--sweep-inputs", type=int, default=64, help="calibration inputs of the sweep workload")
    ap.add_argument("--no-fp8-probe", dest="fp8_probe", action="store_false")
    ap.add_argument("--calib-only", action="store_true",
                    help="only the calibration kernels on --heads heads of the Wan-720p shape (profiling case)")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="dram bytes per launch of the sparse kernel from an ncu capture")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    args.configs = [] if args.configs in ("", "none") else [c.strip() for c in args.configs.split(",")]
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.calib_only:
            run_calib_only(args)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
