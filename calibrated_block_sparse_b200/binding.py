"""ctypes binding of libcalibatt (include/calibatt.h): argument marshalling only.

Every step of the hot path runs in the CUDA library; this module turns torch
tensors into pointers, sizes and the current CUDA stream, allocates outputs
with torch when the caller does not pass them, and raises ``CalibattError``
on a nonzero status. There is no CPU fallback: if the library is missing the
import of a compute function fails loudly.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import numpy as np
import torch

from . import build as _build

_lock = threading.Lock()
_lib = None

BLOCK = 128
HEAD_DIM = 128


class CalibattError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})" if what else f"{strerror(code)} ({code})")


def library_path() -> str:
    """Path of libcalibatt.so: CALIBATT_LIBRARY if set, else the in-tree build."""
    return os.environ.get("CALIBATT_LIBRARY") or _build.LIB


def load(build_if_missing: bool = False):
    """Load libcalibatt.so (optionally building it first). Raises if absent."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if build_if_missing and _build.needs_build():
            _build.build()
        if not os.path.exists(path):
            raise ImportError(f"libcalibatt.so is not built ({path}); run python -m calibrated_block_sparse_b200.build")
        lib = ctypes.CDLL(path)
        P, i32, i64, f32, f64, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                                     ctypes.c_double, ctypes.c_size_t)
        sig = {
            "calibatt_strerror": (ctypes.c_char_p, [i32]),
            "calibatt_version": (i32, []),
            "calibatt_get_status": (i32, [P]),
            "calibatt_set_wait_limit": (i32, [f64]),
            "calibatt_eps_schedule": (f64, [f64, f64, f64, f64, f64]),
            "calibatt_validate_csr": (i32, [P, P, i32, i32, i64]),
            "calibatt_build_plan": (i32, [P, i32, i32, P, P, P]),
            "calibatt_anchor_rows": (i32, [i32, i32, P]),
            "calibatt_rho_threshold": (i32, [i32, f64, P]),
            "calibatt_sparse_attn_fwd": (i32, [P, P, P, i32, i32, i32, f32, P, P, i64, P, i32, P, P, P]),
            "calibatt_repeat_workspace_size": (sz, [i32, i32, i32, i32, i32]),
            "calibatt_repeat_attn_fwd": (i32, [P, P, P, i32, i32, i32, i32, i32, i32, f32, P, i32, P, P, P, sz, P]),
            "calibatt_block_energy": (i32, [P, P, i32, i32, i32, f32, P, P, i32, f64, P, P, P, P, f64, P]),
            "calibatt_select_mask": (i32, [P, i32, i32, f64, P, P, P, P, f64, P]),
            "calibatt_accumulate_masks": (i32, [P, i64, P, P]),
            "calibatt_aggregate_workspace_size": (sz, [i32, i32]),
            "calibatt_aggregate_masks": (i32, [P, i32, i32, i32, f64, P, P, P, i64, P, P, sz, P]),
            "calibatt_aggregate_masks_noalloc": (i32, [P, i32, i32, i32, f64, P, P, P, i64, P, P]),
            "calibatt_pixel_row_energy": (i32, [P, P, i32, i32, i32, i32, i32, f32, P, P, P, P]),
            "calibatt_build_mixed_plan": (i32, [P, i32, i32, P, i32, P, i32, i32, i32, i32, P, P]),
            "calibatt_balance_plan": (i32, [P, i32, P, i32, i32, i32]),
            "calibatt_keep_histogram": (i32, [P, i32, i64, i32, P, P]),
            "calibatt_energy_workspace_size": (sz, [i32, i32]),
            "calibatt_shard_heads": (i32, [P, i32, i32, P, i32, i32, i32, i32, i32, P, P]),
            "calibatt_mixed_host_workspace_size": (sz, [i32, i32, i32, i32, i32, i32, i32]),
            "calibatt_mixed_attn_fwd_host": (i32, [P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, P, P, P, i64, P,
                                                   i32, i32, P, P, P, P, P, P, sz, P]),
            "calibatt_block_energy_1pass": (i32, [P, P, i32, i32, i32, f32, P, sz, P, i32, f64, P, P, P, P, f64, P,
                                                  i32, P]),
            "calibatt_bank_create": (P, [i32, i32, i32, i32, i32, i32, i32]),
            "calibatt_bank_destroy": (None, [P]),
            "calibatt_bank_entry_bytes": (sz, [P, i64, i32]),
            "calibatt_bank_put": (i32, [P, i32, i32, f64, P, P, i64, P, i32, P, sz, P]),
            "calibatt_bank_get": (i32, [P, i32, i32, P]),
            "calibatt_mixed_attn_fwd": (i32, [P, P, P, i32, i32, i32, i32, i32, i32, f32, P, P, i64, P, i32, P, i32,
                                              P, P, P, sz, P]),
            "calibatt_spatial_score": (i32, [P, i32, i32, i32, i32, i32, f32, P, P, P]),
            "calibatt_balance_mixed_plan": (i32, [P, i32, P, i32, i32, P, i32, i32, i32, i32, i32]),
            "calibatt_mixed_masked_attn_fwd": (i32, [P, P, P, i32, i32, i32, i32, i32, i32, f32, P, P, i64, P, i32,
                                                     P, P, i64, P, i32, P, P, P, sz, P]),
            "calibatt_anchor_energy_workspace_size": (sz, [i32, i32, i32, i32, i32, i32]),
            "calibatt_anchor_block_energy": (i32, [P, P, i32, i32, i32, i32, i32, i32, f32, P, i32, P, sz, P, i32,
                                                   f64, P, P, P, P, f64, P]),
            "calibatt_aggregate_rows_workspace_size": (sz, [i64]),
            "calibatt_aggregate_mask_rows": (i32, [P, i32, i64, i32, f64, P, P, P, i64, P, P, sz, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def strerror(code: int) -> str:
    return load().calibatt_strerror(int(code)).decode()


def _check(rc: int, what: str):
    if rc != 0:
        raise CalibattError(rc, what)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return ctypes.c_void_p(t.ctypes.data)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _cuda_tensor(t, dtype, name):
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise TypeError(f"{name} must be a contiguous CUDA {dtype} tensor")
    return t


def _bhnd(q, name="q"):
    _cuda_tensor(q, torch.bfloat16, name)
    if q.dim() != 3 or q.shape[-1] != HEAD_DIM:
        raise ValueError(f"{name} must be [heads][n][{HEAD_DIM}]")
    return q.shape[0], q.shape[1]


# ------------------------------------------------------------------ host helpers

def get_status(stream=None) -> int:
    return load().calibatt_get_status(_stream(stream))


def check_status(stream=None, what="kernel"):
    _check(get_status(stream), what)


def set_wait_limit(seconds: float = 0.0):
    """Limit of the bounded in-kernel waits of later launches on the current
    device (0: the default of 2 s)."""
    _check(load().calibatt_set_wait_limit(float(seconds)), "calibatt_set_wait_limit")


TIE_WINDOW = 1e-6  # decisions within this distance of the threshold are counted


def _tie_out(tie, rows_shape, dev):
    if tie is True:
        return torch.empty(rows_shape, dtype=torch.uint8, device=dev)
    if tie is False or tie is None:
        return None
    return tie


def eps_schedule(A, C, k, t, T) -> float:
    return load().calibatt_eps_schedule(float(A), float(C), float(k), float(t), float(T))


def validate_csr(row_ptr: np.ndarray, col_idx: np.ndarray, heads: int, nb: int) -> int:
    rp = np.ascontiguousarray(row_ptr, np.int32)
    ci = np.ascontiguousarray(col_idx, np.int32)
    return load().calibatt_validate_csr(_ptr(rp), _ptr(ci) if ci.size else None, heads, nb, int(ci.size))


def build_plan(row_ptr: np.ndarray, heads: int, nb: int, head_active=None) -> np.ndarray:
    rp = np.ascontiguousarray(row_ptr, np.int32)
    ha = None if head_active is None else np.ascontiguousarray(head_active, np.uint8)
    out = np.empty(heads * nb, np.int32)
    n = np.zeros(1, np.int32)
    _check(load().calibatt_build_plan(_ptr(rp), heads, nb, _ptr(ha), _ptr(out), _ptr(n)), "build_plan")
    return out[: int(n[0])].copy()


def build_mixed_plan(row_ptr: np.ndarray, heads: int, nb: int, rep_heads, F: int, H: int, W: int,
                     k_anchor: int = 5) -> np.ndarray:
    """Work list of the block-sparse units of the heads not in rep_heads and
    the anchor-query units of the repeated heads, head by head."""
    rp = np.ascontiguousarray(row_ptr, np.int32)
    rep = np.ascontiguousarray([int(h) for h in rep_heads], np.int32)
    nbq_b = -(-F * k_anchor * W // BLOCK)
    out = np.empty(heads * nb + len(rep) * nbq_b, np.int32)
    n = np.zeros(1, np.int32)
    _check(load().calibatt_build_mixed_plan(_ptr(rp), heads, nb, None, len(rep), _ptr(rep) if len(rep) else None,
                                            F, H, W, k_anchor, _ptr(out), _ptr(n)), "build_mixed_plan")
    return out[: int(n[0])].copy()


def balance_plan(work_list: np.ndarray, row_ptr: np.ndarray, heads: int, nb: int, n_slots: int = 0) -> np.ndarray:
    """calibatt_balance_plan on a copy of a host work list (n_slots <= 0: two
    per SM of the current device)."""
    w = np.array(work_list, dtype=np.int32, copy=True)
    rp = np.ascontiguousarray(row_ptr, np.int32)
    _check(load().calibatt_balance_plan(_ptr(w), int(w.size), _ptr(rp), int(heads), int(nb), int(n_slots)),
           "calibatt_balance_plan")
    return w


def shard_heads(row_ptr: np.ndarray, heads: int, nb: int, rep_heads, F: int, W: int, k_anchor: int, n_ranks: int):
    """Owner rank of every head and kept tiles per rank (calibatt_shard_heads)."""
    rp = np.ascontiguousarray(row_ptr, np.int32)
    rep = np.ascontiguousarray([int(h) for h in rep_heads], np.int32)
    owner = np.empty(heads, np.int32)
    load_ = np.empty(n_ranks, np.int64)
    _check(load().calibatt_shard_heads(_ptr(rp), heads, nb, _ptr(rep) if len(rep) else None, len(rep), F, W, k_anchor,
                                       n_ranks, _ptr(owner), _ptr(load_)), "shard_heads")
    return owner, load_


def build_rank_plan(row_ptr: np.ndarray, heads: int, nb: int, rep_heads, owner, rank: int, F: int, H: int, W: int,
                    k_anchor: int = 5):
    """Work list and repeated heads of one rank's share of the heads."""
    rp = np.ascontiguousarray(row_ptr, np.int32)
    mine = np.ascontiguousarray(np.asarray(owner) == rank, np.uint8)
    rep = np.ascontiguousarray([int(h) for h in rep_heads if mine[int(h)]], np.int32)
    nbq_b = -(-F * k_anchor * W // BLOCK)
    out = np.empty(heads * nb + len(rep) * nbq_b, np.int32)
    n = np.zeros(1, np.int32)
    _check(load().calibatt_build_mixed_plan(_ptr(rp), heads, nb, _ptr(mine), len(rep), _ptr(rep) if len(rep) else None,
                                            F, H, W, k_anchor, _ptr(out), _ptr(n)), "build_mixed_plan")
    return out[: int(n[0])].copy(), rep.tolist()


def anchor_rows(H: int, k_anchor: int) -> np.ndarray:
    out = np.empty(k_anchor, np.int32)
    _check(load().calibatt_anchor_rows(H, k_anchor, _ptr(out)), "anchor_rows")
    return out


def rho_threshold(n_inputs: int, rho: float) -> int:
    out = np.zeros(1, np.int32)
    _check(load().calibatt_rho_threshold(int(n_inputs), float(rho), _ptr(out)), "rho_threshold")
    return int(out[0])


# ------------------------------------------------------------------ inference

def sparse_attn_fwd(q, k, v, row_ptr, col_idx, work_list, o=None, lse=None, scale=None, want_lse=True,
                    stream=None):
    """Block-sparse attention over a skip list; returns (o, lse)."""
    heads, n = _bhnd(q)
    _bhnd(k, "k")
    _bhnd(v, "v")
    _cuda_tensor(row_ptr, torch.int32, "row_ptr")
    _cuda_tensor(col_idx, torch.int32, "col_idx")
    _cuda_tensor(work_list, torch.int32, "work_list")
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((heads, n), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(HEAD_DIM) if scale is None else float(scale)
    rc = load().calibatt_sparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), heads, n, HEAD_DIM, scale, _ptr(row_ptr),
                                         _ptr(col_idx) if col_idx.numel() else None, col_idx.numel(),
                                         _ptr(work_list) if work_list.numel() else None, work_list.numel(),
                                         _ptr(o), _ptr(lse), _stream(stream))
    _check(rc, "calibatt_sparse_attn_fwd")
    return o, lse


def repeat_workspace_size(n_rep, F, H, W, k_anchor=5) -> int:
    return load().calibatt_repeat_workspace_size(n_rep, F, H, W, k_anchor)


def repeat_attn_fwd(q, k, v, F, H, W, rep_heads, k_anchor=5, o=None, lse=None, ws=None, scale=None,
                    want_lse=True, stream=None):
    """Anchor-row attention of repeated heads broadcast to every row; returns (o, lse)."""
    heads, n = _bhnd(q)
    _cuda_tensor(rep_heads, torch.int32, "rep_heads")
    n_rep = rep_heads.numel()
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((heads, n), dtype=torch.float32, device=q.device)
    need = repeat_workspace_size(max(n_rep, 1), F, H, W, k_anchor)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(HEAD_DIM) if scale is None else float(scale)
    rc = load().calibatt_repeat_attn_fwd(_ptr(q), _ptr(k), _ptr(v), heads, F, H, W, HEAD_DIM, k_anchor, scale,
                                         _ptr(rep_heads), n_rep, _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
                                         _stream(stream))
    _check(rc, "calibatt_repeat_attn_fwd")
    return o, lse


def mixed_attn_fwd(q, k, v, F, H, W, row_ptr, col_idx, rep_heads, work_list, k_anchor=5, o=None, lse=None,
                   ws=None, scale=None, want_lse=True, stream=None):
    """Block-sparse and repeated heads in one persistent launch; returns (o, lse)."""
    heads, n = _bhnd(q)
    _bhnd(k, "k")
    _bhnd(v, "v")
    _cuda_tensor(row_ptr, torch.int32, "row_ptr")
    _cuda_tensor(col_idx, torch.int32, "col_idx")
    _cuda_tensor(rep_heads, torch.int32, "rep_heads")
    _cuda_tensor(work_list, torch.int32, "work_list")
    n_rep = rep_heads.numel()
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((heads, n), dtype=torch.float32, device=q.device)
    if ws is None and n_rep > 0:
        ws = torch.empty(repeat_workspace_size(n_rep, F, H, W, k_anchor), dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(HEAD_DIM) if scale is None else float(scale)
    rc = load().calibatt_mixed_attn_fwd(_ptr(q), _ptr(k), _ptr(v), heads, F, H, W, HEAD_DIM, k_anchor, scale,
                                        _ptr(row_ptr), _ptr(col_idx) if col_idx.numel() else None, col_idx.numel(),
                                        _ptr(rep_heads) if n_rep else None, n_rep,
                                        _ptr(work_list) if work_list.numel() else None, work_list.numel(),
                                        _ptr(o), _ptr(lse), _ptr(ws), ws.numel() if ws is not None else 0,
                                        _stream(stream))
    _check(rc, "calibatt_mixed_attn_fwd")
    return o, lse


def anchor_blocks(F, W, k_anchor=5) -> int:
    """Blocks of 128 packed anchor queries of one repeated head."""
    return -(-F * k_anchor * W // BLOCK)


def balance_mixed_plan(work_list: np.ndarray, row_ptr: np.ndarray, heads: int, nb: int, row_ptr_b, n_rep: int,
                       F: int, W: int, k_anchor: int = 5, n_slots: int = 0) -> np.ndarray:
    """calibatt_balance_mixed_plan on a copy of a host work list (anchor units
    costed by the anchor skip list row_ptr_b, host int32)."""
    w = np.array(work_list, dtype=np.int32, copy=True)
    rp = np.ascontiguousarray(row_ptr, np.int32)
    rpb = None if row_ptr_b is None else np.ascontiguousarray(row_ptr_b, np.int32)
    _check(load().calibatt_balance_mixed_plan(_ptr(w), int(w.size), _ptr(rp), int(heads), int(nb), _ptr(rpb),
                                              int(n_rep), int(F), int(W), int(k_anchor), int(n_slots)),
           "calibatt_balance_mixed_plan")
    return w


def mixed_masked_attn_fwd(q, k, v, F, H, W, row_ptr, col_idx, rep_heads, row_ptr_b, col_idx_b, work_list, k_anchor=5,
                          o=None, lse=None, ws=None, scale=None, want_lse=True, stream=None):
    """calibatt_mixed_masked_attn_fwd: block-sparse heads over their skip lists,
    repeated heads' anchor rows over their own anchor skip list; returns (o, lse)."""
    heads, n = _bhnd(q)
    _bhnd(k, "k")
    _bhnd(v, "v")
    for t, name in ((row_ptr, "row_ptr"), (col_idx, "col_idx"), (rep_heads, "rep_heads"), (row_ptr_b, "row_ptr_b"),
                    (col_idx_b, "col_idx_b"), (work_list, "work_list")):
        _cuda_tensor(t, torch.int32, name)
    n_rep = rep_heads.numel()
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((heads, n), dtype=torch.float32, device=q.device)
    if ws is None and n_rep > 0:
        ws = torch.empty(repeat_workspace_size(n_rep, F, H, W, k_anchor), dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(HEAD_DIM) if scale is None else float(scale)
    rc = load().calibatt_mixed_masked_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), heads, F, H, W, HEAD_DIM, k_anchor, scale, _ptr(row_ptr),
        _ptr(col_idx) if col_idx.numel() else None, col_idx.numel(), _ptr(rep_heads) if n_rep else None, n_rep,
        _ptr(row_ptr_b) if row_ptr_b.numel() else None, _ptr(col_idx_b) if col_idx_b.numel() else None,
        col_idx_b.numel(), _ptr(work_list) if work_list.numel() else None, work_list.numel(), _ptr(o), _ptr(lse),
        _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream))
    _check(rc, "calibatt_mixed_masked_attn_fwd")
    return o, lse


def mixed_attn_fwd_host(q_host, k_host, v_host, o_host, F, H, W, row_ptr_host, row_ptr, col_idx, rep_heads,
                        q_dev, k_dev, v_dev, o_dev, lse_host=None, lse_dev=None, ws=None, heads_per_chunk=2,
                        k_anchor=5, scale=None, stream=None):
    """calibatt_mixed_attn_fwd from host buffers, copies overlapped with compute
    over chunks of heads; o_host (lse_host) hold the result when `stream` is done."""
    for t, name in ((q_host, "q_host"), (k_host, "k_host"), (v_host, "v_host"), (o_host, "o_host")):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host bf16 tensor")
    heads, n = _bhnd(q_dev)
    rp = np.ascontiguousarray(row_ptr_host, np.int32)
    rep = np.ascontiguousarray([int(h) for h in rep_heads], np.int32)
    lib = load()
    if ws is None:
        ws = torch.empty(lib.calibatt_mixed_host_workspace_size(heads, F, H, W, k_anchor, len(rep), heads_per_chunk),
                         dtype=torch.uint8, device=q_dev.device)
    scale = 1.0 / math.sqrt(HEAD_DIM) if scale is None else float(scale)
    rc = lib.calibatt_mixed_attn_fwd_host(q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(), o_host.data_ptr(),
                                          lse_host.data_ptr() if lse_host is not None else None, heads, F, H, W,
                                          HEAD_DIM, k_anchor, scale, _ptr(rp), _ptr(row_ptr),
                                          _ptr(col_idx) if col_idx.numel() else None, col_idx.numel(),
                                          _ptr(rep) if len(rep) else None, len(rep), int(heads_per_chunk),
                                          _ptr(q_dev), _ptr(k_dev), _ptr(v_dev), _ptr(o_dev), _ptr(lse_dev), _ptr(ws),
                                          ws.numel(), _stream(stream))
    _check(rc, "calibatt_mixed_attn_fwd_host")
    return o_host, lse_host


# ------------------------------------------------------------------ calibration

def block_energy(q, k, eps=None, energy=True, mask=None, kept=None, counts=None, lse_ws=None, scale=None,
                 stream=None, tie=None, tie_window=TIE_WINDOW):
    """Block energy of one input; with eps, fused greedy selection too
    (tie=True or a uint8 [heads][nb] tensor: tie-affected rows at tie_window).

    Returns (energy or None, mask, kept, counts) — the outputs that were
    requested; with tie, (energy, mask, kept, counts, tie).
    """
    heads, n = _bhnd(q)
    nb = (n + BLOCK - 1) // BLOCK
    dev = q.device
    if lse_ws is None:
        lse_ws = torch.empty((heads, nb * BLOCK), dtype=torch.float32, device=dev)
    e = None
    if energy is True:
        e = torch.empty((heads, nb, nb), dtype=torch.float32, device=dev)
    elif isinstance(energy, torch.Tensor):
        e = energy
    fuse = eps is not None
    if fuse and mask is None and kept is None and counts is None:
        mask = torch.empty((heads, nb, nb), dtype=torch.uint8, device=dev)
        kept = torch.empty((heads, nb), dtype=torch.int32, device=dev)
    want_tie = tie is not None and tie is not False
    tie = _tie_out(tie, (heads, nb), dev)
    scale = 1.0 / math.sqrt(HEAD_DIM) if scale is None else float(scale)
    rc = load().calibatt_block_energy(_ptr(q), _ptr(k), heads, n, HEAD_DIM, scale, _ptr(lse_ws), _ptr(e),
                                      1 if fuse else 0, float(eps) if fuse else 0.0, _ptr(mask), _ptr(kept),
                                      _ptr(counts), _ptr(tie), float(tie_window), _stream(stream))
    _check(rc, "calibatt_block_energy")
    return (e, mask, kept, counts, tie) if want_tie else (e, mask, kept, counts)


def pixel_row_energy(q, k, F, H, W, energy=False, pix=None, lse_ws=None, scale=None, stream=None):
    """Block-energy profiles of the F*H pixel rows of every head: [heads][F*H][nb]
    (and, with energy=True, the block energies [heads][nb][nb] from the same pass).

    Returns (pix, energy or None)."""
    heads, n = _bhnd(q)
    if n != F * H * W:
        raise ValueError(f"n = {n} is not F*H*W = {F * H * W}")
    nb = (n + BLOCK - 1) // BLOCK
    dev = q.device
    if lse_ws is None:
        lse_ws = torch.empty((heads, nb * BLOCK), dtype=torch.float32, device=dev)
    if pix is None:
        pix = torch.empty((heads, F * H, nb), dtype=torch.float32, device=dev)
    e = torch.empty((heads, nb, nb), dtype=torch.float32, device=dev) if energy is True else (
        energy if isinstance(energy, torch.Tensor) else None)
    scale = 1.0 / math.sqrt(HEAD_DIM) if scale is None else float(scale)
    rc = load().calibatt_pixel_row_energy(_ptr(q), _ptr(k), heads, F, H, W, HEAD_DIM, scale, _ptr(lse_ws), _ptr(e),
                                          _ptr(pix), _stream(stream))
    _check(rc, "calibatt_pixel_row_energy")
    return pix, e


def spatial_score(pix, F, H, k_anchor=5, gamma=0.87, score=None, flag=True, stream=None):
    """Spatial similarity score per head from pixel-row profiles; returns
    (score fp32 [heads], flag uint8 [heads] or None), flag = score > gamma."""
    _cuda_tensor(pix, torch.float32, "pix")
    heads, rows, nb = pix.shape
    if rows != F * H:
        raise ValueError(f"pix has {rows} rows per head, not F*H = {F * H}")
    dev = pix.device
    if score is None:
        score = torch.empty((heads,), dtype=torch.float32, device=dev)
    if flag is True:
        flag = torch.empty((heads,), dtype=torch.uint8, device=dev)
    elif flag is False:
        flag = None
    rc = load().calibatt_spatial_score(_ptr(pix), heads, F, H, nb, k_anchor, float(gamma), _ptr(score), _ptr(flag),
                                       _stream(stream))
    _check(rc, "calibatt_spatial_score")
    return score, flag


def energy_workspace_size(heads: int, n: int) -> int:
    return load().calibatt_energy_workspace_size(heads, n)


def block_energy_1pass(q, k, eps=None, energy=True, mask=None, kept=None, counts=None, pix=None, pix_W=None,
                       ws=None, scale=None, stream=None, tie=None, tie_window=TIE_WINDOW):
    """Block energy of one input in a single pass over the keys (with eps, the
    fused greedy selection too; with pix_W, pixel-row profiles of pix_W
    consecutive queries). Returns (energy or None, mask, kept, counts, pix);
    with tie (True or a uint8 [heads][nb] tensor), (energy, mask, kept,
    counts, pix, tie)."""
    heads, n = _bhnd(q)
    nb = (n + BLOCK - 1) // BLOCK
    dev = q.device
    if ws is None:
        ws = torch.empty(energy_workspace_size(heads, n), dtype=torch.uint8, device=dev)
    e = None
    if energy is True:
        e = torch.empty((heads, nb, nb), dtype=torch.float32, device=dev)
    elif isinstance(energy, torch.Tensor):
        e = energy
    fuse = eps is not None
    if fuse and mask is None and kept is None and counts is None:
        mask = torch.empty((heads, nb, nb), dtype=torch.uint8, device=dev)
        kept = torch.empty((heads, nb), dtype=torch.int32, device=dev)
    if pix_W is not None and pix is None:
        pix = torch.empty((heads, n // pix_W, nb), dtype=torch.float32, device=dev)
    want_tie = tie is not None and tie is not False
    tie = _tie_out(tie, (heads, nb), dev)
    scale = 1.0 / math.sqrt(HEAD_DIM) if scale is None else float(scale)
    rc = load().calibatt_block_energy_1pass(_ptr(q), _ptr(k), heads, n, HEAD_DIM, scale, _ptr(ws), ws.numel(),
                                            _ptr(e), 1 if fuse else 0, float(eps) if fuse else 0.0, _ptr(mask),
                                            _ptr(kept), _ptr(counts), _ptr(tie), float(tie_window), _ptr(pix),
                                            int(pix_W or 0), _stream(stream))
    _check(rc, "calibatt_block_energy_1pass")
    return (e, mask, kept, counts, pix, tie) if want_tie else (e, mask, kept, counts, pix)


def anchor_block_energy(q, k, F, H, W, rep_heads, k_anchor=5, eps=None, energy=True, mask=None, kept=None,
                        counts=None, ws=None, scale=None, stream=None, tie=None, tie_window=TIE_WINDOW):
    """Block energies of the repeated heads' anchor queries, [n_rep][nbq][nb]
    (with eps, the fused greedy selection too). Returns (energy or None, mask,
    kept, counts), plus the tie flags when tie is True or a tensor."""
    heads, n = _bhnd(q)
    if n != F * H * W:
        raise ValueError(f"n = {n} is not F*H*W = {F * H * W}")
    _cuda_tensor(rep_heads, torch.int32, "rep_heads")
    n_rep = rep_heads.numel()
    nb = (n + BLOCK - 1) // BLOCK
    nbq = anchor_blocks(F, W, k_anchor)
    dev = q.device
    lib = load()
    if ws is None:
        ws = torch.empty(lib.calibatt_anchor_energy_workspace_size(heads, n_rep, F, H, W, k_anchor),
                         dtype=torch.uint8, device=dev)
    e = torch.empty((n_rep, nbq, nb), dtype=torch.float32, device=dev) if energy is True else (
        energy if isinstance(energy, torch.Tensor) else None)
    fuse = eps is not None
    if fuse and mask is None and kept is None and counts is None:
        mask = torch.empty((n_rep, nbq, nb), dtype=torch.uint8, device=dev)
        kept = torch.empty((n_rep, nbq), dtype=torch.int32, device=dev)
    want_tie = tie is not None and tie is not False
    tie = _tie_out(tie, (n_rep, nbq), dev)
    scale = 1.0 / math.sqrt(HEAD_DIM) if scale is None else float(scale)
    rc = lib.calibatt_anchor_block_energy(_ptr(q), _ptr(k), heads, F, H, W, HEAD_DIM, k_anchor, scale,
                                          _ptr(rep_heads), n_rep, _ptr(ws), ws.numel(), _ptr(e), 1 if fuse else 0,
                                          float(eps) if fuse else 0.0, _ptr(mask), _ptr(kept), _ptr(counts),
                                          _ptr(tie), float(tie_window), _stream(stream))
    _check(rc, "calibatt_anchor_block_energy")
    return (e, mask, kept, counts, tie) if want_tie else (e, mask, kept, counts)


def aggregate_mask_rows(counts, n_inputs, rho=0.5, nnz_cap=None, ws=None, stream=None, trim=True):
    """Binarise [rows][cols] counts at rho and build their CSR skip list;
    returns (mask, row_ptr, col_idx, nnz)."""
    _cuda_tensor(counts, torch.uint16, "counts")
    cols = counts.shape[-1]
    rows = counts.numel() // cols
    dev = counts.device
    if nnz_cap is None:
        nnz_cap = rows * cols
    mask = torch.empty(counts.shape, dtype=torch.uint8, device=dev)
    row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(max(int(nnz_cap), 1), dtype=torch.int32, device=dev)
    nnz = torch.zeros(1, dtype=torch.int64, device=dev)
    lib = load()
    if ws is None:
        ws = torch.empty(lib.calibatt_aggregate_rows_workspace_size(rows), dtype=torch.uint8, device=dev)
    rc = lib.calibatt_aggregate_mask_rows(_ptr(counts), int(n_inputs), rows, cols, float(rho), _ptr(mask),
                                          _ptr(row_ptr), _ptr(col_idx), int(nnz_cap), _ptr(nnz), _ptr(ws), ws.numel(),
                                          _stream(stream))
    _check(rc, "calibatt_aggregate_mask_rows")
    if trim:
        col_idx = col_idx[:int(nnz.item())]
    return mask, row_ptr, col_idx, nnz


def select_mask(energy, eps, mask=True, kept=True, counts=None, stream=None, tie=None, tie_window=TIE_WINDOW):
    """Greedy eps selection on [heads][nb][nb] energies; returns (mask, kept,
    counts), and the tie-affected row flags when tie is True or a tensor."""
    _cuda_tensor(energy, torch.float32, "energy")
    heads, nb, _ = energy.shape
    dev = energy.device
    if mask is True:
        mask = torch.empty((heads, nb, nb), dtype=torch.uint8, device=dev)
    elif mask is False:
        mask = None
    if kept is True:
        kept = torch.empty((heads, nb), dtype=torch.int32, device=dev)
    elif kept is False:
        kept = None
    want_tie = tie is not None and tie is not False
    tie = _tie_out(tie, (heads, nb), dev)
    rc = load().calibatt_select_mask(_ptr(energy), heads, nb, float(eps), _ptr(mask), _ptr(kept), _ptr(counts),
                                     _ptr(tie), float(tie_window), _stream(stream))
    _check(rc, "calibatt_select_mask")
    return (mask, kept, counts, tie) if want_tie else (mask, kept, counts)


def accumulate_masks(mask, counts, stream=None):
    _cuda_tensor(mask, torch.uint8, "mask")
    _cuda_tensor(counts, torch.uint16, "counts")
    rc = load().calibatt_accumulate_masks(_ptr(mask), mask.numel(), _ptr(counts), _stream(stream))
    _check(rc, "calibatt_accumulate_masks")
    return counts


def aggregate_masks(counts, n_inputs, rho=0.5, nnz_cap=None, ws=None, stream=None, trim=True):
    """Binarise counts at rho and build the CSR skip list.

    Returns (mask, row_ptr, col_idx, nnz). With trim, col_idx is cut to nnz
    (one device-to-host read of the total)."""
    _cuda_tensor(counts, torch.uint16, "counts")
    heads, nb, _ = counts.shape
    dev = counts.device
    if nnz_cap is None:
        nnz_cap = heads * nb * nb
    mask = torch.empty((heads, nb, nb), dtype=torch.uint8, device=dev)
    row_ptr = torch.empty(heads * nb + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(max(int(nnz_cap), 1), dtype=torch.int32, device=dev)
    nnz = torch.zeros(1, dtype=torch.int64, device=dev)
    need = load().calibatt_aggregate_workspace_size(heads, nb)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    rc = load().calibatt_aggregate_masks(_ptr(counts), int(n_inputs), heads, nb, float(rho), _ptr(mask),
                                         _ptr(row_ptr), _ptr(col_idx), int(nnz_cap), _ptr(nnz), _ptr(ws),
                                         ws.numel(), _stream(stream))
    _check(rc, "calibatt_aggregate_masks")
    if trim:
        total = int(nnz.item())
        col_idx = col_idx[:total]
    return mask, row_ptr, col_idx, nnz


def aggregate_masks_noalloc(counts, n_inputs, rho, mask, row_ptr, col_idx, nnz, stream=None):
    """calibatt_aggregate_masks_noalloc: the caller passes every output buffer and
    the library allocates nothing (its scratch is a static device array)."""
    _cuda_tensor(counts, torch.uint16, "counts")
    heads, nb, _ = counts.shape
    rc = load().calibatt_aggregate_masks_noalloc(_ptr(counts), int(n_inputs), heads, nb, float(rho), _ptr(mask),
                                                 _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), _ptr(nnz),
                                                 _stream(stream))
    _check(rc, "calibatt_aggregate_masks_noalloc")
    return mask, row_ptr, col_idx, nnz


# ------------------------------------------------------------------ calibration bank

def keep_histogram(counts, n_inputs, stream=None):
    """Per head, the number of blocks kept by exactly c of the n_inputs inputs: int64 [heads][n_inputs + 1]."""
    _cuda_tensor(counts, torch.uint16, "counts")
    heads = counts.shape[0]
    cells = counts.numel() // heads
    hist = torch.empty((heads, n_inputs + 1), dtype=torch.int64, device=counts.device)
    rc = load().calibatt_keep_histogram(_ptr(counts), heads, cells, int(n_inputs), _ptr(hist), _stream(stream))
    _check(rc, "calibatt_keep_histogram")
    return hist


class BankEntry(ctypes.Structure):
    _fields_ = [("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p), ("nnz", ctypes.c_int64),
                ("work_list", ctypes.c_void_p), ("n_work", ctypes.c_int32), ("rep_heads", ctypes.c_void_p),
                ("n_rep", ctypes.c_int32), ("eps", ctypes.c_double)]


class MaskBank:
    """The (t, l) mask bank (calibatt_bank_*): entry buffers are torch device
    tensors this object keeps alive; lookups return views of them."""

    def __init__(self, timesteps, layers, heads, F, H, W, k_anchor=5):
        self._lib = load()
        self._h = self._lib.calibatt_bank_create(timesteps, layers, heads, F, H, W, k_anchor)
        if not self._h:
            raise CalibattError(-1, "calibatt_bank_create: bad sizes")
        self.shape = (timesteps, layers, heads, F, H, W, k_anchor)
        self._buffers = {}

    def close(self):
        if self._h:
            self._lib.calibatt_bank_destroy(self._h)
            self._h = None
        self._buffers.clear()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def put(self, t, l, eps, row_ptr, col_idx, rep_heads=(), stream=None):
        """Store entry (t, l): row_ptr (device or host int32), col_idx (device int32), rep_heads (ints)."""
        _cuda_tensor(col_idx, torch.int32, "col_idx")
        rp = np.ascontiguousarray(row_ptr.cpu().numpy() if isinstance(row_ptr, torch.Tensor) else row_ptr, np.int32)
        rep = np.ascontiguousarray([int(h) for h in rep_heads], np.int32)
        nnz = col_idx.numel()
        need = self._lib.calibatt_bank_entry_bytes(self._h, nnz, len(rep))
        if need == 0:
            raise CalibattError(-1, "calibatt_bank_entry_bytes")
        buf = torch.empty(need + 256, dtype=torch.uint8, device=col_idx.device)
        off = (-buf.data_ptr()) % 256
        rc = self._lib.calibatt_bank_put(self._h, t, l, float(eps), _ptr(rp), _ptr(col_idx) if nnz else None, nnz,
                                         _ptr(rep) if len(rep) else None, len(rep), buf.data_ptr() + off, need,
                                         _stream(stream))
        _check(rc, "calibatt_bank_put")
        self._buffers[(t, l)] = (buf, off)

    def get(self, t, l):
        """Entry (t, l) as tensors viewing its buffer: dict of row_ptr, col_idx,
        work_list, rep_heads (device int32) and eps."""
        e = BankEntry()
        _check(self._lib.calibatt_bank_get(self._h, t, l, ctypes.byref(e)), "calibatt_bank_get")
        buf, _ = self._buffers[(t, l)]
        base = buf.data_ptr()

        def view(ptr, count):
            if count == 0:
                return torch.empty(0, dtype=torch.int32, device=buf.device)
            start = ptr - base
            return buf[start:start + 4 * count].view(torch.int32)

        _, _, heads, F, H, W, _ = self.shape
        nb = -(-F * H * W // BLOCK)
        return {"row_ptr": view(e.row_ptr, heads * nb + 1), "col_idx": view(e.col_idx, e.nnz),
                "work_list": view(e.work_list, e.n_work), "rep_heads": view(e.rep_heads, e.n_rep), "eps": e.eps}

    def attention(self, q, k, v, t, l, o=None, lse=None, stream=None):
        """Online inference for step t, layer l: one mixed launch over the entry's lists."""
        _, _, _, F, H, W, k_anchor = self.shape
        e = self.get(t, l)
        return mixed_attn_fwd(q, k, v, F, H, W, e["row_ptr"], e["col_idx"], e["rep_heads"], e["work_list"],
                              k_anchor=k_anchor, o=o, lse=lse, stream=stream)
