"""CalibAtt oracle: plain fp64 CPU statement of the hot path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product library
(``calibrated_block_sparse_b200``) never imports it, and this package imports
nothing from the product.

The arithmetic lives in ``oracle.c`` (plain C, fp64, no SIMD intrinsics, no
BLAS); this module compiles it with gcc on first use and wraps each function
with numpy marshalling. Every function cites the passage of the method it
follows: "Accelerating Text-to-Video Generation with Calibrated Sparse
Attention" as explained on the zhichai.net CalibAtt page, section 三 (method)
and section 六 (spatial repetition).

Parity pins: every function here is pinned by ``tests/test_oracle_*.py``
against invariants, closed forms and brute force (no function is unpinned).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
             "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
            lib.oracle_masked_attention.argtypes = [P, P, P, i32, i64, i32, i32, f64, P, P, i64, P, P, i32]
            lib.oracle_masked_attention.restype = None
            lib.oracle_repeat_attention.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f64, P, i64, P, P, i32]
            lib.oracle_repeat_attention.restype = ctypes.c_int
            lib.oracle_anchor_rows.argtypes = [i32, i32, P]
            lib.oracle_anchor_rows.restype = None
            lib.oracle_nearest_anchor.argtypes = [i32, i32, P, P]
            lib.oracle_nearest_anchor.restype = None
            lib.oracle_block_energy.argtypes = [P, P, i32, i64, i32, i32, f64, P, i64, P, P, i32]
            lib.oracle_block_energy.restype = None
            lib.oracle_select.argtypes = [P, i64, i32, f64, P, P, P, P, P, P]
            lib.oracle_select.restype = None
            lib.oracle_aggregate.argtypes = [P, i32, i64, f64, P, P]
            lib.oracle_aggregate.restype = None
            lib.oracle_binarize_counts.argtypes = [P, i32, i64, f64, P]
            lib.oracle_binarize_counts.restype = None
            lib.oracle_mask_to_csr.argtypes = [P, i32, i64, P, P]
            lib.oracle_mask_to_csr.restype = i64
            lib.oracle_mask_rows_to_csr.argtypes = [P, i64, i64, P, P]
            lib.oracle_mask_rows_to_csr.restype = i64
            lib.oracle_eps_schedule.argtypes = [f64, f64, f64, f64, f64]
            lib.oracle_eps_schedule.restype = f64
            lib.oracle_pixel_row_energy.argtypes = [P, P, i32, i32, i32, i32, i32, i32, f64, P, i64, P, i32]
            lib.oracle_pixel_row_energy.restype = None
            lib.oracle_spatial_score.argtypes = [P, i32, i32, i64, i32]
            lib.oracle_spatial_score.restype = f64
            lib.oracle_anchor_block_energy.argtypes = [P, P, i32, i32, i32, i32, i32, i32, i32, f64, P, i64, P, i32]
            lib.oracle_anchor_block_energy.restype = ctypes.c_int
            lib.oracle_repeat_attention_masked.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, f64, P, P,
                                                           i64, P, P, i32]
            lib.oracle_repeat_attention_masked.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _bf16_bits(x) -> np.ndarray:
    """Accept a uint16 array of bf16 bit patterns (or a torch bf16 tensor)."""
    if hasattr(x, "view") and str(getattr(x, "dtype", "")) == "torch.bfloat16":
        import torch  # local: torch is only used to reinterpret the bits
        x = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "bf16 inputs are passed as uint16 bit patterns"
    return x


def _threads(threads):
    return int(threads) if threads else (os.cpu_count() or 1)


def masked_attention(q, k, v, mask, B=128, scale=None, rows=None, threads=None):
    """Attention restricted to the kept B x B key blocks of ``mask`` [h][nb][nb].

    q, k, v: bf16 bits [h][n][d]. ``rows``: optional int64 array of h*n+i to
    evaluate (sampled parity); default all. Returns (O fp64 [rows][d] or
    [h][n][d], LSE fp64). Explainer §三 (online inference, skip list).
    """
    q, k, v = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    h, n, d = q.shape
    nb = (n + B - 1) // B
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    assert mask.shape == (h, nb, nb)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    if rows is None:
        o = np.empty((h, n, d), np.float64)
        lse = np.empty((h, n), np.float64)
        nr = h * n
        rp = None
    else:
        rp = np.ascontiguousarray(rows, dtype=np.int64)
        nr = rp.size
        o = np.empty((nr, d), np.float64)
        lse = np.empty((nr,), np.float64)
    _load().oracle_masked_attention(_ptr(q), _ptr(k), _ptr(v), h, n, d, B, scale, _ptr(mask),
                                    _ptr(rp), nr, _ptr(o), _ptr(lse), _threads(threads))
    return o, lse


def anchor_rows(H, k_anchor):
    """Centres of k equal bands of the H rows of a frame (explainer §三/§六)."""
    a = np.empty(k_anchor, np.int32)
    _load().oracle_anchor_rows(H, k_anchor, _ptr(a))
    return a


def nearest_anchor(H, k_anchor):
    """owner[r] = index j of the anchor row nearest to row r (ties -> lower j)."""
    a = anchor_rows(H, k_anchor)
    owner = np.empty(H, np.int32)
    _load().oracle_nearest_anchor(H, k_anchor, _ptr(a), _ptr(owner))
    return owner


def repeat_attention(q, k, v, F, H, W, k_anchor=5, scale=None, rows=None, threads=None):
    """Spatially repeated head: every row copies its nearest anchor row's dense
    attention output (same frame, same column). Explainer §三 and §六."""
    q, k, v = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    h, n, d = q.shape
    assert n == F * H * W
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    if rows is None:
        o = np.empty((h, n, d), np.float64)
        lse = np.empty((h, n), np.float64)
        nr, rp = h * n, None
    else:
        rp = np.ascontiguousarray(rows, dtype=np.int64)
        nr = rp.size
        o = np.empty((nr, d), np.float64)
        lse = np.empty((nr,), np.float64)
    rc = _load().oracle_repeat_attention(_ptr(q), _ptr(k), _ptr(v), h, F, H, W, d, k_anchor, scale,
                                         _ptr(rp), nr, _ptr(o), _ptr(lse), _threads(threads))
    if rc != 0:
        raise ValueError("k_anchor must be in [1, H]")
    return o, lse


def block_energy(q, k, B=128, scale=None, blockrows=None, threads=None, want_lse=False):
    """E[r,c] = (1/|I_r|) sum_{i in I_r, j in J_c} softmax(scale QK^T)_ij (explainer §三 step 2).

    ``blockrows``: optional int64 array of h*nb+r; default all (returns [h][nb][nb]).
    With want_lse, also the per-row LSE ([..][B], unused tail rows left NaN).
    """
    q, k = _bf16_bits(q), _bf16_bits(k)
    h, n, d = q.shape
    nb = (n + B - 1) // B
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    if blockrows is None:
        br, nbr = None, h * nb
    else:
        br = np.ascontiguousarray(blockrows, dtype=np.int64)
        nbr = br.size
    E = np.empty((nbr, nb), np.float64)
    lse = np.full((nbr, B), np.nan) if want_lse else None
    _load().oracle_block_energy(_ptr(q), _ptr(k), h, n, d, B, scale, _ptr(br), nbr, _ptr(E), _ptr(lse),
                                _threads(threads))
    if blockrows is None:
        E = E.reshape(h, nb, nb)
        if lse is not None:
            lse = lse.reshape(h, nb, B)
    return (E, lse) if want_lse else E


def select(E, eps, with_cut=False):
    """Greedy eps selection per block-row (explainer §三 step 3).

    E: [..., nb] energies (fp64). Returns mask uint8 of E's shape and kept counts;
    with_cut also returns (cum_before, cum_at, e_last, e_next) per row.
    """
    E = np.ascontiguousarray(E, dtype=np.float64)
    shape = E.shape
    nb = shape[-1]
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    mask = np.empty(shape, np.uint8)
    kept = np.empty(rows, np.int32)
    cut = [np.empty(rows, np.float64) for _ in range(4)]
    _load().oracle_select(_ptr(E), rows, nb, float(eps), _ptr(mask), _ptr(kept), *[_ptr(c) for c in cut])
    kept = kept.reshape(shape[:-1])
    if with_cut:
        return mask, kept, tuple(c.reshape(shape[:-1]) for c in cut)
    return mask, kept


def aggregate(masks, rho=0.5):
    """Mbar = mean over inputs of the masks, kept where Mbar >= rho (explainer §三).

    masks: [n_inputs, ...] uint8. Returns (mask uint8, counts int32)."""
    masks = np.ascontiguousarray(masks, dtype=np.uint8)
    n_in = masks.shape[0]
    cells = int(np.prod(masks.shape[1:]))
    out = np.empty(masks.shape[1:], np.uint8)
    counts = np.empty(masks.shape[1:], np.int32)
    _load().oracle_aggregate(_ptr(masks), n_in, cells, float(rho), _ptr(out), _ptr(counts))
    return out, counts


def binarize_counts(counts, n_inputs, rho=0.5):
    """Keep where counts / n_inputs >= rho (the same rule from integer counts)."""
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    out = np.empty(counts.shape, np.uint8)
    _load().oracle_binarize_counts(_ptr(counts), int(n_inputs), counts.size, float(rho), _ptr(out))
    return out


def mask_to_csr(mask):
    """Skip list: per (head, block-row) the kept key blocks, ascending, as CSR."""
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    h, nb, nb2 = mask.shape
    assert nb == nb2
    row_ptr = np.empty(h * nb + 1, np.int32)
    col_idx = np.empty(int(mask.sum()), np.int32)
    nnz = _load().oracle_mask_to_csr(_ptr(mask), h, nb, _ptr(row_ptr), _ptr(col_idx))
    assert nnz == col_idx.size
    return row_ptr, col_idx


def mask_rows_to_csr(mask):
    """Skip list of the rows of a mask [..., cols] (any number of rows): per
    row the kept columns, ascending, as CSR with global offsets."""
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    cols = mask.shape[-1]
    rows = mask.size // cols
    row_ptr = np.empty(rows + 1, np.int32)
    col_idx = np.empty(int(mask.sum()), np.int32)
    nnz = _load().oracle_mask_rows_to_csr(_ptr(mask), rows, cols, _ptr(row_ptr), _ptr(col_idx))
    assert nnz == col_idx.size
    return row_ptr, col_idx


def eps_schedule(A, C, k, t, T):
    """eps(t) = A + (C - A) exp(-k t / T) (explainer §三)."""
    return _load().oracle_eps_schedule(float(A), float(C), float(k), float(t), float(T))


def pixel_row_energy(q, k, F, H, W, B=128, scale=None, prows=None, threads=None):
    """Block-energy profile of every pixel row R = (f, r) of a frame:
    Epx[R][c] = (1/W) sum over the W queries of R and the keys of block c of
    softmax(scale QK^T) (the block energy of explainer §三 step 2, taken over
    pixel rows instead of query blocks; §二 observation 4).

    ``prows``: optional int64 array of h*F*H + R; default all (returns [h][F*H][nb])."""
    q, k = _bf16_bits(q), _bf16_bits(k)
    h, n, d = q.shape
    assert n == F * H * W
    nb = (n + B - 1) // B
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    if prows is None:
        pr, npr = None, h * F * H
    else:
        pr = np.ascontiguousarray(prows, dtype=np.int64)
        npr = pr.size
    E = np.empty((npr, nb), np.float64)
    _load().oracle_pixel_row_energy(_ptr(q), _ptr(k), h, F, H, W, d, B, scale, _ptr(pr), npr, _ptr(E),
                                    _threads(threads))
    return E.reshape(h, F * H, nb) if prows is None else E


def spatial_score(Epx, F, H, k_anchor=5):
    """s of one head: mean over frames and non-anchor rows of the cosine
    similarity between a pixel row's profile and its nearest anchor row's
    (explainer §三, the spatial similarity score; the pages give no formula)."""
    E = np.ascontiguousarray(Epx, dtype=np.float64)
    assert E.ndim == 2 and E.shape[0] == F * H
    if not 1 <= k_anchor <= H:
        raise ValueError("k_anchor must be in [1, H]")
    return _load().oracle_spatial_score(_ptr(E), F, H, E.shape[1], k_anchor)


def repeat_flag(s, gamma=0.87):
    """A head is spatially repeated when its score exceeds gamma (explainer §三)."""
    return bool(s > gamma)


def keep_histogram(counts, n_inputs):
    """Keep-rate histogram of calibrated blocks (explainer §二 observation 3:
    over the calibration inputs a block is almost always kept or almost always
    skipped, so the histogram of count / n is bimodal): for each head, the
    number of blocks kept by exactly c of the n inputs, c = 0..n.

    counts: [heads, ...] integer mask counts over n_inputs inputs.
    Returns int64 [heads][n_inputs + 1]."""
    c = np.asarray(counts).reshape(np.asarray(counts).shape[0], -1).astype(np.int64)
    if c.size and (c.min() < 0 or c.max() > n_inputs):
        raise ValueError("a count lies outside [0, n_inputs]")
    return np.stack([np.bincount(row, minlength=n_inputs + 1) for row in c]).astype(np.int64)


def anchor_blocks(F, H, W, k_anchor, B=128):
    """Number of blocks of B packed anchor queries of one repeated head."""
    return (F * k_anchor * W + B - 1) // B


def anchor_block_energy(q, k, F, H, W, k_anchor=5, B=128, scale=None, blockrows=None, threads=None):
    """Block energy of the anchor queries of a repeated head (explainer §三:
    calibration per (t, l, h); the same energy as block_energy, over the
    head's anchor queries taken in the order frame, anchor, column and grouped
    into blocks of B). Returns [h][nbq][nb] (or [len(blockrows)][nb] for
    blockrows h*nbq + r)."""
    q, k = _bf16_bits(q), _bf16_bits(k)
    h, n, d = q.shape
    assert n == F * H * W
    nb = (n + B - 1) // B
    nbq = anchor_blocks(F, H, W, k_anchor, B)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    if blockrows is None:
        br, nbr = None, h * nbq
    else:
        br = np.ascontiguousarray(blockrows, dtype=np.int64)
        nbr = br.size
    E = np.empty((nbr, nb), np.float64)
    rc = _load().oracle_anchor_block_energy(_ptr(q), _ptr(k), h, F, H, W, d, B, k_anchor, scale, _ptr(br), nbr,
                                            _ptr(E), _threads(threads))
    if rc != 0:
        raise ValueError("k_anchor must be in [1, H]")
    return E.reshape(h, nbq, nb) if blockrows is None else E


def repeat_attention_masked(q, k, v, F, H, W, mask_b, k_anchor=5, B=128, scale=None, rows=None, threads=None):
    """Repeated head whose anchor queries attend only to the key blocks their
    anchor block's mask keeps (mask_b [h][nbq][nb]); every row copies its
    nearest anchor row's output (explainer §三 and §六)."""
    q, k, v = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    h, n, d = q.shape
    assert n == F * H * W
    nb = (n + B - 1) // B
    nbq = anchor_blocks(F, H, W, k_anchor, B)
    mask_b = np.ascontiguousarray(mask_b, dtype=np.uint8)
    assert mask_b.shape == (h, nbq, nb)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    if rows is None:
        o = np.empty((h, n, d), np.float64)
        lse = np.empty((h, n), np.float64)
        nr, rp = h * n, None
    else:
        rp = np.ascontiguousarray(rows, dtype=np.int64)
        nr = rp.size
        o = np.empty((nr, d), np.float64)
        lse = np.empty((nr,), np.float64)
    rc = _load().oracle_repeat_attention_masked(_ptr(q), _ptr(k), _ptr(v), h, F, H, W, d, B, k_anchor, scale,
                                                _ptr(mask_b), _ptr(rp), nr, _ptr(o), _ptr(lse), _threads(threads))
    if rc != 0:
        raise ValueError("k_anchor must be in [1, H]")
    return o, lse
