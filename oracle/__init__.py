"""fp64 CPU oracle for block-causal attention (ctypes wrapper over oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, ``__graft_entry__.smoke()`` and
bench.py's CPU-baseline / reference legs, never by the product path.  It shares
no code with the CUDA library; it takes plain arrays (slice list, video geometry,
head counts) so that it does not depend on the product package either.

Every function recomputes its result from the definitions in oracle.c, in double
precision, from the bf16 input values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so beside it (plain gcc, OpenMP, -O2, no
    target-specific flags so the library runs on any x86-64 host)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.orc_mask_row.argtypes = [_i64p, _int, _i64, _i64, _u8p]
        L.orc_mask_col.argtypes = [_i64p, _int, _i64, _i64, _u8p]
        L.orc_mask_dense.argtypes = [_i64p, _int, _i64, _i64, _u8p]
        L.orc_positions.argtypes = [_i32p, _int, _i32p]
        L.orc_prologue.argtypes = [_f64p, _i64, _int, _int, _i32p, _vp, _f64p, ctypes.c_double, _f64p]
        L.orc_prologue_bwd.argtypes = [_f64p, _i64, _int, _int, _i32p, _vp, _f64p, ctypes.c_double,
                                       _f64p, _f64p]
        L.orc_prologue_param_grads.argtypes = [_f64p, _i64, _int, _int, _i32p, _vp, _f64p, ctypes.c_double,
                                               _f64p, _f64p, _f64p]
        L.orc_fwd_rows.argtypes = [_f64p, _i64p, _i64, _f64p, _f64p, _i64, _i64p, _int, _int, _int,
                                   _int, _f64p, _f64p]
        L.orc_bwd_rows.argtypes = [_f64p, _i64p, _i64, _f64p, _f64p, _i64, _f64p, _i64p, _int, _int,
                                   _int, _int, _f64p, _f64p, _f64p]
        L.orc_bwd_keys.argtypes = [_f64p, _f64p, _f64p, _f64p, _i64, _f64p, _f64p, _i64, _i64p, _i64,
                                   _int, _int, _i64p, _int, _int, _int, _int, _f64p, _f64p]
        L.orc_bwd_dense.argtypes = [_f64p, _f64p, _f64p, _f64p, _i64, _i64, _i64p, _int, _int, _int,
                                    _int, _f64p, _f64p, _f64p, _f64p, _f64p]
        for f in ("orc_mask_row", "orc_mask_col", "orc_mask_dense", "orc_positions", "orc_prologue",
                  "orc_prologue_bwd", "orc_prologue_param_grads", "orc_fwd_rows", "orc_bwd_rows", "orc_bwd_keys", "orc_bwd_dense"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def _f64(x) -> np.ndarray:
    """bf16/float torch tensor or array -> contiguous float64 numpy (exact for bf16)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _slices(sl) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(sl, dtype=np.int64).reshape(-1, 5))


# ---------------------------------------------------------------------------
# mask
# ---------------------------------------------------------------------------

def mask_dense(slices, nq: int, nk: int) -> np.ndarray:
    sl = _slices(slices)
    out = np.zeros((nq, nk), dtype=np.uint8)
    lib().orc_mask_dense(sl, len(sl), nq, nk, out)
    return out.astype(bool)


def mask_row(slices, nk: int, i: int) -> np.ndarray:
    sl = _slices(slices)
    out = np.zeros(nk, dtype=np.uint8)
    lib().orc_mask_row(sl, len(sl), nk, i, out)
    return out.astype(bool)


def mask_col(slices, nq: int, j: int) -> np.ndarray:
    sl = _slices(slices)
    out = np.zeros(nq, dtype=np.uint8)
    lib().orc_mask_col(sl, len(sl), nq, j, out)
    return out.astype(bool)


# ---------------------------------------------------------------------------
# prologue
# ---------------------------------------------------------------------------

def positions(videos) -> np.ndarray:
    vid = np.ascontiguousarray(np.asarray(videos, dtype=np.int32).reshape(-1, 5))
    n = int(sum(int(v[0]) * int(v[1]) * int(v[2]) * int(v[3]) for v in vid))
    out = np.zeros((n, 3), dtype=np.int32)
    lib().orc_positions(vid, len(vid), out)
    return out


def prologue(x, pos, base=(1e4, 1e4, 1e4), eps=1e-6, gain=None) -> np.ndarray:
    """QK-Norm (RMS over D) then 3D RoPE; x: [n, H, D]; pos: [n, 3] int32."""
    x = _f64(x)
    n, H, D = x.shape
    out = np.empty_like(x)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int32).reshape(n, 3))
    g = None if gain is None else _f64(gain)
    lib().orc_prologue(x, n, H, D, pos, None if g is None else g.ctypes.data,
                       np.asarray(base, np.float64), float(eps), out)
    return out


def prologue_bwd(x, pos, dy, base=(1e4, 1e4, 1e4), eps=1e-6, gain=None) -> np.ndarray:
    x = _f64(x)
    dy = _f64(dy)
    n, H, D = x.shape
    out = np.empty_like(x)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int32).reshape(n, 3))
    g = None if gain is None else _f64(gain)
    lib().orc_prologue_bwd(x, n, H, D, pos, None if g is None else g.ctypes.data,
                           np.asarray(base, np.float64), float(eps), dy, out)
    return out


def prologue_param_grads(x, pos, dy, base=(1e4, 1e4, 1e4), eps=1e-6, gain=None):
    """(dL/dgain [D], dL/dbase [3]) of the prologue, summed over all rows of x [n, H, D]
    for the upstream gradient dy = dL/d(prologue output)."""
    x = _f64(x)
    dy = _f64(dy)
    n, H, D = x.shape
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int32).reshape(n, 3))
    g = None if gain is None else _f64(gain)
    dg = np.zeros(D)
    db = np.zeros(3)
    lib().orc_prologue_param_grads(x, n, H, D, pos, None if g is None else g.ctypes.data,
                                   np.asarray(base, np.float64), float(eps), dy, dg, db)
    return dg, db


# ---------------------------------------------------------------------------
# attention on post-prologue operands
# ---------------------------------------------------------------------------

def attn_fwd_rows(qh_rows, rows, kh, v, slices, hq: int, hkv: int):
    """O [nr, Hq, D] and LSE [nr, Hq] for the listed query rows; qh_rows holds the
    post-prologue queries of exactly those rows, in the same order."""
    qh = _f64(qh_rows)
    kh = _f64(kh)
    v = _f64(v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    nr, _, D = qh.shape
    nk = kh.shape[0]
    sl = _slices(slices)
    O = np.zeros((nr, hq, D))
    lse = np.zeros((nr, hq))
    lib().orc_fwd_rows(qh, rows, nr, kh, v, nk, sl, len(sl), hq, hkv, D, O, lse)
    return O, lse


def attn_bwd_rows(qh_rows, rows, kh, v, do_rows, slices, hq: int, hkv: int):
    """dq-hat [nr, Hq, D] (plus O and LSE) for the listed rows."""
    qh = _f64(qh_rows)
    kh = _f64(kh)
    v = _f64(v)
    do = _f64(do_rows)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    nr, _, D = qh.shape
    nk = kh.shape[0]
    sl = _slices(slices)
    dq = np.zeros((nr, hq, D))
    O = np.zeros((nr, hq, D))
    lse = np.zeros((nr, hq))
    lib().orc_bwd_rows(qh, rows, nr, kh, v, nk, do, sl, len(sl), hq, hkv, D, dq, O, lse)
    return dq, O, lse


def attn_bwd_keys(qh, do, lse, dsum, kh, v, keys, slices, hq: int, hkv: int,
                  h_begin: int = 0, h_end: Optional[int] = None):
    """dk-hat and dv [nkeys, Hkv, D] for the listed keys, from ALL query rows; only the
    KV groups of heads [h_begin, h_end) are filled."""
    qh = _f64(qh)
    do = _f64(do)
    lse = _f64(lse)
    dsum = _f64(dsum)
    kh = _f64(kh)
    v = _f64(v)
    keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int64))
    nq, _, D = qh.shape
    nk = kh.shape[0]
    sl = _slices(slices)
    h_end = hq if h_end is None else h_end
    dk = np.zeros((len(keys), hkv, D))
    dv = np.zeros((len(keys), hkv, D))
    lib().orc_bwd_keys(qh, do, lse, dsum, nq, kh, v, nk, keys, len(keys), h_begin, h_end, sl,
                       len(sl), hq, hkv, D, dk, dv)
    return dk, dv


def attn_bwd_dense(qh, kh, v, do, slices, hq: int, hkv: int):
    """Full backward on post-prologue operands: (dqh, dkh, dv, O, LSE)."""
    qh = _f64(qh)
    kh = _f64(kh)
    v = _f64(v)
    do = _f64(do)
    nq, _, D = qh.shape
    nk = kh.shape[0]
    sl = _slices(slices)
    dq = np.zeros_like(qh)
    dk = np.zeros_like(kh)
    dv = np.zeros_like(v)
    O = np.zeros_like(qh)
    lse = np.zeros((nq, hq))
    lib().orc_bwd_dense(qh, kh, v, do, nq, nk, sl, len(sl), hq, hkv, D, dq, dk, dv, O, lse)
    return dq, dk, dv, O, lse


# ---------------------------------------------------------------------------
# end to end on raw inputs (prologue on Q and new K; the cache is post-prologue)
# ---------------------------------------------------------------------------

def full_keys(k_new_hat, k_cache):
    """Key index space = [cache | new]."""
    if k_cache is None:
        return _f64(k_new_hat)
    return np.concatenate([_f64(k_cache), _f64(k_new_hat)], axis=0)


def forward(q, k, v, k_cache, v_cache, videos, slices, hq, hkv,
            base=(1e4, 1e4, 1e4), eps=1e-6, q_gain=None, k_gain=None, rows=None,
            q_rows=None):
    """O, LSE for query rows ``rows`` (default: all).  q may be the full Q (then rows
    are selected from it) or, with ``q_rows``, just those rows' raw values."""
    pos = positions(videos)
    kh = full_keys(prologue(k, pos, base, eps, k_gain), k_cache)
    vv = full_keys(v, v_cache)
    if rows is None:
        rows = np.arange(pos.shape[0], dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    qr = _f64(q_rows) if q_rows is not None else _f64(q)[rows]
    qh = prologue(qr, pos[rows], base, eps, q_gain)
    return attn_fwd_rows(qh, rows, kh, vv, slices, hq, hkv)


def backward(q, k, v, k_cache, v_cache, do, videos, slices, hq, hkv,
             base=(1e4, 1e4, 1e4), eps=1e-6, q_gain=None, k_gain=None, param_grads=False):
    """Full backward w.r.t. the raw inputs: (dq, dk, dv, dk_cache, dv_cache, O, LSE), and
    with param_grads=True also (dq_gain [D], dk_gain [D], dbase [3]) appended: the
    gradients of the two QK-Norm gains and of the RoPE bases (shared by Q and K)."""
    pos = positions(videos)
    nc = 0 if k_cache is None else int(k_cache.shape[0])
    kh = full_keys(prologue(k, pos, base, eps, k_gain), k_cache)
    vv = full_keys(v, v_cache)
    qh = prologue(q, pos, base, eps, q_gain)
    dqh, dkh, dvv, O, lse = attn_bwd_dense(qh, kh, vv, do, slices, hq, hkv)
    dq = prologue_bwd(q, pos, dqh, base, eps, q_gain)
    dk = prologue_bwd(k, pos, dkh[nc:], base, eps, k_gain)
    out = (dq, dk, dvv[nc:], (dkh[:nc] if nc else None), (dvv[:nc] if nc else None), O, lse)
    if not param_grads:
        return out
    dgq, dbq = prologue_param_grads(q, pos, dqh, base, eps, q_gain)
    dgk, dbk = prologue_param_grads(k, pos, dkh[nc:], base, eps, k_gain)
    return out + (dgq, dgk, dbq + dbk)


def backward_rows(q_rows, rows, k, v, k_cache, v_cache, do_rows, videos, slices, hq, hkv,
                  base=(1e4, 1e4, 1e4), eps=1e-6, q_gain=None, k_gain=None):
    """dq (w.r.t. the raw queries, through the prologue) for the listed query rows only;
    q_rows / do_rows hold those rows' raw queries and upstream gradients."""
    pos = positions(videos)
    rows = np.asarray(rows, dtype=np.int64)
    kh = full_keys(prologue(k, pos, base, eps, k_gain), k_cache)
    vv = full_keys(v, v_cache)
    qr = _f64(q_rows)
    qh = prologue(qr, pos[rows], base, eps, q_gain)
    dqh, O, lse = attn_bwd_rows(qh, rows, kh, vv, do_rows, slices, hq, hkv)
    return prologue_bwd(qr, pos[rows], dqh, base, eps, q_gain)
