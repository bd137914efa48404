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


def attn_fwd_rows_blas(qh_rows, rows, kh, v, slices, hq: int, hkv: int, batch: int = 16,
                       workers: Optional[int] = None):
    """The same O [nr, Hq, D] and LSE [nr, Hq] as ``attn_fwd_rows``, with the scores
    s_ij = qh_i . kh_j / sqrt(D) and the sum over j of exp(s_ij - LSE_i) v_j taken as fp64
    matrix products (numpy / BLAS) over batches of ``batch`` query rows, for full-size
    workloads where the per-pair C loops take hours.

    Each row is the plain definition: its mask row comes from the C rasteriser
    (``orc_mask_row``, the union of the slices), masked scores are dropped, LSE_i = m_i +
    log sum_j exp(s_ij - m_i) with m_i the row maximum, and a row that sees no key gets
    O = 0, LSE = -inf.  Batches only group independent rows; every row is complete in
    one batch.  ``workers`` threads run batches concurrently (numpy releases the GIL)."""
    import concurrent.futures as cf
    qh = _f64(qh_rows)
    kh = _f64(kh)
    v = _f64(v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    nr, _, D = qh.shape
    nk = kh.shape[0]
    G = hq // hkv
    scale = 1.0 / np.sqrt(float(D))
    sl = _slices(slices)
    O = np.zeros((nr, hq, D))
    lse = np.full((nr, hq), -np.inf)
    L = lib()

    def run(b0):
        b1 = min(nr, b0 + batch)
        nb = b1 - b0
        m = np.zeros((nb, nk), dtype=np.uint8)
        for r in range(nb):
            L.orc_mask_row(sl, len(sl), nk, int(rows[b0 + r]), m[r])
        cols = np.flatnonzero(m.any(0))
        if len(cols) == 0:
            return
        k0, k1 = int(cols[0]), int(cols[-1]) + 1
        vis = m[:, k0:k1].astype(bool)[:, None, :]                     # [nb, 1, span]
        seen = vis.any(-1)                                              # [nb, 1]
        for g in range(hkv):
            q = qh[b0:b1, g * G:(g + 1) * G, :].reshape(nb * G, D)
            s = (q @ kh[k0:k1, g, :].T).reshape(nb, G, k1 - k0) * scale
            s = np.where(vis, s, -np.inf)
            mx = np.where(seen, s.max(-1), 0.0)                          # [nb, G]
            p = np.exp(s - mx[..., None])
            ell = p.sum(-1)
            o = (p.reshape(nb * G, k1 - k0) @ v[k0:k1, g, :]).reshape(nb, G, D)
            with np.errstate(divide="ignore", invalid="ignore"):
                O[b0:b1, g * G:(g + 1) * G] = np.where(seen[..., None], o / ell[..., None], 0.0)
                lse[b0:b1, g * G:(g + 1) * G] = np.where(seen, mx + np.log(ell), -np.inf)

    workers = workers or (os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        list(ex.map(run, range(0, nr, batch)))
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


# ---------------------------------------------------------------------------
# e4m3 operands (the FP8 forward variant)
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0          # largest finite e4m3 value: 1.75 * 2^8
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_SUBNORMAL_STEP = 2.0 ** -9


def round_e4m3(x) -> np.ndarray:
    """Round to the nearest e4m3 value (ties to an even significand), saturating at
    +-448.  The format (OCP 8-bit floating point, E4M3): 1 sign bit, 4 exponent bits
    with bias 7, 3 significand bits, no infinities; normal values (1 + m/8) * 2^e for
    e in [-6, 8] (the top code of e = 8 is NaN, so the largest is 1.75 * 2^8), and
    subnormals m/8 * 2^-6.  In a binade [2^e, 2^(e+1)) the spacing is 2^(e-3); below
    2^-6 it is 2^-9."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    e = np.floor(np.log2(np.maximum(a, E4M3_MIN_NORMAL)))
    step = np.where(a < E4M3_MIN_NORMAL, E4M3_SUBNORMAL_STEP, 2.0 ** (e - 3))
    r = np.rint(a / step) * step                      # rint: halves go to the even multiple
    r = np.minimum(r, E4M3_MAX)
    return np.where(np.isnan(x), np.nan, np.copysign(r, x))


def e4m3_scale_exponent(amax: float) -> int:
    """Exponent e of the power-of-two scale that brings V into e4m3's range: the e with
    amax / 448 in [2^(e-1), 2^e), so V / 2^e < 448 (0 when amax is 0).  Taken from the
    exact binary exponent of amax: amax = m * 2^f with m in [0.5, 1) and 448 = 0.875 * 2^9,
    so e = f - 8 when m >= 0.875, else f - 9."""
    if not amax > 0:
        return 0
    m, f = np.frexp(float(amax))
    return int(f - 8 if m >= 0.875 else f - 9)


def _e4m3_step(a):
    """Spacing of e4m3 values around |x| = a (2^(e-3) in the binade [2^e, 2^(e+1)))."""
    e = np.floor(np.log2(np.maximum(a, E4M3_MIN_NORMAL)))
    return np.where(a < E4M3_MIN_NORMAL, E4M3_SUBNORMAL_STEP, 2.0 ** (e - 3))


def _e4m3_undecided(x, window=2e-6):
    """Step of the elements whose e4m3 rounding a computation carrying an error of
    window * max(|x|, 1) could take either way (within that distance of a rounding
    midpoint), else 0."""
    a = np.abs(x)
    step = _e4m3_step(a)
    frac = a / step - np.floor(a / step)
    near = np.abs(frac - 0.5) * step < window * np.maximum(a, 1.0)
    return np.where(near & (a > 0), step, 0.0)


def forward_fp8(q, k, v, k_cache, v_cache, videos, slices, hq, hkv,
                base=(1e4, 1e4, 1e4), eps=1e-6, q_gain=None, k_gain=None, rows=None, q_rows=None):
    """The forward with e4m3 operands, and the spread its last rounding leaves.

    FP8 on the pages: MAGI-1 research notes, inference infrastructure (real-time streaming
    scenario): the linear layers run W8A8 in FP8 (SmoothQuant).  The attention variant
    modelled here puts the same 8-bit format on the attention operands.

    Same method as ``forward`` with the tensor-core operands rounded to e4m3: Q-hat and
    K-hat after the prologue (unscaled; the softmax scale 1/sqrt(D) multiplies the
    fp64 score), and V divided by 2^e per KV head (``e4m3_scale_exponent`` of max|V|
    over the new and the cache rows), rounded, and multiplied back.  The scores, the
    softmax and P V are then exact (fp64).  Cache keys are used as given (post-prologue).

    The GPU kernel also rounds P to e4m3 before P V, at a per-row reference that the
    online softmax chooses (P <= 2^8), so its P differs from this P by a relative
    rounding error of at most 2^-4 per element in e4m3's normal range, and by at most
    2^-10 (half the subnormal step) in the kernel's P units below it, a unit at least
    exp(lse - max s) in normalised probability.  The row sum that normalises O is
    formed from the unrounded fp32 P, so the errors do not cancel in the division:
    O_gpu - O = sum_j p_ij e_ij v_jd.  Treating the e_ij as independent and uniform
    gives the standard deviation returned as ``sd``:
        sd[i,h,d]^2 = sum_j ((2^-4/sqrt 3)^2 p_ij^2 + (2^-10/sqrt 3)^2 exp(2 (max_j s_ij - lse_i)))
                      * v_jd^2.
    A Q-hat or K-hat element computed in fp32 (the kernel's prologue) within about 2e-6
    of an e4m3 rounding midpoint may round to the other neighbour, moving score s_ij by
    at most that element's step times its partner's magnitude / sqrt(D).  ``flip`` is
    the p-weighted sum of those possible score moves per (row, head), a first-order bound
    of the LSE change they can cause (and, times max_j |v_jd - o_id|, of the O change);
    it is 0 for rows no undecided element reaches.
    Returns (O [nr,Hq,D], LSE [nr,Hq], sd [nr,Hq,D], flip [nr,Hq], vdev [nr,Hq,D] =
    max_j |v_jd| over the KV group plus |o_id|, a bound of max_j |v_jd - o_id|)."""
    pos = positions(videos)
    if rows is None:
        rows = np.arange(pos.shape[0], dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    qr = _f64(q_rows) if q_rows is not None else _f64(q)[rows]
    D = qr.shape[-1]
    nc = 0 if k_cache is None else int(k_cache.shape[0])
    kh = full_keys(prologue(k, pos, base, eps, k_gain), k_cache)
    vv = full_keys(v, v_cache)
    qh = prologue(qr, pos[rows], base, eps, q_gain)
    uq = _e4m3_undecided(qh)
    uk = _e4m3_undecided(kh)
    uk[:nc] = 0.0                                   # cache keys are bf16 values: rounded exactly alike
    q8 = round_e4m3(qh)
    k8 = round_e4m3(kh)
    v8 = np.empty_like(vv)
    for g in range(hkv):
        e = e4m3_scale_exponent(np.abs(vv[:, g, :]).max() if vv.shape[0] else 0.0)
        v8[:, g, :] = round_e4m3(vv[:, g, :] / 2.0 ** e) * 2.0 ** e
    nk = kh.shape[0]
    vis = np.stack([mask_row(slices, nk, int(i)) for i in rows]) if len(rows) else np.zeros((0, nk), bool)
    G = hq // hkv
    nr = len(rows)
    O = np.zeros((nr, hq, D))
    lse = np.full((nr, hq), -np.inf)
    sd = np.zeros((nr, hq, D))
    flip = np.zeros((nr, hq))
    vdev = np.zeros((nr, hq, D))
    rel = 2.0 ** -4 / np.sqrt(3.0)
    absu = 2.0 ** -10 / np.sqrt(3.0)
    for h in range(hq):
        g = h // G
        s = (q8[:, h, :] @ k8[:, g, :].T) / np.sqrt(D)
        s = np.where(vis, s, -np.inf)
        smax = s.max(axis=1, initial=-np.inf)
        live = np.isfinite(smax)
        sm = np.where(live, smax, 0.0)
        ex = np.exp(s - sm[:, None])
        tot = ex.sum(axis=1)
        l_ = np.where(live, sm + np.log(np.where(live, tot, 1.0)), -np.inf)
        p = ex / np.where(live, tot, 1.0)[:, None]
        vg = v8[:, g, :]
        o = p @ vg
        w = (rel * p) ** 2 + (absu * np.where(live, np.exp(sm - l_), 0.0))[:, None] ** 2 * vis
        var = w @ (vg * vg)
        ds = (uq[:, h, :] @ np.abs(k8[:, g, :]).T + np.abs(q8[:, h, :]) @ uk[:, g, :].T) / np.sqrt(D)
        O[:, h, :] = o
        lse[:, h] = l_
        sd[:, h, :] = np.sqrt(np.maximum(var, 0.0))
        flip[:, h] = (p * ds).sum(axis=1)
        if nk:
            vdev[:, h, :] = np.where(live[:, None], np.abs(vg).max(axis=0)[None, :] + np.abs(o), 0.0)
    return O, lse, sd, flip, vdev
