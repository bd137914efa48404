"""Expected dK / dV of seeded key rows of the full-size backward workloads, from the fp64
oracle alone.

For one KV group g of a workload, the gradient of key j sums over every (query row i,
query head h of g) that sees j:  dV_j = sum P_ij dO_i,  dK^_j = sum dS_ij q^_i / sqrt(D),
dS_ij = P_ij (dO_i . v_j - Dsum_i),  P_ij = exp(s_ij - LSE_i),  Dsum_i = dO_i . O_i.  It
needs LSE_i and O_i of exactly the rows that see a sampled key, so this script
  1. finds those rows (the oracle's mask columns of the sampled keys),
  2. runs the oracle forward on them for the group's heads (``attn_fwd_rows_blas``),
  3. forms Dsum from the exact O and calls the oracle's key backward (``attn_bwd_keys``),
  4. maps dK^ of new keys through the prologue backward (w.r.t. the raw keys); cache keys
     are given post-prologue, so their dK is dK^ itself.
Rows that see no sampled key do not enter (their LSE is +inf for the key backward, so
P = 0).  Inputs are the workloads' seeded tensors (the same bits the GPU tests use).

Writes tests/golden/key_grads_<workload>.npz (float32 values, int64 key indices in the
[cache | new] key space) with a JSON note of the command, the duration and the host.

    python tests/golden/make_key_grads.py [workload ...]      # default: all three
"""
from __future__ import annotations

import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from block_causal_attention_b200 import workloads as W  # noqa: E402

# (KV group, key sets).  A key set is (first key, last key + 1, how many, seed) in the
# [cache | new] key space; the first and last key of every set are always included.
SPECS = {
    "p720_pipelined": (5, [
        (0, 8 * 21600, 128, 31),                        # the 8 cached chunks (dK_cache, dV_cache)
        (8 * 21600, 12 * 21600, 128, 32),               # the 4 new chunks
    ]),
    "packed_varlen": (2, [
        (22 * 6144, 24 * 6144, 64, 41),                 # video 0 (24 chunks): its last two chunks
        (24 * 6144, 25 * 6144, 32, 42),                 # video 1 (12 chunks): its first chunk
        (44 * 6144, 48 * 6144, 64, 43),                 # video 3 (4 chunks): all of it
    ]),
    "long_kvrange": (7, [
        (127 * 8192, 128 * 8192, 64, 51),               # the last chunk
        (32 * 8192, 33 * 8192, 64, 52),                 # transition chunk 32
        (1 * 8192, 2 * 8192, 64, 53),                   # chunk 1, also seen by the transition chunks
    ]),
}


def sample_keys(sets) -> np.ndarray:
    out = []
    for (k0, k1, n, seed) in sets:
        rng = np.random.default_rng(seed)
        inner = rng.choice(np.arange(k0 + 1, k1 - 1), size=n - 2, replace=False)
        out.append(np.concatenate([[k0, k1 - 1], inner]))
    return np.unique(np.concatenate(out).astype(np.int64))


def key_grads(w, g: int, keys, workers=None):
    """dK and dV [len(keys), D] (fp64) of KV group g for the listed keys of workload w."""
    keys = np.asarray(keys, np.int64)
    G = w.hq // w.hkv
    nc, nq, nk = w.num_cache_keys, w.nq, w.nk
    sl = w.slices_array()
    heads = (g * G, (g + 1) * G)
    # 1. rows that see any sampled key
    seen = np.zeros(nq, bool)
    for j in keys:
        seen |= oracle.mask_col(sl, nq, int(j))
    rows = np.flatnonzero(seen).astype(np.int64)
    # 2. forward of those rows (post-prologue queries of the group's heads)
    pos = oracle.positions(w.videos_array())
    qh = oracle.prologue(W.make_input_rows(w, W.T_Q, rows, heads=heads), pos[rows], w.rope_base, w.eps)
    k_new = W.make_input_rows(w, W.T_K, np.arange(nq), heads=(g, g + 1))
    kh = oracle.prologue(k_new, pos, w.rope_base, w.eps)
    v = oracle._f64(W.make_input_rows(w, W.T_V, np.arange(nq), heads=(g, g + 1)))
    if nc:
        kc = oracle._f64(W.make_input_rows(w, W.T_KC, np.arange(nc), heads=(g, g + 1)))
        vc = oracle._f64(W.make_input_rows(w, W.T_VC, np.arange(nc), heads=(g, g + 1)))
        kh = np.concatenate([kc, kh], 0)
        v = np.concatenate([vc, v], 0)
    O, lse = oracle.attn_fwd_rows_blas(qh, rows, kh, v, sl, G, 1, workers=workers)
    do = oracle._f64(W.make_input_rows(w, W.T_DO, rows, heads=heads))
    # 3. key backward over the full row space (rows not computed: LSE = +inf, P = 0)
    qh_all = np.zeros((nq, G, w.d))
    do_all = np.zeros((nq, G, w.d))
    lse_all = np.full((nq, G), np.inf)
    dsum_all = np.zeros((nq, G))
    qh_all[rows], do_all[rows], lse_all[rows] = qh, do, lse
    dsum_all[rows] = (do * O).sum(-1)
    del qh, do, O
    dkh, dv = oracle.attn_bwd_keys(qh_all, do_all, lse_all, dsum_all, kh, v, keys, sl, G, 1)
    dkh, dv = dkh[:, 0], dv[:, 0]
    # 4. new keys: through the prologue backward, w.r.t. the raw keys
    new = keys >= nc
    dk = dkh.copy()
    if new.any():
        kn = keys[new] - nc
        dk[new] = oracle.prologue_bwd(k_new[kn], pos[kn], dkh[new][:, None], w.rope_base, w.eps)[:, 0]
    return dk, dv, len(rows)


def main(names):
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)  # one BLAS thread per worker thread
    except Exception:
        pass
    for name in names:
        w = W.WORKLOADS[name]
        g, sets = SPECS[name]
        keys = sample_keys(sets)
        t0 = time.time()
        dk, dv, nrows = key_grads(w, g, keys)
        dt = time.time() - t0
        note = {"command": "python tests/golden/make_key_grads.py " + name, "workload": name, "group": g,
                "keys": int(len(keys)), "rows_forwarded": int(nrows), "seconds": round(dt, 1),
                "host_cores": os.cpu_count()}
        out = os.path.join(HERE, f"key_grads_{name}.npz")
        np.savez_compressed(out, keys=keys, group=np.int64(g), dk=dk.astype(np.float32),
                            dv=dv.astype(np.float32), note=np.asarray(json.dumps(note)))
        print(json.dumps(note), flush=True)


if __name__ == "__main__":
    main(sys.argv[1:] or list(SPECS))
