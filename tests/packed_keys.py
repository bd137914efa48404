"""Exact dK / dV for sampled key rows of one packed video, from the fp64 oracle (test
support for the full-size backward checks).

In a packed workload each video's slices reference only its own tokens, so one video
with one KV group is a problem of its own: its queries, keys and positions (restarting at
the video's t0) are the same as in the whole pack.  A key of chunk c is seen only by
the rows of chunks >= c, so the keys of a video's last chunks need the LSE and Dsum of
only those rows: exact dK / dV at full size without the whole forward."""
import numpy as np

import oracle
from block_causal_attention_b200 import workloads as W


def video_span(w, vi):
    """(first token, tokens per chunk, chunks) of packed video vi."""
    vids = np.asarray(w.videos_array(), np.int64).reshape(-1, 5)
    start = int(sum(int(v[0] * v[1] * v[2] * v[3]) for v in vids[:vi]))
    nc, f, h, wd, _ = (int(x) for x in vids[vi])
    return start, f * h * wd, nc


def video_key_grads(w, vi, g, keys_local):
    """dK (w.r.t. the raw keys, through QK-Norm and RoPE) and dV [nkeys, D] of KV group g
    for the listed keys of video vi (indices within the video)."""
    vids = np.asarray(w.videos_array(), np.int64).reshape(-1, 5)
    start, C, nch = video_span(w, vi)
    n = nch * C
    rows = np.arange(start, start + n)
    G = w.hq // w.hkv
    q = W.make_input_rows(w, W.T_Q, rows)[:, g * G:(g + 1) * G]
    k = W.make_input_rows(w, W.T_K, rows)[:, g:g + 1]
    v = W.make_input_rows(w, W.T_V, rows)[:, g:g + 1]
    do = W.make_input_rows(w, W.T_DO, rows)[:, g * G:(g + 1) * G]
    sub_vid = vids[vi:vi + 1].astype(np.int32)
    sub_sl = np.asarray([[c * C, (c + 1) * C, 0, (c + 1) * C, 0] for c in range(nch)], np.int64)
    pos = oracle.positions(sub_vid)
    qh = oracle.prologue(q, pos, w.rope_base, w.eps)
    kh = oracle.prologue(k, pos, w.rope_base, w.eps)
    keys_local = np.asarray(keys_local, np.int64)
    r0 = int(keys_local.min()) // C * C              # first row that sees any listed key
    O, lse = oracle.attn_fwd_rows(qh[r0:], np.arange(r0, n), kh, v, sub_sl, G, 1)
    dsum = (do.double().numpy()[r0:] * O).sum(-1)
    lse_all = np.full((n, G), np.inf)
    dsum_all = np.zeros((n, G))
    lse_all[r0:], dsum_all[r0:] = lse, dsum
    dkh, dv = oracle.attn_bwd_keys(qh, do, lse_all, dsum_all, kh, v, keys_local, sub_sl, G, 1)
    dk = oracle.prologue_bwd(k.double().numpy()[keys_local], pos[keys_local], dkh, w.rope_base, w.eps)
    return dk[:, 0], dv[:, 0]
