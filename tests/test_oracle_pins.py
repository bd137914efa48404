"""Pins for the fp64 oracle: each test checks the oracle against something other than
itself (numpy/torch library routines on special cases, closed forms, invariants,
brute force, finite differences, hand-written fixtures)."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _block_causal(sizes_per_video, C, cache=0):
    """Slices for packed block-causal videos (chunk size C) built here, in the test."""
    out, q = [], 0
    for vi, n in enumerate(sizes_per_video):
        for c in range(n):
            k0 = 0 if (vi == 0 and cache) else cache + q
            out.append((q + c * C, q + (c + 1) * C, k0, cache + q + (c + 1) * C, 0))
        q += n * C
    return np.asarray(out, np.int64)


# --------------------------------------------------------------------------- mask

def test_mask_one_chunk_is_full():
    sl = _block_causal([1], 37)
    assert oracle.mask_dense(sl, 37, 37).all()


def test_mask_chunk_size_one_is_lower_triangle():
    n = 29
    sl = _block_causal([n], 1)
    assert np.array_equal(oracle.mask_dense(sl, n, n), np.tril(np.ones((n, n), bool)))


@pytest.mark.parametrize("nchunks,C", [(3, 64), (5, 7), (2, 1)])
def test_mask_block_causal_is_kron_of_tril(nchunks, C):
    n = nchunks * C
    want = np.kron(np.tril(np.ones((nchunks, nchunks), int)), np.ones((C, C), int)).astype(bool)
    assert np.array_equal(oracle.mask_dense(_block_causal([nchunks], C), n, n), want)


def test_mask_packed_videos_block_diagonal():
    sizes, C = [4, 2, 3, 1], 5
    n = sum(sizes) * C
    blocks = [np.kron(np.tril(np.ones((s, s), int)), np.ones((C, C), int)) for s in sizes]
    want = np.zeros((n, n), int)
    o = 0
    for b in blocks:
        want[o:o + len(b), o:o + len(b)] = b
        o += len(b)
    assert np.array_equal(oracle.mask_dense(_block_causal(sizes, C), n, n), want.astype(bool))


def test_mask_cache_prefix_visible_to_all():
    C, nc, nqch = 6, 3, 4
    sl = _block_causal([nqch], C, cache=nc * C)
    nq, nk = nqch * C, (nc + nqch) * C
    want = np.concatenate([np.ones((nq, nc * C), int),
                           np.kron(np.tril(np.ones((nqch, nqch), int)), np.ones((C, C), int))], 1)
    assert np.array_equal(oracle.mask_dense(sl, nq, nk), want.astype(bool))


@pytest.mark.parametrize("qlen,klen", [(5, 5), (3, 8), (8, 3), (1, 4)])
def test_mask_causal_slice_bottom_right(qlen, klen):
    sl = np.asarray([(2, 2 + qlen, 1, 1 + klen, 1)], np.int64)
    nq, nk = 2 + qlen + 3, 1 + klen + 2
    want = np.zeros((nq, nk), bool)
    want[2:2 + qlen, 1:1 + klen] = np.tril(np.ones((qlen, klen), bool), k=klen - qlen)
    assert np.array_equal(oracle.mask_dense(sl, nq, nk), want)


def test_mask_union_of_random_slices_bruteforce():
    for trial in range(20):
        nq, nk = int(RNG.integers(1, 40)), int(RNG.integers(1, 40))
        ns = int(RNG.integers(0, 6))
        sl = []
        want = np.zeros((nq, nk), bool)
        for _ in range(ns):
            q0 = int(RNG.integers(0, nq)); q1 = int(RNG.integers(q0, nq + 1))
            k0 = int(RNG.integers(0, nk)); k1 = int(RNG.integers(k0, nk + 1))
            t = int(RNG.integers(0, 2))
            sl.append((q0, q1, k0, k1, t))
            blk = np.ones((q1 - q0, k1 - k0), bool)
            if t == 1:
                blk = np.tril(blk, k=(k1 - k0) - (q1 - q0))
            want[q0:q1, k0:k1] |= blk
        got = oracle.mask_dense(np.asarray(sl, np.int64).reshape(-1, 5), nq, nk)
        assert np.array_equal(got, want), trial
        # rows and columns agree with the dense mask
        for i in range(nq):
            assert np.array_equal(oracle.mask_row(sl, nk, i), want[i])
        for j in range(nk):
            assert np.array_equal(oracle.mask_col(sl, nq, j), want[:, j])


def test_mask_workload_pair_counts_closed_form():
    # 720p pipelined replica: query chunk j sees 8 cached chunks + chunks 0..j
    w = W.WORKLOADS["p720_replica"]
    C = w.videos[0].chunk_tokens
    m = oracle.mask_dense(w.slices_array(), w.nq, w.nk)
    assert m.sum() == C * C * sum(8 + j + 1 for j in range(4))
    # KV-range replica: chunk c sees min(c,16)+1 chunks, a transition chunk sees 3
    w = W.WORKLOADS["kvrange_replica"]
    C = w.videos[0].chunk_tokens
    m = oracle.mask_dense(w.slices_array(), w.nq, w.nk)
    per = [3 if c in (12, 24, 36) else min(c, 16) + 1 for c in range(40)]
    assert m.sum() == C * C * sum(per)
    # full-size long-context row sample: row in chunk c sees exactly per-chunk closed form
    w = W.WORKLOADS["long_kvrange"]
    C = w.videos[0].chunk_tokens
    for c in (0, 5, 16, 31, 32, 33, 64, 96, 127):
        row = oracle.mask_row(w.slices_array(), w.nk, c * C + 17)
        if c in (32, 64, 96):
            want = np.zeros(w.nk, bool); want[:2 * C] = True; want[c * C:(c + 1) * C] = True
        else:
            want = np.zeros(w.nk, bool); want[max(0, c - 16) * C:(c + 1) * C] = True
        assert np.array_equal(row, want), c


# --------------------------------------------------------------------------- positions

def test_positions_golden_fixture():
    pos = oracle.positions([[2, 2, 3, 4, 5]])
    assert pos.shape == (48, 3)
    rows = np.loadtxt(os.path.join(GOLDEN, "positions_2x2x3x4_t0_5.txt"), dtype=np.int64)
    for n, t, h, w in rows:
        assert tuple(pos[n]) == (t, h, w), n


def test_positions_restart_per_video():
    pos = oracle.positions([[2, 1, 2, 2, 0], [1, 2, 1, 3, 0]])
    assert tuple(pos[8]) == (0, 0, 0) and tuple(pos[13]) == (1, 0, 2)


# --------------------------------------------------------------------------- prologue

def _rand(shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def test_prologue_rms_norm_gives_norm_sqrt_d():
    for D in (24, 32, 48):
        x = _rand((7, 3, D), 3.0)
        pos = RNG.integers(0, 50, size=(7, 3)).astype(np.int32)
        y = oracle.prologue(x, pos, eps=0.0)
        assert np.allclose(np.linalg.norm(y, axis=-1), math.sqrt(D), rtol=1e-12)


def test_prologue_zero_position_is_plain_rms_norm():
    D = 48
    x = _rand((5, 2, D))
    g = RNG.uniform(0.5, 2.0, D)
    y = oracle.prologue(x, np.zeros((5, 3), np.int32), eps=1e-6, gain=g)
    rms = np.sqrt((x ** 2).mean(-1, keepdims=True) + 1e-6)
    assert np.allclose(y, g * x / rms, rtol=1e-13, atol=0)


@pytest.mark.parametrize("D", [24, 48])
def test_prologue_huge_base_leaves_only_the_first_pair_of_each_axis_rotating(D):
    """Pair k of an axis rotates by pos * base^(-k/p): as the base grows every pair but
    the first (k = 0, frequency 1 for any base) stops rotating, so the output is the plain
    RMS norm except channels (0, 1) of each axis segment, rotated by that axis's position."""
    p = (D // 2) // 3
    x = _rand((6, 1, D))
    pos = np.asarray([[3, 1, 2], [0, 5, 7], [9, 0, 0], [1, 1, 1], [4, 2, 6], [2, 3, 0]], np.int32)
    y = oracle.prologue(x, pos, base=(1e300, 1e300, 1e300), eps=1e-6)
    z = x / np.sqrt((x ** 2).mean(-1, keepdims=True) + 1e-6)
    want = z.copy()
    for a in range(3):
        c0 = 2 * p * a
        th = pos[:, a].astype(np.float64)[:, None]
        x0, x1 = z[:, :, c0], z[:, :, c0 + 1]
        want[:, :, c0] = x0 * np.cos(th) - x1 * np.sin(th)
        want[:, :, c0 + 1] = x0 * np.sin(th) + x1 * np.cos(th)
    assert np.allclose(y, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("D", [24, 32, 48])
def test_prologue_rope_pairs_are_adjacent_channels(D):
    """A basis vector on channel 2k of axis a rotates into channel 2k+1 of the same
    segment only, by the angle pos * base^(-k/p); channels past 6p never move."""
    p = (D // 2) // 3
    base = (10000.0, 500.0, 77.0)
    for a in range(3):
        for k in range(p):
            c0 = 2 * p * a + 2 * k
            x = np.zeros((1, 1, D)); x[0, 0, c0] = 1.0  # rms norm maps it to sqrt(D) e_c0
            pos = np.zeros((1, 3), np.int32); pos[0, a] = 9
            y = oracle.prologue(x, pos, base=base, eps=0.0)[0, 0]
            ang = 9 * base[a] ** (-k / p)
            want = np.zeros(D); want[c0] = math.cos(ang); want[c0 + 1] = math.sin(ang)
            want *= math.sqrt(D)
            assert np.allclose(y, want, atol=1e-12), (a, k)
    if 6 * p < D:
        x = np.zeros((1, 1, D)); x[0, 0, 6 * p:] = 1.0
        y = oracle.prologue(x, np.full((1, 3), 13, np.int32), eps=0.0)
        assert np.allclose(y[0, 0, :6 * p], 0) and np.allclose(y[0, 0, 6 * p:], y[0, 0, -1])


def test_prologue_relative_position_invariance():
    D = 48
    q = _rand((6, 1, D)); k = _rand((6, 1, D))
    pq = RNG.integers(0, 40, (6, 3)).astype(np.int32)
    pk = RNG.integers(0, 40, (6, 3)).astype(np.int32)
    shift = np.asarray([[11, 3, 7]], np.int32)
    s0 = (oracle.prologue(q, pq) * oracle.prologue(k, pk)).sum(-1)
    s1 = (oracle.prologue(q, pq + shift) * oracle.prologue(k, pk + shift)).sum(-1)
    assert np.allclose(s0, s1, atol=1e-10)
    # but not invariant to shifting only one side
    s2 = (oracle.prologue(q, pq + shift) * oracle.prologue(k, pk)).sum(-1)
    assert not np.allclose(s0, s2, atol=1e-3)


# --------------------------------------------------------------------------- attention

def _sdpa(qh, kh, v, mask=None, causal=False):
    """torch's reference SDPA (math backend, fp64, CPU); [n, H, D] in, [n, H, D] out."""
    q = torch.from_numpy(qh).permute(1, 0, 2)[None]
    k = torch.from_numpy(kh).permute(1, 0, 2)[None]
    vv = torch.from_numpy(v).permute(1, 0, 2)[None]
    G = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(G, dim=1)
    vv = vv.repeat_interleave(G, dim=1)
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, vv, attn_mask=m, is_causal=causal)
    return o[0].permute(1, 0, 2).numpy()


def test_attention_one_chunk_equals_full_attention():
    n, Hq, Hkv, D = 40, 4, 2, 32
    qh, kh, v = _rand((n, Hq, D)), _rand((n, Hkv, D)), _rand((n, Hkv, D))
    O, lse = oracle.attn_fwd_rows(qh, np.arange(n), kh, v, _block_causal([1], n), Hq, Hkv)
    assert np.allclose(O, _sdpa(qh, kh, v), atol=1e-12)
    # LSE closed form on a row
    s = (qh[3, 1] @ kh[:, 0].T) / math.sqrt(D)
    assert abs(lse[3, 1] - (s.max() + math.log(np.exp(s - s.max()).sum()))) < 1e-12


def test_attention_chunk_size_one_equals_causal():
    n, Hq, Hkv, D = 33, 4, 4, 24
    qh, kh, v = _rand((n, Hq, D)), _rand((n, Hkv, D)), _rand((n, Hkv, D))
    O, _ = oracle.attn_fwd_rows(qh, np.arange(n), kh, v, _block_causal([n], 1), Hq, Hkv)
    assert np.allclose(O, _sdpa(qh, kh, v, causal=True), atol=1e-12)


def test_attention_block_causal_equals_masked_sdpa_gqa():
    C, nch, Hq, Hkv, D = 9, 4, 8, 2, 48
    n = C * nch
    qh, kh, v = _rand((n, Hq, D)), _rand((n, Hkv, D)), _rand((n, Hkv, D))
    mask = np.kron(np.tril(np.ones((nch, nch), int)), np.ones((C, C), int)).astype(bool)
    O, _ = oracle.attn_fwd_rows(qh, np.arange(n), kh, v, _block_causal([nch], C), Hq, Hkv)
    assert np.allclose(O, _sdpa(qh, kh, v, mask=mask), atol=1e-12)


def test_gqa_with_groups_equal_heads_is_mha():
    """Hkv = Hq (one head per group) equals per-head attention; and GQA equals MHA on
    K/V repeated contiguously over each group's heads."""
    n, Hq, Hkv, D = 24, 6, 3, 32
    sl = _block_causal([3], 8)
    qh, kh, v = _rand((n, Hq, D)), _rand((n, Hkv, D)), _rand((n, Hkv, D))
    O_gqa, l_gqa = oracle.attn_fwd_rows(qh, np.arange(n), kh, v, sl, Hq, Hkv)
    kr, vr = np.repeat(kh, 2, axis=1), np.repeat(v, 2, axis=1)
    O_mha, l_mha = oracle.attn_fwd_rows(qh, np.arange(n), kr, vr, sl, Hq, Hq)
    assert np.array_equal(O_gqa, O_mha) and np.array_equal(l_gqa, l_mha)
    for h in range(Hq):
        O1, _ = oracle.attn_fwd_rows(qh[:, h:h + 1].copy(), np.arange(n), kr[:, h:h + 1].copy(),
                                     vr[:, h:h + 1].copy(), sl, 1, 1)
        assert np.array_equal(O1[:, 0], O_mha[:, h])


def test_attention_bruteforce_tiny():
    """Explicit python sums over <= 8 tokens."""
    n, D = 7, 24
    sl = np.asarray([(0, 3, 0, 3, 0), (3, 7, 0, 7, 0), (5, 7, 2, 4, 1)], np.int64)
    qh, kh, v = _rand((n, 1, D)), _rand((n, 1, D)), _rand((n, 1, D))
    O, lse = oracle.attn_fwd_rows(qh, np.arange(n), kh, v, sl, 1, 1)
    vis = [[0, 1, 2]] * 3 + [list(range(7))] * 4
    for i in range(n):
        s = [sum(qh[i, 0, d] * kh[j, 0, d] for d in range(D)) / math.sqrt(D) for j in vis[i]]
        z = sum(math.exp(x) for x in s)
        o = [sum(math.exp(s[a]) / z * v[j, 0, d] for a, j in enumerate(vis[i])) for d in range(D)]
        assert abs(lse[i, 0] - math.log(z)) < 1e-12
        assert np.allclose(O[i, 0], o, atol=1e-12)


def test_attention_rows_sum_to_one_and_empty_rows():
    n, D = 20, 32
    sl = np.asarray([(0, 10, 0, 10, 0), (12, 20, 5, 18, 1)], np.int64)  # rows 10, 11 see nothing
    qh, kh = _rand((n, 2, D)), _rand((n, 1, D))
    O, lse = oracle.attn_fwd_rows(qh, np.arange(n), kh, np.ones((n, 1, D)), sl, 2, 1)
    live = [i for i in range(n) if i not in (10, 11)]
    assert np.allclose(O[live], 1.0, atol=1e-13)
    assert np.all(O[[10, 11]] == 0) and np.all(np.isneginf(lse[[10, 11]]))


def test_causality_later_chunks_do_not_change_earlier_outputs():
    w = W.WORKLOADS["tiny"]
    x = W.make_inputs(w)
    C = w.videos[0].chunk_tokens
    O0, l0 = oracle.forward(x["q"], x["k"], x["v"], None, None, w.videos_array(), w.slices_array(),
                            w.hq, w.hkv)
    q2, k2, v2 = x["q"].clone(), x["k"].clone(), x["v"].clone()
    q2[2 * C:] = q2[2 * C:] * 3 + 1
    k2[2 * C:] = -k2[2 * C:]
    v2[2 * C:] = v2[2 * C:] + 5
    O1, l1 = oracle.forward(q2, k2, v2, None, None, w.videos_array(), w.slices_array(), w.hq, w.hkv)
    assert np.array_equal(O0[:2 * C], O1[:2 * C]) and np.array_equal(l0[:2 * C], l1[:2 * C])
    assert not np.allclose(O0[2 * C:], O1[2 * C:])


# --------------------------------------------------------------------------- backward

def test_backward_matches_central_finite_differences():
    """Gradients w.r.t. the raw inputs (through QK-Norm + RoPE) against central
    differences of the forward, fp64.  Loss = sum(O * R) for a fixed random R."""
    Hq, Hkv, D = 4, 2, 24
    videos = np.asarray([[2, 1, 2, 3, 4]], np.int32)          # 2 chunks x 6 tokens, t0=4
    nq, nc = 12, 6
    sl = _block_causal([2], 6, cache=nc)
    q, k, v = _rand((nq, Hq, D)), _rand((nq, Hkv, D)), _rand((nq, Hkv, D))
    kc, vc = _rand((nc, Hkv, D)), _rand((nc, Hkv, D))
    R = _rand((nq, Hq, D))
    g_q, g_k = RNG.uniform(0.5, 1.5, D), RNG.uniform(0.5, 1.5, D)
    base = (100.0, 50.0, 20.0)

    def loss(q, k, v, kc, vc):
        O, _ = oracle.forward(q, k, v, kc, vc, videos, sl, Hq, Hkv, base=base, q_gain=g_q,
                              k_gain=g_k)
        return float((O * R).sum())

    dq, dk, dv, dkc, dvc, _, _ = oracle.backward(q, k, v, kc, vc, R, videos, sl, Hq, Hkv, base=base,
                                                 q_gain=g_q, k_gain=g_k)
    args = [q, k, v, kc, vc]
    grads = [dq, dk, dv, dkc, dvc]
    h = 1e-6
    for ai, (a, g) in enumerate(zip(args, grads)):
        idx = [tuple(RNG.integers(0, s) for s in a.shape) for _ in range(12)]
        for ix in idx:
            ap, am = a.copy(), a.copy()
            ap[ix] += h; am[ix] -= h
            fa = list(args); fa[ai] = ap
            fb = list(args); fb[ai] = am
            fd = (loss(*fa) - loss(*fb)) / (2 * h)
            assert abs(fd - g[ix]) <= 1e-6 * max(1.0, abs(fd)), (ai, ix, fd, g[ix])


@pytest.mark.parametrize("D", [24, 32])
def test_parameter_gradients_match_central_finite_differences(D):
    """Gradients of the QK-Norm gains (Q and K) and of the three RoPE bases against
    central differences of the forward in fp64.  D = 32 leaves one pair unrotated, and
    the cache keys (already post-prologue) must not contribute to the K gain."""
    Hq, Hkv = 4, 2
    videos = np.asarray([[2, 1, 2, 3, 4]], np.int32)
    nq, nc = 12, 6
    sl = _block_causal([2], 6, cache=nc)
    q, k, v = _rand((nq, Hq, D)), _rand((nq, Hkv, D)), _rand((nq, Hkv, D))
    kc, vc = _rand((nc, Hkv, D)), _rand((nc, Hkv, D))
    R = _rand((nq, Hq, D))
    g_q, g_k = RNG.uniform(0.5, 1.5, D), RNG.uniform(0.5, 1.5, D)
    base = np.asarray([100.0, 50.0, 20.0])

    def loss(gq, gk, b):
        O, _ = oracle.forward(q, k, v, kc, vc, videos, sl, Hq, Hkv, base=tuple(b), q_gain=gq, k_gain=gk)
        return float((O * R).sum())

    out = oracle.backward(q, k, v, kc, vc, R, videos, sl, Hq, Hkv, base=tuple(base), q_gain=g_q,
                          k_gain=g_k, param_grads=True)
    dgq, dgk, db = out[7], out[8], out[9]
    for name, vec, grad in (("q_gain", 0, dgq), ("k_gain", 1, dgk), ("base", 2, db)):
        for i in range(len(grad)):
            vals = [g_q.copy(), g_k.copy(), base.copy()]
            h = 1e-6 * max(1.0, abs(vals[vec][i]))
            vp = [x.copy() for x in vals]; vp[vec][i] += h
            vm = [x.copy() for x in vals]; vm[vec][i] -= h
            fd = (loss(*vp) - loss(*vm)) / (2 * h)
            assert abs(fd - grad[i]) <= 2e-6 * max(1.0, abs(fd)), (name, i, fd, grad[i])
    assert np.any(np.abs(db) > 1e-3) and np.any(np.abs(dgk) > 1e-3)


def test_backward_dv_sums_to_do_sum():
    """Rows of P sum to one, so sum_j dV_j = sum over the group's heads and rows with a
    visible key of dO_i; and sum_j dS_ij = 0, so sum_j dkh_j = 0 per group."""
    n, Hq, Hkv, D = 30, 4, 2, 32
    sl = _block_causal([3], 10)
    qh, kh, v, do = _rand((n, Hq, D)), _rand((n, Hkv, D)), _rand((n, Hkv, D)), _rand((n, Hq, D))
    dq, dk, dv, O, lse = oracle.attn_bwd_dense(qh, kh, v, do, sl, Hq, Hkv)
    for g in range(Hkv):
        assert np.allclose(dv[:, g].sum(0), do[:, 2 * g:2 * g + 2].sum((0, 1)), atol=1e-10)
        assert np.allclose(dk[:, g].sum(0), 0, atol=1e-10)


def test_video_key_grads_equal_the_dense_backward():
    """The per-video key-row helper of the full-size backward checks (packed_keys) gives
    the dense oracle backward's dK and dV, for videos of a packed workload and each group."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from packed_keys import video_key_grads, video_span
    w = W.WORKLOADS["packed_replica"]
    x = W.make_inputs(w, "cpu", with_grad=True)
    _, dk, dv, _, _, _, _ = oracle.backward(x["q"], x["k"], x["v"], None, None, x["do"], w.videos_array(),
                                            w.slices_array(), w.hq, w.hkv, base=w.rope_base, eps=w.eps)
    for vi in (1, 2):
        start, C, nch = video_span(w, vi)
        keys = np.unique(np.random.default_rng(vi).integers(max(0, nch - 2) * C, nch * C, 40))
        for g in range(w.hkv):
            k_dk, k_dv = video_key_grads(w, vi, g, keys)
            assert np.abs(k_dk - dk[start + keys, g]).max() <= 1e-12
            assert np.abs(k_dv - dv[start + keys, g]).max() <= 1e-12


# --------------------------------------------------------------------------- full-size helpers

def test_blas_rows_equal_the_loop_rows_on_random_slice_unions():
    """attn_fwd_rows_blas (fp64 matrix products over row batches) gives the per-pair C
    loops' O and LSE on random FULL/CAUSAL slice unions with empty rows, GQA and MHA,
    rows in any order and batches that split the rows raggedly."""
    rng = np.random.default_rng(77)
    for trial in range(6):
        nq, nc = int(rng.integers(20, 90)), int(rng.integers(0, 40))
        nk = nq + nc
        Hq, Hkv = ((8, 2), (4, 4), (6, 1))[trial % 3]
        D = (24, 32, 48)[trial % 3]
        sl = []
        for _ in range(int(rng.integers(1, 5))):
            q0 = int(rng.integers(0, nq)); q1 = int(rng.integers(q0, nq + 1))
            k0 = int(rng.integers(0, nk)); k1 = int(rng.integers(k0, nk + 1))
            sl.append((q0, q1, k0, k1, int(rng.integers(0, 2))))
        sl = np.asarray(sl, np.int64)
        qh, kh, v = _rand((nq, Hq, D)), _rand((nk, Hkv, D)), _rand((nk, Hkv, D))
        rows = rng.permutation(nq)[:int(rng.integers(1, nq + 1))]
        O1, l1 = oracle.attn_fwd_rows(qh[rows], rows, kh, v, sl, Hq, Hkv)
        O2, l2 = oracle.attn_fwd_rows_blas(qh[rows], rows, kh, v, sl, Hq, Hkv, batch=7, workers=3)
        assert np.array_equal(np.isneginf(l1), np.isneginf(l2))
        fin = np.isfinite(l1)
        assert np.abs(l1[fin] - l2[fin]).max(initial=0) <= 1e-12
        assert np.abs(O1 - O2).max() <= 1e-12


def test_blas_rows_one_chunk_equals_full_attention():
    n, Hq, Hkv, D = 45, 8, 2, 48
    qh, kh, v = _rand((n, Hq, D)), _rand((n, Hkv, D)), _rand((n, Hkv, D))
    O, lse = oracle.attn_fwd_rows_blas(qh, np.arange(n), kh, v, _block_causal([1], n), Hq, Hkv, batch=8)
    assert np.allclose(O, _sdpa(qh, kh, v), atol=1e-12)
    s = (qh[7, 5] @ kh[:, 1].T) / math.sqrt(D)   # head 5 of 8 over 2 KV heads uses KV head 1
    assert abs(lse[7, 5] - (s.max() + math.log(np.exp(s - s.max()).sum()))) < 1e-12


@pytest.mark.parametrize("name", ["kvrange_replica", "packed_replica", "cache_small"])
def test_golden_key_grads_script_equals_the_dense_backward(name):
    """The script that writes the full-size dK / dV expectations (tests/golden/
    make_key_grads.py: rows that see the sampled keys only, forward by row batches, key
    backward) gives the dense oracle backward's dK, dV and cache gradients on small
    workloads of the same structure (KV-range transitions, packed videos, a KV cache)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_key_grads", os.path.join(GOLDEN, "make_key_grads.py"))
    mk = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mk)
    if name == "cache_small":
        w = W._c3_like("cache_small", 98, 1, 5, 5, 4, 1, backward=True)    # 8 cached + 4 new chunks of 25
    else:
        w = W.WORKLOADS[name]
    x = W.make_inputs(w, "cpu", with_grad=True)
    _, dk, dv, dkc, dvc, _, _ = oracle.backward(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], x["do"],
                                                w.videos_array(), w.slices_array(), w.hq, w.hkv,
                                                base=w.rope_base, eps=w.eps)
    rng = np.random.default_rng(5)
    keys = np.unique(np.concatenate([[0, w.nk - 1], rng.integers(0, w.nk, 40)]))
    nc = w.num_cache_keys
    for g in sorted({0, w.hkv - 1}):
        k_dk, k_dv, _ = mk.key_grads(w, g, keys, workers=2)
        for a, j in enumerate(keys):
            want_k = dkc[j, g] if j < nc else dk[j - nc, g]
            want_v = dvc[j, g] if j < nc else dv[j - nc, g]
            assert np.abs(k_dk[a] - want_k).max() <= 1e-12, (g, j)
            assert np.abs(k_dv[a] - want_v).max() <= 1e-12, (g, j)


@pytest.mark.parametrize("D", [32, 48])
def test_row_backward_equals_the_dense_backward(D):
    """backward_rows (the per-row C backward behind the full-size dQ row samples, through
    the prologue) gives the dense backward's dq, and attn_bwd_rows its O and LSE, on rows
    in any order: GQA with a KV cache, a FULL and a CAUSAL slice that overlap, and a row
    that sees no key (dq = 0).  The dense backward is pinned by central differences."""
    Hq, Hkv = 4, 2
    videos = np.asarray([[2, 1, 2, 3, 4]], np.int32)      # 2 chunks of 6 tokens, t0 = 4
    nq, nc = 12, 6
    sl = np.asarray([(0, 5, 0, 12, 0), (6, 12, 6, 18, 1), (8, 12, 0, 9, 0)], np.int64)  # row 5 sees nothing
    q, k, v = _rand((nq, Hq, D)), _rand((nq, Hkv, D)), _rand((nq, Hkv, D))
    kc, vc, do = _rand((nc, Hkv, D)), _rand((nc, Hkv, D)), _rand((nq, Hq, D))
    g_q, g_k = RNG.uniform(0.5, 1.5, D), RNG.uniform(0.5, 1.5, D)
    base = (100.0, 50.0, 20.0)
    dq, _, _, _, _, O, lse = oracle.backward(q, k, v, kc, vc, do, videos, sl, Hq, Hkv, base=base,
                                             q_gain=g_q, k_gain=g_k)
    rows = np.asarray([11, 5, 0, 7, 3, 6], np.int64)
    dq_r = oracle.backward_rows(q[rows], rows, k, v, kc, vc, do[rows], videos, sl, Hq, Hkv, base=base,
                                q_gain=g_q, k_gain=g_k)
    assert np.abs(dq_r - dq[rows]).max() <= 1e-12
    assert np.all(dq_r[1] == 0.0)
    pos = oracle.positions(videos)
    kh = oracle.full_keys(oracle.prologue(k, pos, base, 1e-6, g_k), kc)
    qh = oracle.prologue(q[rows], pos[rows], base, 1e-6, g_q)
    _, O_r, lse_r = oracle.attn_bwd_rows(qh, rows, kh, oracle.full_keys(v, vc), do[rows], sl, Hq, Hkv)
    assert np.abs(O_r - O[rows]).max() <= 1e-12
    assert np.array_equal(np.isneginf(lse_r), np.isneginf(lse[rows]))
    fin = np.isfinite(lse_r)
    assert np.abs(lse_r[fin] - lse[rows][fin]).max() <= 1e-12
