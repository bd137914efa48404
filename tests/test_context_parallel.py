"""Context parallelism: dispatch and local problems (host), the exchange through
torch.distributed with gloo ranks on CPU (attention by the fp64 oracle, injected as the
engine), and the CUDA entry points it uses.  The N > 1 path cannot run on one GPU, so
its collectives are exercised here with gloo."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_b200 import context_parallel as CP
from block_causal_attention_b200 import workloads as W

NAMES = ["tiny", "b45_replica", "packed_replica", "kvrange_replica", "p720_replica"]


def _local_mask(cp, r):
    """The rank's local mask mapped back to global (query token, global key) pairs."""
    lp = cp.local[r]
    nq_l, nc_l = len(lp.tokens), lp.num_cache_keys
    m = oracle.mask_dense(lp.slices, nq_l, nc_l + nq_l)
    key_of = np.concatenate([lp.cache_rows, cp.nc + lp.remote_rows, cp.nc + lp.tokens]).astype(np.int64)
    g = np.zeros((cp.nq, cp.nc + cp.nq), bool)
    qi, kj = np.nonzero(m)
    g[lp.tokens[qi], key_of[kj]] = True
    return g


@pytest.mark.parametrize("name", NAMES)
@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_local_problems_reproduce_the_global_mask(name, world):
    w = W.WORKLOADS[name]
    cp = CP.ContextParallelPlan(world, w.videos_array(), w.num_cache_keys, w.slices_array())
    ref = oracle.mask_dense(w.slices_array(), w.nq, w.nk).astype(bool)
    union = np.zeros_like(ref)
    for r in range(world):
        lm = _local_mask(cp, r)
        assert not (union & lm).any()                        # every query row has one owner
        union |= lm
        assert cp.local[r].area == int(lm.sum())
    assert np.array_equal(union, ref)
    assert sorted(np.concatenate([cp.local[r].tokens for r in range(world)]).tolist()) == list(range(w.nq))


def test_dispatch_balances_area():
    areas = [9, 7, 6, 5, 5, 4, 2, 1]
    ch = [CP.Chunk(i, i + 1, 1, 1, 1, 0) for i in range(len(areas))]
    owner = CP.dispatch(ch, areas, 3)
    load = [sum(a for a, o in zip(areas, owner) if o == r) for r in range(3)]
    assert max(load) - min(load) <= 1 and sum(load) == sum(areas)


def test_causal_piece_equals_the_restricted_slice_by_brute_force():
    """A CAUSAL slice restricted to rows [qa, qb) and keys [a, b) is exactly the union of
    the returned pieces (pair by pair), and the pieces do not overlap."""
    rng = np.random.default_rng(7)
    for _ in range(3000):
        n, m = int(rng.integers(1, 24)), int(rng.integers(1, 24))
        q0 = int(rng.integers(0, n)); q1 = int(rng.integers(q0, n + 1))
        k0 = int(rng.integers(0, m)); k1 = int(rng.integers(k0, m + 1))
        qa = int(rng.integers(0, n)); qb = int(rng.integers(qa, n + 1))
        a = int(rng.integers(0, m)); b = int(rng.integers(a, m + 1))
        want = oracle.mask_dense(np.asarray([[q0, q1, k0, k1, 1]], np.int64), n, m).astype(bool)
        want[:qa] = want[qb:] = False
        want[:, :a] = want[:, b:] = False
        got = np.zeros((n, m), np.int32)
        for piece in CP.causal_piece(q0, q1, k0, k1, qa, qb, a, b):
            got += oracle.mask_dense(np.asarray([piece], np.int64), n, m)
        assert got.max(initial=0) <= 1 and np.array_equal(got.astype(bool), want), (q0, q1, k0, k1, qa, qb, a, b)


def _random_slices(rng, nq, nk, count):
    sl = []
    for _ in range(count):
        q0 = int(rng.integers(0, nq)); q1 = int(rng.integers(q0 + 1, nq + 1))
        k0 = int(rng.integers(0, nk)); k1 = int(rng.integers(k0 + 1, nk + 1))
        sl.append((q0, q1, k0, k1, int(rng.integers(0, 2))))
    return np.asarray(sl, np.int64).reshape(-1, 5)


@pytest.mark.parametrize("seed", range(8))
@pytest.mark.parametrize("world", [1, 2, 3])
def test_local_problems_reproduce_random_full_and_causal_masks(seed, world):
    """Random overlapping FULL and CAUSAL slices over a cache and several chunks: the
    ranks' local masks (and their held / borrowed splits) map back onto the global mask
    exactly, each query row on one rank."""
    rng = np.random.default_rng(100 + seed)
    nchunks, nc = int(rng.integers(2, 6)), int(rng.integers(0, 20))
    vid = np.asarray([[nchunks, 1, 2, 4, 0]], np.int32)          # chunks of 8 tokens
    nq = nchunks * 8
    sl = _random_slices(rng, nq, nc + nq, int(rng.integers(1, 7)))
    cp = CP.ContextParallelPlan(world, vid, nc, sl)
    ref = oracle.mask_dense(sl, nq, nc + nq).astype(bool)
    union = np.zeros_like(ref)
    for r in range(world):
        lm = _local_mask(cp, r)
        assert not (union & lm).any()
        union |= lm
        assert cp.local[r].area == int(lm.sum())
        lp = cp.local[r]
        nql, ncache, nrem = len(lp.tokens), len(lp.cache_rows), len(lp.remote_rows)
        g = np.zeros_like(ref)
        for sls, keys in ((lp.slices_held, np.concatenate([lp.cache_rows, nc + lp.tokens])),
                          (lp.slices_borrowed, np.concatenate([nc + lp.remote_rows, nc + lp.tokens]))):
            m = oracle.mask_dense(sls, nql, len(keys)).astype(bool) if nql else np.zeros((0, len(keys)), bool)
            qi, kj = np.nonzero(m)
            part = np.zeros_like(ref)
            part[lp.tokens[qi], keys[kj].astype(np.int64)] = True
            assert not (g & part).any()                      # held and borrowed do not overlap
            g |= part
        assert np.array_equal(g, lm)
    assert np.array_equal(union, ref)


# --------------------------------------------------------------------------- gloo ranks

class OracleEngine:
    """The attention engine on the fp64 oracle (test infrastructure only).  Its backward
    takes the O and LSE of the whole problem, as the CUDA plan's does, so that a plan over
    a subset of the keys yields that subset's share of the gradients."""

    o_fp32 = True

    def __init__(self, hq, hkv, d, videos, nc, slices, base, eps, o_fp32):
        self.hq, self.hkv, self.d, self.nc = hq, hkv, d, nc
        self.videos, self.slices, self.base, self.eps = np.asarray(videos), np.asarray(slices), base, eps
        self.pos = oracle.positions(self.videos) if len(self.videos) else np.zeros((0, 3), np.int32)

    def k_prologue(self, k, k_gain=None):
        return torch.from_numpy(oracle.prologue(k, self.pos, self.base, self.eps, k_gain))

    def k_prologue_bwd(self, k, dk_hat, k_gain=None, dk=None, accumulate=False):
        g = torch.from_numpy(oracle.prologue_bwd(k, self.pos, dk_hat, self.base, self.eps, k_gain))
        return dk + g if accumulate else g

    def fwd(self, q, k, v, kc, vc, q_gain=None, k_gain=None):
        o, lse = oracle.forward(q, k, v, kc, vc, self.videos, self.slices, self.hq, self.hkv, base=self.base,
                                eps=self.eps, q_gain=q_gain, k_gain=k_gain)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def attn_merge(self, o_a, lse_a, o_b, lse_b):
        la, lb = lse_a.numpy(), lse_b.numpy()
        m = np.maximum(la, lb)
        fin = np.isfinite(m)
        ms = np.where(fin, m, 0.0)
        wa = np.where(np.isfinite(la), np.exp(la - ms), 0.0)
        wb = np.where(np.isfinite(lb), np.exp(lb - ms), 0.0)
        tot = wa + wb
        lse = np.where(fin, ms + np.log(np.where(fin, tot, 1.0)), -np.inf)
        sa, sb = np.where(fin, wa / np.where(fin, tot, 1.0), 0.0), np.where(fin, wb / np.where(fin, tot, 1.0), 0.0)
        o = o_a.numpy() * sa[..., None] + o_b.numpy() * sb[..., None]
        return torch.from_numpy(o), torch.from_numpy(lse)

    def bwd(self, q, k, v, kc, vc, o, lse, do, q_gain=None, k_gain=None, dq=None, dk=None, dv=None,
            dk_cache=None, dv_cache=None, accumulate=False):
        nq, nc = q.shape[0], self.nc
        qh = oracle.prologue(q, self.pos, self.base, self.eps, q_gain)
        kh = oracle.prologue(k, self.pos, self.base, self.eps, k_gain)
        if nc:
            kh = np.concatenate([np.asarray(kc, np.float64), kh])
            vv = np.concatenate([np.asarray(vc, np.float64), np.asarray(v, np.float64)])
        else:
            vv = np.asarray(v, np.float64)
        M = oracle.mask_dense(self.slices, nq, nc + nq).astype(bool)
        O, L, dO = np.asarray(o, np.float64), np.asarray(lse, np.float64), np.asarray(do, np.float64)
        G = self.hq // self.hkv
        dqh, dkh, dvv = np.zeros_like(qh), np.zeros_like(kh), np.zeros_like(vv)
        sc = 1.0 / np.sqrt(self.d)
        for h in range(self.hq):
            g = h // G
            S = qh[:, h] @ kh[:, g].T * sc
            Lh = L[:, h][:, None]
            P = np.where(M & np.isfinite(Lh), np.exp(S - np.where(np.isfinite(Lh), Lh, 0.0)), 0.0)
            dP = dO[:, h] @ vv[:, g].T
            dS = P * (dP - (dO[:, h] * O[:, h]).sum(-1)[:, None])
            dqh[:, h] = dS @ kh[:, g] * sc
            dkh[:, g] += dS.T @ qh[:, h] * sc
            dvv[:, g] += P.T @ dO[:, h]
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        gq = t(oracle.prologue_bwd(q, self.pos, dqh, self.base, self.eps, q_gain))
        gk = t(oracle.prologue_bwd(k, self.pos, dkh[nc:], self.base, self.eps, k_gain))
        out = [gq, gk, t(dvv[nc:]), t(dkh[:nc]) if nc else None, t(dvv[:nc]) if nc else None]
        if accumulate:
            for dst, add in zip((dq, dk, dv, dk_cache, dv_cache), out):
                if dst is not None:
                    dst += add
            return dq, dk, dv, dk_cache, dv_cache
        return tuple(out)


def _small_cached():
    """2 cached chunks + 3 query chunks of 16 tokens (1 x 4 x 4), block-causal over
    (cache + queries): query chunk c sees the cache and query chunks 0..c."""
    from types import SimpleNamespace
    C, nc = 16, 32
    sl = np.asarray([[C * c, C * (c + 1), 0, nc + C * (c + 1), 0] for c in range(3)], np.int64)
    vid = np.asarray([[3, 1, 4, 4, 2]], np.int32)
    return SimpleNamespace(nq=3 * C, nk=nc + 3 * C, hq=4, hkv=2, d=24, num_cache_keys=nc, rope_base=(50.0, 30.0, 20.0),
                           eps=1e-6, videos_array=lambda: vid, slices_array=lambda: sl)


def _small_causal():
    """A cache of 24 keys and 3 query chunks of 16 tokens with overlapping FULL and
    CAUSAL slices, including causal slices with |q| != |k| (bottom-right aligned)."""
    from types import SimpleNamespace
    C, nc = 16, 24
    sl = np.asarray([[0, 48, 0, nc, 0],                  # every query sees the cache
                     [0, 48, nc, nc + 48, 1],            # token-causal over the new tokens
                     [16, 32, nc, nc + 16, 0],           # chunk 1 also sees chunk 0 fully
                     [32, 48, 8, nc + 40, 1],            # |q| = 16, |k| = 56: bottom-right aligned
                     [20, 28, 0, 6, 1]], np.int64)       # |q| = 8 > |k| = 6: early rows see nothing
    vid = np.asarray([[3, 1, 4, 4, 0]], np.int32)
    return SimpleNamespace(nq=3 * C, nk=nc + 3 * C, hq=4, hkv=2, d=24, num_cache_keys=nc, rope_base=(50.0, 30.0, 20.0),
                           eps=1e-6, videos_array=lambda: vid, slices_array=lambda: sl)


def _workload(name):
    if name == "small_cached":
        return _small_cached()
    if name == "small_causal":
        return _small_causal()
    return W.WORKLOADS[name]


def _inputs(w):
    g = torch.Generator().manual_seed(5)
    r = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)
    nc = w.num_cache_keys
    x = {"q": r(w.nq, w.hq, w.d), "k": r(w.nq, w.hkv, w.d), "v": r(w.nq, w.hkv, w.d), "do": r(w.nq, w.hq, w.d),
         "kc": r(nc, w.hkv, w.d) if nc else None, "vc": r(nc, w.hkv, w.d) if nc else None,
         "qg": (0.5 + torch.rand(w.d, generator=g, dtype=torch.float64)),
         "kg": (0.5 + torch.rand(w.d, generator=g, dtype=torch.float64))}
    return x


def _rank_main(rank, world, port, name, out_dir, overlap=False):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _workload(name)
        x = _inputs(w)
        att = CP.ContextParallelAttention(None, rank, world, w.hq, w.hkv, w.d, w.videos_array(), w.num_cache_keys,
                                          w.slices_array(), w.rope_base, w.eps, engine=OracleEngine,
                                          overlap=overlap)
        tok = torch.as_tensor(att.local.tokens, dtype=torch.long)
        ql, kl, vl, dol = (x[n].index_select(0, tok) for n in ("q", "k", "v", "do"))
        o, lse = att.forward(ql, kl, vl, x["kc"], x["vc"], q_gain=x["qg"], k_gain=x["kg"])
        dq, dk, dv, dkc, dvc = att.backward(ql, kl, vl, x["kc"], x["vc"], o, lse, dol, q_gain=x["qg"],
                                            k_gain=x["kg"])
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), tokens=att.local.tokens, o=o.numpy(), lse=lse.numpy(),
                 dq=dq.numpy(), dk=dk.numpy(), dv=dv.numpy(),
                 dkc=np.zeros(0) if dkc is None else dkc.numpy(), dvc=np.zeros(0) if dvc is None else dvc.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("name,world,overlap", [("b45_replica", 2, False), ("packed_replica", 3, False),
                                                ("kvrange_replica", 2, True), ("tiny", 3, True),
                                                ("small_cached", 2, False), ("small_cached", 3, True),
                                                ("small_causal", 1, False), ("small_causal", 2, False),
                                                ("small_causal", 3, True)])
def test_gloo_ranks_match_the_single_process_oracle(name, world, overlap, tmp_path):
    """overlap=True: each rank attends to the keys it holds while the borrowed ones are in
    flight and merges the two partial results by their log-sum-exps."""
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(world, _free_port(), name, str(tmp_path), overlap), nprocs=world,
                       join=True, start_method="spawn")
    w = _workload(name)
    x = _inputs(w)
    ro, rl = oracle.forward(x["q"], x["k"], x["v"], x["kc"], x["vc"], w.videos_array(), w.slices_array(), w.hq,
                            w.hkv, base=w.rope_base, eps=w.eps, q_gain=x["qg"], k_gain=x["kg"])
    rq, rk, rv, rkc, rvc, _, _ = oracle.backward(x["q"], x["k"], x["v"], x["kc"], x["vc"], x["do"],
                                                 w.videos_array(), w.slices_array(), w.hq, w.hkv, base=w.rope_base,
                                                 eps=w.eps, q_gain=x["qg"], k_gain=x["kg"])
    seen = np.zeros(w.nq, bool)
    for r in range(world):
        z = np.load(os.path.join(tmp_path, f"r{r}.npz"))
        t = z["tokens"]
        seen[t] = True
        np.testing.assert_allclose(z["o"], ro[t], atol=1e-10)
        fin = np.isfinite(rl[t])
        assert np.array_equal(np.isfinite(z["lse"]), fin)
        np.testing.assert_allclose(z["lse"][fin], rl[t][fin], atol=1e-10)
        np.testing.assert_allclose(z["dq"], rq[t], atol=1e-10)
        np.testing.assert_allclose(z["dk"], rk[t], atol=1e-10)
        np.testing.assert_allclose(z["dv"], rv[t], atol=1e-10)
        if w.num_cache_keys:
            np.testing.assert_allclose(z["dkc"], rkc, atol=1e-10)
            np.testing.assert_allclose(z["dvc"], rvc, atol=1e-10)
    assert seen.all()
    if name == "small_cached":
        assert np.abs(rkc).max() > 1e-3          # the cache-gradient path carried something


# --------------------------------------------------------------------------- CUDA pieces

@pytest.mark.gpu
@pytest.mark.parametrize("name", ["b45_replica", "p720_replica"])
def test_k_prologue_passes_match_the_oracle(name):
    from block_causal_attention_b200 import Plan
    w = W.WORKLOADS[name]
    p = Plan.from_workload(w)
    k = W.make_input(w, W.T_K, "cuda")
    g = torch.Generator().manual_seed(3)
    kg = (0.5 + torch.rand(w.d, generator=g)).float()
    dkh = torch.randn((w.nq, w.hkv, w.d), generator=g).float()
    kh = p.k_prologue(k, kg.cuda())
    base = torch.randn((w.nq, w.hkv, w.d), generator=g).float()
    dk = p.k_prologue_bwd(k, dkh.cuda(), kg.cuda(), dk=base.clone().cuda(), accumulate=True)
    torch.cuda.synchronize()
    pos = oracle.positions(w.videos_array())
    ref = oracle.prologue(k.cpu(), pos, w.rope_base, w.eps, kg.double().numpy())
    assert np.abs(kh.double().cpu().numpy() - ref).max() <= 2 ** -8 * np.abs(ref).max()   # bf16 rounding
    refd = oracle.prologue_bwd(k.cpu(), pos, dkh.double().numpy(), w.rope_base, w.eps, kg.double().numpy())
    assert np.abs(dk.double().cpu().numpy() - (refd + base.double().numpy())).max() <= 1e-4


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["packed_replica", "kvrange_replica"])
def test_cuda_engine_one_rank_equals_plain_plan(name):
    """With one rank the context-parallel path (own keys through k_prologue, needed cache
    rows gathered, local slices) must give the plain plan's results."""
    from block_causal_attention_b200 import Plan
    w = W.WORKLOADS[name]
    x = W.make_inputs(w, "cuda", with_grad=True)
    att = CP.ContextParallelAttention(None, 0, 1, w.hq, w.hkv, w.d, w.videos_array(), w.num_cache_keys,
                                      w.slices_array(), w.rope_base, w.eps, w.o_fp32)
    o, lse = att.forward(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"])
    dq, dk, dv, dkc, dvc = att.backward(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], o, lse, x["do"])
    p = Plan.from_workload(w)
    o2, l2 = p.fwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"])
    g2 = p.bwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], o2, l2, x["do"])
    torch.cuda.synchronize()
    assert (o.float() - o2.float()).abs().max().item() <= 1e-2
    assert (lse - l2).abs().max().item() <= 1e-3
    for a, b in zip((dq, dk, dv), g2[:3]):
        assert (a - b).abs().max().item() <= 1e-2
    if w.num_cache_keys:
        assert (dkc - g2[3]).abs().max().item() <= 1e-2 and (dvc - g2[4]).abs().max().item() <= 1e-2


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["p720_replica", "packed_replica"])
def test_cuda_split_by_key_location_equals_unsplit(name):
    """Rank 0 of a 2-rank split, on one GPU: the plans over held and borrowed keys, merged
    by their log-sum-exps (bca_attn_merge), and their backwards added into the same arrays
    (accumulate), give the unsplit local plan's O, LSE and gradients."""
    from block_causal_attention_b200 import Plan
    w = W.WORKLOADS[name]
    x = W.make_inputs(w, "cuda", with_grad=True)
    lp = CP.ContextParallelPlan(2, w.videos_array(), w.num_cache_keys, w.slices_array()).local[0]
    assert len(lp.remote_rows) > 0
    mk = lambda nc, sl, f32: Plan(w.hq, w.hkv, w.d, lp.videos, nc, sl, w.rope_base, w.eps, f32)
    full = mk(lp.num_cache_keys, lp.slices, True)
    held = mk(len(lp.cache_rows), lp.slices_held, True)
    bor = mk(len(lp.remote_rows), lp.slices_borrowed, True)
    dev = "cuda"
    tok = torch.as_tensor(lp.tokens, device=dev)
    ql, kl, vl, dol = (x[n].index_select(0, tok) for n in ("q", "k", "v", "do"))
    khat_all = Plan.from_workload(w).k_prologue(x["k"])
    rr = torch.as_tensor(lp.remote_rows, device=dev)
    rk, rv = khat_all.index_select(0, rr), x["v"].index_select(0, rr)
    if len(lp.cache_rows):
        cr = torch.as_tensor(lp.cache_rows, device=dev)
        kch, vch = x["k_cache"].index_select(0, cr), x["v_cache"].index_select(0, cr)
        kcf, vcf = torch.cat([kch, rk]), torch.cat([vch, rv])
    else:
        kch = vch = None
        kcf, vcf = rk, rv
    of, lf = full.fwd(ql, kl, vl, kcf, vcf)
    oh, lh = held.fwd(ql, kl, vl, kch, vch)
    ob, lb = bor.fwd(ql, kl, vl, rk, rv)
    om, lm = held.attn_merge(oh, lh, ob, lb)
    gf = full.bwd(ql, kl, vl, kcf, vcf, of, lf, dol)
    dq, dk, dv, rem_k, rem_v = bor.bwd(ql, kl, vl, rk, rv, om, lm, dol)
    dkc = torch.zeros(kch.shape, dtype=torch.float32, device=dev) if kch is not None else None
    dvc = torch.zeros(vch.shape, dtype=torch.float32, device=dev) if vch is not None else None
    held.bwd(ql, kl, vl, kch, vch, om, lm, dol, dq=dq, dk=dk, dv=dv, dk_cache=dkc, dv_cache=dvc, accumulate=True)
    torch.cuda.synchronize()
    for p in (full, held, bor):
        assert p.status() == 0
    fin = torch.isfinite(lf)
    assert torch.equal(fin, torch.isfinite(lm))
    assert (lm[fin] - lf[fin]).abs().max().item() <= 1e-3
    assert (om - of).abs().max().item() <= 1e-2
    for a, b in ((dq, gf[0]), (dk, gf[1]), (dv, gf[2])):
        assert (a - b).abs().max().item() <= 1e-2
    ncl = len(lp.cache_rows)
    assert (rem_k - gf[3][ncl:]).abs().max().item() <= 1e-2 and (rem_v - gf[4][ncl:]).abs().max().item() <= 1e-2
    if ncl:
        assert (dkc - gf[3][:ncl]).abs().max().item() <= 1e-2 and (dvc - gf[4][:ncl]).abs().max().item() <= 1e-2


def test_exchange_keeps_the_key_and_value_types():
    """K-hat in fp16 (the CUDA engine's cache-key type) and V in bf16 travel together and
    come back with their own types and bits (one rank: the exchange is a local copy)."""
    w = W.WORKLOADS["packed_replica"]

    class Strict:
        """Stands in for the CUDA plan's type checks (no computation)."""
        def __init__(self, *a, **k):
            pass

    att = CP.ContextParallelAttention(None, 0, 1, w.hq, w.hkv, w.d, w.videos_array(), w.num_cache_keys,
                                      w.slices_array(), engine=Strict)
    n = len(att.local.tokens)
    g = torch.Generator().manual_seed(3)
    kh = torch.randn((n, w.hkv, w.d), generator=g).to(torch.float16)
    v = torch.randn((n, w.hkv, w.d), generator=g).to(torch.bfloat16)
    rk, rv = att._gather_keys(kh, v)
    assert rk.dtype == torch.float16 and rv.dtype == torch.bfloat16
    assert rk.is_contiguous() and rv.is_contiguous()
    assert rk.shape[0] == len(att.local.remote_rows) == 0
    # with rows to move: a 2-rank plan's send rows of rank 0, exchanged with itself
    cp = CP.ContextParallelPlan(2, w.videos_array(), w.num_cache_keys, w.slices_array())
    att2 = CP.ContextParallelAttention(None, 1, 2, w.hq, w.hkv, w.d, w.videos_array(), w.num_cache_keys,
                                       w.slices_array(), engine=Strict)
    att2.world = 1                      # emulate the exchange as a local copy of what rank 0 sends
    own = att2.local.tokens
    assert len(cp.send_rows[1][0]) > 0
    att2.send_idx = [np.searchsorted(own, cp.send_rows[1][0])]
    att2.recv_counts = [len(cp.send_rows[1][0])]
    att2.recv_order = np.arange(len(cp.send_rows[1][0]))
    import dataclasses
    att2.local = dataclasses.replace(att2.local, remote_rows=np.asarray(cp.send_rows[1][0]))
    kh2 = torch.randn((len(own), w.hkv, w.d), generator=g).to(torch.float16)
    v2 = torch.randn((len(own), w.hkv, w.d), generator=g).to(torch.bfloat16)
    rk2, rv2 = att2._gather_keys(kh2, v2)
    idx = torch.as_tensor(att2.send_idx[0])
    assert rk2.dtype == torch.float16 and rv2.dtype == torch.bfloat16
    assert torch.equal(rk2.view(torch.int16), kh2.index_select(0, idx).view(torch.int16))
    assert torch.equal(rv2.view(torch.int16), v2.index_select(0, idx).view(torch.int16))
