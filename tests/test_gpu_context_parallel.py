"""Context parallelism on the CUDA engine against the fp64 oracle.

Two or three ranks, each a process driving the real CUDA plans (bca_k_prologue, bca_fwd,
bca_bwd_ex with accumulate, bca_attn_merge, bca_k_prologue_bwd) on the same GPU; their
exchanges (the group-cast of post-prologue keys, the group-reduce of key gradients and the
sum of cache gradients; MAGI-1 research notes, "Infra > MagiAttention") run through a gloo
process group on host copies.  No kernel waits on another rank's kernel: ranks meet only in
the host collectives between launches.  The results of all ranks, put together, must match
the single-process fp64 oracle within the tolerances of every other parity test (O, dQ, dK,
dV max-abs 1e-2 and mean-abs 1e-3, LSE max-abs 1e-3).  Borrowed keys travel as bf16 K-hat,
which those tolerances cover.

Also: bca_attn_merge of the oracle's own partial results over two disjoint key subsets
equals the oracle over the union."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_b200 import context_parallel as CP
from block_causal_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3


def _mixed():
    """A KV cache of 96 keys and 3 query chunks of 64 tokens whose slices overlap and mix
    FULL and CAUSAL, including causal slices with |q| != |k| (bottom-right aligned) and rows
    that see few keys."""
    from types import SimpleNamespace
    C, nc = 64, 96
    sl = np.asarray([[0, 192, 0, nc, 0],                 # every query sees the cache
                     [0, 192, nc, nc + 192, 1],          # token-causal over the new tokens
                     [64, 128, nc, nc + 64, 0],          # chunk 1 also sees chunk 0 fully
                     [128, 192, 32, nc + 160, 1],        # |q| = 64, |k| = 224: bottom-right aligned
                     [80, 112, 0, 24, 1]], np.int64)     # |q| = 32 > |k| = 24: early rows see little
    vid = np.asarray([[3, 1, 8, 8, 4]], np.int32)
    return SimpleNamespace(name="mixed", seed_ns=61, nq=3 * C, nk=nc + 3 * C, hq=8, hkv=2, d=48,
                           num_cache_keys=nc, rope_base=(1e4, 1e4, 1e4), eps=1e-6, o_fp32=False,
                           videos_array=lambda: vid, slices_array=lambda: sl)


def _workload(name):
    return _mixed() if name == "mixed" else W.WORKLOADS[name]


def _inputs(w, device):
    def t(tid, shape):
        return W.seeded_normal_bf16(1000 * w.seed_ns + tid, shape, device)
    nc = w.num_cache_keys
    x = {"q": t(W.T_Q, (w.nq, w.hq, w.d)), "k": t(W.T_K, (w.nq, w.hkv, w.d)), "v": t(W.T_V, (w.nq, w.hkv, w.d)),
         "do": t(W.T_DO, (w.nq, w.hq, w.d)),
         "kc": t(W.T_KC, (nc, w.hkv, w.d)) if nc else None, "vc": t(W.T_VC, (nc, w.hkv, w.d)) if nc else None}
    g = torch.Generator().manual_seed(17)
    x["qg"] = (0.5 + torch.rand(w.d, generator=g)).float()
    x["kg"] = (0.5 + torch.rand(w.d, generator=g)).float()
    return x


def _rank_main(rank, world, port, name, out_dir, overlap):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _workload(name)
        x = _inputs(w, "cuda")
        qg, kg = x["qg"].cuda(), x["kg"].cuda()
        att = CP.ContextParallelAttention(None, rank, world, w.hq, w.hkv, w.d, w.videos_array(), w.num_cache_keys,
                                          w.slices_array(), w.rope_base, w.eps, w.o_fp32, overlap=overlap)
        tok = torch.as_tensor(att.local.tokens, dtype=torch.long, device="cuda")
        ql, kl, vl, dol = (x[n].index_select(0, tok) for n in ("q", "k", "v", "do"))
        o, lse = att.forward(ql, kl, vl, x["kc"], x["vc"], q_gain=qg, k_gain=kg)
        dq, dk, dv, dkc, dvc = att.backward(ql, kl, vl, x["kc"], x["vc"], o, lse, dol, q_gain=qg, k_gain=kg)
        torch.cuda.synchronize()
        plans = [att.plan] + ([att.plan_held, att.plan_borrowed] if att.overlap else [])
        status = [p.status() for p in plans]
        f = lambda t: np.zeros(0) if t is None else t.double().cpu().numpy()
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), tokens=att.local.tokens, o=f(o), lse=f(lse), dq=f(dq),
                 dk=f(dk), dv=f(dv), dkc=f(dkc), dvc=f(dvc), status=np.asarray(status),
                 overlap=np.asarray(att.overlap))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _close(name, got, want):
    e = np.abs(got - want)
    assert e.max() <= O_MAX and e.mean() <= O_MEAN, f"{name}: max {e.max():.3e} mean {e.mean():.3e}"


@pytest.mark.parametrize("name,world,overlap", [("mixed", 2, False), ("mixed", 2, True), ("mixed", 3, True),
                                                ("kvrange_replica", 2, True), ("p720_replica", 2, False)])
def test_cuda_context_parallel_ranks_match_the_oracle(name, world, overlap, tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(world, _free_port(), name, str(tmp_path), overlap), nprocs=world,
                       join=True, start_method="spawn")
    w = _workload(name)
    x = _inputs(w, "cpu")
    qg, kg = x["qg"].double().numpy(), x["kg"].double().numpy()
    rq, rk, rv, rkc, rvc, ro, rl = oracle.backward(x["q"], x["k"], x["v"], x["kc"], x["vc"], x["do"],
                                                   w.videos_array(), w.slices_array(), w.hq, w.hkv,
                                                   base=w.rope_base, eps=w.eps, q_gain=qg, k_gain=kg)
    seen = np.zeros(w.nq, bool)
    any_overlap = False
    for r in range(world):
        z = np.load(os.path.join(tmp_path, f"r{r}.npz"))
        assert (z["status"] == 0).all()
        any_overlap |= bool(z["overlap"])
        t = z["tokens"]
        seen[t] = True
        _close("o", z["o"], ro[t])
        fin = np.isfinite(rl[t])
        assert np.array_equal(np.isfinite(z["lse"]).T, fin)
        assert np.abs(z["lse"].T[fin] - rl[t][fin]).max() <= LSE_MAX
        _close("dq", z["dq"], rq[t])
        _close("dk", z["dk"], rk[t])
        _close("dv", z["dv"], rv[t])
        if w.num_cache_keys:
            _close("dk_cache", z["dkc"], rkc)
            _close("dv_cache", z["dvc"], rvc)
    assert seen.all()
    assert any_overlap == overlap          # the split held / borrowed path really ran


def test_attn_merge_of_oracle_parts_equals_the_oracle_over_the_union():
    """bca_attn_merge given the oracle's O and LSE over two disjoint key subsets (fp32)
    returns the oracle's O and LSE over their union; rows that see no key in either part
    get O = 0 and LSE = -inf."""
    from block_causal_attention_b200 import Plan
    w = _mixed()
    x = _inputs(w, "cpu")
    nc = w.num_cache_keys
    sl = w.slices_array()
    # split the key space at an off-tile boundary, keys [0, 150) and [150, nk): each part
    # is written as one FULL slice per (row, run of visible keys) of the oracle's dense mask
    cut = 150
    full_mask = oracle.mask_dense(sl, w.nq, w.nk)
    part_a, part_b = [], []
    for i in range(w.nq):
        cols = np.flatnonzero(full_mask[i])
        for run in np.split(cols, np.flatnonzero(np.diff(cols) != 1) + 1):
            if len(run) == 0:
                continue
            a, b = int(run[0]), int(run[-1]) + 1
            if a < cut:
                part_a.append((i, i + 1, a, min(b, cut), 0))
            if b > cut:
                part_b.append((i, i + 1, max(a, cut), b, 0))
    part_a, part_b = np.asarray(part_a, np.int64), np.asarray(part_b, np.int64)
    ma = oracle.mask_dense(part_a, w.nq, w.nk)
    mb = oracle.mask_dense(part_b, w.nq, w.nk)
    assert not (ma & mb).any() and np.array_equal(ma | mb, oracle.mask_dense(sl, w.nq, w.nk))
    run = lambda s: oracle.forward(x["q"], x["k"], x["v"], x["kc"], x["vc"], w.videos_array(), s, w.hq, w.hkv,
                                   base=w.rope_base, eps=w.eps)
    oa, la = run(part_a)
    ob, lb = run(part_b)
    of, lf = run(sl)
    # rows 5 and 6 are made to see no key in either part (the merge's empty-row case)
    empty = np.asarray([5, 6])
    la[empty], lb[empty] = -np.inf, -np.inf
    oa[empty], ob[empty] = 0.0, 0.0
    lf[empty], of[empty] = -np.inf, 0.0
    p = Plan(w.hq, w.hkv, w.d, w.videos_array(), nc, sl, w.rope_base, w.eps, o_fp32=True)
    dev = lambda a: torch.as_tensor(np.ascontiguousarray(a), dtype=torch.float32, device="cuda")
    om, lm = p.attn_merge(dev(oa), dev(la.T), dev(ob), dev(lb.T))
    torch.cuda.synchronize()
    om, lm = om.double().cpu().numpy(), lm.double().cpu().numpy().T
    fin = np.isfinite(lf)
    assert np.array_equal(np.isfinite(lm), fin)
    assert np.abs(lm[fin] - lf[fin]).max() <= 1e-5           # fp32 arithmetic on fp32 inputs
    assert np.abs(om - of).max() <= 1e-5
    assert (om[empty] == 0).all()
