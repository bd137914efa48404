"""GPU parity of the head groupings and plan modes beyond the default 128/8 GQA:

* odd query-head group sizes and MHA (Hkv = Hq), which run one query head per forward
  work item, against the fp64 oracle (forward and backward);
* BCA_NO_PROLOGUE: q and k given post-prologue, compared with the oracle's attention on
  the given operands (no QK-Norm, no RoPE), forward and backward;
* head-parallel sharding (one rank's KV groups and their query heads per plan, run one
  after another on one GPU): the pieces put back together equal the unsharded plan bit for
  bit (O, LSE, dK, dV; dQ, which is summed with atomics, to 1e-5) and match the oracle.

Tolerances: O, dQ, dK, dV max-abs <= 1e-2 and mean-abs <= 1e-3, LSE max-abs <= 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_b200 import BcaError, Plan, _abi
from block_causal_attention_b200 import workloads as W
from block_causal_attention_b200.sharding import shard_heads

pytestmark = pytest.mark.gpu

G_MAX, G_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3


def _err(name, got, want):
    e = np.abs(got.double().cpu().numpy() - want)
    assert e.max() <= G_MAX and e.mean() <= G_MEAN, f"{name}: max {e.max():.3e} mean {e.mean():.3e}"


def _lse_err(got, want):
    l = got.double().cpu().numpy().T
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(l), fin)
    assert np.abs(l[fin] - want[fin]).max(initial=0) <= LSE_MAX


def _problem(seed, hq, hkv, d, C=80, nchunks=3, nc=50):
    """3 chunks of C tokens after a cache of nc keys, block-causal, with a ragged last tile."""
    vids = np.asarray([[nchunks, 1, 8, C // 8, 3]], np.int32)
    nq = nchunks * C
    sl = np.asarray([(c * C, (c + 1) * C, 0, nc + (c + 1) * C, 0) for c in range(nchunks)], np.int64)
    t = lambda k, shape: W.seeded_normal_bf16(seed + k, shape, "cuda")
    x = {"q": t(0, (nq, hq, d)), "k": t(1, (nq, hkv, d)), "v": t(2, (nq, hkv, d)), "do": t(5, (nq, hq, d)),
         "kc": t(3, (nc, hkv, d)), "vc": t(4, (nc, hkv, d))}
    return vids, sl, nc, x


@pytest.mark.parametrize("hq,hkv,d", [(4, 4, 48), (6, 2, 24), (3, 1, 32), (10, 2, 48)])
def test_odd_group_sizes_and_mha_match_the_oracle(hq, hkv, d):
    vids, sl, nc, x = _problem(6000 + hq * 10 + hkv, hq, hkv, d)
    p = Plan(hq, hkv, d, vids, nc, sl)
    assert p.info()["num_items"] == p.info()["num_q_tiles"] * hq // (2 if (hq // hkv) % 2 == 0 else 1)
    o, lse = p.fwd(x["q"], x["k"], x["v"], x["kc"], x["vc"])
    dq, dk, dv, dkc, dvc = p.bwd(x["q"], x["k"], x["v"], x["kc"], x["vc"], o, lse, x["do"])
    torch.cuda.synchronize()
    assert p.status() == _abi.BCA_OK
    c = {k: v.cpu() for k, v in x.items()}
    rq, rk, rv, rkc, rvc, ro, rl = oracle.backward(c["q"], c["k"], c["v"], c["kc"], c["vc"], c["do"], vids, sl,
                                                   hq, hkv)
    _err("o", o, ro)
    _lse_err(lse, rl)
    for name, a, b in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv), ("dk_cache", dkc, rkc), ("dv_cache", dvc, rvc)):
        _err(name, a, b)


@pytest.mark.parametrize("hq,hkv,d,causal", [(8, 2, 48, False), (4, 2, 24, True)])
def test_no_prologue_matches_the_oracle_attention_on_the_given_operands(hq, hkv, d, causal):
    vids, sl, nc, x = _problem(6500 + d, hq, hkv, d)
    if causal:   # token-causal over the new tokens plus the whole cache
        nq = x["q"].shape[0]
        sl = np.asarray([(0, nq, 0, nc, 0), (0, nq, nc, nc + nq, 1)], np.int64)
    p = Plan(hq, hkv, d, vids, nc, sl, no_prologue=True)
    o, lse = p.fwd(x["q"], x["k"], x["v"], x["kc"], x["vc"])
    dq, dk, dv, dkc, dvc = p.bwd(x["q"], x["k"], x["v"], x["kc"], x["vc"], o, lse, x["do"])
    torch.cuda.synchronize()
    assert p.status() == _abi.BCA_OK
    c = {k: v.cpu() for k, v in x.items()}
    kh = oracle.full_keys(c["k"], c["kc"])
    vv = oracle.full_keys(c["v"], c["vc"])
    dqh, dkh, dvv, ro, rl = oracle.attn_bwd_dense(c["q"], kh, vv, c["do"], sl, hq, hkv)
    _err("o", o, ro)
    _lse_err(lse, rl)
    _err("dq", dq, dqh)
    _err("dk", dk, dkh[nc:])
    _err("dv", dv, dvv[nc:])
    _err("dk_cache", dkc, dkh[:nc])
    _err("dv_cache", dvc, dvv[:nc])
    # the prologue's parameters do not exist in this mode
    g = torch.ones(d, device="cuda")
    with pytest.raises(BcaError) as e:
        p.fwd(x["q"], x["k"], x["v"], x["kc"], x["vc"], q_gain=g)
    assert e.value.code == _abi.BCA_ERR_INVALID_ARGUMENT
    with pytest.raises(BcaError) as e:
        p.bwd(x["q"], x["k"], x["v"], x["kc"], x["vc"], o, lse, x["do"], param_grads=True)
    assert e.value.code == _abi.BCA_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("world", [2, 4, 8])
def test_head_parallel_shards_reassemble_to_the_unsharded_plan(world):
    hq, hkv, d = 16, 8, 24
    vids, sl, nc, x = _problem(7000, hq, hkv, d, C=96)
    full = Plan(hq, hkv, d, vids, nc, sl)
    o, lse = full.fwd(x["q"], x["k"], x["v"], x["kc"], x["vc"])
    g = full.bwd(x["q"], x["k"], x["v"], x["kc"], x["vc"], o, lse, x["do"])
    parts = []
    for r in range(world):
        h0, h1, g0, g1 = shard_heads(hq, hkv, r, world)
        xs = {"q": x["q"][:, h0:h1].contiguous(), "do": x["do"][:, h0:h1].contiguous()}
        for n in ("k", "v", "kc", "vc"):
            xs[n] = x[n][:, g0:g1].contiguous()
        p = Plan(h1 - h0, g1 - g0, d, vids, nc, sl)
        os_, ls = p.fwd(xs["q"], xs["k"], xs["v"], xs["kc"], xs["vc"])
        gs = p.bwd(xs["q"], xs["k"], xs["v"], xs["kc"], xs["vc"], os_, ls, xs["do"])
        parts.append(((h0, h1, g0, g1), os_, ls, gs, p))
    torch.cuda.synchronize()
    assert full.status() == _abi.BCA_OK and all(pp[4].status() == _abi.BCA_OK for pp in parts)
    cat = lambda ts, dim: torch.cat(ts, dim)
    o_r = cat([pp[1] for pp in parts], 1)
    l_r = cat([pp[2] for pp in parts], 0)
    assert torch.equal(o_r, o) and torch.equal(l_r, lse)
    for i in (1, 2, 3, 4):          # dk, dv, dk_cache, dv_cache: fixed reduction order
        assert torch.equal(cat([pp[3][i] for pp in parts], 1), g[i]), i
    dq_r = cat([pp[3][0] for pp in parts], 1)
    assert (dq_r - g[0]).abs().max().item() <= 1e-5
    c = {k: v.cpu() for k, v in x.items()}
    rq, rk, rv, rkc, rvc, ro, rl = oracle.backward(c["q"], c["k"], c["v"], c["kc"], c["vc"], c["do"], vids, sl,
                                                   hq, hkv)
    _err("o", o_r, ro)
    _lse_err(l_r, rl)
    _err("dq", dq_r, rq)


def test_fp16_cache_keys_equal_bf16_cache_keys_when_exact():
    """BCA_CACHE_K_FP16: cache keys given as fp16.  The kernels stage K-hat as fp16, so
    bf16 cache keys converted exactly to fp16 give bit-identical results; and
    bca_k_prologue writes the fp16 rounding of the fp32 K-hat (exactly the key images'
    rounding), within one fp16 step of the oracle's prologue."""
    hq, hkv, d = 8, 2, 48
    vids, sl, nc, x = _problem(7500, hq, hkv, d)
    pb = Plan(hq, hkv, d, vids, nc, sl)
    ph = Plan(hq, hkv, d, vids, nc, sl, cache_k_fp16=True)
    kc16 = x["kc"].to(torch.float16)
    assert torch.equal(kc16.to(torch.bfloat16), x["kc"])         # the conversion is exact
    ob, lb = pb.fwd(x["q"], x["k"], x["v"], x["kc"], x["vc"])
    oh, lh = ph.fwd(x["q"], x["k"], x["v"], kc16, x["vc"])
    gb = pb.bwd(x["q"], x["k"], x["v"], x["kc"], x["vc"], ob, lb, x["do"])
    gh = ph.bwd(x["q"], x["k"], x["v"], kc16, x["vc"], oh, lh, x["do"])
    kh = ph.k_prologue(x["k"])
    torch.cuda.synchronize()
    assert pb.status() == _abi.BCA_OK and ph.status() == _abi.BCA_OK
    assert torch.equal(ob, oh) and torch.equal(lb, lh)
    for i in (1, 2, 3, 4):
        assert torch.equal(gb[i], gh[i]), i
    assert (gb[0] - gh[0]).abs().max().item() <= 1e-5
    assert kh.dtype == torch.float16
    pos = oracle.positions(vids)
    ref = oracle.prologue(x["k"].cpu(), pos, (1e4, 1e4, 1e4), 1e-6)
    assert np.abs(kh.double().cpu().numpy() - ref).max() <= 2 ** -11 * np.abs(ref).max()


def test_degenerate_problems():
    """No new tokens (a cache only), rows that see no key at all, and a single token."""
    f32 = torch.float32
    # (1) no new token: the forward launches nothing, the backward zeroes the cache gradients
    hq, hkv, d, nc = 4, 2, 32, 64
    p = Plan(hq, hkv, d, np.zeros((0, 5), np.int32), nc, np.zeros((0, 5), np.int64))
    e = lambda *s: torch.empty(s, dtype=torch.bfloat16, device="cuda")
    kc, vc = W.seeded_normal_bf16(7701, (nc, hkv, d), "cuda"), W.seeded_normal_bf16(7702, (nc, hkv, d), "cuda")
    o, lse = p.fwd(e(0, hq, d), e(0, hkv, d), e(0, hkv, d), kc, vc)
    dkc = torch.full((nc, hkv, d), 7.0, dtype=f32, device="cuda")
    dvc = torch.full((nc, hkv, d), 7.0, dtype=f32, device="cuda")
    p.bwd(e(0, hq, d), e(0, hkv, d), e(0, hkv, d), kc, vc, o, lse, e(0, hq, d), dk_cache=dkc, dv_cache=dvc)
    torch.cuda.synchronize()
    assert p.status() == _abi.BCA_OK and o.numel() == 0
    assert (dkc == 0).all() and (dvc == 0).all()
    # (2) an explicit empty slice list: no row sees a key -> O = 0, LSE = -inf, gradients 0
    vids, _, nc2, x = _problem(7710, 4, 2, 48, C=80)
    p2 = Plan(4, 2, 48, vids, nc2, np.zeros((0, 5), np.int64))
    o2, l2 = p2.fwd(x["q"], x["k"], x["v"], x["kc"], x["vc"])
    g2 = p2.bwd(x["q"], x["k"], x["v"], x["kc"], x["vc"], o2, l2, x["do"])
    torch.cuda.synchronize()
    assert p2.status() == _abi.BCA_OK
    assert (o2 == 0).all() and torch.isneginf(l2).all()
    for t in g2:
        assert (t == 0).all()
    # (3) one token, one key: P = 1 exactly, so O is the token's V row
    p3 = Plan(4, 2, 48, np.asarray([[1, 1, 1, 1, 0]], np.int32), 0, None)
    q3, k3, v3 = (W.seeded_normal_bf16(7720 + i, (1, h, 48), "cuda") for i, h in enumerate((4, 2, 2)))
    o3, l3 = p3.fwd(q3, k3, v3)
    torch.cuda.synchronize()
    assert p3.status() == _abi.BCA_OK
    assert torch.equal(o3, v3.repeat_interleave(2, dim=1))
    ro, rl = oracle.forward(q3.cpu(), k3.cpu(), v3.cpu(), None, None, np.asarray([[1, 1, 1, 1, 0]], np.int32),
                            np.asarray([[0, 1, 0, 1, 0]], np.int64), 4, 2)
    assert np.abs(l3.double().cpu().numpy().T - rl).max() <= 1e-3
