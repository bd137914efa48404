"""GPU parity of the backward (CUDA path through the C ABI) against the fp64 oracle.

Tolerances: dQ, dK, dV (and the cache gradients) max-abs <= 1e-2 and mean-abs <= 1e-3
on the same seeded bf16 inputs, with the GPU's own forward outputs (O, LSE) fed to its
backward, as a training step does."""
import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_b200 import Plan, _abi
from block_causal_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu

G_MAX, G_MEAN = 1e-2, 1e-3


def _err(name, got, want):
    e = np.abs(got.double().cpu().numpy() - want)
    msg = f"{name}: max {e.max():.3e} mean {e.mean():.3e} (|ref| max {np.abs(want).max():.3e})"
    assert e.max() <= G_MAX and e.mean() <= G_MEAN, msg
    return msg


def _gpu_fwd_bwd(w, x, plan=None, **kw):
    plan = plan or Plan.from_workload(w)
    o, lse = plan.fwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], **kw)
    grads = plan.bwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], o, lse, x["do"], **kw)
    torch.cuda.synchronize()
    assert plan.status() == _abi.BCA_OK
    return grads


@pytest.mark.parametrize("name", ["tiny", "b45_replica", "p720_replica", "packed_replica", "kvrange_replica"])
def test_bwd_parity_full(name):
    w = W.WORKLOADS[name]
    x = W.make_inputs(w, "cuda", with_grad=True)
    dq, dk, dv, dkc, dvc = _gpu_fwd_bwd(w, x)
    c = {k: (None if t is None else t.cpu()) for k, t in x.items()}
    rq, rk, rv, rkc, rvc, _, _ = oracle.backward(c["q"], c["k"], c["v"], c["k_cache"], c["v_cache"], c["do"],
                                                 w.videos_array(), w.slices_array(), w.hq, w.hkv,
                                                 base=w.rope_base, eps=w.eps)
    msgs = [_err("dq", dq, rq), _err("dk", dk, rk), _err("dv", dv, rv)]
    if w.num_cache_keys:
        msgs += [_err("dk_cache", dkc, rkc), _err("dv_cache", dvc, rvc)]
    print(name, "; ".join(msgs))


def test_bwd_dk_dv_are_deterministic():
    w = W.WORKLOADS["p720_replica"]
    x = W.make_inputs(w, "cuda", with_grad=True)
    p = Plan.from_workload(w)
    a = _gpu_fwd_bwd(w, x, p)
    b = _gpu_fwd_bwd(w, x, p)
    for i in (1, 2, 3, 4):
        assert torch.equal(a[i], b[i]), i
    assert (a[0] - b[0]).abs().max().item() < 1e-5  # dq: atomics, order may vary


def test_bwd_with_gains_random_slices_and_empty_rows():
    rng = np.random.default_rng(11)
    for trial in range(4):
        nq = int(rng.integers(1, 300))
        nc = int(rng.integers(0, 200))
        nk = nq + nc
        sl = []
        for _ in range(int(rng.integers(1, 6))):
            q0 = int(rng.integers(0, nq)); q1 = int(rng.integers(q0, nq + 1))
            k0 = int(rng.integers(0, nk)); k1 = int(rng.integers(k0, nk + 1))
            sl.append((q0, q1, k0, k1, int(rng.integers(0, 2))))
        sl = np.asarray(sl, np.int64).reshape(-1, 5)
        hq, hkv, d = 4, 2, (24, 32, 48)[trial % 3]
        vids = np.asarray([[1, nq, 1, 1, 2]], np.int32)
        sd = 9000 + 10 * trial
        x = {"q": W.seeded_normal_bf16(sd, (nq, hq, d), "cuda"),
             "k": W.seeded_normal_bf16(sd + 1, (nq, hkv, d), "cuda"),
             "v": W.seeded_normal_bf16(sd + 2, (nq, hkv, d), "cuda"),
             "k_cache": W.seeded_normal_bf16(sd + 3, (nc, hkv, d), "cuda") if nc else None,
             "v_cache": W.seeded_normal_bf16(sd + 4, (nc, hkv, d), "cuda") if nc else None,
             "do": W.seeded_normal_bf16(sd + 5, (nq, hq, d), "cuda")}
        gen = torch.Generator().manual_seed(sd)
        qg = (0.5 + torch.rand(d, generator=gen)).float()
        kg = (0.5 + torch.rand(d, generator=gen)).float()
        p = Plan(hq, hkv, d, vids, nc, sl, o_fp32=bool(trial % 2))
        dq, dk, dv, dkc, dvc = _gpu_fwd_bwd(None, x, p, q_gain=qg.cuda(), k_gain=kg.cuda())
        c = {k: (None if t is None else t.cpu()) for k, t in x.items()}
        rq, rk, rv, rkc, rvc, _, _ = oracle.backward(c["q"], c["k"], c["v"], c["k_cache"], c["v_cache"], c["do"],
                                                     vids, sl, hq, hkv, q_gain=qg.double().numpy(),
                                                     k_gain=kg.double().numpy())
        _err("dq", dq, rq); _err("dk", dk, rk); _err("dv", dv, rv)
        if nc:
            _err("dk_cache", dkc, rkc); _err("dv_cache", dvc, rvc)


@pytest.mark.parametrize("name", ["tiny", "b45_replica", "p720_replica", "kvrange_replica"])
def test_bwd_parameter_gradients(name):
    """Gradients of the QK-Norm gains and the RoPE bases (bca_bwd_ex) against the oracle.
    They are sums over every row and head, so they are compared relative to the largest
    reference entry: max-abs error <= 1e-2 x max|ref| (the per-element dQ / dK tolerance
    of 1e-2 relative to |dq| ~ 1 carried over to the sums); the ordinary gradients of the
    same call must still meet their own tolerances."""
    w = W.WORKLOADS[name]
    x = W.make_inputs(w, "cuda", with_grad=True)
    gen = torch.Generator().manual_seed(77)
    qg = (0.5 + torch.rand(w.d, generator=gen)).float()
    kg = (0.5 + torch.rand(w.d, generator=gen)).float()
    p = Plan.from_workload(w)
    o, lse = p.fwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], q_gain=qg.cuda(), k_gain=kg.cuda())
    out = p.bwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], o, lse, x["do"], q_gain=qg.cuda(),
                k_gain=kg.cuda(), param_grads=True)
    torch.cuda.synchronize()
    assert p.status() == _abi.BCA_OK
    c = {k: (None if t is None else t.cpu()) for k, t in x.items()}
    ref = oracle.backward(c["q"], c["k"], c["v"], c["k_cache"], c["v_cache"], c["do"], w.videos_array(),
                          w.slices_array(), w.hq, w.hkv, base=w.rope_base, eps=w.eps, q_gain=qg.double().numpy(),
                          k_gain=kg.double().numpy(), param_grads=True)
    _err("dq", out[0], ref[0]); _err("dk", out[1], ref[1]); _err("dv", out[2], ref[2])
    msgs = []
    for nm, got, want in (("dq_gain", out[5], ref[7]), ("dk_gain", out[6], ref[8]), ("drope_base", out[7], ref[9])):
        e = np.abs(got.double().cpu().numpy() - want).max()
        scale = np.abs(want).max()
        msgs.append(f"{nm}: max err {e:.3e} of max|ref| {scale:.3e}")
        assert e <= 1e-2 * scale, msgs[-1]
    print(name, "; ".join(msgs))


@pytest.mark.parametrize("name", ["tiny", "b45_replica"])
def test_bwd_large_upstream_gradient(name):
    """dO scaled by 2^12 (exact in bf16) pushes the bound 2 max|dO| max|v| on |dS| past
    fp16's safe range, so the kernel applies a power-of-two scale to dS (and to P, through
    the shifted LSE) and undoes it on dQ, dK, dV.  Gradients are linear in dO, so they
    must equal 2^12 times the oracle's for the unscaled dO."""
    w = W.WORKLOADS[name]
    x = W.make_inputs(w, "cuda", with_grad=True)
    x["do"] = x["do"] * 4096.0
    dq, dk, dv, dkc, dvc = _gpu_fwd_bwd(w, x)
    c = {k: (None if t is None else t.cpu()) for k, t in x.items()}
    c["do"] = c["do"] / 4096.0
    rq, rk, rv, rkc, rvc, _, _ = oracle.backward(c["q"], c["k"], c["v"], c["k_cache"], c["v_cache"], c["do"],
                                                 w.videos_array(), w.slices_array(), w.hq, w.hkv,
                                                 base=w.rope_base, eps=w.eps)
    _err("dq", dq / 4096.0, rq); _err("dk", dk / 4096.0, rk); _err("dv", dv / 4096.0, rv)
    if w.num_cache_keys:
        _err("dk_cache", dkc / 4096.0, rkc); _err("dv_cache", dvc / 4096.0, rvc)


@pytest.mark.parametrize("name,nrows", [("p720_pipelined", 24), ("packed_varlen", 24), ("long_kvrange", 12)])
def test_bwd_full_size_sampled_rows_and_key_rows(name, nrows):
    """Full-size workloads in the benchmark's launch configuration:
    * dK and dV (and dK_cache, dV_cache) of seeded key rows of one KV group, element by
      element, against the fp64 oracle's values stored in tests/golden/key_grads_<name>.npz
      (written by tests/golden/make_key_grads.py from the oracle alone; the keys include
      chunk edges, cache keys and keys that transition chunks see);
    * dq on a seeded row sample computed exactly by the oracle;
    * per KV group, sum_j dV_j equals the sum of dO over the group's heads (rows of P sum
      to one), an extra whole-tensor check."""
    import os
    w = W.WORKLOADS[name]
    x = W.make_inputs(w, "cuda", with_grad=True)
    dq, dk, dv, dkc, dvc = _gpu_fwd_bwd(w, x)
    gold = np.load(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", f"key_grads_{name}.npz"))
    keys, g, nc = gold["keys"], int(gold["group"]), w.num_cache_keys
    new, old = keys >= nc, keys < nc
    assert new.any()
    kn = torch.as_tensor(keys[new] - nc, device="cuda")
    print(name, _err("dk key rows", dk[kn, g], gold["dk"][new].astype(np.float64)),
          _err("dv key rows", dv[kn, g], gold["dv"][new].astype(np.float64)))
    if old.any():
        ko = torch.as_tensor(keys[old], device="cuda")
        print(name, _err("dk_cache key rows", dkc[ko, g], gold["dk"][old].astype(np.float64)),
              _err("dv_cache key rows", dvc[ko, g], gold["dv"][old].astype(np.float64)))
    rows = W.sample_rows(w, nrows)
    xc = {k: (None if t is None else t.cpu()) for k, t in x.items() if k in ("k", "v", "k_cache", "v_cache")}
    rq = oracle.backward_rows(W.make_input_rows(w, W.T_Q, rows), rows, xc["k"], xc["v"], xc["k_cache"],
                              xc["v_cache"], W.make_input_rows(w, W.T_DO, rows), w.videos_array(),
                              w.slices_array(), w.hq, w.hkv, base=w.rope_base, eps=w.eps)
    r = torch.as_tensor(rows, device="cuda")
    print(name, _err("dq rows", dq[r], rq))
    G = w.hq // w.hkv
    sdv = dv.double().sum(0) + (dvc.double().sum(0) if dvc is not None else 0)   # [Hkv, D]
    sdo = x["do"].double().view(w.nq, w.hkv, G, w.d).sum((0, 2))                # [Hkv, D]
    rel = ((sdv - sdo).abs().max() / sdo.abs().max()).item()
    # P enters dV rounded to bf16 (relative 2^-9 per element), so the identity holds to
    # about that precision, not to fp32 rounding
    assert rel < 1e-2, rel


@pytest.mark.parametrize("name,groups", [("b45_infer", (0, 5))])
def test_bwd_full_size_sampled_key_rows(name, groups):
    """Full size, in the benchmark's launch configuration: dK (w.r.t. the raw keys) and dV
    of seeded key rows of the last two chunks, for two KV groups, computed exactly by the
    oracle from only the query rows that see those keys (tests/packed_keys.py)."""
    import sys, os
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from packed_keys import video_key_grads, video_span
    w = W.WORKLOADS[name]
    x = W.make_inputs(w, "cuda", with_grad=True)
    dq, dk, dv, dkc, dvc = _gpu_fwd_bwd(w, x)
    start, C, nch = video_span(w, 0)
    keys = np.sort(np.random.default_rng(11).choice(np.arange((nch - 2) * C, nch * C), 96, replace=False))
    kr = torch.as_tensor(start + keys, device="cuda")
    for g in groups:
        rk, rv = video_key_grads(w, 0, g, keys)
        print(name, g, _err("dk rows", dk[kr, g], rk), _err("dv rows", dv[kr, g], rv))


@pytest.mark.parametrize("name", ["tiny", "p720_replica", "kvrange_replica", "b45_replica"])
def test_bwd_deterministic_dq_pass(name):
    """BCA_DQ_DETERMINISTIC: dQ from the separate fixed-order pass is bit-identical over
    two runs, matches the oracle, and agrees with the reduce-add path to fp32 rounding;
    dK and dV are the same as without the flag, bit for bit."""
    w = W.WORKLOADS[name]
    x = W.make_inputs(w, "cuda", with_grad=True)
    pd = Plan(w.hq, w.hkv, w.d, w.videos_array(), w.num_cache_keys, w.slices_array(), w.rope_base, w.eps, w.o_fp32,
              dq_deterministic=True)
    a = _gpu_fwd_bwd(w, x, pd)
    b = _gpu_fwd_bwd(w, x, pd)
    for i in range(5):
        if a[i] is not None:
            assert torch.equal(a[i], b[i]), i
    ref = _gpu_fwd_bwd(w, x, Plan.from_workload(w))
    for i in (1, 2, 3, 4):
        if a[i] is not None:
            assert torch.equal(a[i], ref[i]), i
    assert (a[0] - ref[0]).abs().max().item() <= 1e-5
    c = {k: (None if t is None else t.cpu()) for k, t in x.items()}
    rq, _, _, _, _, _, _ = oracle.backward(c["q"], c["k"], c["v"], c["k_cache"], c["v_cache"], c["do"],
                                           w.videos_array(), w.slices_array(), w.hq, w.hkv, base=w.rope_base,
                                           eps=w.eps)
    print(name, _err("dq (deterministic pass)", a[0], rq))
