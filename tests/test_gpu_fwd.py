"""GPU parity of the forward (CUDA path through the C ABI) against the fp64 oracle.

Tolerances (those stated with the method's definition): O max-abs <= 1e-2 and
mean-abs <= 1e-3, LSE max-abs <= 1e-3, on the same seeded bf16 inputs.  Small
workloads are compared element by element over every row and head; full-size ones
on a seeded row sample that always includes every slice edge."""
import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_b200 import Plan, _abi
from block_causal_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3


def _dev_inputs(w):
    return {k: (None if v is None else v.cuda()) for k, v in W.make_inputs(w, "cuda").items()}


def _run(w, x, plan=None):
    plan = plan or Plan.from_workload(w)
    o, lse = plan.fwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"])
    torch.cuda.synchronize()
    assert plan.status() == _abi.BCA_OK
    return o, lse


def _compare(o_gpu, lse_gpu, O_ref, lse_ref, what):
    o = o_gpu.double().cpu().numpy()
    l = lse_gpu.double().cpu().numpy().T  # [Nq, Hq]
    finite = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(l), finite), what
    err_o = np.abs(o - O_ref)
    err_l = np.abs(l[finite] - lse_ref[finite])
    msg = f"{what}: O max {err_o.max():.3e} mean {err_o.mean():.3e}, LSE max {err_l.max(initial=0):.3e}"
    assert err_o.max() <= O_MAX and err_o.mean() <= O_MEAN and err_l.max(initial=0) <= LSE_MAX, msg
    return msg


def _oracle_full(w, x):
    c = {k: (None if v is None else v.cpu()) for k, v in x.items()}
    return oracle.forward(c["q"], c["k"], c["v"], c["k_cache"], c["v_cache"], w.videos_array(),
                          w.slices_array(), w.hq, w.hkv, base=w.rope_base, eps=w.eps)


@pytest.mark.parametrize("name", ["tiny", "b45_replica", "p720_replica", "packed_replica",
                                  "kvrange_replica"])
def test_fwd_parity_full(name):
    w = W.WORKLOADS[name]
    x = _dev_inputs(w)
    o, lse = _run(w, x)
    O_ref, lse_ref = _oracle_full(w, x)
    print(_compare(o, lse, O_ref, lse_ref, name))


@pytest.mark.parametrize("name,nrows", [("b45_infer", 96), ("p720_pipelined", 40),
                                        ("packed_varlen", 48), ("long_kvrange", 24)])
def test_fwd_parity_full_size_sampled(name, nrows):
    """Full-size workloads, in the launch configuration the benchmark times; the
    oracle computes a seeded row sample (all heads) exactly."""
    w = W.WORKLOADS[name]
    x = _dev_inputs(w)
    o, lse = _run(w, x)
    rows = W.sample_rows(w, nrows)
    xc = {k: (None if v is None else v.cpu()) for k, v in x.items() if k != "q"}
    q_rows = W.make_input_rows(w, W.T_Q, rows)
    O_ref, lse_ref = oracle.forward(None, xc["k"], xc["v"], xc["k_cache"], xc["v_cache"], w.videos_array(),
                                    w.slices_array(), w.hq, w.hkv, base=w.rope_base, eps=w.eps,
                                    rows=rows, q_rows=q_rows)
    r = torch.as_tensor(rows, device="cuda")
    print(_compare(o[r], lse[:, r], O_ref, lse_ref, name))


def test_fwd_later_chunks_do_not_change_earlier_outputs():
    for name in ("tiny", "p720_replica"):
        w = W.WORKLOADS[name]
        x = _dev_inputs(w)
        o0, l0 = _run(w, x)
        C = w.videos[0].chunk_tokens
        cut = 2 * C  # new-token index where chunk 2 starts
        y = dict(x)
        y["q"] = x["q"].clone(); y["q"][cut:] = -y["q"][cut:] * 2
        y["k"] = x["k"].clone(); y["k"][cut:] = y["k"][cut:].flip(-1)
        y["v"] = x["v"].clone(); y["v"][cut:] = y["v"][cut:] + 3
        o1, l1 = _run(w, y)
        assert torch.equal(o0[:cut], o1[:cut]) and torch.equal(l0[:, :cut], l1[:, :cut]), name
        assert not torch.equal(o0[cut:], o1[cut:])


def test_fwd_is_deterministic():
    w = W.WORKLOADS["p720_replica"]
    x = _dev_inputs(w)
    p = Plan.from_workload(w)
    o0, l0 = _run(w, x, p)
    o1, l1 = _run(w, x, p)
    assert torch.equal(o0, o1) and torch.equal(l0, l1)


def test_fwd_random_slices_with_empty_rows_and_causal():
    """Overlapping FULL/CAUSAL slices with ragged, off-tile edges and rows that see
    nothing (O = 0, LSE = -inf)."""
    rng = np.random.default_rng(5)
    for trial in range(6):
        nq = int(rng.integers(1, 400))
        nc = int(rng.integers(0, 300))
        nk = nq + nc
        sl = []
        for _ in range(int(rng.integers(0, 7))):
            q0 = int(rng.integers(0, nq)); q1 = int(rng.integers(q0, nq + 1))
            k0 = int(rng.integers(0, nk)); k1 = int(rng.integers(k0, nk + 1))
            sl.append((q0, q1, k0, k1, int(rng.integers(0, 2))))
        sl = np.asarray(sl, np.int64).reshape(-1, 5)
        hq, hkv, d = 4, 2, (24, 32, 48)[trial % 3]
        vids = np.asarray([[1, nq, 1, 1, 3]], np.int32)
        seeds = 7000 + 10 * trial
        q = W.seeded_normal_bf16(seeds, (nq, hq, d), "cuda")
        k = W.seeded_normal_bf16(seeds + 1, (nq, hkv, d), "cuda")
        v = W.seeded_normal_bf16(seeds + 2, (nq, hkv, d), "cuda")
        kc = W.seeded_normal_bf16(seeds + 3, (nc, hkv, d), "cuda") if nc else None
        vc = W.seeded_normal_bf16(seeds + 4, (nc, hkv, d), "cuda") if nc else None
        p = Plan(hq, hkv, d, vids, nc, sl, o_fp32=bool(trial % 2))
        o, lse = p.fwd(q, k, v, kc, vc)
        torch.cuda.synchronize()
        assert p.status() == 0
        O_ref, lse_ref = oracle.forward(q.cpu(), k.cpu(), v.cpu(), None if kc is None else kc.cpu(),
                                        None if vc is None else vc.cpu(), vids, sl, hq, hkv)
        _compare(o, lse, O_ref, lse_ref, f"trial {trial}")


def test_fwd_rejects_misaligned_and_foreign_arguments():
    w = W.WORKLOADS["tiny"]
    x = _dev_inputs(w)
    p = Plan.from_workload(w)
    o = torch.empty((w.nq, w.hq, w.d), device="cuda", dtype=torch.float32)
    lse = torch.empty((w.hq, w.nq), device="cuda", dtype=torch.float32)
    ws = p.alloc_workspace()
    buf = torch.empty(x["q"].numel() + 8, dtype=torch.bfloat16, device="cuda")
    qmis = buf[1:1 + x["q"].numel()]  # 2-byte offset
    L = _abi.lib()
    rc = L.bca_fwd(p._h, qmis.data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), None, None, None, None,
                   o.data_ptr(), lse.data_ptr(), ws.data_ptr(), None)
    assert rc == _abi.BCA_ERR_MISALIGNED
    rc = L.bca_fwd(p._h, x["q"].data_ptr(), None, x["v"].data_ptr(), None, None, None, None,
                   o.data_ptr(), lse.data_ptr(), ws.data_ptr(), None)
    assert rc == _abi.BCA_ERR_INVALID_ARGUMENT
    # a plan with a cache needs the cache tensors
    wc = W.WORKLOADS["p720_replica"]
    pc = Plan.from_workload(wc)
    xc = _dev_inputs(wc)
    with pytest.raises(ValueError):
        pc.fwd(xc["q"], xc["k"], xc["v"], None, None)


def test_fwd_with_qk_norm_gains():
    w = W.WORKLOADS["tiny"]
    x = _dev_inputs(w)
    g = torch.Generator().manual_seed(3)
    qg = (0.5 + torch.rand(w.d, generator=g)).float()
    kg = (0.5 + torch.rand(w.d, generator=g)).float()
    p = Plan.from_workload(w)
    o, lse = p.fwd(x["q"], x["k"], x["v"], q_gain=qg.cuda(), k_gain=kg.cuda())
    torch.cuda.synchronize()
    c = {k: v.cpu() for k, v in x.items() if v is not None}
    O_ref, lse_ref = oracle.forward(c["q"], c["k"], c["v"], None, None, w.videos_array(), w.slices_array(),
                                    w.hq, w.hkv, q_gain=qg.double().numpy(), k_gain=kg.double().numpy())
    _compare(o, lse, O_ref, lse_ref, "gains")
