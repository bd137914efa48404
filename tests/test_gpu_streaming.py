"""Streaming inference step: a plan reused as the window slides (only the start frames
move) and forward/backward captured in a CUDA graph.

The sliding window (MAGI-1 research notes, "Inference tricks > KV Cache"): every step
the same shapes repeat with later frames, so the compiled mask and work items stay valid
and only the RoPE positions change."""
import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_b200 import BcaError, Plan, _abi
from block_causal_attention_b200 import workloads as W


def _shifted(videos, dt):
    v = np.asarray(videos, np.int32).copy().reshape(-1, 5)
    v[:, 4] += dt
    return v


def _inputs(w, seed_shift=0):
    return W.make_inputs(w, "cuda", with_grad=True)


def test_update_positions_argument_checks_on_host():
    w = W.WORKLOADS["packed_replica"]
    p = Plan.from_workload(w, host_only=True)
    vids = w.videos_array()
    info0 = p.info()
    p.update_positions(_shifted(vids, 3))                 # same geometry, later frames
    assert p.info() == info0                              # tiles and items unchanged
    bad = np.asarray(vids, np.int32).copy().reshape(-1, 5)
    bad[0, 2] += 1                                        # height changed
    with pytest.raises(BcaError) as e:
        p.update_positions(bad)
    assert e.value.code == _abi.BCA_ERR_INVALID_ARGUMENT
    with pytest.raises(BcaError) as e:
        p.update_positions(_shifted(vids, -10_000))       # negative t0
    assert e.value.code == _abi.BCA_ERR_INVALID_ARGUMENT
    with pytest.raises(BcaError) as e:
        p.update_positions(np.asarray(vids, np.int32).reshape(-1, 5)[:-1])   # fewer videos
    assert e.value.code == _abi.BCA_ERR_INVALID_ARGUMENT


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["b45_replica", "kvrange_replica"])
def test_updated_plan_equals_fresh_plan(name):
    """A plan moved by update_positions gives bit-identical O, LSE, dK, dV to a plan
    compiled for the moved videos, and both match the oracle at the new positions."""
    w = W.WORKLOADS[name]
    x = _inputs(w)
    vids = w.videos_array()
    dt = int(np.asarray(vids).reshape(-1, 5)[0, 1]) * 2   # two chunks later
    moved = _shifted(vids, dt)
    pa = Plan.from_workload(w)
    o0, _ = pa.fwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"])
    pa.update_positions(moved)
    pb = Plan(w.hq, w.hkv, w.d, moved, w.num_cache_keys, w.slices_array(), w.rope_base, w.eps, w.o_fp32)
    oa, la = pa.fwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"])
    ob, lb = pb.fwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"])
    ga = pa.bwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], oa, la, x["do"])
    gb = pb.bwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], ob, lb, x["do"])
    torch.cuda.synchronize()
    assert pa.status() == _abi.BCA_OK and pb.status() == _abi.BCA_OK
    assert torch.equal(oa, ob) and torch.equal(la, lb)
    assert not torch.equal(oa, o0)                        # the positions did change
    for i in (1, 2):
        assert torch.equal(ga[i], gb[i])
    assert (ga[0] - gb[0]).abs().max().item() < 1e-5      # dQ: reduction order may vary
    c = {k: (None if t is None else t.cpu()) for k, t in x.items()}
    ro, rl = oracle.forward(c["q"], c["k"], c["v"], c["k_cache"], c["v_cache"], moved, w.slices_array(), w.hq,
                            w.hkv, base=w.rope_base, eps=w.eps)
    e = np.abs(oa.double().cpu().numpy() - ro)
    assert e.max() <= 1e-2 and e.mean() <= 1e-3
    assert np.nanmax(np.abs(np.where(np.isinf(rl), 0, la.cpu().numpy().T - rl))) <= 1e-3


@pytest.mark.gpu
def test_fwd_bwd_in_cuda_graph():
    """Forward and backward of a small first-chunk problem captured once in a CUDA graph
    and replayed: bit-identical to eager launches, also after the window moves."""
    w = W.WORKLOADS["tiny"]
    x = _inputs(w)
    p = Plan.from_workload(w)
    wsf = p.alloc_workspace(_abi.BCA_PASS_FWD)
    wsb = p.alloc_workspace(_abi.BCA_PASS_BWD)
    f32 = torch.float32
    o = torch.empty((w.nq, w.hq, w.d), device="cuda", dtype=f32 if w.o_fp32 else torch.bfloat16)
    lse = torch.empty((w.hq, w.nq), device="cuda", dtype=f32)
    dq = torch.empty((w.nq, w.hq, w.d), device="cuda", dtype=f32)
    dk = torch.empty((w.nq, w.hkv, w.d), device="cuda", dtype=f32)
    dv = torch.empty((w.nq, w.hkv, w.d), device="cuda", dtype=f32)

    def step():
        p.fwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], o=o, lse=lse, workspace=wsf)
        p.bwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"], o, lse, x["do"], dq=dq, dk=dk, dv=dv,
              workspace=wsb)

    step()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (o, lse, dk, dv, dq)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                          # warm-up on the capture stream
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in (o, lse, dk, dv, dq):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert p.status() == _abi.BCA_OK
    for a, b in zip((o, lse, dk, dv), ref[:4]):
        assert torch.equal(a, b)
    assert (dq - ref[4]).abs().max().item() < 1e-5
    # the window moves: the same graph reads the rewritten tables
    moved = _shifted(w.videos_array(), 5)
    p.update_positions(moved)
    g.replay()
    fresh = Plan(w.hq, w.hkv, w.d, moved, w.num_cache_keys, w.slices_array(), w.rope_base, w.eps, w.o_fp32)
    of, lf = fresh.fwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"])
    torch.cuda.synchronize()
    assert torch.equal(o, of) and torch.equal(lse, lf)
    del g
