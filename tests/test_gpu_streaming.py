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


@pytest.mark.gpu
def test_graph_replay_after_videos_move_by_different_amounts():
    """Two packed videos whose start frames move by different amounts, so the span of
    frames they cover shrinks: a forward and a backward with the gain and RoPE-base
    gradients, captured in a CUDA graph before the move and replayed after it, equal a plan
    compiled for the moved videos (the table layout and the first frame used by the base
    gradient are read from device memory, not from the captured launch arguments)."""
    hq, hkv, d = 4, 2, 48
    vids = np.asarray([[2, 2, 4, 6, 0], [2, 2, 4, 6, 10]], np.int32)    # frames 0-3 and 10-13
    moved = np.asarray([[2, 2, 4, 6, 3], [2, 2, 4, 6, 6]], np.int32)    # frames 3-6 and 6-9
    nq = 2 * 2 * 2 * 4 * 6
    x = {"q": W.seeded_normal_bf16(7100, (nq, hq, d), "cuda"),
         "k": W.seeded_normal_bf16(7101, (nq, hkv, d), "cuda"),
         "v": W.seeded_normal_bf16(7102, (nq, hkv, d), "cuda"),
         "do": W.seeded_normal_bf16(7105, (nq, hq, d), "cuda")}
    gen = torch.Generator().manual_seed(71)
    qg = (0.5 + torch.rand(d, generator=gen)).float().cuda()
    kg = (0.5 + torch.rand(d, generator=gen)).float().cuda()
    p = Plan(hq, hkv, d, vids, 0, None)
    wsf = p.alloc_workspace(_abi.BCA_PASS_FWD)
    wsb = p.alloc_workspace(_abi.BCA_PASS_BWD)

    def step(plan, wf, wb):
        o, lse = plan.fwd(x["q"], x["k"], x["v"], q_gain=qg, k_gain=kg, workspace=wf)
        g = plan.bwd(x["q"], x["k"], x["v"], None, None, o, lse, x["do"], q_gain=qg, k_gain=kg, workspace=wb,
                     param_grads=True)
        return (o, lse) + tuple(g)

    step(p, wsf, wsb)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(p, wsf, wsb)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = step(p, wsf, wsb)
    p.update_positions(moved)
    graph.replay()
    torch.cuda.synchronize()
    assert p.status() == _abi.BCA_OK
    fresh = Plan(hq, hkv, d, moved, 0, None)
    ref = step(fresh, fresh.alloc_workspace(_abi.BCA_PASS_FWD), fresh.alloc_workspace(_abi.BCA_PASS_BWD))
    torch.cuda.synchronize()
    names = ("o", "lse", "dq", "dk", "dv", "dk_cache", "dv_cache", "dq_gain", "dk_gain", "drope_base")
    for name, a, b in zip(names, outs, ref):
        if a is None:
            continue
        if name in ("o", "lse", "dk", "dv"):          # fixed reduction order: bit-identical
            assert torch.equal(a, b), name
        else:                                         # sums formed with atomics
            assert (a - b).abs().max().item() <= 1e-5 * max(1.0, b.abs().max().item()), name
    # and the moved plan really differs from the unmoved one
    still = Plan(hq, hkv, d, vids, 0, None)
    o0, _ = still.fwd(x["q"], x["k"], x["v"], q_gain=qg, k_gain=kg)
    torch.cuda.synchronize()
    assert not torch.equal(o0, outs[0])
    del graph


@pytest.mark.gpu
def test_kv_range_stage_schedule_over_a_sliding_window():
    """A stage schedule over a sliding window (KV range 4 normally; range 1 for chunk 10 at
    the two noisiest stages, a shot change, and for chunk 13 at the least noisy stage, a
    detail change): every step's forward on the reused plans matches the oracle, plans are
    compiled once per range layout, and each later step costs only a position update."""
    from block_causal_attention_b200.streaming import PipelinedWindow
    F, H, Wd, win_chunks, cache_chunks = 3, 15, 15, 4, 8
    hq, hkv, d = 32, 2, 48
    C = F * H * Wd
    win = PipelinedWindow(hq, hkv, d, F, H, Wd, win_chunks, cache_chunks, 4)
    win.add_transition(10, stages=(2, 3), kv_range=1)
    win.add_transition(13, stages=(0,), kv_range=1)

    def chunk_rows(seed, chunks, heads):      # seeded rows of absolute chunks (same data in every window)
        return torch.cat([W.seeded_normal_bf16(seed + 97 * c, (C, heads, d), "cuda") for c in chunks])

    host_ms = []
    for first in range(6, 14):
        p = win.plan(first)
        host_ms.append(win.last_host_ms)
        chunks = range(first, first + win_chunks)
        q, k, v = chunk_rows(8100, chunks, hq), chunk_rows(8200, chunks, hkv), chunk_rows(8300, chunks, hkv)
        cached = range(first - cache_chunks, first)
        kc, vc = chunk_rows(8400, cached, hkv), chunk_rows(8500, cached, hkv)
        o, lse = p.fwd(q, k, v, kc, vc)
        torch.cuda.synchronize()
        assert p.status() == _abi.BCA_OK
        ro, rl = oracle.forward(q.cpu(), k.cpu(), v.cpu(), kc.cpu(), vc.cpu(), win.videos(first),
                                win.slices(win.ranges(first)), hq, hkv)
        e = np.abs(o.double().cpu().numpy() - ro)
        assert e.max() <= 1e-2 and e.mean() <= 1e-3, (first, e.max(), e.mean())
        assert np.abs(lse.double().cpu().numpy().T - rl).max() <= 1e-3
    layouts = {win.ranges(f) for f in range(6, 14)}
    assert win.compiles == len(layouts) and len(layouts) > 1
    print("per-step host ms:", [round(x, 2) for x in host_ms], "layouts:", len(layouts))
    win.close()
