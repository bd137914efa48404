"""Out-of-bounds write detection without a fault: every output array and workspace that
the library writes is placed inside a larger device buffer whose guard bands before and
after hold a known byte pattern; after the forward and the backward the guard bands must
be unchanged (a kernel that wrote past an array's end, or before its start, would have
changed them).  Workloads with ragged last tiles, empty rows, caches and partial tiles,
in every plan mode that changes what the kernels write."""
import numpy as np
import pytest
import torch

from block_causal_attention_b200 import Plan, _abi
from block_causal_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side
PATTERN = 0xA5


class Guarded:
    """Tensors carved out of one buffer, each between two guard bands."""

    def __init__(self):
        self.bufs = []

    def empty(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.bufs.append((raw, n))
        return raw[GUARD:GUARD + n].view(dtype).view(shape)

    def check(self):
        torch.cuda.synchronize()
        for raw, n in self.bufs:
            assert (raw[:GUARD] == PATTERN).all().item(), "write before an array's start"
            assert (raw[GUARD + n:] == PATTERN).all().item(), "write past an array's end"


def _run(plan, x, nq, hq, hkv, d, nc, o_fp32, param_grads=False):
    g = Guarded()
    f32 = torch.float32
    o = g.empty((nq, hq, d), f32 if o_fp32 else torch.bfloat16)
    lse = g.empty((hq, nq), f32)
    wsf = g.empty((max(16, plan.workspace_bytes(_abi.BCA_PASS_FWD)),), torch.uint8)
    plan.fwd(x["q"], x["k"], x["v"], x["kc"], x["vc"], o=o, lse=lse, workspace=wsf)
    if plan.fp8:
        g.check()
        assert plan.status() == _abi.BCA_OK
        return
    wsb = g.empty((max(16, plan.workspace_bytes(_abi.BCA_PASS_BWD)),), torch.uint8)
    dq, dk, dv = g.empty((nq, hq, d), f32), g.empty((nq, hkv, d), f32), g.empty((nq, hkv, d), f32)
    dkc = g.empty((nc, hkv, d), f32) if nc else None
    dvc = g.empty((nc, hkv, d), f32) if nc else None
    plan.bwd(x["q"], x["k"], x["v"], x["kc"], x["vc"], o, lse, x["do"], dq=dq, dk=dk, dv=dv, dk_cache=dkc,
             dv_cache=dvc, workspace=wsb, param_grads=param_grads)
    g.check()
    assert plan.status() == _abi.BCA_OK


def _inputs(seed, nq, nc, hq, hkv, d):
    t = lambda k, shape: W.seeded_normal_bf16(seed + k, shape, "cuda")
    return {"q": t(0, (nq, hq, d)), "k": t(1, (nq, hkv, d)), "v": t(2, (nq, hkv, d)), "do": t(5, (nq, hq, d)),
            "kc": t(3, (nc, hkv, d)) if nc else None, "vc": t(4, (nc, hkv, d)) if nc else None}


@pytest.mark.parametrize("name", ["tiny", "b45_replica", "p720_replica", "packed_replica", "kvrange_replica"])
def test_workloads_write_only_their_arrays(name):
    w = W.WORKLOADS[name]
    x = _inputs(8800, w.nq, w.num_cache_keys, w.hq, w.hkv, w.d)
    for kw in ({}, {"dq_deterministic": True}):
        p = Plan(w.hq, w.hkv, w.d, w.videos_array(), w.num_cache_keys, w.slices_array(), w.rope_base, w.eps,
                 w.o_fp32, **kw)
        _run(p, x, w.nq, w.hq, w.hkv, w.d, w.num_cache_keys, w.o_fp32, param_grads=not kw)
    p8 = Plan.from_workload(w, fp8=True)
    _run(p8, x, w.nq, w.hq, w.hkv, w.d, w.num_cache_keys, w.o_fp32)


def test_random_slices_ragged_sizes_write_only_their_arrays():
    rng = np.random.default_rng(21)
    for trial in range(6):
        nq, nc = int(rng.integers(1, 400)), int(rng.integers(0, 300))
        nk = nq + nc
        sl = []
        for _ in range(int(rng.integers(1, 6))):
            q0 = int(rng.integers(0, nq)); q1 = int(rng.integers(q0, nq + 1))
            k0 = int(rng.integers(0, nk)); k1 = int(rng.integers(k0, nk + 1))
            sl.append((q0, q1, k0, k1, int(rng.integers(0, 2))))
        hq, hkv = ((4, 2), (3, 1), (2, 2))[trial % 3]
        d = (24, 32, 48)[trial % 3]
        x = _inputs(8900 + 10 * trial, nq, nc, hq, hkv, d)
        vids = np.asarray([[1, nq, 1, 1, 0]], np.int32)
        p = Plan(hq, hkv, d, vids, nc, np.asarray(sl, np.int64), o_fp32=bool(trial % 2),
                 dq_deterministic=bool(trial % 3 == 0), no_prologue=bool(trial % 2))
        _run(p, x, nq, hq, hkv, d, nc, bool(trial % 2))
