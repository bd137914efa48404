"""The allocation-free forward, bca_fwd_static_workspace, against bca_fwd.

Some callers cannot allocate device memory on their own (a plug-in inside a host
whose allocator owns all device memory, or a C caller without an allocator), so
they cannot supply bca_fwd's workspace; bca_fwd_static_workspace keeps that scratch
in a fixed device array inside the library instead.  These tests call it through
the C ABI and check, on consecutive calls that share that array, that it gives the
same results as bca_fwd: bit for bit, since both run the same deterministic kernels on
the same inputs (a looser check could hide a scratch offset that shifts results only
slightly).  Plans with bf16 operands and with e4m3 operands (whose scratch also holds
the max|V| words that each call clears) are both covered.  This file is collected last
on purpose."""
import numpy as np
import pytest
import torch

from block_causal_attention_b200 import Plan, _abi
from block_causal_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _ptr(t):
    return None if t is None else t.data_ptr()


def _static_fwd(plan, x, o, lse):
    rc = _abi.lib().bca_fwd_static_workspace(plan._h, _ptr(x["q"]), _ptr(x["k"]), _ptr(x["v"]),
                                             _ptr(x["k_cache"]), _ptr(x["v_cache"]), None, None,
                                             _ptr(o), _ptr(lse), torch.cuda.current_stream().cuda_stream)
    assert rc == _abi.BCA_OK, _abi.error_string(rc)
    torch.cuda.synchronize()
    assert plan.status() == _abi.BCA_OK


def test_static_workspace_matches_bca_fwd_on_consecutive_calls():
    runs = []
    for name, fp8 in (("p720_replica", False), ("b45_replica", False), ("p720_replica", True)):
        w = W.WORKLOADS[name]
        x = W.make_inputs(w, "cuda")
        plan = Plan.from_workload(w, fp8=fp8)
        assert plan.workspace_bytes() <= _abi.BCA_STATIC_WORKSPACE_BYTES
        o_ref, lse_ref = plan.fwd(x["q"], x["k"], x["v"], x["k_cache"], x["v_cache"])
        torch.cuda.synchronize()
        runs.append((plan, x, o_ref, lse_ref))
    # two calls in a row on the same problem, then one on a different problem (other
    # head_dim and key count) that reuses the same static array, two with e4m3 operands,
    # then the first again
    for plan, x, o_ref, lse_ref in (runs[0], runs[0], runs[1], runs[2], runs[2], runs[0]):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        _static_fwd(plan, x, o, lse)
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_static_workspace_rejects_problems_beyond_its_size():
    w = W.WORKLOADS["p720_pipelined"]
    plan = Plan.from_workload(w)
    assert plan.workspace_bytes() > _abi.BCA_STATIC_WORKSPACE_BYTES
    rc = _abi.lib().bca_fwd_static_workspace(plan._h, *([None] * 10))
    assert rc == _abi.BCA_ERR_TOO_LARGE
    assert "static workspace" in _abi.error_string(rc)
