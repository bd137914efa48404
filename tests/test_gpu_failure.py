"""Failure detection without a GPU fault: every device-side wait in the forward is
bounded; with BCA_TEST_FORCE_TIMEOUT the K/V loads are withheld (a barrier nothing
completes) and the waits give up after 1 ms, so the kernel records a timeout in the
plan's status word and returns.  The context must stay usable afterwards."""
import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_b200 import Plan, _abi
from block_causal_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _plan(w, **kw):
    return Plan(w.hq, w.hkv, w.d, w.videos_array(), w.num_cache_keys, w.slices_array(), w.rope_base, w.eps,
                w.o_fp32, **kw)


def test_forced_timeout_is_reported_and_context_stays_usable():
    w = W.WORKLOADS["tiny"]
    x = W.make_inputs(w, "cuda")
    bad = _plan(w, test_force_timeout=True)
    bad.fwd(x["q"], x["k"], x["v"])
    torch.cuda.synchronize()
    assert bad.status() == _abi.BCA_ERR_DEVICE_TIMEOUT
    assert bad.status() == _abi.BCA_OK  # reading the status clears it
    good = _plan(w)
    o, lse = good.fwd(x["q"], x["k"], x["v"])
    torch.cuda.synchronize()
    assert good.status() == _abi.BCA_OK
    c = {k: v.cpu() for k, v in x.items() if v is not None}
    O_ref, _ = oracle.forward(c["q"], c["k"], c["v"], None, None, w.videos_array(), w.slices_array(), w.hq, w.hkv)
    assert np.abs(o.double().cpu().numpy() - O_ref).max() < 1e-2


def test_forced_timeout_in_the_backward_is_reported_and_context_stays_usable():
    """The same for the backward kernel: with its tile loads withheld every CTA gives up
    after 1 ms, records the timeout and returns; a normal plan then still computes the
    right gradients."""
    w = W.WORKLOADS["tiny"]
    x = W.make_inputs(w, "cuda", with_grad=True)
    good = _plan(w)
    o, lse = good.fwd(x["q"], x["k"], x["v"])
    bad = _plan(w, test_force_timeout=True)
    bad.bwd(x["q"], x["k"], x["v"], None, None, o, lse, x["do"])
    torch.cuda.synchronize()
    assert bad.status() == _abi.BCA_ERR_DEVICE_TIMEOUT
    assert bad.status() == _abi.BCA_OK
    dq, dk, dv, _, _ = good.bwd(x["q"], x["k"], x["v"], None, None, o, lse, x["do"])
    torch.cuda.synchronize()
    assert good.status() == _abi.BCA_OK
    c = {k: v.cpu() for k, v in x.items() if v is not None}
    rq, rk, rv, _, _, _, _ = oracle.backward(c["q"], c["k"], c["v"], None, None, c["do"], w.videos_array(),
                                             w.slices_array(), w.hq, w.hkv)
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(a.double().cpu().numpy() - b).max() < 1e-2


def test_forced_timeout_in_the_deterministic_dq_pass_is_reported():
    """The deterministic dQ pass waits with the same bounded waits (loads withheld too)."""
    w = W.WORKLOADS["tiny"]
    x = W.make_inputs(w, "cuda", with_grad=True)
    good = _plan(w)
    o, lse = good.fwd(x["q"], x["k"], x["v"])
    bad = _plan(w, test_force_timeout=True, dq_deterministic=True)
    bad.bwd(x["q"], x["k"], x["v"], None, None, o, lse, x["do"])
    torch.cuda.synchronize()
    assert bad.status() == _abi.BCA_ERR_DEVICE_TIMEOUT
    assert bad.status() == _abi.BCA_OK
    good.bwd(x["q"], x["k"], x["v"], None, None, o, lse, x["do"])
    torch.cuda.synchronize()
    assert good.status() == _abi.BCA_OK
