"""Host-side tests of the C-ABI library: exported symbols, argument checks, and the
mask compiler against the fp64 oracle's dense mask (bit-exact, each visible pair
covered exactly once).  No GPU needed: plans are built with BCA_PLAN_HOST_ONLY."""
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

import oracle
from block_causal_attention_b200 import Plan, BcaError, _abi
from block_causal_attention_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_causal_attention_b200 import build
    build.build()


def test_library_exports_every_declared_symbol():
    hdr = open(os.path.join(ROOT, "include", "bca.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    declared = set(re.findall(r"\b(bca_[a-z_0-9]+)\s*\(", hdr))
    assert {"bca_plan_create", "bca_fwd", "bca_status"} <= declared
    L = ctypes.CDLL(_abi.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(L, name), name
    assert set(_abi.EXPORTS) == declared


def _plan(w, **kw):
    return Plan.from_workload(w, host_only=True, **kw)


@pytest.mark.parametrize("name", ["tiny", "b45_infer", "b45_replica", "p720_replica",
                                  "packed_replica", "kvrange_replica"])
def test_compiled_mask_equals_oracle_mask(name):
    w = W.WORKLOADS[name]
    p = _plan(w)
    got = p.expand_rows(0, w.nq)
    want = oracle.mask_dense(w.slices_array(), w.nq, w.nk)
    assert got.max() <= 1
    assert np.array_equal(got.astype(bool), want)
    assert p.info()["visible_pairs"] == int(want.sum())


@pytest.mark.parametrize("name", ["tiny", "b45_replica", "p720_replica", "packed_replica",
                                  "kvrange_replica"])
def test_transposed_tables_equal_oracle_mask(name):
    """The backward's per-key-tile runs cover exactly the oracle's mask columns."""
    w = W.WORKLOADS[name]
    p = _plan(w)
    got = p.expand_cols(0, w.nk)
    want = oracle.mask_dense(w.slices_array(), w.nq, w.nk).T
    assert got.max() <= 1
    assert np.array_equal(got.astype(bool), want)


@pytest.mark.parametrize("name", ["p720_pipelined", "packed_varlen", "long_kvrange"])
def test_transposed_tables_full_size_columns(name):
    w = W.WORKLOADS[name]
    p = _plan(w)
    rng = np.random.default_rng(3)
    for j in list(rng.choice(w.nk, 6, replace=False)) + [0, w.nk - 1]:
        got = p.expand_cols(int(j), int(j) + 1)[0]
        assert got.max() <= 1
        assert np.array_equal(got.astype(bool), oracle.mask_col(w.slices_array(), w.nq, int(j))), j


@pytest.mark.parametrize("name", ["p720_pipelined", "packed_varlen", "long_kvrange"])
def test_compiled_mask_full_size_rows(name):
    w = W.WORKLOADS[name]
    p = _plan(w)
    inf = p.info()
    assert inf["visible_pairs"] == w.visible_pairs()
    rows = W.sample_rows(w, 48 if name != "long_kvrange" else 24)
    for r in rows:
        got = p.expand_rows(int(r), int(r) + 1)[0]
        assert got.max() <= 1
        assert np.array_equal(got.astype(bool), oracle.mask_row(w.slices_array(), w.nk, int(r))), r


def test_compiled_mask_random_slices():
    rng = np.random.default_rng(99)
    for trial in range(40):
        nq = int(rng.integers(1, 700))
        nc = int(rng.integers(0, 300))
        nk = nq + nc
        ns = int(rng.integers(0, 9))
        sl = []
        for _ in range(ns):
            q0 = int(rng.integers(0, nq)); q1 = int(rng.integers(q0, nq + 1))
            k0 = int(rng.integers(0, nk)); k1 = int(rng.integers(k0, nk + 1))
            sl.append((q0, q1, k0, k1, int(rng.integers(0, 2))))
        sl = np.asarray(sl, np.int64).reshape(-1, 5)
        p = Plan(4, 2, 32, [[1, nq, 1, 1, 0]], nc, sl, host_only=True)
        got = p.expand_rows(0, nq)
        want = oracle.mask_dense(sl, nq, nk)
        assert got.max(initial=0) <= 1, trial
        assert np.array_equal(got.astype(bool), want), trial
        gotc = p.expand_cols(0, nk)
        assert gotc.max(initial=0) <= 1, trial
        assert np.array_equal(gotc.astype(bool), want.T), trial


def test_default_slices_are_block_causal():
    vids = [[3, 2, 4, 8, 0]]
    p = Plan(4, 2, 32, vids, 0, None, host_only=True)
    want = oracle.mask_dense(W.block_causal_slices([W.Video(3, 2, 4, 8)]), 192, 192)
    assert np.array_equal(p.expand_rows(0, 192).astype(bool), want)


def test_tile_classes_of_720p_pipelined():
    w = W.WORKLOADS["p720_pipelined"]
    inf = _plan(w).info()
    assert (inf["num_q_tiles"], inf["num_k_tiles"]) == (675, 2025)
    tiles = inf["num_full_tiles"] + inf["num_partial_tiles"]
    # every visible pair lies in a compiled tile and partial tiles are rare
    assert inf["num_partial_tiles"] < 0.001 * tiles
    assert inf["num_items"] == 675 * 64  # 2 query heads per item


# ---------------------------------------------------------------- argument checks

def _create(hq=4, hkv=2, d=32, videos=((2, 1, 4, 4, 0),), nc=0, slices=None, flags=_abi.BCA_PLAN_HOST_ONLY,
            base=(1e4, 1e4, 1e4), eps=1e-6):
    prob, keep = _abi.make_problem(hq, hkv, d, videos, nc, slices, base, eps, flags)
    h = ctypes.c_void_p()
    rc = _abi.lib().bca_plan_create(ctypes.byref(prob), ctypes.byref(h))
    if rc == 0:
        _abi.lib().bca_plan_destroy(h)
    else:
        assert not h.value
    return rc


def test_argument_checks_return_codes():
    E = _abi
    assert _create() == E.BCA_OK
    assert _create(hq=6, hkv=4) == E.BCA_ERR_UNSUPPORTED           # Hq % Hkv != 0
    assert _create(hq=6, hkv=2) == E.BCA_OK                        # odd group size: one head per item
    assert _create(hq=4, hkv=4) == E.BCA_OK                        # MHA
    H = E.BCA_PLAN_HOST_ONLY
    assert _create(flags=H | E.BCA_NO_PROLOGUE) == E.BCA_OK
    assert _create(flags=H | E.BCA_NO_PROLOGUE | E.BCA_FWD_FP8_E4M3) == E.BCA_ERR_UNSUPPORTED
    assert _create(flags=H | E.BCA_DQ_DETERMINISTIC) == E.BCA_OK
    assert _create(flags=H | E.BCA_CACHE_K_FP16) == E.BCA_OK
    assert _create(flags=H | E.BCA_CACHE_K_FP16 | E.BCA_FWD_FP8_E4M3) == E.BCA_ERR_UNSUPPORTED
    assert _create(d=64) == E.BCA_ERR_UNSUPPORTED
    assert _create(d=40) == E.BCA_ERR_UNSUPPORTED
    assert _create(hq=0) == E.BCA_ERR_INVALID_ARGUMENT
    assert _create(flags=0x80 | E.BCA_PLAN_HOST_ONLY) == E.BCA_ERR_INVALID_ARGUMENT
    assert _create(base=(1e4, -1.0, 1e4)) == E.BCA_ERR_INVALID_ARGUMENT
    assert _create(eps=float("nan")) == E.BCA_ERR_INVALID_ARGUMENT
    assert _create(videos=((2, 0, 4, 4, 0),)) == E.BCA_ERR_INVALID_ARGUMENT
    assert _create(videos=((2, 1, 300, 4, 0),)) == E.BCA_ERR_UNSUPPORTED
    n = 32
    assert _create(slices=[(0, n, 0, n, 0)]) == E.BCA_OK
    assert _create(slices=[(0, n + 1, 0, n, 0)]) == E.BCA_ERR_BAD_SLICE   # q out of range
    assert _create(slices=[(0, n, 0, n + 1, 0)]) == E.BCA_ERR_BAD_SLICE   # k out of range
    assert _create(slices=[(5, 4, 0, n, 0)]) == E.BCA_ERR_BAD_SLICE       # begin > end
    assert _create(slices=[(-1, 4, 0, n, 0)]) == E.BCA_ERR_BAD_SLICE
    assert _create(slices=[(0, 4, 0, n, 2)]) == E.BCA_ERR_BAD_SLICE       # unknown type
    assert _create(nc=-1) == E.BCA_ERR_INVALID_ARGUMENT
    assert _abi.lib().bca_plan_create(None, None) == E.BCA_ERR_INVALID_ARGUMENT



def test_maximum_sizes_are_refused_before_any_allocation():
    """Token counts past the 31-bit index space, frames past the 8-bit packed positions
    and time positions past int32 are refused by validation (nothing is allocated)."""
    E = _abi
    assert _create(videos=((1, 1, 256, 256, 0),)) == E.BCA_OK                   # largest frame: 65,536 tokens
    assert _create(videos=((1, 1, 4, 257, 0),)) == E.BCA_ERR_UNSUPPORTED        # width > 256
    assert _create(videos=((32768, 1, 256, 256, 0),)) == E.BCA_ERR_UNSUPPORTED  # 2^31 tokens
    assert _create(videos=((16384, 1, 256, 256, 0),) * 2) == E.BCA_ERR_UNSUPPORTED  # 2^30 + 2^30
    assert _create(videos=((2, 1, 4, 4, 2 ** 31 - 2),)) == E.BCA_ERR_UNSUPPORTED    # t past int32
    assert _create(videos=((2, 1, 4, 4, 0),), nc=2 ** 31 - 16) == E.BCA_ERR_UNSUPPORTED  # Nc + Nq = 2^31


def test_host_only_plan_refuses_device_calls():
    p = _plan(W.WORKLOADS["tiny"])
    rc = _abi.lib().bca_fwd(p._h, *([None] * 11))
    assert rc == _abi.BCA_ERR_HOST_ONLY_PLAN
    assert _abi.lib().bca_status(p._h, None) == _abi.BCA_ERR_HOST_ONLY_PLAN
    with pytest.raises(BcaError):
        p.fwd(None, None, None)


def test_empty_problem():
    p = Plan(4, 2, 32, np.zeros((0, 5), np.int32), 0, None, host_only=True)
    inf = p.info()
    assert inf["num_q"] == 0 and inf["num_items"] == 0 and inf["visible_pairs"] == 0


def test_error_strings():
    for c in range(0, -10, -1):
        assert _abi.error_string(c) != "unknown error"
    assert _abi.error_string(-100) == "unknown error"


def test_header_flag_and_error_constants_match_the_binding():
    hdr = open(os.path.join(ROOT, "include", "bca.h")).read()
    # plain numeric defines only (a value followed by a comment or the end of the line)
    defs = dict(re.findall(r"^#define\s+(BCA_[A-Z0-9_]+)\s+\(?(-?(?:0x[0-9a-fA-F]+|\d+))u?\)?\s*(?:/\*.*)?$",
                           hdr, flags=re.M))
    for name, val in defs.items():
        if hasattr(_abi, name):
            assert getattr(_abi, name) == int(val, 0), name
    for name in ("BCA_O_FP32", "BCA_PLAN_HOST_ONLY", "BCA_TEST_FORCE_TIMEOUT", "BCA_FWD_FP8_E4M3",
                 "BCA_ERR_UNSUPPORTED"):
        assert name in defs and hasattr(_abi, name), name


def test_fp8_plan_compiles_on_host_and_refuses_the_backward():
    w = W.WORKLOADS["tiny"]
    p = Plan.from_workload(w, host_only=True, fp8=True)
    assert p.info() == Plan.from_workload(w, host_only=True).info()
    vp = [None] * 18                                      # every tensor pointer NULL
    rc = p._lib.bca_bwd_ex(p._h, *vp, 0, None, None)
    assert rc == _abi.BCA_ERR_UNSUPPORTED


def test_missing_library_fails_loudly():
    """With the native library absent the binding raises instead of falling back: there
    is no CPU path behind Plan."""
    code = ("import block_causal_attention_b200._abi as A, sys\n"
            "A.LIB_PATH = '/nonexistent/libbca.so'\nA._lib = None\n"
            "from block_causal_attention_b200 import Plan, workloads as W\n"
            "try:\n    Plan.from_workload(W.WORKLOADS['tiny'], host_only=True)\n"
            "except ImportError as e:\n    print('raised', e)\n    sys.exit(0)\n"
            "sys.exit(1)\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "raised" in r.stdout, r.stdout + r.stderr


def test_plan_is_a_context_manager_and_close_is_idempotent():
    with Plan.from_workload(W.WORKLOADS["tiny"], host_only=True) as p:
        assert p.info()["num_q"] == 192
    assert not p._h.value                       # destroyed on exit
    p.close()                                   # a second close is a no-op
