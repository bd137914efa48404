"""Pins of the oracle's e4m3 model (the FP8 forward variant), without a GPU.

The e4m3 rounding is pinned against PyTorch's float8_e4m3fn conversion (a library
routine) and against values the format definition fixes; the forward model against
properties of the method: a power-of-two change of V scales O exactly, the model's O
stays within the first-order bound of the operand roundings around the exact O, and
the spread ``sd`` matches a Monte-Carlo of independent P rounding errors."""
import numpy as np
import pytest
import torch

import oracle
from block_causal_attention_b200 import workloads as W


def test_round_e4m3_matches_torch_float8_on_random_values():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(300_000) * np.exp(rng.uniform(-12, 6.5, 300_000))
    x = x[np.abs(x) <= 448].astype(np.float32).astype(np.float64)
    ref = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.round_e4m3(x), ref)


def test_round_e4m3_every_code_and_midpoint():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vals = np.unique(codes[np.isfinite(codes)])
    assert len(vals) == 253 and vals.max() == 448 and vals.min() == -448   # +-0 merge, NaN codes dropped
    assert np.array_equal(oracle.round_e4m3(vals), vals)                    # representable values are fixed
    pos = vals[vals >= 0]
    mids = (pos[:-1] + pos[1:]) / 2
    got = oracle.round_e4m3(mids)
    ref = torch.tensor(mids, dtype=torch.float64).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(got, ref)
    # ties go to the neighbour with an even significand (last bit 0)
    lo_even = (np.searchsorted(pos, got) % 2) == 0
    assert lo_even.all()


def test_round_e4m3_values_fixed_by_the_format():
    x = np.array([448, 464, 1e6, -1e6, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10, 1.0625, 1.1875, 0.0,
                  2.0 ** -6, 1.9375, 232.0, 0.3])
    want = np.array([448, 448, 448, -448, 2.0 ** -9, 0.0, 2.0 ** -8, 1.0, 1.25, 0.0,
                     2.0 ** -6, 2.0, 224.0, 0.3125])
    assert np.array_equal(oracle.round_e4m3(x), want)
    assert np.isnan(oracle.round_e4m3(np.array([np.nan])))[0]


@pytest.mark.parametrize("amax", [448.0, 447.0, 449.0, 1.0, 3.5, 1e-3, 6.0e4, 2.0 ** -20, 0.875, 0.8749])
def test_scale_exponent_brings_max_into_upper_half_of_range(amax):
    e = oracle.e4m3_scale_exponent(amax)
    assert 224.0 <= amax / 2.0 ** e < 448.0
    assert oracle.e4m3_scale_exponent(0.0) == 0


def _small(seed=5, nq=160, nk=160, hq=4, hkv=2, D=48):
    """A two-chunk video problem, block-causal, with random inputs."""
    rng = np.random.default_rng(seed)
    videos = np.array([[2, 2, 8, 5, 0]], np.int32)     # chunks, frames/chunk, h, w, t0 -> 160 tokens
    slices = np.array([[0, 80, 0, 80, 0], [80, 160, 0, 160, 0]], np.int64)
    bf = lambda a: torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)
    q = bf(rng.standard_normal((nq, hq, D)))
    k = bf(rng.standard_normal((nk, hkv, D)))
    v = bf(rng.standard_normal((nk, hkv, D)) * 1.7)
    return q, k, v, videos, slices, hq, hkv


def test_forward_fp8_power_of_two_v_scale_is_exact():
    q, k, v, videos, slices, hq, hkv = _small()
    O1, L1, sd1, f1, _ = oracle.forward_fp8(q, k, v, None, None, videos, slices, hq, hkv)
    O2, L2, sd2, f2, _ = oracle.forward_fp8(q, k, v * 8, None, None, videos, slices, hq, hkv)
    assert np.array_equal(O2, 8 * O1) and np.array_equal(L2, L1) and np.array_equal(sd2, 8 * sd1)


def test_forward_fp8_within_first_order_bound_of_exact():
    """|O_e4m3 - O| <= 2 * (sum_j p_j |ds_j - E_p ds| |v_j - o| + sum_j p_j |dv_j|), the
    first-order effect of the operand roundings (score change ds from rounding Q-hat and
    K-hat, dv from rounding V / 2^e), with 2x for second-order terms."""
    q, k, v, videos, slices, hq, hkv = _small(seed=7)
    O8, L8, _, _, _ = oracle.forward_fp8(q, k, v, None, None, videos, slices, hq, hkv)
    O, L = oracle.forward(q, k, v, None, None, videos, slices, hq, hkv)
    pos = oracle.positions(videos)
    D = q.shape[-1]
    qh = oracle.prologue(q, pos)
    kh = oracle.prologue(k, pos)
    vv = v.double().numpy()
    mask = oracle.mask_dense(slices, q.shape[0], k.shape[0])
    G = hq // hkv
    for h in range(hq):
        g = h // G
        s = np.where(mask, qh[:, h] @ kh[:, g].T / np.sqrt(D), -np.inf)
        p = np.exp(s - L[:, h:h + 1])
        ds = (oracle.round_e4m3(qh[:, h]) @ oracle.round_e4m3(kh[:, g]).T - qh[:, h] @ kh[:, g].T) / np.sqrt(D)
        ds = np.where(mask, ds, 0.0)
        dsc = ds - (p * ds).sum(axis=1, keepdims=True)
        e = oracle.e4m3_scale_exponent(np.abs(vv[:, g]).max())
        dv = oracle.round_e4m3(vv[:, g] / 2.0 ** e) * 2.0 ** e - vv[:, g]
        o = O[:, h]
        bound = np.einsum("ij,ij,ijd->id", p, np.abs(dsc), np.abs(vv[None, :, g] - o[:, None, :])) + p @ np.abs(dv)
        err = np.abs(O8[:, h] - o)
        assert (err <= 2 * bound + 1e-12).all(), (h, (err / (bound + 1e-30)).max())
        assert err.max() > 0.05 * bound.max()          # the model is not the exact result
        assert np.abs(L8[:, h] - L[:, h]).max() <= 2 * np.abs(p * ds).sum(axis=1).max() + 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_forward_fp8_sd_matches_monte_carlo_of_p_rounding(causal):
    """sd is the standard deviation of O under independent relative errors of P drawn
    uniformly from +-2^-4 (the worst-case e4m3 spacing), with O normalised by the
    unrounded row sum as the kernel does: Monte-Carlo over 400 draws.  The causal mask
    gives rows that see 1 to 160 keys, where O is far from 0 and an error model built on
    v - o instead of v would be off."""
    q, k, v, videos, slices, hq, hkv = _small(seed=11, hq=2, hkv=1)
    if causal:
        slices = np.array([[0, 160, 0, 160, 1]], np.int64)
    O8, L8, sd, _, _ = oracle.forward_fp8(q, k, v, None, None, videos, slices, hq, hkv)
    pos = oracle.positions(videos)
    D = q.shape[-1]
    q8 = oracle.round_e4m3(oracle.prologue(q, pos))
    k8 = oracle.round_e4m3(oracle.prologue(k, pos))
    vv = v.double().numpy()[:, 0]
    e = oracle.e4m3_scale_exponent(np.abs(vv).max())
    v8 = oracle.round_e4m3(vv / 2.0 ** e) * 2.0 ** e
    mask = oracle.mask_dense(slices, q.shape[0], k.shape[0])
    rng = np.random.default_rng(0)
    for h in range(hq):
        s = np.where(mask, q8[:, h] @ k8[:, 0].T / np.sqrt(D), -np.inf)
        p = np.exp(s - L8[:, h:h + 1])
        draws = []
        for _ in range(400):
            pe = p * (1 + rng.uniform(-2.0 ** -4, 2.0 ** -4, p.shape))
            draws.append(pe @ v8 / p.sum(axis=1, keepdims=True))   # normalised by the exact sum
        emp = np.std(np.stack(draws), axis=0)
        # the subnormal term of sd is negligible here; the relative term alone is the MC spread
        ratio = (emp / sd[:, h])[:, :][sd[:, h] > 0]
        assert 0.85 < np.median(ratio) < 1.15 and 0.5 < ratio.min() and ratio.max() < 1.6, \
            (np.median(ratio), ratio.min(), ratio.max())


def test_forward_fp8_flip_bound_is_zero_without_undecided_elements():
    q, k, v, videos, slices, hq, hkv = _small(seed=13)
    _, _, _, flip, vdev = oracle.forward_fp8(q, k, v, None, None, videos, slices, hq, hkv)
    pos = oracle.positions(videos)
    uq = oracle._e4m3_undecided(oracle.prologue(q, pos))
    uk = oracle._e4m3_undecided(oracle.prologue(k, pos))
    rows_hit = (uq > 0).any(axis=2)                      # [nq, hq] rows with an undecided Q-hat element
    assert np.all(flip[rows_hit] > 0)
    if not (uk > 0).any():
        assert np.all(flip[~rows_hit] == 0)
    assert (vdev >= 0).all()
