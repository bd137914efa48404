"""Host checks of the seeded input generator and workload definitions."""
import numpy as np
import torch

from block_causal_attention_b200 import workloads as W


def test_generator_slabs_and_rows_match_whole_tensor():
    shape = (300, 4, 24)
    full = W.seeded_normal_bf16(77, shape)
    assert torch.equal(W.seeded_normal_bf16(77, shape, row_start=123, nrows=50), full[123:173])
    rows = [299, 0, 17, 17, 150]
    assert torch.equal(W.seeded_rows_bf16(77, shape, rows), full[rows])
    # chunked generation is identical
    assert torch.equal(W.seeded_normal_bf16(77, shape, chunk_elems=1000), full)


def test_generator_is_standard_normal_ish_and_seed_dependent():
    x = W.seeded_normal_bf16(5, (1 << 20,)).float()
    assert abs(x.mean().item()) < 5e-3 and abs(x.std().item() - 1) < 5e-3
    y = W.seeded_normal_bf16(6, (1 << 20,)).float()
    assert (x != y).float().mean().item() > 0.99


def test_workload_sizes_match_the_stated_configs():
    w = W.WORKLOADS
    assert (w["tiny"].nq, w["tiny"].nk, w["tiny"].hq, w["tiny"].hkv, w["tiny"].d) == (192, 192, 4, 2, 32)
    assert (w["b45_infer"].nq, w["b45_infer"].d) == (6144, 24)
    p = w["p720_pipelined"]
    assert (p.nq, p.nk, p.num_cache_keys) == (86400, 259200, 172800)
    assert p.visible_pairs() == 21600 * 21600 * (9 + 10 + 11 + 12)
    assert w["packed_varlen"].nq == 294912 and len(w["packed_varlen"].slices) == 48
    l5 = w["long_kvrange"]
    assert l5.nq == 1 << 20 and len(l5.slices) == 131
    assert l5.visible_pairs() == 1998 * 8192 * 8192


def test_sample_rows_contains_slice_edges():
    w = W.WORKLOADS["long_kvrange"]
    r = W.sample_rows(w, 400)
    for (q0, q1, *_rest) in w.slices:
        assert q0 in r and (q1 - 1) in r
