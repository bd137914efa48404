"""Seeded synthetic workloads for block-causal attention.

This module is the one place that both the CUDA path (through the binding) and
the fp64 oracle get their inputs from.  It holds workload *data* only: token
geometry, AttnSlice lists and seeded random tensors.  It holds none of the
method's arithmetic (no masking, no positions, no normalisation, no RoPE, no
softmax); each side derives those from this data on its own.

Workloads follow the shapes the MAGI-1 pages give:

* chunk = 24 raw frames, i.e. 6 latent frames after the VAE's 4x temporal
  compression (MAGI-1 research notes (zhao9797.github.io), "Model architecture
  > Overall pipeline" and "Transformer-based VAE");
* block-causal mask = full attention inside a chunk, causal across chunks, with
  the mask written as a list of AttnSlices (q-range, k-range, full|causal)
  (same page, "Infra > Training infra > MagiAttention > Flex-Flash-Attention");
* GQA with 128 query heads over 8 KV groups; model dims 3072 / 6144 over 128
  heads give head_dim 24 / 48 (same page, "Model specs (Table 2)");
* up to 4 chunks denoised concurrently, attending to a KV cache of earlier
  chunks, and a KV range that limits how many earlier chunks are visible
  (same page, "Inference tricks > KV Cache").

Random inputs are "N(0,1) rounded to bf16", drawn by a counter-based generator
so that any row of any tensor can be produced on its own, on the CPU or on the
GPU, with identical bits: a 32-bit integer hash of (seed, element index)
selects one of 65536 equiprobable normal quantiles, each rounded to bf16.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch

SLICE_FULL = 0
SLICE_CAUSAL = 1

# tensor ids inside a workload's seed namespace
T_Q, T_K, T_V, T_KC, T_VC, T_DO = 0, 1, 2, 3, 4, 5


@dataclasses.dataclass(frozen=True)
class Video:
    """New-token geometry of one (packed) video: chunks x frames x height x width.

    ``t0`` is the latent-frame index of the first new frame, so that new chunks
    that follow cached chunks of the same video continue its time axis.
    """
    num_chunks: int
    frames: int
    height: int
    width: int
    t0: int = 0

    @property
    def chunk_tokens(self) -> int:
        return self.frames * self.height * self.width

    @property
    def tokens(self) -> int:
        return self.num_chunks * self.chunk_tokens


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed_ns: int                 # seed namespace: seed = 1000*seed_ns + tensor id
    hq: int
    hkv: int
    d: int
    videos: tuple
    num_cache_keys: int
    slices: tuple                # tuple of (q0, q1, k0, k1, type)
    rope_base: tuple = (10000.0, 10000.0, 10000.0)
    eps: float = 1e-6
    o_fp32: bool = False
    backward: bool = False
    description: str = ""

    @property
    def nq(self) -> int:
        return sum(v.tokens for v in self.videos)

    @property
    def nk(self) -> int:
        return self.num_cache_keys + self.nq

    def slices_array(self) -> np.ndarray:
        return np.asarray(self.slices, dtype=np.int64).reshape(-1, 5)

    def videos_array(self) -> np.ndarray:
        return np.asarray([[v.num_chunks, v.frames, v.height, v.width, v.t0]
                           for v in self.videos], dtype=np.int32).reshape(-1, 5)

    def visible_pairs(self) -> int:
        """Visible (query, key) pairs per head for slice lists whose slices are
        FULL and pairwise disjoint (true of every workload built here); used only
        for FLOP accounting."""
        tot = 0
        for (q0, q1, k0, k1, t) in self.slices:
            assert t == SLICE_FULL
            tot += (q1 - q0) * (k1 - k0)
        return tot


# ---------------------------------------------------------------------------
# slice-list builders (workload data: which query range sees which key range)
# ---------------------------------------------------------------------------

def block_causal_slices(videos: Sequence[Video], num_cache_keys: int = 0) -> tuple:
    """One FULL slice per chunk: chunk c of a video sees the cache (first video
    only) plus chunks 0..c of its own video.  Videos are packed back to back and
    never see each other."""
    out = []
    qoff = 0
    for vi, v in enumerate(videos):
        C = v.chunk_tokens
        kbase = num_cache_keys + qoff
        for c in range(v.num_chunks):
            q0, q1 = qoff + c * C, qoff + (c + 1) * C
            k0 = 0 if (vi == 0 and num_cache_keys) else kbase
            out.append((q0, q1, k0, kbase + (c + 1) * C, SLICE_FULL))
        qoff += v.tokens
    return tuple(out)


def kv_range_slices(num_chunks: int, C: int, kv_range: int,
                    transitions: Sequence[int], transition_keep: int) -> tuple:
    """Chunk c sees chunks [c-kv_range, c]; a transition chunk sees only chunks
    [0, transition_keep) and itself."""
    out = []
    for c in range(num_chunks):
        q0, q1 = c * C, (c + 1) * C
        if c in transitions:
            out.append((q0, q1, 0, transition_keep * C, SLICE_FULL))
            out.append((q0, q1, c * C, (c + 1) * C, SLICE_FULL))
        else:
            out.append((q0, q1, max(0, c - kv_range) * C, (c + 1) * C, SLICE_FULL))
    return tuple(out)


def _wl(name, seed_ns, hq, hkv, d, videos, cache=0, slices=None, **kw) -> Workload:
    videos = tuple(videos)
    if slices is None:
        slices = block_causal_slices(videos, cache)
    return Workload(name=name, seed_ns=seed_ns, hq=hq, hkv=hkv, d=d, videos=videos,
                    num_cache_keys=cache, slices=tuple(slices), **kw)


def _c3_like(name, seed_ns, frames, h, w, hq, hkv, cache_chunks=8, q_chunks=4, **kw):
    C = frames * h * w
    v = Video(q_chunks, frames, h, w, t0=cache_chunks * frames)
    return _wl(name, seed_ns, hq, hkv, 48, [v], cache=cache_chunks * C, **kw)


def _c5_like(name, seed_ns, nchunks, frames, h, w, hq, hkv, kv_range, transitions, **kw):
    C = frames * h * w
    v = Video(nchunks, frames, h, w)
    return _wl(name, seed_ns, hq, hkv, 48, [v],
               slices=kv_range_slices(nchunks, C, kv_range, transitions, 2), **kw)


WORKLOADS = {
    # 1: tiny, CPU-in-seconds
    "tiny": _wl("tiny", 1, 4, 2, 32, [Video(3, 2, 4, 8)], o_fp32=True, backward=True,
                description="3 chunks x 64 tokens (t=3x2, h=4, w=8), 4/2 heads, D=32"),
    # 2: 4.5B-shaped inference step
    "b45_infer": _wl("b45_infer", 2, 128, 8, 24, [Video(4, 6, 16, 16)],
                     description="4 chunks x 1536 tokens (6x16x16), 128/8 heads, D=24, fwd"),
    # 3: 720p pipelined inference at 24B shape
    "p720_pipelined": _c3_like("p720_pipelined", 3, 6, 45, 80, 128, 8, backward=True,
                               description="4 query chunks x 21600 (6x45x80) + 8 cached "
                                           "chunks, 128/8 heads, D=48"),
    # 4: training-shaped packed varlen
    "packed_varlen": _wl("packed_varlen", 4, 128, 8, 48,
                         [Video(n, 6, 32, 32) for n in (24, 12, 8, 4)], backward=True,
                         description="videos of 24/12/8/4 chunks x 6144 (6x32x32), "
                                     "128/8 heads, D=48"),
    # 5: long context with KV-range control
    "long_kvrange": _c5_like("long_kvrange", 5, 128, 8, 32, 32, 128, 8, 16, (32, 64, 96),
                             backward=True,
                             description="128 chunks x 8192 (8x32x32), KV range 16, "
                                         "transitions at 32/64/96, 128/8 heads, D=48"),
    # scaled replicas of 3-5 (same slice structure, smaller chunks, fewer heads;
    # small enough for full fp64 parity).  G = 16 query heads per KV head is kept.
    "p720_replica": _c3_like("p720_replica", 13, 3, 15, 15, 32, 2, backward=True,
                             description="8 cached + 4 query chunks of 675 (3x15x15)"),
    "packed_replica": _wl("packed_replica", 14, 32, 2, 48,
                          [Video(n, 3, 8, 8) for n in (8, 4, 2, 1)], backward=True,
                          description="videos of 8/4/2/1 chunks x 192 (3x8x8)"),
    "kvrange_replica": _c5_like("kvrange_replica", 15, 40, 1, 8, 8, 16, 1, 16, (12, 24, 36),
                                backward=True,
                                description="40 chunks x 64 (1x8x8), KV range 16, "
                                            "transitions at 12/24/36"),
    # one KV group of the 720p pipelined workload (16 query heads / 1 KV head): the
    # same per-head work and mask at 1/8 of the size, for kernel profiling
    "p720_1group": _c3_like("p720_1group", 3, 6, 45, 80, 16, 1,
                            description="p720_pipelined restricted to one KV group"),
    "b45_replica": _wl("b45_replica", 12, 32, 2, 24, [Video(4, 2, 8, 12)],
                       description="4 chunks x 192 (2x8x12), D=24"),
}

# ---------------------------------------------------------------------------
# counter-based N(0,1)->bf16 generator
# ---------------------------------------------------------------------------

_M32 = 0xFFFFFFFF
_HASH_MUL = 0x45D9F3B          # < 2**31, so (x < 2**32) * mul never overflows int64
_SEED_MUL = 0x2C1B3C6D          # < 2**31
_TABLE_CACHE: dict = {}


def _quantile_table(device) -> torch.Tensor:
    """65536 equiprobable N(0,1) quantiles ((k+0.5)/65536), rounded to bf16."""
    key = str(device)
    t = _TABLE_CACHE.get(key)
    if t is None:
        if "cpu" not in _TABLE_CACHE:
            p = (torch.arange(65536, dtype=torch.float64) + 0.5) / 65536.0
            _TABLE_CACHE["cpu"] = torch.special.ndtri(p).to(torch.bfloat16)
        t = _TABLE_CACHE["cpu"].to(device)
        _TABLE_CACHE[key] = t
    return t


def _mix32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = (x * _HASH_MUL) & _M32
    x = x ^ (x >> 16)
    x = (x * _HASH_MUL) & _M32
    x = x ^ (x >> 16)
    return x


def _normal_bf16_flat(seed: int, start: int, count: int, device) -> torch.Tensor:
    e = torch.arange(start, start + count, dtype=torch.int64, device=device)
    lo = e & _M32
    hi = e >> 32
    key = _mix32(((hi + 1) * _SEED_MUL + seed) & _M32)
    h = _mix32(lo ^ key)
    h = _mix32((h + seed * 0x9E37) & _M32)
    return _quantile_table(device)[h >> 16]


def seeded_normal_bf16(seed: int, shape: Sequence[int], device="cpu",
                       row_start: int = 0, nrows: Optional[int] = None,
                       chunk_elems: int = 1 << 26) -> torch.Tensor:
    """Rows [row_start, row_start+nrows) of a tensor of ``shape`` whose element with
    flat index e is N(0,1)->bf16 drawn from (seed, e).  Any slab of rows is
    bit-identical to the same rows of the whole tensor, on any device."""
    shape = tuple(int(s) for s in shape)
    row_elems = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    if nrows is None:
        nrows = shape[0] - row_start
    total = nrows * row_elems
    out = torch.empty(total, dtype=torch.bfloat16, device=device)
    base = row_start * row_elems
    for s in range(0, total, chunk_elems):
        n = min(chunk_elems, total - s)
        out[s:s + n] = _normal_bf16_flat(seed, base + s, n, device)
    return out.view((nrows,) + shape[1:])


def seeded_rows_bf16(seed: int, shape: Sequence[int], rows, device="cpu", heads=None) -> torch.Tensor:
    """Selected rows (any order) of the same seeded tensor; with ``heads`` = (h0, h1) only
    heads [h0, h1) of a [rows, heads, D] tensor (the same elements as the full rows')."""
    shape = tuple(int(s) for s in shape)
    row_elems = int(np.prod(shape[1:]))
    cols = torch.arange(row_elems, device=device)
    out_shape = shape[1:]
    if heads is not None:
        h0, h1 = int(heads[0]), int(heads[1])
        cols = cols[h0 * shape[2]:h1 * shape[2]]
        out_shape = (h1 - h0,) + shape[2:]
    rows = torch.as_tensor(np.asarray(rows, dtype=np.int64), device=device)
    out = torch.empty((len(rows), len(cols)), dtype=torch.bfloat16, device=device)
    step = max(1, (1 << 24) // max(1, len(cols)))
    for r0 in range(0, len(rows), step):
        e = (rows[r0:r0 + step, None] * row_elems + cols[None, :]).reshape(-1)
        lo = e & _M32
        hi = e >> 32
        key = _mix32(((hi + 1) * _SEED_MUL + seed) & _M32)
        h = _mix32(lo ^ key)
        h = _mix32((h + seed * 0x9E37) & _M32)
        out[r0:r0 + step] = _quantile_table(device)[h >> 16].view(-1, len(cols))
    return out.view((len(rows),) + tuple(out_shape))


def tensor_shape(w: Workload, tid: int) -> tuple:
    if tid == T_Q or tid == T_DO:
        return (w.nq, w.hq, w.d)
    if tid in (T_K, T_V):
        return (w.nq, w.hkv, w.d)
    if tid in (T_KC, T_VC):
        return (w.num_cache_keys, w.hkv, w.d)
    raise ValueError(tid)


def seed_of(w: Workload, tid: int) -> int:
    return 1000 * w.seed_ns + tid


def make_input(w: Workload, tid: int, device="cpu", row_start=0, nrows=None) -> torch.Tensor:
    return seeded_normal_bf16(seed_of(w, tid), tensor_shape(w, tid), device, row_start, nrows)


def make_input_rows(w: Workload, tid: int, rows, device="cpu", heads=None) -> torch.Tensor:
    return seeded_rows_bf16(seed_of(w, tid), tensor_shape(w, tid), rows, device, heads)


def make_inputs(w: Workload, device="cpu", with_grad: bool = False) -> dict:
    d = {
        "q": make_input(w, T_Q, device),
        "k": make_input(w, T_K, device),
        "v": make_input(w, T_V, device),
        "k_cache": make_input(w, T_KC, device) if w.num_cache_keys else None,
        "v_cache": make_input(w, T_VC, device) if w.num_cache_keys else None,
    }
    if with_grad:
        d["do"] = make_input(w, T_DO, device)
    return d


def sample_rows(w: Workload, n: int, seed: int = 7) -> np.ndarray:
    """A seeded sample of query rows that always contains the first and last row
    of every slice's query range (chunk and video edges, transition chunks)."""
    must = set()
    for (q0, q1, k0, k1, t) in w.slices:
        must.update((q0, q1 - 1))
    must = sorted(x for x in must if 0 <= x < w.nq)
    rng = np.random.default_rng(seed)
    extra = max(0, n - len(must))
    rnd = rng.choice(w.nq, size=min(extra, w.nq), replace=False) if extra else []
    return np.unique(np.concatenate([np.asarray(must, np.int64), np.asarray(rnd, np.int64)]))
