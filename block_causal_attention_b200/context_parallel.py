"""Context parallelism: one block-causal attention problem spread over the ranks of a
process group, by query chunk.

The route of the pages (MAGI-1 research notes, "Infra > MagiAttention": the dispatch
solver balances the unmasked area per rank, then key/value chunks are group-cast to the
ranks whose queries see them and the gradients are group-reduced back; the Interview's
answer on the dispatch solver gives the same cost model):

1. dispatch: every chunk of every video goes to one rank, longest-first onto the least
   loaded rank, where a chunk's load is its number of visible (query, key) pairs;
2. each rank builds a local problem: its chunks are the new tokens (one single-chunk
   video each, at the chunk's frames), the keys it needs from other ranks' tokens and
   from the global cache become its cache (post-prologue keys), and every FULL slice is
   cut into pieces that map contiguous global key ranges onto contiguous local ones;
3. forward: each rank computes the post-prologue keys of its own tokens
   (``k_prologue``) and one all-to-all-v sends the rows each other rank needs;
4. backward: the local backward returns gradients for the borrowed rows as cache
   gradients; a second all-to-all-v sends them to the owners, which add them (K through
   ``k_prologue_bwd``); gradients of the global cache are summed over ranks.

Every rank derives the whole dispatch from the same inputs, so no metadata is exchanged.
CAUSAL slices (bottom-right aligned) are cut too: a causal slice restricted to a key
sub-range [a, b) is exactly one CAUSAL band (the rows whose diagonal ends inside the
range, with the band's own bottom-right corner on the diagonal) plus one FULL band (the
rows that see all of [a, b)), and both forms survive the shift to local indices.
The attention engine is pluggable: the default is this package's CUDA ``Plan``.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional, Sequence

import numpy as np

SLICE_FULL = 0
SLICE_CAUSAL = 1


@dataclasses.dataclass(frozen=True)
class Chunk:
    """One chunk of one video: new tokens [start, end) in the global token order."""
    start: int
    end: int
    frames: int
    height: int
    width: int
    t0: int  # first frame of the chunk


def chunks_of(videos) -> List[Chunk]:
    out = []
    n = 0
    for nc, f, h, w, t0 in np.asarray(videos, np.int64).reshape(-1, 5):
        size = int(f * h * w)
        for c in range(int(nc)):
            out.append(Chunk(n, n + size, int(f), int(h), int(w), int(t0 + c * f)))
            n += size
    return out


def _merge(iv):
    iv = sorted(iv)
    out = []
    for a, b in iv:
        if a >= b:
            continue
        if out and a <= out[-1][1]:
            out[-1][1] = max(out[-1][1], b)
        else:
            out.append([a, b])
    return [(a, b) for a, b in out]


def causal_piece(q0: int, q1: int, k0: int, k1: int, qa: int, qb: int, a: int, b: int):
    """The pairs of the CAUSAL slice (q0, q1, k0, k1) with rows in [qa, qb) and keys in
    [a, b), as at most one CAUSAL and one FULL slice (same coordinates).

    Bottom-right alignment: row i sees keys j in [k0, k1) with j - k0 <= (i - q0) +
    (k1 - k0) - (q1 - q0), i.e. j < e(i) = i + k1 - q1 + 1.  Restricted to keys [lo, hi):
    rows with e(i) <= lo see nothing, rows with e(i) >= hi see all of [lo, hi) (FULL),
    and the rows between see [lo, e(i)): a CAUSAL slice whose bottom-right corner is
    (last row, e(last row) - 1), so its own alignment gives the same e(i)."""
    r0, r1 = max(q0, qa), min(q1, qb)
    lo, hi = max(k0, a), min(k1, b)
    if r0 >= r1 or lo >= hi:
        return []
    c = k1 - q1 + 1                               # e(i) = i + c
    r_start = max(r0, lo - c + 1)                 # first row that sees a key of [lo, hi)
    if r_start >= r1:
        return []
    r_full = min(r1, max(r_start, hi - c))        # first row that sees all of [lo, hi)
    out = []
    if r_start < r_full:
        out.append((r_start, r_full, lo, r_full - 1 + c, SLICE_CAUSAL))
    if r_full < r1:
        out.append((r_full, r1, lo, hi, SLICE_FULL))
    return out


def _causal_of(slices, chunk: Chunk):
    """The CAUSAL slices that reach the chunk's rows, as (q0, q1, k0, k1)."""
    sl = np.asarray(slices, np.int64).reshape(-1, 5)
    return [tuple(int(x) for x in r[:4]) for r in sl
            if r[4] == SLICE_CAUSAL and max(int(r[0]), chunk.start) < min(int(r[1]), chunk.end)
            and r[2] < r[3]]


def chunk_rows(slices, chunk: Chunk, nc: int):
    """Row groups of a chunk with the merged key intervals of its FULL slices: a list of
    (q_begin, q_end, [(k_begin, k_end), ...]) in global query / key indices.  CAUSAL
    slices are taken separately (``_causal_of``)."""
    sl = np.asarray(slices, np.int64).reshape(-1, 5)
    cuts = {chunk.start, chunk.end}
    mine = []
    for q0, q1, k0, k1, t in sl:
        if t != SLICE_FULL:
            continue
        a, b = max(int(q0), chunk.start), min(int(q1), chunk.end)
        if a < b and k0 < k1:
            mine.append((a, b, int(k0), int(k1)))
            cuts.update((a, b))
    cuts = sorted(cuts)
    groups = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        iv = _merge([(k0, k1) for (s0, s1, k0, k1) in mine if s0 <= a and b <= s1])
        if iv:
            groups.append((a, b, iv))
    return groups


def _row_intervals(groups, causal, chunk: Chunk):
    """Per row of the chunk, the merged visible key intervals of its FULL row groups and
    its CAUSAL slices (used only when the chunk has CAUSAL slices)."""
    per = [[] for _ in range(chunk.end - chunk.start)]
    for a, b, iv in groups:
        for i in range(a, b):
            per[i - chunk.start].extend(iv)
    for q0, q1, k0, k1 in causal:
        c = k1 - q1 + 1
        for i in range(max(q0, chunk.start), min(q1, chunk.end)):
            e = min(k1, i + c)
            if e > k0:
                per[i - chunk.start].append((k0, e))
    return [_merge(x) for x in per]


def chunk_area(slices, chunk: Chunk, nc: int) -> int:
    """Visible (query, key) pairs of the chunk's rows (the union over all slices)."""
    groups = chunk_rows(slices, chunk, nc)
    causal = _causal_of(slices, chunk)
    if not causal:
        return sum((b - a) * sum(k1 - k0 for k0, k1 in iv) for a, b, iv in groups)
    return sum(k1 - k0 for row in _row_intervals(groups, causal, chunk) for k0, k1 in row)


def dispatch(chunks: Sequence[Chunk], areas: Sequence[int], world: int) -> List[int]:
    """Owner rank of each chunk: longest first onto the least loaded rank (ties: the
    lower rank), so every rank computes the same answer."""
    order = sorted(range(len(chunks)), key=lambda i: (-areas[i], i))
    load = [0] * world
    owner = [0] * len(chunks)
    for i in order:
        r = min(range(world), key=lambda x: (load[x], x))
        owner[i] = r
        load[r] += areas[i]
    return owner


@dataclasses.dataclass
class LocalProblem:
    rank: int
    chunks: List[int]            # indices of this rank's chunks, in global order
    tokens: np.ndarray           # global token index of each local new token
    videos: np.ndarray           # [n_chunks, 5] single-chunk videos
    cache_rows: np.ndarray       # global cache rows needed, sorted
    remote_rows: np.ndarray      # global token indices of borrowed keys, sorted
    slices: np.ndarray           # [m, 5] local slices (FULL and CAUSAL)
    area: int
    slices_held: np.ndarray      # the slices restricted to keys held locally: keys [cache rows | own]
    slices_borrowed: np.ndarray  # restricted to borrowed keys: keys [borrowed rows | own (unused)]

    @property
    def num_cache_keys(self) -> int:
        return len(self.cache_rows) + len(self.remote_rows)


class ContextParallelPlan:
    """The dispatch and the local problem of every rank, computed identically on all."""

    def __init__(self, world: int, videos, num_cache_keys: int, slices):
        self.world = int(world)
        self.nc = int(num_cache_keys)
        self.chunks = chunks_of(videos)
        self.nq = self.chunks[-1].end if self.chunks else 0
        self.rows = [chunk_rows(slices, c, self.nc) for c in self.chunks]
        self.causal = [_causal_of(slices, c) for c in self.chunks]
        self.areas = [self._area(i) for i in range(len(self.chunks))]
        self.owner = dispatch(self.chunks, self.areas, self.world)
        self.token_owner = np.zeros(self.nq, np.int64)
        for c, r in zip(self.chunks, self.owner):
            self.token_owner[c.start:c.end] = r
        self.local = [self._local(r) for r in range(self.world)]
        # exchange plan: rows[src][dst] = global tokens src sends to dst (in dst's order)
        self.send_rows = [[np.zeros(0, np.int64) for _ in range(self.world)] for _ in range(self.world)]
        for dst in range(self.world):
            rr = self.local[dst].remote_rows
            own = self.token_owner[rr] if len(rr) else np.zeros(0, np.int64)
            for src in range(self.world):
                self.send_rows[src][dst] = rr[own == src]

    def _area(self, i: int) -> int:
        """Visible pairs of chunk i's rows: the union of its FULL row groups and CAUSAL
        slices (per row only when the chunk has CAUSAL slices)."""
        if not self.causal[i]:
            return sum((b - a) * sum(k1 - k0 for k0, k1 in iv) for a, b, iv in self.rows[i])
        return sum(k1 - k0 for row in _row_intervals(self.rows[i], self.causal[i], self.chunks[i])
                   for k0, k1 in row)

    def _local(self, r: int) -> LocalProblem:
        mine = [i for i, o in enumerate(self.owner) if o == r]
        spans = [(self.chunks[i].start, self.chunks[i].end) for i in mine]
        tokens = np.concatenate([np.arange(a, b) for a, b in spans]) if mine else np.zeros(0, np.int64)
        first_local = np.cumsum([0] + [b - a for a, b in spans])
        videos = np.asarray([[1, self.chunks[i].frames, self.chunks[i].height, self.chunks[i].width,
                              self.chunks[i].t0] for i in mine], np.int32).reshape(-1, 5)
        nk = self.nc + self.nq
        own = np.zeros(nk, bool)
        own[self.nc + tokens] = True
        need = np.zeros(nk, bool)
        for i in mine:
            for a, b, iv in self.rows[i]:
                for k0, k1 in iv:
                    need[k0:k1] = True
            c = self.chunks[i]
            for q0, q1, k0, k1 in self.causal[i]:   # rows see [k0, e(i)), e growing with i
                need[k0:min(k1, min(q1, c.end) - 1 + k1 - q1 + 1)] = True
        need &= ~own
        cache_rows = np.flatnonzero(need[:self.nc]).astype(np.int64)
        remote_rows = np.flatnonzero(need[self.nc:]).astype(np.int64)
        nc_loc = len(cache_rows) + len(remote_rows)
        # global key -> local key: needed cache rows, then borrowed tokens, then own tokens
        lk = np.full(nk, -1, np.int64)
        lk[cache_rows] = np.arange(len(cache_rows))
        lk[self.nc + remote_rows] = len(cache_rows) + np.arange(len(remote_rows))
        lk[self.nc + tokens] = nc_loc + np.arange(len(tokens))
        def runs(k0, k1):
            """Maximal runs of global keys [k0, k1) whose local index advances by one:
            (global start, global end, local start)."""
            seg = lk[k0:k1]
            cuts = np.flatnonzero(np.diff(seg) != 1) + 1
            starts = np.concatenate([[0], cuts])
            ends = np.concatenate([cuts, [k1 - k0]])
            return [(k0 + int(s0), k0 + int(s1), int(seg[s0])) for s0, s1 in zip(starts, ends)]

        out = []
        area = 0
        for ci, i in enumerate(mine):
            c = self.chunks[i]
            dq = first_local[ci] - c.start                # global row -> local row
            area += self.areas[i]
            for a, b, iv in self.rows[i]:
                for k0, k1 in iv:
                    for ga, gb, la in runs(k0, k1):
                        out.append((a + dq, b + dq, la, la + gb - ga, SLICE_FULL))
            for q0, q1, k0, k1 in self.causal[i]:
                e_last = min(k1, min(q1, c.end) - 1 + k1 - q1 + 1)
                if e_last <= k0:
                    continue
                for ga, gb, la in runs(k0, e_last):
                    for ra, rb, ka, kb, t in causal_piece(q0, q1, k0, k1, c.start, c.end, ga, gb):
                        out.append((ra + dq, rb + dq, ka - ga + la, kb - ga + la, t))
        sl = np.asarray(out, np.int64).reshape(-1, 5)
        # split at the region boundaries: [0, ncache) cache, [ncache, nc_loc) borrowed, own
        ncache, nrem = len(cache_rows), len(remote_rows)
        held, borrowed = [], []
        for qa, qb, k0, k1, t in out:
            for lo, hi, dst, shift in ((0, ncache, held, 0), (ncache, nc_loc, borrowed, -ncache),
                                       (nc_loc, nc_loc + len(tokens), held, -nrem)):
                if t == SLICE_FULL:
                    a0, a1 = max(k0, lo), min(k1, hi)
                    if a0 < a1:
                        dst.append((qa, qb, a0 + shift, a1 + shift, t))
                else:
                    for ra, rb, ka, kb, tt in causal_piece(qa, qb, k0, k1, qa, qb, lo, hi):
                        dst.append((ra, rb, ka + shift, kb + shift, tt))
        sh = np.asarray(held, np.int64).reshape(-1, 5)
        sb = np.asarray(borrowed, np.int64).reshape(-1, 5)
        return LocalProblem(r, mine, tokens, videos, cache_rows, remote_rows, sl, area, sh, sb)


# ----------------------------------------------------------------------------- runtime

def _default_engine(hq, hkv, d, videos, num_cache_keys, slices, rope_base, eps, o_fp32):
    """CUDA plans whose cache keys (the global cache's and the borrowed ones) are fp16:
    the owner's K-hat reaches the kernels with the same fp16 rounding as a key of the
    plan's own tokens, instead of passing through bf16 on the way."""
    from . import Plan
    return Plan(hq, hkv, d, videos, num_cache_keys, slices, rope_base, eps, o_fp32, cache_k_fp16=True)


def _host_staged(group, t) -> bool:
    """True when the collectives of `group` cannot take `t` where it lives: device tensors
    on a gloo group (gloo moves host memory) go through host copies."""
    import torch.distributed as dist
    return t.is_cuda and dist.get_backend(group) == "gloo"


def _all_to_all_rows(group, send: List, recv_counts: List[int], row_shape, like, async_op: bool = False):
    """Rows of `send[dst]` go to rank dst; returns the received rows per source rank (and,
    with async_op, the pending work to wait on before reading them).  Rows are moved
    bit-exactly: 16-bit rows (an even count of elements per row) travel as 32-bit words,
    a type every backend has (gloo and NCCL have no 16-bit integer type)."""
    import torch
    import torch.distributed as dist
    world = len(send)
    width = int(np.prod(row_shape))
    flat = [s.reshape(-1, width) for s in send]
    sbuf = torch.cat(flat, 0) if flat else like.new_zeros((0, width))
    rbuf = like.new_empty((sum(recv_counts), width))
    pack = sbuf.element_size() == 2 and width % 2 == 0
    sview = sbuf.view(torch.int32) if pack else sbuf
    rview = rbuf.view(torch.int32) if pack else rbuf
    work = None
    if world == 1:
        rview.copy_(sview)
    elif _host_staged(group, sview):
        rhost = torch.empty(rview.shape, dtype=rview.dtype)
        dist.all_to_all_single(rhost, sview.cpu(), output_split_sizes=list(recv_counts),
                               input_split_sizes=[int(f.shape[0]) for f in flat], group=group)
        rview.copy_(rhost)
    else:
        work = dist.all_to_all_single(rview, sview, output_split_sizes=list(recv_counts),
                                      input_split_sizes=[int(f.shape[0]) for f in flat], group=group,
                                      async_op=async_op)
    out, o = [], 0
    for c in recv_counts:
        out.append(rbuf[o:o + c].reshape((c,) + tuple(row_shape)))
        o += c
    return (out, work) if async_op else out


class ContextParallelAttention:
    """One rank's part of a context-parallel attention problem.  `q_local`, `k_local`,
    `v_local`, `do_local` hold this rank's tokens (``local.tokens``); the cache is given
    whole on every rank (post-prologue keys and values)."""

    def __init__(self, group, rank: int, world: int, hq: int, hkv: int, d: int, videos, num_cache_keys: int,
                 slices, rope_base=(1e4, 1e4, 1e4), eps: float = 1e-6, o_fp32: bool = False,
                 engine: Optional[Callable] = None, overlap: bool = False):
        """overlap=True: attend to the keys held locally while the borrowed ones are in
        flight, then to the borrowed ones, and merge the two partial results by their
        log-sum-exps (plans with fp32 O for the parts); the backward runs the borrowed part
        first so that its gradients travel while the held part computes."""
        self.group, self.rank, self.world = group, int(rank), int(world)
        self.hq, self.hkv, self.d = hq, hkv, d
        self.cp = ContextParallelPlan(world, videos, num_cache_keys, slices)
        self.local = self.cp.local[self.rank]
        eng = engine or _default_engine
        lp = self.local
        self.plan = eng(hq, hkv, d, lp.videos, lp.num_cache_keys, lp.slices, rope_base, eps, o_fp32)
        self.overlap = bool(overlap) and len(lp.remote_rows) > 0
        if self.overlap:
            self.plan_held = eng(hq, hkv, d, lp.videos, len(lp.cache_rows), lp.slices_held, rope_base, eps, True)
            self.plan_borrowed = eng(hq, hkv, d, lp.videos, len(lp.remote_rows), lp.slices_borrowed, rope_base, eps,
                                     True)
        self._saved = None
        self._index_maps()
        self._dev_idx = {}

    def _index_maps(self):
        """Row indices of the exchanges, fixed by the dispatch (``local.tokens`` and
        ``local.remote_rows`` are sorted, so every lookup is a binary search):
        - send_idx[dst]: rows of this rank's tokens that dst borrows (its K-hat / V);
        - recv_order: for each borrowed row, in remote_rows order, its place in the
          concatenated receive buffer (sources in rank order, each in global order);
        - ret_send_idx[dst]: rows of remote_rows that belong to dst (their gradients);
        - ret_recv_idx[src]: rows of this rank's tokens that src returns gradients for."""
        cp, r, lp = self.cp, self.rank, self.local
        tok, rr = lp.tokens.astype(np.int64), lp.remote_rows.astype(np.int64)
        self.send_idx = [np.searchsorted(tok, cp.send_rows[r][dst]) for dst in range(self.world)]
        self.recv_counts = [len(cp.send_rows[src][r]) for src in range(self.world)]
        own = cp.token_owner[rr] if len(rr) else np.zeros(0, np.int64)
        offs = np.cumsum([0] + self.recv_counts)
        j = np.zeros(len(rr), np.int64)
        for src in range(self.world):
            m = own == src
            j[m] = np.arange(int(m.sum()))
        self.recv_order = (offs[own] + j) if len(rr) else np.zeros(0, np.int64)
        self.ret_send_idx = [np.searchsorted(rr, cp.send_rows[dst][r]) for dst in range(self.world)]
        self.ret_recv_idx = [np.searchsorted(tok, cp.send_rows[r][src]) for src in range(self.world)]

    def _idx(self, name, arr, device):
        """The index array as a torch tensor on the device (made once per device)."""
        import torch
        key = (name, str(device))
        t = self._dev_idx.get(key)
        if t is None:
            t = torch.as_tensor(arr, dtype=torch.long, device=device)
            self._dev_idx[key] = t
        return t

    def _gather_keys(self, khat_local, v_local):
        return self._gather_keys_finish(self._gather_keys_start(khat_local, v_local))

    def _gather_keys_start(self, khat_local, v_local):
        """Send the rows of [K-hat | V] of this rank's tokens that the other ranks need;
        returns a handle for _gather_keys_finish (the receive may still be in flight).
        K-hat (fp16 for the CUDA engine) and V (bf16) travel together as 16-bit words."""
        import torch
        self._kv_types = (khat_local.dtype, v_local.dtype)
        if khat_local.dtype != v_local.dtype and khat_local.element_size() == v_local.element_size() == 2:
            khat_local, v_local = khat_local.view(torch.int16), v_local.view(torch.int16)
        kv = torch.stack([khat_local, v_local], 1)                      # [n, 2, Hkv, D]
        send = [kv.index_select(0, self._idx(("send", dst), self.send_idx[dst], kv.device))
                for dst in range(self.world)]
        recv_counts = self.recv_counts
        return _all_to_all_rows(self.group, send, recv_counts, kv.shape[1:], kv, async_op=True), recv_counts, kv

    def _gather_keys_finish(self, handle):
        """The borrowed rows, in the order of local.remote_rows."""
        import torch
        (got, work), recv_counts, kv = handle
        if work is not None:
            work.wait()
        # reorder to local.remote_rows: each source sent its subset in global order
        if len(self.local.remote_rows):
            cat = torch.cat(got, 0)
            rem = cat.index_select(0, self._idx("recv", self.recv_order, kv.device))
        else:
            rem = kv.new_zeros((0,) + tuple(kv.shape[1:]))
        kt, vt = self._kv_types
        rk, rv = rem[:, 0].contiguous(), rem[:, 1].contiguous()
        if rk.dtype != kt:
            rk, rv = rk.view(kt), rv.view(vt)
        return rk, rv

    def _cache_grads(self, dkc, dvc, ncl, like):
        """Gradients of the global cache: this rank's rows scattered, summed over ranks."""
        import torch
        import torch.distributed as dist
        if not self.cp.nc:
            return None, None
        gk = like.new_zeros((self.cp.nc, self.hkv, self.d))
        gv = like.new_zeros((self.cp.nc, self.hkv, self.d))
        if ncl:
            rows = torch.as_tensor(self.local.cache_rows, dtype=torch.long, device=like.device)
            gk.index_add_(0, rows, dkc[:ncl])
            gv.index_add_(0, rows, dvc[:ncl])
        if self.world > 1:
            for t in (gk, gv):
                if _host_staged(self.group, t):
                    h = t.cpu()
                    dist.all_reduce(h, group=self.group)
                    t.copy_(h)
                else:
                    dist.all_reduce(t, group=self.group)
        return gk, gv

    def _return_grads_start(self, rem_k, rem_v):
        """Send the borrowed rows' (dK-hat, dV) back to their owners (in flight on return)."""
        import torch
        cp, r = self.cp, self.rank
        grads = torch.stack([rem_k, rem_v], 1)                             # [n_remote, 2, Hkv, D]
        send = [grads.index_select(0, self._idx(("ret_send", dst), self.ret_send_idx[dst], grads.device))
                for dst in range(self.world)]
        recv_counts = [len(cp.send_rows[r][src]) for src in range(self.world)]
        return _all_to_all_rows(self.group, send, recv_counts, grads.shape[1:], grads, async_op=True)

    def _return_grads_finish(self, handle, k_local, dk, dv, k_gain):
        """Add what the other ranks returned for this rank's keys (dK through the prologue)."""
        import torch
        got, work = handle
        if work is not None:
            work.wait()
        dkh = dk.new_zeros(dk.shape)
        for src in range(self.world):
            if len(self.ret_recv_idx[src]):
                idx = self._idx(("ret_recv", src), self.ret_recv_idx[src], dk.device)
                dkh.index_add_(0, idx, got[src][:, 0])
                dv.index_add_(0, idx, got[src][:, 1])
        dk = self.plan.k_prologue_bwd(k_local, dkh, k_gain, dk=dk, accumulate=True)
        return dk, dv

    def _local_cache(self, k_cache, v_cache, rk, rv):
        """Cache rows of the local problem: the global cache rows it needs, then the
        borrowed rows; keys in the type of this rank's K-hat (the engine's cache type)."""
        import torch
        rows = torch.as_tensor(self.local.cache_rows, dtype=torch.long, device=rk.device)
        if len(self.local.cache_rows):
            kc, vc = k_cache.index_select(0, rows).to(rk.dtype), v_cache.index_select(0, rows)
            return torch.cat([kc, rk], 0), torch.cat([vc, rv], 0)
        return rk, rv

    def _held_cache(self, k_cache, v_cache, key_dtype):
        import torch
        if not len(self.local.cache_rows):
            return None, None
        rows = torch.as_tensor(self.local.cache_rows, dtype=torch.long, device=k_cache.device)
        return k_cache.index_select(0, rows).to(key_dtype), v_cache.index_select(0, rows)

    def forward(self, q_local, k_local, v_local, k_cache=None, v_cache=None, q_gain=None, k_gain=None):
        khat = self.plan.k_prologue(k_local, k_gain)
        if self.overlap:
            handle = self._gather_keys_start(khat, v_local)
            kc_h, vc_h = self._held_cache(k_cache, v_cache, khat.dtype)
            o_h, l_h = self.plan_held.fwd(q_local, k_local, v_local, kc_h, vc_h, q_gain=q_gain, k_gain=k_gain)
            rk, rv = self._gather_keys_finish(handle)
            o_b, l_b = self.plan_borrowed.fwd(q_local, k_local, v_local, rk, rv, q_gain=q_gain, k_gain=k_gain)
            o32, lse = self.plan_held.attn_merge(o_h, l_h, o_b, l_b)
            o = o32 if self.plan.o_fp32 else self.plan.attn_merge(o_h, l_h, o_b, l_b)[0]
            self._saved = (kc_h, vc_h, rk, rv, o32)
            return o, lse
        rk, rv = self._gather_keys(khat, v_local)
        kc, vc = self._local_cache(k_cache, v_cache, rk, rv)
        if self.local.num_cache_keys == 0:
            kc = vc = None
        o, lse = self.plan.fwd(q_local, k_local, v_local, kc, vc, q_gain=q_gain, k_gain=k_gain)
        self._saved = (kc, vc)
        return o, lse

    def backward(self, q_local, k_local, v_local, k_cache, v_cache, o, lse, do_local, q_gain=None, k_gain=None):
        """(dq, dk, dv) of this rank's tokens and (dk_cache, dv_cache) of the global cache
        (summed over ranks, on every rank; None without a cache)."""
        import torch
        import torch.distributed as dist
        ncl = len(self.local.cache_rows)
        if self.overlap:
            kc_h, vc_h, rk, rv, o32 = self._saved
            # borrowed part first: its key gradients leave while the held part computes
            dq, dk, dv, rem_k, rem_v = self.plan_borrowed.bwd(q_local, k_local, v_local, rk, rv, o32, lse, do_local,
                                                              q_gain=q_gain, k_gain=k_gain)
            handle = self._return_grads_start(rem_k, rem_v)
            if ncl:
                dkc = torch.zeros(kc_h.shape, dtype=dk.dtype, device=dk.device)
                dvc = torch.zeros(vc_h.shape, dtype=dk.dtype, device=dk.device)
            else:
                dkc = dvc = None
            self.plan_held.bwd(q_local, k_local, v_local, kc_h, vc_h, o32, lse, do_local, dq=dq, dk=dk, dv=dv,
                               dk_cache=dkc, dv_cache=dvc, q_gain=q_gain, k_gain=k_gain, accumulate=True)
            gk, gv = self._cache_grads(dkc, dvc, ncl, dk)
            dk, dv = self._return_grads_finish(handle, k_local, dk, dv, k_gain)
            return dq, dk, dv, gk, gv
        kc, vc = self._saved
        dq, dk, dv, dkc, dvc = self.plan.bwd(q_local, k_local, v_local, kc, vc, o, lse, do_local,
                                             q_gain=q_gain, k_gain=k_gain)
        # the same collective order as the overlapped path (ranks may differ in which path
        # they take): the returning all-to-all first, then the cache all-reduce
        rem_k = dkc[ncl:] if dkc is not None else dk.new_zeros((0, self.hkv, self.d))
        rem_v = dvc[ncl:] if dvc is not None else dv.new_zeros((0, self.hkv, self.d))
        handle = self._return_grads_start(rem_k, rem_v)
        gk, gv = self._cache_grads(dkc, dvc, ncl, dk)
        dk, dv = self._return_grads_finish(handle, k_local, dk, dv, k_gain)
        return dq, dk, dv, gk, gv
