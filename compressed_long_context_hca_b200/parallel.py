"""The HCA path over several GPUs: one process per GPU, torch.distributed for the
exchanges (NCCL over NVLink / NVSwitch on GPUs; the same calls run over gloo on CPU).

Three partitions. The workloads are batches of independent sequences, so the first is
plain data parallelism; the other two cut ONE long sequence over the ranks.

* ``seq_range`` -- a decode (or prefill) batch dealt out in contiguous ranges of
  sequences. No exchange at all: every rank serves its own sequences.

* ``decode_split_entries`` -- one long context per sequence, its compressed entries cut
  into contiguous ranges of whole 128-entry tiles, one range per rank; the last rank also
  holds the raw window. Every rank computes the unnormalised partial softmax sums
  (m, l, O) over its range, the partials are all-gathered (hq x (2 + head_dim) float32
  per sequence, ~130 KB at 64 heads) and every rank merges them into the output. One
  softmax over disjoint key parts equals that merge (log-sum-exp algebra), so the result
  is the decode of the whole key set.

* ``prefill_rows`` -- the query rows of a sequence cut into contiguous ranges of whole
  blocks. Each rank compresses the blocks of its own rows, the entries are all-gathered
  (ceil(T/128) entries in all, 2 MB at 128K), each rank receives the window-1 raw tokens
  that precede its range (the halo, from the ranks before it), then runs the prefill of
  its rows against the full entry list and its halo + own tokens.

The compute steps go through a backend object with the methods ``compress``,
``prefill_range``, ``decode_partial`` and ``merge``; ``GpuBackend`` runs them on the
kernels of libhca. The exchanges are plain collectives on the given process group, taken
in the same order on every rank.
"""

from __future__ import annotations

from typing import List, Optional, Tuple

import torch
import torch.distributed as dist

from . import binding as B
from . import ops


# ------------------------------------------------------------------------------ ranges

def split_range(n: int, world: int, rank: int, align: int = 1) -> Tuple[int, int]:
    """[lo, hi) of ``rank`` when n items are cut into ``world`` contiguous ranges made of
    whole units of ``align`` items (the last unit may be short), as even as possible:
    the first (units % world) ranks take one unit more."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside the world")
    units = -(-n // align) if n > 0 else 0
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return min(n, u0 * align), min(n, u1 * align)


def seq_range(nseq: int, world: int, rank: int) -> Tuple[int, int]:
    """Sequences [lo, hi) a rank serves in the batch partition (no exchange)."""
    return split_range(nseq, world, rank)


def entry_range(n_entries: int, world: int, rank: int) -> Tuple[int, int]:
    """Compressed entries [lo, hi) of a rank in the split-entries decode: whole 128-entry
    tiles (the decode kernel's tile; entry_begin must be a multiple of 128). The last
    rank's range is open-ended (it also takes entries past n_entries, should a sequence
    have more) and holds the raw window."""
    units = -(-n_entries // 128) if n_entries > 0 else 0
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return u0 * 128, (1 << 30) if rank == world - 1 else u1 * 128


def row_range(T: int, world: int, rank: int, block: int) -> Tuple[int, int]:
    """Query rows [lo, hi) of a rank in the row-partitioned prefill: whole blocks, so
    every block (and its compressed entry) belongs to exactly one rank."""
    return split_range(T, world, rank, block)


def _world(group) -> Tuple[int, int]:
    """(world size, rank) of the group; a single process without a process group is a
    world of one."""
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def _all_gather(t: torch.Tensor, group) -> List[torch.Tensor]:
    world, _ = _world(group)
    if world == 1:
        return [t]
    out = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(out, t.contiguous(), group=group)
    return out


# ------------------------------------------------------------------------------ decode

def decode_split_entries(backend, group, q, ctx_len, cache, ring_k, ring_v,
                         n_entries: int, desc=None):
    """One decode step whose key list is cut over the ranks of ``group``.

    Every rank holds the queries, the context lengths and the compressed entries of its
    own ``entry_range`` (its cache may hold nothing else; the entries are addressed by
    absolute index); the last rank also holds the ring of raw tokens. ``n_entries`` is
    the largest visible entry count of the batch. Returns the output on every rank."""
    world, rank = _world(group)
    if world == 1:  # one rank holds every key: the plain decode step
        return backend.decode(q, ctx_len, cache, ring_k, ring_v, desc)
    e0, e1 = entry_range(n_entries, world, rank)
    part = backend.decode_partial(q, ctx_len, cache, ring_k, ring_v, e0, e1,
                                  rank == world - 1, desc)
    parts = torch.stack(_all_gather(part, group))
    return backend.merge(parts, desc)


# ------------------------------------------------------------------------------ prefill

def prefill_rows(backend, group, Q, K, V, T: int, block: int, window: int, G=None,
                 desc=None, out=None):
    """Prefill of the rows [row_range) of every sequence, cut over the ranks of
    ``group``.

    Q, K, V (and G): this rank's rows only, [b, rows, h, D]. T is the full sequence
    length. Returns this rank's output rows (in ``out`` if given)."""
    world, rank = _world(group)
    ranges = [row_range(T, world, r, block) for r in range(world)]
    t0, t1 = ranges[rank]
    if Q.shape[1] != t1 - t0 or K.shape[1] != t1 - t0:
        raise ValueError("rows do not match this rank's range")
    # 1. entries of this rank's blocks, all-gathered (padded to the largest range)
    nb = [-(-(hi - lo) // block) for lo, hi in ranges]
    nb_max = max(nb)
    Kc, Vc = backend.compress(K, V, block)                      # [b, nb[rank], hkv, D]
    if world == 1:
        Kc_all, Vc_all = Kc, Vc
    else:
        pad = nb_max - Kc.shape[1]
        if pad:
            z = Kc.new_zeros((Kc.shape[0], pad) + tuple(Kc.shape[2:]))
            Kc, Vc = torch.cat([Kc, z], 1), torch.cat([Vc, z], 1)
        KVc = _all_gather(torch.stack([Kc, Vc]), group)         # world x [2, b, nb_max, ...]
        Kc_all = torch.cat([KVc[r][0][:, :nb[r]] for r in range(world)], 1)
        Vc_all = torch.cat([KVc[r][1][:, :nb[r]] for r in range(world)], 1)
    # 2. halo: every rank's last window-1 rows, zero rows in front when it has fewer; the
    # rows [t0 - (window-1), t0) this rank needs lie in the tails of the ranks before it
    h = window - 1
    kv0 = max(0, t0 - h)
    pieces_k, pieces_v = [], []
    if h > 0:
        n = K.shape[1]
        tail = torch.stack([K[:, max(0, n - h):], V[:, max(0, n - h):]])
        if tail.shape[2] < h:
            z = tail.new_zeros(tail.shape[:2] + (h - tail.shape[2],) + tuple(tail.shape[3:]))
            tail = torch.cat([z, tail], 2)
        tails = _all_gather(tail, group)
        for r in range(rank):
            lo, hi = ranges[r]
            a = max(kv0, lo)
            if a >= hi:
                continue
            # rank r's tail holds positions hi - h .. hi - 1 (hi <= t0, so a >= hi - h)
            pieces_k.append(tails[r][0][:, a - (hi - h):])
            pieces_v.append(tails[r][1][:, a - (hi - h):])
    Kloc = torch.cat(pieces_k + [K], 1)
    Vloc = torch.cat(pieces_v + [V], 1)
    return backend.prefill_range(Q, Kloc, Vloc, Kc_all, Vc_all, t0, kv0, block, window, G,
                                 desc, out)


# ------------------------------------------------------------------------------ backend

class GpuBackend:
    """The compute steps on the kernels of libhca (bf16, head_dim 512, 1 KV head).

    Device buffers (caches, partial results) are kept per shape and reused by later calls
    of the same shape, so a loop of steps allocates nothing after its first step."""

    def __init__(self, scale: Optional[float] = None):
        self.scale = scale
        self._caches = {}
        self._parts = {}
        self._ws = {}
        self._outs = {}
        # a list to receive a (start, end) CUDA event pair around every prefill kernel
        self.kernel_events = None

    def _cache(self, key, b, n, hkv, D, dtype, device):
        c = self._caches.get(key)
        if c is None:
            c = B.PagedCache(b, max(n, 1), hkv, D, dtype, 128, device=device)
            self._caches[key] = c
        return c

    def compress(self, K, V, block: int):
        b, n, hkv, D = K.shape
        nb = -(-n // block)
        cache = self._cache(("own", b, nb, hkv, D, K.dtype), b, nb, hkv, D, K.dtype, K.device)
        desc = B.make_desc(b, n, 1, hkv, D, block, 128, self.scale, B.dtype_code(K))
        ops.compress(desc, K, V, cache)
        # identity page table: sequence b's entries are pool rows b * cap .. b * cap + nb - 1
        cap = cache.max_pages * cache.page_entries
        return cache.kc.view(b, cap, hkv, D)[:, :nb], cache.vc.view(b, cap, hkv, D)[:, :nb]

    def _cache_from(self, Kc, Vc):
        b, n, hkv, D = Kc.shape
        own = self._caches.get(("own", b, n, hkv, D, Kc.dtype))
        if own is not None and Kc.data_ptr() == own.kc.data_ptr():
            return own  # the entries this backend's compress wrote (a world of one)
        cache = self._cache(("all", b, n, hkv, D, Kc.dtype), b, n, hkv, D, Kc.dtype,
                            Kc.device)
        cap = cache.max_pages * cache.page_entries
        cache.kc.view(b, cap, hkv, D)[:, :n].copy_(Kc)
        cache.vc.view(b, cap, hkv, D)[:, :n].copy_(Vc)
        cache.n_entries.fill_(n)
        return cache

    def prefill_range(self, Q, K, V, Kc, Vc, q_pos0: int, kv_pos0: int, block: int,
                      window: int, G=None, desc=None, out=None):
        cache = self._cache_from(Kc, Vc)
        d = ops.desc_for_prefill(Q, K, block, window, self.scale)
        ops.attach_gate(d, G)
        if out is None:
            out = self._outs.get(tuple(Q.shape))
            if out is None:
                out = self._outs[tuple(Q.shape)] = torch.empty_like(Q)
        if self.kernel_events is not None:  # a caller timing the prefill kernel alone
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
        ops.prefill_range(d, q_pos0, kv_pos0, Q, K, V, cache, O=out)
        if self.kernel_events is not None:
            b.record()
            self.kernel_events.append((a, b))
        return out

    def decode(self, q, ctx_len, cache, ring_k, ring_v, desc):
        key = (desc.batch, desc.seqlen, desc.hq, desc.decode_splits, q.device)
        if key not in self._ws:
            self._ws[key] = (ops.decode_workspace(desc, q.device), torch.empty_like(q))
        ws, O = self._ws[key]
        ops.decode(desc, q, ctx_len, cache, ring_k, ring_v, O=O, workspace=ws)
        return O

    def decode_partial(self, q, ctx_len, cache, ring_k, ring_v, e0: int, e1: int,
                       with_window: bool, desc):
        key = (desc.batch, desc.seqlen, desc.hq, desc.decode_splits, q.device)
        if key not in self._parts:
            self._parts[key] = (ops.decode_partial_buffer(desc, 1, q.device),
                                ops.decode_workspace(desc, q.device))
        buf, ws = self._parts[key]
        ops.decode_partial(desc, q, ctx_len, cache, ring_k, ring_v, e0, e1, with_window,
                           buf[0], workspace=ws)
        return buf[0]

    def merge(self, parts, desc):
        key = ("merge", desc.batch, desc.hq, parts.device)
        O = self._outs.get(key)
        if O is None:
            O = self._outs[key] = torch.empty((desc.batch, desc.hq, desc.head_dim),
                                              dtype=torch.bfloat16, device=parts.device)
        ops.decode_merge(desc, parts, O)
        return O
