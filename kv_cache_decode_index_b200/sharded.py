"""Context-sharded pool of long requests (host side).

One request's context is split into consecutive whole-page slices, one per
device.  Each device scans its slice and keeps its own top pool_blocks blocks
(csa2_index_full, csa2_pool_select), turns them into (block max, global block
id) candidates (csa2_pool_candidates), the devices all-gather the candidates
(pool_blocks x 8 bytes per request and device: 16 KB for the pages' 2048-block
pool) and each merges them into the request's exact pool (csa2_pool_merge),
the pool of the unsharded request, bit for bit.  [alphalab analysis, limits
section: a 1M-token context may have to be sharded across machines; the cost
is the exchange between them.]

The exchange is torch.distributed's all_gather (NCCL between GPUs: plain
device buffers, nothing multicast; gloo on CPU in the tests).  What follows
the pool on a sharded request (the re-score and attention over rows that live
on other devices) needs those rows fetched first and is not built here.
"""
from __future__ import annotations

import ctypes

import torch

from . import csa2


def slice_pages(max_pages: int, n_shards: int):
    """(first_page, n_pages) of each of n_shards consecutive slices of a
    request's page table: whole pages, as even as possible, earlier slices
    never shorter than later ones."""
    if n_shards < 1:
        raise ValueError("n_shards must be >= 1")
    per, extra = divmod(max_pages, n_shards)
    out, first = [], 0
    for g in range(n_shards):
        n = per + (1 if g < extra else 0)
        out.append((first, n))
        first += n
    return out


def slice_view(cache: csa2.Cache, first_page: int, n_pages: int) -> csa2.Cache:
    """A cache over pages [first_page, first_page + n_pages) of every request's
    page table, sharing the storage of `cache`: its positions count from the
    slice start (first_page * page_size) and its ctx_len is the part of each
    request's visible context inside the slice.  (On a real multi-device
    deployment every device holds its slice in a cache of its own.)"""
    v = csa2.Cache.__new__(csa2.Cache)
    v.device, v.num_pages, v.page_size = cache.device, cache.num_pages, cache.page_size
    v.kv_codes, v.kv_scales, v.ik_codes, v.ik_exp = cache.kv_codes, cache.kv_scales, cache.ik_codes, cache.ik_exp
    v.page_table = cache.page_table[:, first_page:first_page + n_pages].contiguous()
    start = first_page * cache.page_size
    v.ctx_len = (cache.ctx_len.to(torch.int64) - start).clamp(0, n_pages * cache.page_size).to(torch.int32)
    v.batch, v.max_pages_per_req = v.page_table.shape
    v.err_word = cache.err_word
    v._struct = None
    return v


def pool_candidates(shard: csa2.Cache, blockmax, pool, block_offset: int, values=None, ids=None):
    """csa2_pool_candidates: (values float32 [batch, P], ids int32 [batch, P])."""
    B, P = pool.shape
    csa2._need(blockmax, torch.float32, (B, shard.capacity // csa2.BLOCK), "blockmax")
    csa2._need(pool, torch.int32, (B, P), "pool")
    values = torch.empty(B, P, dtype=torch.float32, device=shard.device) if values is None else values
    ids = torch.empty(B, P, dtype=torch.int32, device=shard.device) if ids is None else ids
    csa2._need(values, torch.float32, (B, P), "values")
    csa2._need(ids, torch.int32, (B, P), "ids")
    csa2._check(csa2._lib.csa2_pool_candidates(ctypes.byref(shard.struct), csa2._ptr(blockmax), csa2._ptr(pool),
                                               P, int(block_offset), csa2._ptr(values), csa2._ptr(ids),
                                               csa2._stream(shard.device)), "csa2_pool_candidates")
    return values, ids


def pool_merge(values, ids, pool=None):
    """csa2_pool_merge of candidates [G, batch, P] (slices in ascending order)
    -> pool int32 [batch, P]."""
    G, B, P = values.shape
    csa2._need(values, torch.float32, (G, B, P), "values")
    csa2._need(ids, torch.int32, (G, B, P), "ids")
    pool = torch.empty(B, P, dtype=torch.int32, device=values.device) if pool is None else pool
    csa2._need(pool, torch.int32, (B, P), "pool")
    csa2._check(csa2._lib.csa2_pool_merge(G, B, P, csa2._ptr(values), csa2._ptr(ids), csa2._ptr(pool),
                                          csa2._stream(values.device)), "csa2_pool_merge")
    return pool


def exchange_candidates(values, ids, group=None):
    """All-gather every rank's candidates: returns (values [G, batch, P], ids
    [G, batch, P]) with rank g's lists at index g.  Ranks must own the slices
    in rank order (rank g: slice g), so that index order is slice order."""
    import torch.distributed as dist
    G = dist.get_world_size(group)
    all_v = torch.empty((G * values.shape[0], *values.shape[1:]), dtype=values.dtype, device=values.device)
    all_i = torch.empty((G * ids.shape[0], *ids.shape[1:]), dtype=ids.dtype, device=ids.device)
    dist.all_gather_into_tensor(all_v, values.contiguous(), group=group)   # rank g's rows at [g * batch, ...)
    dist.all_gather_into_tensor(all_i, ids.contiguous(), group=group)
    return all_v.view(G, *values.shape), all_i.view(G, *ids.shape)


class ShardedPool:
    """The pool step of one device that holds slice `rank` of every request
    (rank order = slice order): scan the slice, keep its top pool_blocks
    blocks, exchange candidates with the other ranks, merge."""

    def __init__(self, shard: csa2.Cache, block_offset: int, pool_blocks: int = 2048, group=None):
        dev, B = shard.device, shard.batch
        self.shard, self.block_offset, self.pool_blocks, self.group = shard, int(block_offset), pool_blocks, group
        self.blockmax = torch.empty(B, shard.capacity // csa2.BLOCK, dtype=torch.float32, device=dev)
        self.hist = csa2.pool_hist(shard)
        self.local = torch.empty(B, pool_blocks, dtype=torch.int32, device=dev)
        self.values = torch.empty(B, pool_blocks, dtype=torch.float32, device=dev)
        self.ids = torch.empty(B, pool_blocks, dtype=torch.int32, device=dev)
        self.pool = torch.empty(B, pool_blocks, dtype=torch.int32, device=dev)

    def step(self, q, w):
        csa2.index_full(self.shard, q, w, self.blockmax, hist=self.hist)
        csa2.pool_select(self.shard, self.blockmax, self.pool_blocks, self.local, hist=self.hist)
        pool_candidates(self.shard, self.blockmax, self.local, self.block_offset, self.values, self.ids)
        all_v, all_i = exchange_candidates(self.values, self.ids, self.group)
        return pool_merge(all_v, all_i, self.pool)


def emulated_sharded_pool(cache: csa2.Cache, q, w, n_shards: int, pool_blocks: int = 2048):
    """The sharded pool step with every slice on this one device (each slice's
    scan and pool run over a view of `cache`; the gather is a copy into
    [G, batch, P]): the single-device check of the sharded path."""
    B, dev = cache.batch, cache.device
    if not 1 <= n_shards <= cache.max_pages_per_req:
        raise ValueError(f"n_shards {n_shards} outside [1, {cache.max_pages_per_req}] (slices are whole pages)")
    all_v = torch.empty(n_shards, B, pool_blocks, dtype=torch.float32, device=dev)
    all_i = torch.empty(n_shards, B, pool_blocks, dtype=torch.int32, device=dev)
    for g, (first, n) in enumerate(slice_pages(cache.max_pages_per_req, n_shards)):
        v = slice_view(cache, first, n)
        bm = torch.empty(B, v.capacity // csa2.BLOCK, dtype=torch.float32, device=dev)
        hist = csa2.pool_hist(v)
        csa2.index_full(v, q, w, bm, hist=hist)
        local = csa2.pool_select(v, bm, pool_blocks, hist=hist)
        pool_candidates(v, bm, local, first * cache.page_size // csa2.BLOCK, all_v[g], all_i[g])
    return pool_merge(all_v, all_i)
