"""Seeded synthetic workloads for the CSA2 decode step.

This module only draws random inputs and lays out page tables; it holds none of
the method's arithmetic (no quantisation, scoring, selection or attention), so
the CUDA path and the float64 oracle can both be fed from it.

Every random array is drawn from numpy's PCG64 seeded by
``SeedSequence([workload seed, stream tag, request, chunk])``.  Cache rows are
drawn one page-sized chunk at a time, so any row can be regenerated on its own
(the parity tests use this to check sampled rows of 1M-position caches).

Distributions (the pages give none; these follow the workload descriptions):

* indexer query q ~ N(0,1) fp32 [32,128] per request and non-Reuse layer;
  head weights w ~ U(0,1) [32].
* indexer key k ~ N(0,1) fp32 [128] per position.
* main KV row x = z * c with z ~ N(0,1) [512] per position and a per-workload
  channel scale c = exp(0.5 * N(0,1)), times 8 on 5 outlier channels (1 %).
* main query ~ N(0,1) rounded to bf16, [H,512] per request and layer.
* needles (decode at 1M): 64 distinct positions per request, uniform; the key
  there gets + 4 * u, where u is the unit vector along sum_h w_h q_h of the
  request's first (Full) layer: the key's component along the query direction is
  raised by 4 standard deviations of N(0,1).
* ragged serving batch: context lengths log-uniform in [4096, 1048576]; pages
  of 4096 positions handed out from a shuffled free list.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

INDEX_HEADS = 32
INDEX_DIM = 128
KV_DIM = 512

_TAG_IDX_Q, _TAG_MAIN_Q, _TAG_CHAN, _TAG_IK, _TAG_KV, _TAG_LEN, _TAG_PAGES, _TAG_NEEDLE = range(1, 9)


def _rng(*entropy: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(e) for e in entropy])))


@dataclass(frozen=True)
class Workload:
    """One synthetic workload.  `modes` lists the layer group ("F", "Ri", "Ru")."""
    name: str
    batch: int
    modes: tuple
    heads: int                      # main-attention query heads (d = 512)
    seed: int
    ctx: int = 0                    # fixed context length (0: drawn per request)
    ctx_range: tuple = (0, 0)       # log-uniform range when ctx == 0
    pool_blocks: int | None = 2048  # None: no hierarchical pool
    topk: int = 512
    page_size: int = 4096
    needles: int = 0
    append: bool = False            # one new token appended per request first
    shuffle_pages: bool = False
    prefill_queries: int = 0        # >0: causal prefill chunk (one request)
    prefill_tokens: int = 0
    scale: float = field(default=1.0 / math.sqrt(KV_DIM))

    @property
    def index_layers(self):
        """Layer numbers that run an indexer (every non-Reuse layer)."""
        return [i for i, m in enumerate(self.modes) if m != "Ru"]


WORKLOADS = {
    # single Full layer, 1 query, 4K context, flat Top-512, 16 heads
    "full_4k_b1": Workload("full_4k_b1", batch=1, modes=("F",), heads=16, seed=0,
                           ctx=4096, pool_blocks=None),
    # 1 Full + 2 Reindex + 3 Reuse, batch 8, 64K contexts, 64 heads
    "group_64k_b8": Workload("group_64k_b8", batch=8, modes=("F", "Ri", "Ri", "Ru", "Ru", "Ru"),
                             heads=64, seed=1, ctx=65536),
    # same group at 1M context, batch 4, 64 needles per request
    "group_1m_b4": Workload("group_1m_b4", batch=4, modes=("F", "Ri", "Ri", "Ru", "Ru", "Ru"),
                            heads=64, seed=2, ctx=1048576, needles=64),
    # encoder-style causal prefill: 8192 queries over 262144 m=2 entries, 1F + 5Ru
    "prefill_256k_q8192": Workload("prefill_256k_q8192", batch=1,
                                   modes=("F", "Ru", "Ru", "Ru", "Ru", "Ru"), heads=16, seed=3,
                                   ctx=262144, pool_blocks=None, prefill_queries=8192,
                                   prefill_tokens=524288),
    # ragged serving batch: 64 requests, 1F + 4Ri + 1Ru, shuffled 4096-position pages
    "ragged_b64": Workload("ragged_b64", batch=64, modes=("F", "Ri", "Ri", "Ri", "Ri", "Ru"),
                           heads=64, seed=7, ctx=0, ctx_range=(4096, 1048576), append=True,
                           shuffle_pages=True),
}


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of `wl` with some fields replaced (smaller parity cases)."""
    d = {f: getattr(wl, f) for f in wl.__dataclass_fields__}
    d.update(changes)
    return Workload(**d)


# ----------------------------------------------------------- shapes / pages --

def ctx_lengths(wl: Workload) -> np.ndarray:
    """Visible context length of each request (after the append, if any)."""
    if wl.ctx:
        return np.full(wl.batch, wl.ctx, dtype=np.int64)
    lo, hi = wl.ctx_range
    u = _rng(wl.seed, _TAG_LEN).random(wl.batch)
    return np.floor(np.exp(np.log(lo) + u * (np.log(hi) - np.log(lo)))).astype(np.int64)


def page_layout(wl: Workload, lengths=None):
    """(page_table int32 [B, max_pages], num_pages).  Unused slots hold -1.
    `lengths` overrides the workload's context lengths."""
    n = ctx_lengths(wl) if lengths is None else np.asarray(lengths, dtype=np.int64)
    per = -(-n // wl.page_size)
    max_pages = int(per.max())
    num_pages = int(per.sum())
    ids = np.arange(num_pages, dtype=np.int32)
    if wl.shuffle_pages:
        ids = _rng(wl.seed, _TAG_PAGES).permutation(ids).astype(np.int32)
    table = np.full((wl.batch, max_pages), -1, dtype=np.int32)
    off = 0
    for b in range(wl.batch):
        table[b, :per[b]] = ids[off:off + per[b]]
        off += per[b]
    return table, num_pages


# ------------------------------------------------------------------ queries --

def index_query(wl: Workload, layer: int, rows: int | None = None):
    """(q fp32 [R,32,128], w fp32 [R,32]) of one indexer layer; R = batch, or
    the number of prefill queries."""
    r = rows if rows is not None else (wl.prefill_queries or wl.batch)
    g = _rng(wl.seed, _TAG_IDX_Q, layer)
    q = g.standard_normal((r, INDEX_HEADS, INDEX_DIM), dtype=np.float32)
    w = g.random((r, INDEX_HEADS), dtype=np.float32)
    return q, w


def main_query(wl: Workload, layer: int, rows: int | None = None):
    """Main-attention query [R,H,512] as a torch bfloat16 tensor (CPU)."""
    import torch
    r = rows if rows is not None else (wl.prefill_queries or wl.batch)
    g = _rng(wl.seed, _TAG_MAIN_Q, layer)
    q = g.standard_normal((r, wl.heads, KV_DIM), dtype=np.float32)
    return torch.from_numpy(q).to(torch.bfloat16)


def prefill_positions(wl: Workload) -> np.ndarray:
    """Token positions (int32) of the prefill queries: the last
    `prefill_queries` tokens of a `prefill_tokens`-token stream."""
    return np.arange(wl.prefill_tokens - wl.prefill_queries, wl.prefill_tokens, dtype=np.int32)


def prefill_ratio(wl: Workload) -> int:
    """Tokens per compressed entry of a prefill workload (m = 2 on the pages)."""
    return wl.prefill_tokens // wl.ctx


# -------------------------------------------------------------- cache rows --

def channel_scale(wl: Workload) -> np.ndarray:
    """Per-channel scale of the main KV: exp(0.5 N(0,1)), x8 on 1 % of channels."""
    g = _rng(wl.seed, _TAG_CHAN)
    c = np.exp(0.5 * g.standard_normal(KV_DIM)).astype(np.float32)
    out = g.choice(KV_DIM, size=round(0.01 * KV_DIM), replace=False)
    c[out] *= 8.0
    return c


def needle_positions(wl: Workload, b: int) -> np.ndarray:
    """Sorted needle positions of request b (empty when the workload has none)."""
    if not wl.needles:
        return np.zeros(0, dtype=np.int64)
    n = int(ctx_lengths(wl)[b])
    g = _rng(wl.seed, _TAG_NEEDLE, b)
    return np.sort(g.choice(n, size=min(wl.needles, n), replace=False)).astype(np.int64)


def needle_direction(wl: Workload, b: int) -> np.ndarray:
    """Unit vector along sum_h w_h q_h of request b's first layer (fp32 [128])."""
    q, w = index_query(wl, wl.index_layers[0])
    v = (w[b].astype(np.float64)[:, None] * q[b].astype(np.float64)).sum(axis=0)
    return (v / np.linalg.norm(v)).astype(np.float32)


def indexer_key_chunk(wl: Workload, b: int, chunk: int) -> np.ndarray:
    """Indexer keys fp32 [page_size,128] for positions [chunk*P, (chunk+1)*P)."""
    P = wl.page_size
    k = _rng(wl.seed, _TAG_IK, b, chunk).standard_normal((P, INDEX_DIM), dtype=np.float32)
    if wl.needles:
        pos = needle_positions(wl, b)
        sel = pos[(pos >= chunk * P) & (pos < (chunk + 1) * P)] - chunk * P
        if len(sel):
            k[sel] += np.float32(4.0) * needle_direction(wl, b)
    return k


def main_kv_chunk(wl: Workload, b: int, chunk: int, cscale: np.ndarray | None = None) -> np.ndarray:
    """Main KV rows fp32 [page_size,512] for positions [chunk*P, (chunk+1)*P)."""
    c = channel_scale(wl) if cscale is None else cscale
    z = _rng(wl.seed, _TAG_KV, b, chunk).standard_normal((wl.page_size, KV_DIM), dtype=np.float32)
    z *= c
    return z


def rows_at(wl: Workload, b: int, positions, which: str = "ik") -> np.ndarray:
    """Regenerate the rows of request b at the given positions ("ik" or "kv")."""
    positions = np.asarray(positions, dtype=np.int64)
    P = wl.page_size
    width = INDEX_DIM if which == "ik" else KV_DIM
    out = np.empty((len(positions), width), dtype=np.float32)
    cscale = channel_scale(wl)
    for chunk in np.unique(positions // P):
        m = positions // P == chunk
        rows = indexer_key_chunk(wl, b, int(chunk)) if which == "ik" else main_kv_chunk(wl, b, int(chunk), cscale)
        out[m] = rows[positions[m] - chunk * P]
    return out


def request_rows(wl: Workload, b: int, n: int | None = None, which: str = "ik",
                 threads: int = 8) -> np.ndarray:
    """All rows [0, n) of request b (default n = its context length)."""
    n = int(ctx_lengths(wl)[b]) if n is None else n
    P = wl.page_size
    chunks = -(-n // P)
    cscale = channel_scale(wl)

    def one(c):
        return indexer_key_chunk(wl, b, c) if which == "ik" else main_kv_chunk(wl, b, c, cscale)

    with ThreadPoolExecutor(threads) as ex:
        parts = list(ex.map(one, range(chunks)))
    return np.concatenate(parts)[:n]


def iter_chunks(wl: Workload, threads: int = 8, lengths=None):
    """Yield (b, chunk, rows_ik fp32 [P,128], rows_kv fp32 [P,512], n_valid) for
    every page-sized chunk of every request, drawn on a thread pool in order."""
    n = ctx_lengths(wl) if lengths is None else np.asarray(lengths)
    P = wl.page_size
    cscale = channel_scale(wl)
    jobs = [(b, c) for b in range(wl.batch) for c in range(-(-int(n[b]) // P))]

    def one(job):
        b, c = job
        return b, c, indexer_key_chunk(wl, b, c), main_kv_chunk(wl, b, c, cscale), \
            int(min(P, n[b] - c * P))

    with ThreadPoolExecutor(threads) as ex:
        window = []
        for job in jobs:
            window.append(ex.submit(one, job))
            if len(window) >= 2 * threads:
                yield window.pop(0).result()
        for f in window:
            yield f.result()
