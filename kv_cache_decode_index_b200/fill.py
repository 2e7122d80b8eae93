"""Fill a CSA2 cache with a synthetic workload through csa2_append_kv.

The rows are drawn on the host (kv_cache_decode_index_b200.workloads), one
page-sized chunk at a time on a thread pool, copied to the device and
quantised there by the append kernel.
"""
from __future__ import annotations

import numpy as np
import torch

from . import workloads as W


def build_cache(wl, csa2, append_last: bool = False, lengths=None, device="cuda", fp4_indexer: bool = False):
    """Allocate a cache for `wl` and fill it chunk by chunk.  With append_last,
    each request's last position is left out (a decode step appends it).
    With fp4_indexer, the same indexer keys are also stored in the FP4
    indexer format (cache.ik4)."""
    n = W.ctx_lengths(wl) if lengths is None else np.asarray(lengths)
    table, num_pages = W.page_layout(wl, n)
    cache = csa2.Cache(num_pages, wl.page_size, table, n, device=device)
    dev = cache.device
    cache.ik4 = csa2.Ik4(cache) if fp4_indexer else None
    for b, c, ik, kv, nvalid in W.iter_chunks(wl, lengths=n):
        stop = nvalid - (1 if append_last and c * wl.page_size + nvalid == n[b] else 0)
        if stop <= 0:
            continue
        pos = torch.arange(c * wl.page_size, c * wl.page_size + stop, dtype=torch.int32, device=dev)
        req = torch.full((stop,), b, dtype=torch.int32, device=dev)
        tik = torch.from_numpy(ik[:stop]).to(dev)
        csa2.append_kv(cache, torch.from_numpy(kv[:stop]).to(dev, non_blocking=False), tik, pos, req)
        if fp4_indexer:
            csa2.append_ik4(cache, cache.ik4, tik, pos, req)
    torch.cuda.synchronize(dev)
    return cache
