"""The context-sharded pool on one GPU: every slice of a request scanned and
pooled over a view of the cache, the slices' candidates merged by
csa2_pool_merge.  The merged pool must be the unsharded pool bit for bit, and
the oracle's pool under the parity rules.  Needs a B200 and libcsa2.so."""
import numpy as np
import pytest
import torch

from kv_cache_decode_index_b200 import workloads as W
from oracle import csa2 as C
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    from kv_cache_decode_index_b200 import csa2 as lib
    from kv_cache_decode_index_b200 import sharded
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib, sharded


@pytest.mark.parametrize("G", [1, 2, 3, 8])
def test_sharded_pool_equals_unsharded(libs, G):
    csa2, sharded = libs
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=3, ctx=0, ctx_range=(4096, 4096), shuffle_pages=True,
                  page_size=4096)
    lengths = [262144, 250001, 9000]
    cache = U.build_cache(wl, csa2, lengths=lengths)
    dev = cache.device
    q, w = W.index_query(wl, 0)
    tq, tw = torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev)
    bm = csa2.index_full(cache, tq, tw)
    whole = csa2.pool_select(cache, bm, 2048)
    merged = sharded.emulated_sharded_pool(cache, tq, tw, G, 2048)
    assert torch.equal(merged, whole)
    assert csa2.get_error(cache)[0] == csa2.OK
    if G == 3:
        bmh = bm.cpu().numpy()
        for b, n in enumerate(lengths):
            codes, exp = U.oracle_request(wl, b, n)
            bm64 = C.block_max(C.indexer_scores(q[b], w[b], codes, exp), n)
            gp = merged[b].cpu().numpy()
            U.assert_sorted_padded(gp, f"merged pool b={b}")
            U.assert_set_parity(gp, C.pool_select(bm64, 2048), lambda j: bm64[j], U.threshold(bm64, 2048),
                                what=f"merged pool b={b}")
            # the merge of the GPU's candidates equals the oracle's merge of the same candidates
            vals, ids = [], []
            for first, npg in sharded.slice_pages(cache.max_pages_per_req, G):
                lo, hi = first * cache.page_size // 8, min((first + npg) * cache.page_size, n)
                v, i = C.slice_candidates(bmh[b, lo:max(lo, -(-hi // 8))].astype(np.float64), lo, 2048)
                vals.append(v)
                ids.append(i)
            np.testing.assert_array_equal(gp, C.pool_merge(vals, ids, 2048))


def test_sharded_pool_1m_eight_slices(libs):
    """The 1M-position request split into 8 slices of 131,072 positions."""
    csa2, sharded = libs
    wl = W.scaled(W.WORKLOADS["group_1m_b4"], batch=2)
    cache = U.build_cache(wl, csa2)
    dev = cache.device
    q, w = W.index_query(wl, 0)
    tq, tw = torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev)
    bm = csa2.index_full(cache, tq, tw)
    whole = csa2.pool_select(cache, bm, 2048)
    for G in (2, 8):
        assert torch.equal(sharded.emulated_sharded_pool(cache, tq, tw, G, 2048), whole), f"G={G}"
    assert csa2.get_error(cache)[0] == csa2.OK


def test_pool_merge_ties_go_to_the_lower_global_id(libs):
    """Hand-built candidates with equal block maxima in every slice."""
    csa2, sharded = libs
    dev = torch.device("cuda")
    G, B, P = 3, 2, 8
    vals = torch.ones(G, B, P, dtype=torch.float32)
    ids = torch.arange(G * P, dtype=torch.int32).view(G, 1, P).repeat(1, B, 1).contiguous()
    ids[:, 1, 6:] = -1                         # request 1: two empty entries per slice
    vals[1, 0, 3] = 2.0                        # one clear winner in slice 1
    got = sharded.pool_merge(vals.to(dev), ids.to(dev)).cpu().numpy()
    np.testing.assert_array_equal(got[0], [0, 1, 2, 3, 4, 5, 6, 11])
    np.testing.assert_array_equal(got[1], [0, 1, 2, 3, 4, 5, 8, 9])
