"""csa2_prefill_index_static (candidate lists in the library's static device
array, no workspace) against csa2_prefill_index (caller workspace) on the
same inputs, two calls in a row.  Collected last on purpose; passes alone too.
Needs a B200 and libcsa2.so."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa2():
    from kv_cache_decode_index_b200 import csa2 as lib
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib


def _cache(csa2, n_ent, seed):
    rng = np.random.default_rng(seed)
    ik = rng.standard_normal((n_ent, 128), dtype=np.float32)
    page = 1024
    per = -(-n_ent // page)
    cache = csa2.Cache(per, page, np.arange(per, dtype=np.int32)[::-1].copy()[None, :], [n_ent])
    dev = cache.device
    csa2.append_kv(cache, torch.zeros(n_ent, 512, device=dev), torch.from_numpy(ik).to(dev),
                   torch.arange(n_ent, dtype=torch.int32, device=dev), torch.zeros(n_ent, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    return cache, rng


def test_static_scratch_matches_workspace_twice(csa2):
    cache, rng = _cache(csa2, 6000, 77)
    dev = cache.device
    for call, (n_q, k) in enumerate([(csa2.PREFILL_STATIC_MAX_QUERIES, 512), (37, 64)]):
        q = torch.from_numpy(rng.standard_normal((n_q, 32, 128), dtype=np.float32)).to(dev)
        w = torch.from_numpy(rng.random((n_q, 32), dtype=np.float32)).to(dev)
        pos = torch.from_numpy(np.linspace(0, 2 * 6000 + 9, n_q).astype(np.int32)).to(dev)
        ref = csa2.prefill_index(cache, 0, pos, q, w, k=k)
        got = csa2.prefill_index_static(cache, 0, pos, q, w, k=k)
        st, word = csa2.get_error(cache)
        assert st == csa2.OK, word
        assert torch.equal(ref, got), f"call {call}: static-scratch result differs from the workspace result"


def test_static_scratch_rejects_too_many_queries(csa2):
    cache, _ = _cache(csa2, 1000, 5)
    dev = cache.device
    n_q = csa2.PREFILL_STATIC_MAX_QUERIES + 1
    with pytest.raises(csa2.Csa2Error):
        csa2.prefill_index_static(cache, 0, torch.zeros(n_q, dtype=torch.int32, device=dev),
                                  torch.zeros(n_q, 32, 128, device=dev), torch.zeros(n_q, 32, device=dev))
