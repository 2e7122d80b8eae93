"""Parity of the causal prefill indexer (csa2_prefill_index) and of the
prefill layer group (indexer, then attention of every layer over the Top-k)
against the float64 oracle.  Needs a B200 and libcsa2.so."""
import numpy as np
import pytest
import torch

from kv_cache_decode_index_b200 import workloads as W
from oracle import csa2 as C
from oracle import formats as F
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

PREFILL = W.WORKLOADS["prefill_256k_q8192"]


@pytest.fixture(scope="module")
def csa2():
    from kv_cache_decode_index_b200 import csa2 as lib
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib


def _cache_from_rows(csa2, ik_rows, page_size=4096, shuffle=True):
    """One request whose indexer keys are `ik_rows` (fp32 [N,128]), written by
    the append kernel into pages handed out in reverse order."""
    n = ik_rows.shape[0]
    per = -(-n // page_size)
    ids = np.arange(per, dtype=np.int32)[::-1].copy() if shuffle else np.arange(per, dtype=np.int32)
    cache = csa2.Cache(per, page_size, ids[None, :], [n])
    dev = cache.device
    for c0 in range(0, n, page_size):
        c1 = min(n, c0 + page_size)
        m = c1 - c0
        csa2.append_kv(cache, torch.zeros(m, 512, dtype=torch.float32, device=dev),
                       torch.from_numpy(np.ascontiguousarray(ik_rows[c0:c1])).to(dev),
                       torch.arange(c0, c1, dtype=torch.int32, device=dev),
                       torch.zeros(m, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    return cache


def _check_query(gpu_row, q, w, codes, exp, p, k, ratio, what, exact=False):
    v = min(C.prefill_visible(int(p), ratio), len(codes))
    U.assert_sorted_padded(gpu_row, what)
    g = gpu_row[gpu_row >= 0]
    assert len(g) == min(k, v), f"{what}: {len(g)} selected, {min(k, v)} visible"
    if v == 0:
        return 0
    assert g.max() < v, f"{what}: selects an entry the query cannot see"
    s = C.indexer_scores(q, w, codes[:v], exp[:v])
    ora = C.top_k_ascending(np.arange(v), s, k)
    if exact:
        np.testing.assert_array_equal(gpu_row, ora, err_msg=what)
        return 0
    return U.assert_set_parity(gpu_row, ora, lambda t: s[t], U.threshold(s, k), what=what)


@pytest.mark.parametrize("k", [1, 64, 512, 1024])
def test_prefill_index_ragged_causal(csa2, k):
    """5,000 entries (39 full tiles and a ragged tail) over reversed pages;
    37 queries (a partial CTA of queries) whose positions sweep the whole
    causal range, so that the visible count runs from 0 to all entries."""
    rng = np.random.default_rng(41 + k)
    n_ent, n_q, ratio = 5000, 37, 2
    ik = rng.standard_normal((n_ent, 128), dtype=np.float32)
    cache = _cache_from_rows(csa2, ik)
    codes, exp = F.quantize_indexer(ik)
    q = rng.standard_normal((n_q, 32, 128), dtype=np.float32)
    w = rng.random((n_q, 32), dtype=np.float32)
    pos = np.linspace(-3, 2 * n_ent + 40, n_q).astype(np.int32)
    dev = cache.device
    topk = csa2.prefill_index(cache, 0, torch.from_numpy(pos).to(dev), torch.from_numpy(q).to(dev),
                              torch.from_numpy(w).to(dev), k=k, ratio=ratio)
    st, word = csa2.get_error(cache)
    assert st == csa2.OK, word
    got = topk.cpu().numpy()
    for j in range(n_q):
        _check_query(got[j], q[j], w[j], codes, exp, pos[j], k, ratio, f"query {j} p={pos[j]} k={k}")


def test_prefill_index_ties_go_to_lower_entries(csa2):
    """Keys repeat with period 13, so every score value is shared by hundreds
    of entries: the candidate lists overflow and are compacted with whole tie
    classes at the threshold; the lower entries must win, bit-exactly."""
    rng = np.random.default_rng(5)
    base = rng.standard_normal((13, 128), dtype=np.float32)
    n_ent = 12288 + 77
    ik = base[np.arange(n_ent) % 13]
    cache = _cache_from_rows(csa2, ik, shuffle=False)
    codes, exp = F.quantize_indexer(ik)
    n_q = 9
    q = rng.standard_normal((n_q, 32, 128), dtype=np.float32)
    w = rng.random((n_q, 32), dtype=np.float32)
    pos = np.full(n_q, 2 * n_ent, dtype=np.int32)
    pos[3] = 2 * 3000
    dev = cache.device
    for k in (512, 1000):
        topk = csa2.prefill_index(cache, 0, torch.from_numpy(pos).to(dev), torch.from_numpy(q).to(dev),
                                  torch.from_numpy(w).to(dev), k=k)
        got = topk.cpu().numpy()
        for j in range(n_q):
            s13 = np.sort(C.indexer_scores(q[j], w[j], codes[:13], exp[:13]))
            gaps = np.diff(s13) / np.maximum(s13[1:], 1e-30)
            assert gaps.min() > 2e-5, "the 13 score classes must lie outside each other's tie band"
            _check_query(got[j], q[j], w[j], codes, exp, pos[j], k, 2, f"ties query {j} k={k}", exact=True)


def test_prefill_index_ratio_and_request(csa2):
    """Another compression ratio (m = 4) and the second request of a batch."""
    rng = np.random.default_rng(9)
    n_ent = 3000
    page = 1024
    ik0 = rng.standard_normal((n_ent, 128), dtype=np.float32)
    ik1 = rng.standard_normal((n_ent, 128), dtype=np.float32)
    per = -(-n_ent // page)
    table = np.stack([np.arange(per), np.arange(per, 2 * per)[::-1]]).astype(np.int32)
    cache = csa2.Cache(2 * per, page, table, [n_ent, n_ent - 100])
    dev = cache.device
    for b, rows in ((0, ik0), (1, ik1)):
        csa2.append_kv(cache, torch.zeros(n_ent, 512, device=dev), torch.from_numpy(rows).to(dev),
                       torch.arange(n_ent, dtype=torch.int32, device=dev),
                       torch.full((n_ent,), b, dtype=torch.int32, device=dev))
    codes, exp = F.quantize_indexer(ik1[:n_ent - 100])
    n_q = 16
    q = rng.standard_normal((n_q, 32, 128), dtype=np.float32)
    w = rng.random((n_q, 32), dtype=np.float32)
    pos = np.linspace(0, 4 * n_ent, n_q).astype(np.int32)
    topk = csa2.prefill_index(cache, 1, torch.from_numpy(pos).to(dev), torch.from_numpy(q).to(dev),
                              torch.from_numpy(w).to(dev), k=256, ratio=4)
    got = topk.cpu().numpy()
    for j in range(n_q):
        _check_query(got[j], q[j], w[j], codes, exp, pos[j], 256, 4, f"m=4 query {j}")


def test_prefill_group_full_size(csa2):
    """The pages' encoder chunk at full size: 8,192 queries over 262,144 m=2
    entries, 1 Full + 5 Reuse layers of 16 heads.  Every query's Top-512 is
    checked for structure; sampled queries against the oracle's Top-512 and
    attention outputs."""
    from kv_cache_decode_index_b200.fill import build_cache
    wl = PREFILL
    cache = build_cache(wl, csa2)
    dev = cache.device
    n = wl.prefill_queries
    pos = W.prefill_positions(wl)
    ratio = W.prefill_ratio(wl)
    q, w = W.index_query(wl, 0)
    q_main = [W.main_query(wl, layer).to(dev) for layer in range(len(wl.modes))]
    group = csa2.PrefillGroup(cache, 0, wl.modes, wl.heads, n, wl.topk, ratio, wl.scale)
    out = [torch.empty_like(m) for m in q_main]
    tq = [torch.from_numpy(q).to(dev)] + [None] * (len(wl.modes) - 1)
    tw = [torch.from_numpy(w).to(dev)] + [None] * (len(wl.modes) - 1)
    group.step(torch.from_numpy(pos).to(dev), tq, tw, q_main, out)
    st, word = csa2.get_error(cache)
    assert st == csa2.OK, word
    got = group.topk[0].cpu().numpy()
    for layer in range(1, len(wl.modes)):
        assert group.topk[layer] is group.topk[0]
    # structure of every row
    vis = np.minimum((pos.astype(np.int64) + 1) // ratio, wl.ctx)
    valid = got >= 0
    assert valid.all(), "every query sees more than 512 entries"
    assert np.all(np.diff(got, axis=1) > 0), "rows not strictly ascending"
    assert np.all(got.max(axis=1) < vis), "an entry past the causal limit"
    # sampled rows against the oracle
    codes, exp = U.oracle_request(wl, 0, wl.ctx)
    sample = [0, 1, 7, 8, 1234, 4095, 4096, 6001, 8190, 8191]
    for j in sample:
        _check_query(got[j], q[j], w[j], codes, exp, pos[j], wl.topk, ratio, f"prefill query {j}")
    for j in (0, 4096, 8191):
        kv_codes, kv_scales = U.oracle_kv_rows(wl, 0, got[j])
        for layer in (0, 5):
            qm = q_main[layer][j].float().cpu().numpy().astype(np.float64)
            o64 = C.sparse_attention(qm, kv_codes, kv_scales, np.arange(len(got[j])), wl.scale)
            U.assert_attention_close(out[layer][j].float().cpu().numpy(), o64, f"attn layer {layer} query {j}")
