"""The FP4 indexer variant on the GPU (through the C ABI) against the float64
oracle: quantise-on-append bit-exact, the block-scaled FP4 tensor-core scan's
scores within an fp32 bound, the pool and every layer's Top-k under the parity
rules, and the whole decode group.  Needs a B200 and libcsa2.so."""
import numpy as np
import pytest
import torch

from kv_cache_decode_index_b200 import workloads as W
from oracle import csa2 as C
from oracle import formats as F
from tests import gpu_util as U

# the pool histogram bins the leading 12 bits of a block max's order key
HIST_SHIFT = 20

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa2():
    from kv_cache_decode_index_b200 import csa2 as lib
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib


def _scales_of_rows(csa2, ik4, rows):
    """Block scales [len(rows), 8] of cache rows, read from the tile blocks."""
    sc = ik4.scales.cpu().numpy()
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), 8), np.uint8)
    for g in range(8):
        out[:, g] = sc[rows // 128, [csa2.ik4_scale_offset(int(m), g) for m in rows % 128]]
    return out


def _oracle_fp4(wl, b, n):
    return F.quantize_indexer_fp4(W.request_rows(wl, b, n, "ik"))


def test_append_ik4_bitexact(csa2):
    """Random rows, rows on E2M1 / E4M3 midpoints, zero rows, saturation."""
    rng = np.random.default_rng(21)
    rows = [rng.standard_normal(128) * np.exp(rng.uniform(-8, 8)) for _ in range(300)]
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.0])
    for _ in range(40):
        r = np.zeros(128)
        for g in range(8):
            s = F.e4m3_value(rng.integers(1, 127))
            v = rng.choice(mids, 16) * s * rng.choice([-1, 1], 16)
            v[rng.integers(16)] = 6 * s
            r[16 * g:16 * g + 16] = v
        rows.append(r)
    rows += [np.zeros(128), np.full(128, -0.0), np.full(128, 1e6), np.full(128, 1e-9)]
    x = np.stack(rows).astype(np.float32)
    n = len(x)
    page = 128
    per = -(-n // page)
    table = rng.permutation(per).astype(np.int32)[None, :]
    cache = csa2.Cache(per, page, table, [n])
    ik4 = csa2.Ik4(cache)
    dev = cache.device
    pos = rng.permutation(n).astype(np.int32)
    csa2.append_ik4(cache, ik4, torch.from_numpy(x[pos]).to(dev), torch.from_numpy(pos).to(dev),
                    torch.zeros(n, dtype=torch.int32, device=dev))
    assert csa2.get_error(cache)[0] == csa2.OK
    codes, scales = F.quantize_indexer_fp4(x)
    crow = cache.rows_of(0, np.arange(n)).numpy()
    np.testing.assert_array_equal(ik4.codes.cpu().numpy()[crow], codes)
    np.testing.assert_array_equal(_scales_of_rows(csa2, ik4, crow), scales)


def _fp4_bound(q, w, codes, scales):
    """fp32 bound of the block-scaled tensor-core score: every head dot
    product within 2^-20 of its absolute sum, plus the 32-term fp32 sum."""
    qc, qs = F.quantize_indexer_fp4(q)
    qa = np.abs(F.dequantize_indexer_fp4(qc, qs))
    ka = np.abs(F.dequantize_indexer_fp4(codes, scales))
    return (ka @ qa.T) @ np.abs(w.astype(np.float64)) * 2.0 ** -20


# Many short requests: about four requests per CTA's range of units, so the
# scan's query buffers rotate (segment x in buffer x % 3) inside a CTA.
MANY_SHORT = [int(n) for n in np.random.default_rng(77).integers(1, 1100, size=600)]


# Pages of 128 or 384 rows: a unit's two tiles on two pages (or the second
# absent), copied tile by tile instead of in one 256-row box.
@pytest.mark.parametrize("lengths,page_size", [([4096, 1, 1000, 9999, 128 * 37], 512), (MANY_SHORT, 512),
                                               ([4096, 1, 1000, 9999, 128 * 37], 128),
                                               ([4096, 1, 1000, 9999, 128 * 37], 384)],
                         ids=["five", "many_short", "five_page128", "five_page384"])
def test_index_full_fp4_scores_ragged(csa2, lengths, page_size):
    B = len(lengths)
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=B, page_size=page_size, shuffle_pages=True)
    from kv_cache_decode_index_b200.fill import build_cache
    cache = build_cache(wl, csa2, lengths=lengths, fp4_indexer=True)
    q, w = W.index_query(wl, 0)
    dev = cache.device
    bm = torch.full((B, cache.capacity // 8), float("nan"), device=dev)
    sc = torch.full((B, cache.capacity), float("nan"), device=dev)
    hist = csa2.pool_hist(cache)
    csa2.index_full_fp4(cache, cache.ik4, torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev), bm, sc, hist)
    assert csa2.get_error(cache)[0] == csa2.OK
    bm, sc, h = bm.cpu().numpy(), sc.cpu().numpy(), hist.cpu().numpy()
    worst = 0.0
    for b, n in enumerate(lengths):
        codes, scales = _oracle_fp4(wl, b, n)
        s64 = C.indexer_scores_fp4(q[b], w[b], codes, scales)
        err = np.abs(sc[b, :n].astype(np.float64) - s64)
        assert np.all(err <= _fp4_bound(q[b], w[b], codes, scales) + 1e-30), f"request {b}: score beyond the bound"
        worst = max(worst, float((err / np.maximum(s64, 1e-30)).max()))
        assert np.all(np.isnan(sc[b, n:]))
        nb = -(-n // 8)
        np.testing.assert_array_equal(bm[b, :nb].astype(np.float64), C.block_max(sc[b, :n].astype(np.float64), n))
        assert np.all(np.isnan(bm[b, nb:]))
        keys = bm[b, :nb].view(np.uint32).astype(np.uint64)
        keys = np.where(keys & 0x80000000, ~keys & 0xFFFFFFFF, keys | 0x80000000)
        np.testing.assert_array_equal(h[b], np.bincount(keys >> HIST_SHIFT, minlength=1 << (32 - HIST_SHIFT)))
    print(f"FP4 scan: max relative score error {worst:.3e}")


@pytest.mark.parametrize("n_layers,lengths", [(3, [65536, 20000, 4000]), (4, [30000]), (1, [65536, 9000])])
def test_reindex_layers_fp4_parity(csa2, n_layers, lengths):
    """Every layer's Top-k over a pool against the oracle's FP4 scores (tie
    band), on two calls in a row; a Full layer's Top-k equals the Top-k of
    its own FP4 scan's stored scores."""
    from kv_cache_decode_index_b200.fill import build_cache
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=len(lengths), shuffle_pages=True)
    cache = build_cache(wl, csa2, lengths=lengths, fp4_indexer=True)
    rng = np.random.default_rng(60 + n_layers)
    nb = [-(-n // 8) for n in lengths]
    pool = np.full((len(lengths), 2048), -1, np.int32)
    for b, k in enumerate(nb):
        ids = np.sort(rng.choice(k, size=min(2048, k), replace=False))
        pool[b, :len(ids)] = ids
    dev = cache.device
    tp = torch.from_numpy(pool).to(dev)
    qs, ws = [], []
    for layer in range(n_layers):
        q, w = W.index_query(wl, layer)
        qs.append(q)
        ws.append(w)
    tq = [torch.from_numpy(x).to(dev) for x in qs]
    tw = [torch.from_numpy(x).to(dev) for x in ws]
    wsb = torch.zeros(csa2.reindex_layers_workspace_bytes(len(lengths), n_layers, 2048), dtype=torch.uint8, device=dev)
    first = [t.cpu().numpy() for t in csa2.reindex_layers(cache, tp, tq, tw, 512, workspace=wsb, ik4=cache.ik4)]
    second = [t.cpu().numpy() for t in csa2.reindex_layers(cache, tp, tq, tw, 512, workspace=wsb, ik4=cache.ik4)]
    for l in range(n_layers):
        np.testing.assert_array_equal(first[l], second[l])
    assert csa2.get_error(cache)[0] == csa2.OK
    for b, n in enumerate(lengths):
        codes, scales = _oracle_fp4(wl, b, n)
        cand = C.pool_positions(pool[b], n)
        for l in range(n_layers):
            s64 = C.indexer_scores_fp4(qs[l][b], ws[l][b], codes[cand], scales[cand])
            ref = C.top_k_ascending(cand, s64, 512)
            score_of = dict(zip(cand.tolist(), s64.tolist())).get
            U.assert_sorted_padded(first[l][b], f"layer {l} b={b}")
            U.assert_set_parity(first[l][b], ref, score_of, U.threshold(s64, 512), what=f"fp4 reindex l={l} b={b}")
    sc = torch.empty(len(lengths), cache.capacity, device=dev)
    csa2.index_full_fp4(cache, cache.ik4, tq[0], tw[0], scores=sc)
    full_st = csa2.reindex(cache, csa2.FULL, 512, tp, full_scores=sc).cpu().numpy()
    np.testing.assert_array_equal(first[0], full_st)


def test_group_fp4_64k_b8(csa2):
    """The decode group (1 Full + 2 Reindex + 3 Reuse, pool 2048 x 8, 64 heads)
    over the FP4 indexer: pool and every layer's Top-k against the oracle's FP4
    scores, attention fed the oracle's indices."""
    from kv_cache_decode_index_b200.fill import build_cache
    wl = W.WORKLOADS["group_64k_b8"]
    cache = build_cache(wl, csa2, fp4_indexer=True)
    dev = cache.device
    q_idx, w_idx, tq, tw, tm = [], [], [], [], []
    for layer, m in enumerate(wl.modes):
        if m == "Ru":
            q_idx.append(None)
            w_idx.append(None)
            tq.append(None)
            tw.append(None)
        else:
            q, w = W.index_query(wl, layer)
            q_idx.append(q)
            w_idx.append(w)
            tq.append(torch.from_numpy(q).to(dev))
            tw.append(torch.from_numpy(w).to(dev))
        tm.append(W.main_query(wl, layer).to(dev))
    out = [torch.empty_like(m) for m in tm]
    group = csa2.DecodeGroup(cache, wl.modes, wl.heads, wl.topk, wl.pool_blocks, wl.scale, ik4=cache.ik4)
    group.step(tq, tw, tm, out)
    torch.cuda.synchronize()
    assert csa2.get_error(cache)[0] == csa2.OK
    n = wl.ctx
    for b in range(wl.batch):
        codes, scales = _oracle_fp4(wl, b, n)
        s_full = C.indexer_scores_fp4(q_idx[0][b], w_idx[0][b], codes, scales)
        bm64 = C.block_max(s_full, n)
        pool64 = C.pool_select(bm64, wl.pool_blocks)
        gp = group.pool[b].cpu().numpy()
        U.assert_sorted_padded(gp, f"pool b={b}")
        U.assert_set_parity(gp, pool64, lambda j: bm64[j], U.threshold(bm64, wl.pool_blocks), what=f"fp4 pool b={b}")
        pool_diff = set(gp[gp >= 0].tolist()) ^ set(pool64[pool64 >= 0].tolist())
        excused = lambda t: (t // 8) in pool_diff
        gpu_pool_pos = set(C.pool_positions(gp, n).tolist())
        cand = C.pool_positions(pool64, n)
        for layer, m in enumerate(wl.modes):
            gt = group.topk[layer][b].cpu().numpy()
            U.assert_sorted_padded(gt, f"topk layer {layer} b={b}")
            if m == "Ru":
                np.testing.assert_array_equal(gt, group.topk[layer - 1][b].cpu().numpy())
                continue
            assert set(gt[gt >= 0].tolist()) <= gpu_pool_pos
            s = s_full if m == "F" else C.indexer_scores_fp4(q_idx[layer][b], w_idx[layer][b], codes, scales)
            ref = C.top_k_ascending(cand, s[cand], wl.topk)
            U.assert_set_parity(gt, ref, lambda t: s[t], U.threshold(s[cand], wl.topk), excused,
                                what=f"fp4 topk layer {layer} ({m}) b={b}")
    # attention over the group's own Top-k equals the FP8 group's attention kernel on the same indices
    for layer in range(len(wl.modes)):
        ref = csa2.sparse_attn(cache, group.topk[layer], tm[layer], wl.scale)
        assert torch.equal(ref, out[layer]), f"attention layer {layer}"
