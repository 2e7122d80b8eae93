"""Stage-by-stage parity of the CUDA kernels (through the C ABI) against the
float64 oracle, on the same seeded inputs.  Needs a B200 and libcsa2.so."""
import json
import os

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


def _flat_cache(csa2, rows, batch=1, page_size=512):
    """One request (or `batch` requests) over contiguous pages, no data."""
    per = -(-rows // page_size)
    table = np.arange(batch * per, dtype=np.int32).reshape(batch, per)
    return csa2.Cache(batch * per, page_size, table, [rows] * batch)


# ------------------------------------------------------------ append (a1) --

def _special_kv_rows(rng, golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "fp4_hand_cases.json")) as f:
        for g in json.load(f)["groups"]:
            r = np.zeros(512, np.float32)
            r[:16] = g["x"]
            rows.append(r)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1, 1.5, 2, 3, 4, 6, 0, 7])
    for _ in range(64):
        r = np.zeros(512, np.float32)
        for g in range(32):
            c = rng.integers(1, 127)
            s = F.e4m3_value(c)
            v = rng.choice(mids, 16) * s * rng.choice([-1, 1], 16)
            v[rng.integers(16)] = 6 * s                      # amax/6 = s exactly
            if g % 4 == 0 and c < 126:                        # amax/6 on an E4M3 midpoint
                v[0] = 3 * (s + F.e4m3_value(c + 1))
            r[16 * g:16 * g + 16] = v
        rows.append(r)
    rows.append(np.zeros(512, np.float32))
    rows.append(np.full(512, -0.0, np.float32))
    return np.stack(rows).astype(np.float32)


def _special_ik_rows(rng, golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "fp8_indexer_hand_cases.json")) as f:
        for g in json.load(f)["rows"]:
            r = np.zeros(128, np.float32)
            r[:len(g["k_head"])] = g["k_head"]
            rows.append(r)
    vals = np.unique(np.abs(F.e4m3_value(np.arange(127))))
    mids = (vals[:-1] + vals[1:]) / 2
    for _ in range(64):
        e = rng.integers(-20, 20)
        r = rng.choice(np.concatenate([vals, mids]), 128) * np.exp2(float(e)) * rng.choice([-1, 1], 128)
        r[rng.integers(128)] = 448 * np.exp2(float(e))
        rows.append(r)
    rows += [np.zeros(128), np.full(128, 1e-40), np.full(128, 3e38)]
    return np.stack(rows).astype(np.float32)


def test_append_bitexact(csa2, golden_dir):
    rng = np.random.default_rng(0)
    kv_s = _special_kv_rows(rng, golden_dir)
    ik_s = _special_ik_rows(rng, golden_dir)
    n_rand = 700
    kv = np.concatenate([kv_s, (rng.standard_normal((n_rand, 512)) *
                                np.exp(rng.standard_normal(512) * 2)).astype(np.float32)])
    ik = np.concatenate([ik_s, (rng.standard_normal((n_rand + len(kv_s) - len(ik_s), 128)) *
                                np.exp(rng.uniform(-25, 25, (n_rand + len(kv_s) - len(ik_s), 1)))).astype(np.float32)])
    n = len(kv)
    cache = _flat_cache(csa2, n)
    dev = cache.device
    perm = rng.permutation(n).astype(np.int32)          # scattered positions
    csa2.append_kv(cache, torch.from_numpy(kv).to(dev), torch.from_numpy(ik).to(dev),
                   torch.from_numpy(perm).to(dev), torch.zeros(n, dtype=torch.int32, device=dev))
    codes, scales = F.quantize_main_kv(kv)
    ikc, ike = F.quantize_indexer(ik)
    inv = np.argsort(perm)
    g_codes = cache.kv_codes[:n].cpu().numpy()[perm]
    g_scales = cache.kv_scales[:n].cpu().numpy()[perm]
    g_ikc = cache.ik_codes[:n].cpu().numpy()[perm]
    g_ike = cache.ik_exp[:n].cpu().numpy()[perm]
    np.testing.assert_array_equal(g_scales, scales)
    np.testing.assert_array_equal(g_codes, codes)
    np.testing.assert_array_equal(g_ike, ike)
    np.testing.assert_array_equal(g_ikc, ikc)
    assert inv is not None
    assert csa2.get_error(cache)[0] == csa2.OK


@pytest.mark.parametrize("m", [1, 2, 4, 8])
def test_compress_append_bitexact(csa2, golden_dir, m):
    """Sequence compressor + quantise-on-append against the oracle's mean and
    quantisation: codes, scales, indexer codes and exponents bit-exact.  The
    first entries are the special rows of the append test written as m equal
    tokens (their mean is the row itself), then pairs of tokens whose mean
    lands exactly on E2M1 midpoints, then log-normal random tokens."""
    rng = np.random.default_rng(40 + m)
    kv_s = _special_kv_rows(rng, golden_dir)
    ik_s = _special_ik_rows(rng, golden_dir)
    n_s = min(len(kv_s), len(ik_s))
    kv_tok = [np.repeat(kv_s[:n_s], m, axis=0)]
    ik_tok = [np.repeat(ik_s[:n_s], m, axis=0)]
    if m >= 2:
        # mean exactly on a midpoint of the E2M1 grid (scale s = 1 by a 6 in the group)
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
        for _ in range(16):
            base = np.zeros((m, 512), np.float32)
            base[:, ::16] = 6.0
            target = rng.choice(mids, (512,)) * rng.choice([-1.0, 1.0], (512,))
            d = rng.integers(-8, 9, 512).astype(np.float32) * np.float32(0.0625)   # target +- d exact in fp32
            base[0] += target + d
            base[1] += target - d
            base[2:] += target
            base[:, ::16] = 6.0
            kv_tok.append(base)
            ik_tok.append(np.repeat(rng.standard_normal((1, 128)).astype(np.float32), m, axis=0))
    n_rand = 300
    kv_tok.append((rng.standard_normal((n_rand * m, 512)) * np.exp(rng.standard_normal(512) * 2)).astype(np.float32))
    ik_tok.append((rng.standard_normal((n_rand * m, 128)) *
                   np.exp(rng.uniform(-20, 20, (n_rand * m, 1)))).astype(np.float32))
    kv_tok = np.concatenate(kv_tok)
    ik_tok = np.concatenate(ik_tok)
    n = kv_tok.shape[0] // m
    cache = _flat_cache(csa2, n)
    dev = cache.device
    perm = rng.permutation(n).astype(np.int32)
    csa2.compress_append(cache, torch.from_numpy(kv_tok).to(dev), torch.from_numpy(ik_tok).to(dev),
                         torch.from_numpy(perm).to(dev), m=m)
    kv_e = C.compress_tokens(kv_tok, m)
    ik_e = C.compress_tokens(ik_tok, m)
    codes, scales = F.quantize_main_kv(kv_e)
    ikc, ike = F.quantize_indexer(ik_e)
    np.testing.assert_array_equal(cache.kv_scales[:n].cpu().numpy()[perm], scales)
    np.testing.assert_array_equal(cache.kv_codes[:n].cpu().numpy()[perm], codes)
    np.testing.assert_array_equal(cache.ik_exp[:n].cpu().numpy()[perm], ike)
    np.testing.assert_array_equal(cache.ik_codes[:n].cpu().numpy()[perm], ikc)
    assert csa2.get_error(cache)[0] == csa2.OK


def test_append_one_row_per_request(csa2):
    """req = NULL: row i goes to request i (the decode-step append)."""
    rng = np.random.default_rng(1)
    B = 5
    cache = _flat_cache(csa2, 256, batch=B, page_size=128)
    kv = rng.standard_normal((B, 512)).astype(np.float32)
    ik = rng.standard_normal((B, 128)).astype(np.float32)
    pos = np.array([0, 255, 128, 7, 200], np.int32)
    dev = cache.device
    csa2.append_kv(cache, torch.from_numpy(kv).to(dev), torch.from_numpy(ik).to(dev), torch.from_numpy(pos).to(dev))
    codes, scales = F.quantize_main_kv(kv)
    ikc, ike = F.quantize_indexer(ik)
    for b in range(B):
        row = int(cache.rows_of(b, [pos[b]])[0])
        np.testing.assert_array_equal(cache.kv_codes[row].cpu().numpy(), codes[b])
        np.testing.assert_array_equal(cache.kv_scales[row].cpu().numpy(), scales[b])
        np.testing.assert_array_equal(cache.ik_codes[row].cpu().numpy(), ikc[b])
        assert int(cache.ik_exp[row]) == int(ike[b])


# --------------------------------------------------------- index_full (a2) --

def _score_bound(q, w, codes, exp):
    """fp32 error bound of the tensor-core score: every head dot product within
    2^-22 of its absolute sum, plus the 32-term fp32 sum (32 * 2^-24)."""
    qc, sq = C.quantize_index_query(q)
    qa = np.abs(F.e4m3_value(qc))
    ka = np.abs(F.e4m3_value(codes))
    absdot = ka @ qa.T * sq
    sig = F.indexer_sigma(exp)
    w64 = np.abs(w.astype(np.float64))
    return sig * (absdot @ w64) * 2.0 ** -22 * 2, sig


# Many short requests: about four requests per CTA's range of units, so the
# scan's query-code buffers rotate (segment x in buffer x % 3) inside a CTA.
MANY_SHORT = [int(n) for n in np.random.default_rng(77).integers(1, 1100, size=600)]


# Pages of 128 or 384 rows: a unit's two tiles on two pages (or the second
# absent), copied tile by tile instead of in one 256-row box.
@pytest.mark.parametrize("lengths,page_size", [([4096, 1, 1000, 9999, 128 * 37], 512), (MANY_SHORT, 512),
                                               ([4096, 1, 1000, 9999, 128 * 37], 128),
                                               ([4096, 1, 1000, 9999, 128 * 37], 384)],
                         ids=["five", "many_short", "five_page128", "five_page384"])
def test_index_full_scores_ragged(csa2, lengths, page_size):
    B = len(lengths)
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=B, page_size=page_size, shuffle_pages=True)
    cache = U.build_cache(wl, csa2, lengths=lengths)
    q, w = W.index_query(wl, 0)
    dev = cache.device
    bm = torch.full((B, cache.capacity // 8), float("nan"), device=dev)
    sc = torch.full((B, cache.capacity), float("nan"), device=dev)
    csa2.index_full(cache, torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev), bm, sc)
    bm, sc = bm.cpu().numpy(), sc.cpu().numpy()
    worst = 0.0
    for b, n in enumerate(lengths):
        codes, exp = U.oracle_request(wl, b, n)
        s64 = C.indexer_scores(q[b], w[b], codes, exp)
        bound, _ = _score_bound(q[b], w[b], codes, exp)
        err = np.abs(sc[b, :n].astype(np.float64) - s64)
        assert np.all(err <= bound + 1e-30), f"request {b}: score error beyond the fp32 bound"
        worst = max(worst, float((err / np.maximum(s64, 1e-30)).max()))
        assert np.all(np.isnan(sc[b, n:]))                          # nothing written past ctx
        nb = -(-n // 8)
        ref = C.block_max(sc[b, :n].astype(np.float64), n)
        np.testing.assert_array_equal(bm[b, :nb].astype(np.float64), ref)   # GPU blockmax = max of GPU scores
        assert np.all(np.isnan(bm[b, nb:]))
        bm64 = C.block_max(s64, n)
        assert np.all(np.abs(bm[b, :nb] - bm64) <= np.abs(bm64) * 1e-5)
    print(f"max relative score error {worst:.3e}")
    assert csa2.get_error(cache)[0] == csa2.OK


# ------------------------------------------------------- pool_select (a3) --

@pytest.mark.parametrize("lengths,P,kind", [([1048576, 300000], 2048, "ties"), ([16384, 16383, 8, 0], 2048, "ties"),
                                            ([200000, 5000], 64, "ties"), ([1500000], 2048, "ties"),
                                            ([1048576, 700000], 2048, "on_sample_grid"),
                                            ([1048576], 2048, "all_equal")])
def test_pool_select_bitexact(csa2, lengths, P, kind):
    """Synthetic block maxima with many ties (and negative values), fed to both.
    "on_sample_grid": 4096 evenly spaced blocks far above the rest, in a few
    histogram bins; "all_equal": every block ties (the threshold's bin holds
    every block: more keys than the kernel gathers in one CTA, so it takes
    the general cluster select)."""
    rng = np.random.default_rng(len(lengths) * 1000 + P)
    B = len(lengths)
    page = 4096
    per = max(-(-max(lengths) // page), 1)
    table = np.arange(B * per, dtype=np.int32).reshape(B, per)
    cache = csa2.Cache(B * per, page, table, lengths)
    cap8 = cache.capacity // 8
    vals = rng.standard_normal((B, cap8)).astype(np.float32)
    vals[:, ::3] = np.round(vals[:, ::3] * 4) / 4                       # ties
    vals[:, 5::7] = 2.0                                                  # a big tie group
    if kind == "on_sample_grid":
        for b, n in enumerate(lengths):
            nb = -(-n // 8)
            grid = (np.arange(4096, dtype=np.int64) * nb) // 4096
            vals[b, grid] = 100.0 + rng.random(4096).astype(np.float32)
    elif kind == "all_equal":
        vals[:] = 3.5
    dev = cache.device
    tv = torch.from_numpy(vals).to(dev)
    pool = csa2.pool_select(cache, tv, P).cpu().numpy()
    for b, n in enumerate(lengths):
        nb = -(-n // 8)
        ref = C.pool_select(vals[b, :nb].astype(np.float64), P)
        np.testing.assert_array_equal(pool[b], ref, err_msg=f"request {b} (n={n})")
    # with the block maxima's histogram (as the scan writes it): the same pool,
    # and the histogram is left zeroed; a histogram that does not match the
    # block maxima (stale) is ignored, with the same result
    hist = np.zeros((B, csa2.POOL_HIST_BINS), np.int64)
    for b, n in enumerate(lengths):
        hist[b] = np.bincount(_order_keys(vals[b, :-(-n // 8)]) >> HIST_SHIFT, minlength=1 << (32 - HIST_SHIFT))
    th = torch.from_numpy(hist.astype(np.int32)).to(dev)
    pool_h = csa2.pool_select(cache, tv, P, hist=th).cpu().numpy()
    np.testing.assert_array_equal(pool_h, pool)
    assert int(th.abs().sum()) == 0
    th = torch.from_numpy((hist + rng.integers(0, 3, hist.shape)).astype(np.int32)).to(dev)
    np.testing.assert_array_equal(csa2.pool_select(cache, tv, P, hist=th).cpu().numpy(), pool)
    assert int(th.abs().sum()) == 0
    # the right total in the wrong bin (every count in the top bin): the
    # per-CTA counts of the bin's keys contradict it, and the result is exact
    wrong = np.zeros_like(hist)
    wrong[:, -1] = hist.sum(axis=1)
    th = torch.from_numpy(wrong.astype(np.int32)).to(dev)
    np.testing.assert_array_equal(csa2.pool_select(cache, tv, P, hist=th).cpu().numpy(), pool)
    assert int(th.abs().sum()) == 0
    assert csa2.get_error(cache)[0] == csa2.OK


def _order_keys(v):
    """The kernels' order-preserving uint32 key of an fp32 score (sign bit
    flipped for positive values, all bits for negative ones; 0 -> 1)."""
    bits = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    k = np.where(bits & 0x80000000, ~bits & 0xFFFFFFFF, bits | 0x80000000)
    return np.where(k == 0, 1, k).astype(np.uint64)


def test_scan_histogram_drives_the_pool(csa2):
    """The scan's histogram holds one count per visible block in the bin of
    its block max's leading 12 key bits; the pool selected from it equals the
    pool selected without it, and the histogram is zero again afterwards."""
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=3, page_size=512, shuffle_pages=True)
    lengths = [65536, 40001, 777]
    cache = U.build_cache(wl, csa2, lengths=lengths)
    q, w = W.index_query(wl, 0)
    dev = cache.device
    tq, tw = torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev)
    hist = csa2.pool_hist(cache)
    bm = csa2.index_full(cache, tq, tw, hist=hist)
    h = hist.cpu().numpy().astype(np.int64)
    bmh = bm.cpu().numpy()
    for b, n in enumerate(lengths):
        want = np.bincount(_order_keys(bmh[b, :-(-n // 8)]) >> HIST_SHIFT, minlength=1 << (32 - HIST_SHIFT))
        np.testing.assert_array_equal(h[b], want, err_msg=f"request {b}")
    pool_h = csa2.pool_select(cache, bm, 512, hist=hist)
    assert int(hist.abs().sum()) == 0
    pool = csa2.pool_select(cache, bm, 512)
    assert torch.equal(pool_h, pool)
    assert csa2.get_error(cache)[0] == csa2.OK


# ---------------------------------------------------------- reindex (a4-a6) --

def _synthetic_pool(rng, n, P):
    nb = -(-n // 8)
    k = min(P, nb)
    ids = np.sort(rng.choice(nb, size=k, replace=False)) if nb else np.zeros(0, np.int64)
    out = np.full(P, -1, np.int32)
    out[:k] = ids
    return out


def test_full_topk_from_stored_scores_bitexact(csa2):
    rng = np.random.default_rng(3)
    lengths = [65536, 3000, 100]
    B, page = 3, 4096
    per = 16
    cache = csa2.Cache(B * per, page, np.arange(B * per, dtype=np.int32).reshape(B, per), lengths)
    scores = rng.standard_normal((B, cache.capacity)).astype(np.float32)
    scores[:, ::5] = np.round(scores[:, ::5])                       # ties
    pool = np.stack([_synthetic_pool(rng, n, 2048) for n in lengths])
    dev = cache.device
    topk = csa2.reindex(cache, csa2.FULL, 512, torch.from_numpy(pool).to(dev),
                        full_scores=torch.from_numpy(scores).to(dev)).cpu().numpy()
    for b, n in enumerate(lengths):
        ref = C.full_topk(scores[b].astype(np.float64), pool[b], n, 512)
        np.testing.assert_array_equal(topk[b], ref, err_msg=f"request {b}")
    # without a pool: flat Top-k over every visible position
    cache2 = csa2.Cache(B * 4, page, np.arange(B * 4, dtype=np.int32).reshape(B, 4), [16384, 5000, 100])
    sc2 = scores[:, :cache2.capacity].copy()
    topk2 = csa2.reindex(cache2, csa2.FULL, 512, None, full_scores=torch.from_numpy(sc2).to(dev)).cpu().numpy()
    for b, n in enumerate([16384, 5000, 100]):
        np.testing.assert_array_equal(topk2[b], C.full_topk(sc2[b].astype(np.float64), None, n, 512))


def test_reindex_rescore_parity(csa2):
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=3, shuffle_pages=True)
    lengths = [65536, 20000, 4000]
    cache = U.build_cache(wl, csa2, lengths=lengths)
    rng = np.random.default_rng(4)
    pool = np.stack([_synthetic_pool(rng, n, 2048) for n in lengths])
    q, w = W.index_query(wl, 1)
    dev = cache.device
    tq, tw, tp = torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev), torch.from_numpy(pool).to(dev)
    topk = csa2.reindex(cache, csa2.REINDEX, 512, tp, tq, tw).cpu().numpy()
    # Full recompute: same arithmetic as the scan -> identical to Top-k of the scan's scores
    sc = torch.empty(3, cache.capacity, device=dev)
    csa2.index_full(cache, tq, tw, scores=sc)
    full_re = csa2.reindex(cache, csa2.FULL, 512, tp, tq, tw).cpu().numpy()
    full_st = csa2.reindex(cache, csa2.FULL, 512, tp, full_scores=sc).cpu().numpy()
    np.testing.assert_array_equal(full_re, full_st)
    np.testing.assert_array_equal(full_re, topk)
    for b, n in enumerate(lengths):
        codes, exp = U.oracle_request(wl, b, n)
        ref = C.reindex_topk(q[b], w[b], codes, exp, pool[b], n, 512)
        cand = C.pool_positions(pool[b], n)
        s64 = C.indexer_scores(q[b], w[b], codes[cand], exp[cand])
        score_of = dict(zip(cand.tolist(), s64.tolist())).get
        U.assert_sorted_padded(topk[b], f"request {b}")
        assert set(topk[b][topk[b] >= 0]) <= set(cand.tolist())
        U.assert_set_parity(topk[b], ref, score_of, U.threshold(s64, 512), what=f"reindex b={b}")


@pytest.mark.parametrize("n_layers,lengths,P", [(3, [65536, 20000, 4000], 2048), (5, [65536, 3001], 2048),
                                                 (8, [9000, 300], 64), (1, [65536], 1000)])
def test_reindex_layers_equal_per_layer_reindex(csa2, n_layers, lengths, P):
    """csa2_reindex_layers (all layers gathered and scored at once, histogram
    select) returns for every layer exactly what csa2_reindex returns for that
    layer alone, on two calls in a row with the same workspace (whose
    histograms each call leaves zeroed) and with a workspace whose histograms
    were not zero; the first layer is checked against the oracle too."""
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=len(lengths), shuffle_pages=True)
    cache = U.build_cache(wl, csa2, lengths=lengths)
    rng = np.random.default_rng(40 + n_layers)
    pool = np.stack([_synthetic_pool(rng, n, P) for n in lengths])
    dev = cache.device
    tp = torch.from_numpy(pool).to(dev)
    qs, ws = [], []
    for layer in range(n_layers):
        q, w = W.index_query(wl, layer)
        qs.append(torch.from_numpy(q).to(dev))
        ws.append(torch.from_numpy(w).to(dev))
    want = [csa2.reindex(cache, csa2.REINDEX, 512, tp, qs[l], ws[l]).cpu().numpy() for l in range(n_layers)]
    B = len(lengths)
    nbytes = csa2.reindex_layers_workspace_bytes(B, n_layers, P)
    ws_buf = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    hist_part = ws_buf[B * n_layers * P * 8 * 4:]
    for attempt in range(3):
        if attempt == 2:   # histograms that do not match the keys
            hist_part.copy_(torch.randint(0, 255, hist_part.shape, dtype=torch.uint8, device=dev))
        got = csa2.reindex_layers(cache, tp, qs, ws, 512, workspace=ws_buf)
        for l in range(n_layers):
            np.testing.assert_array_equal(got[l].cpu().numpy(), want[l], err_msg=f"layer {l}, call {attempt}")
        assert int(hist_part.sum()) == 0
    assert csa2.get_error(cache)[0] == csa2.OK
    q0, w0 = W.index_query(wl, 0)
    for b, n in enumerate(lengths):
        codes, exp = U.oracle_request(wl, b, n)
        cand = C.pool_positions(pool[b], n)
        s64 = C.indexer_scores(q0[b], w0[b], codes[cand], exp[cand])
        score_of = dict(zip(cand.tolist(), s64.tolist())).get
        U.assert_sorted_padded(want[0][b], f"request {b}")
        U.assert_set_parity(want[0][b], C.reindex_topk(q0[b], w0[b], codes, exp, pool[b], n, 512), score_of,
                            U.threshold(s64, 512), what=f"reindex_layers b={b}")


def test_reindex_layers_full_layer_equals_stored_scores(csa2):
    """A Full layer's Top-k from csa2_reindex_layers equals the Top-k of its
    own scan's stored scores (bit-identical scoring arithmetic)."""
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=2, shuffle_pages=True)
    lengths = [65536, 12345]
    cache = U.build_cache(wl, csa2, lengths=lengths)
    dev = cache.device
    q, w = W.index_query(wl, 0)
    q1, w1 = W.index_query(wl, 1)
    tq, tw = torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev)
    sc = torch.empty(2, cache.capacity, device=dev)
    bm = csa2.index_full(cache, tq, tw, scores=sc)
    pool = csa2.pool_select(cache, bm, 2048)
    full_st = csa2.reindex(cache, csa2.FULL, 512, pool, full_scores=sc)
    got = csa2.reindex_layers(cache, pool, [tq, torch.from_numpy(q1).to(dev)], [tw, torch.from_numpy(w1).to(dev)], 512)
    assert torch.equal(got[0], full_st)


def test_reuse_copy_and_alias(csa2):
    cache = _flat_cache(csa2, 1024, batch=2)
    dev = cache.device
    prev = torch.randint(-1, 1000, (2, 512), dtype=torch.int32, device=dev)
    out = torch.zeros_like(prev)
    csa2.reindex(cache, csa2.REUSE, 512, prev_topk=prev, topk=out)
    assert torch.equal(out, prev)
    same = prev.clone()
    csa2.reindex(cache, csa2.REUSE, 512, prev_topk=same, topk=same)
    assert torch.equal(same, prev)


# ------------------------------------------------------------ attention (a7) --

@pytest.mark.parametrize("H,k,n", [(64, 512, 65536), (16, 512, 4096), (32, 100, 3000), (64, 7, 50),
                                   (16, 1024, 9000), (64, 512, 300)])
def test_sparse_attention_parity(csa2, H, k, n):
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=3, heads=H, page_size=1024, shuffle_pages=True, seed=11 + k)
    lengths = [n, max(n // 3, 1), n]
    cache = U.build_cache(wl, csa2, lengths=lengths)
    rng = np.random.default_rng(H + k)
    topk = np.full((3, k), -1, np.int32)
    for b, nb in enumerate(lengths):
        m = min(k, nb) - (1 if b == 1 and min(k, nb) > 1 else 0)     # request 1 keeps some -1 padding
        topk[b, :m] = np.sort(rng.choice(nb, m, replace=False))
    topk[2] = rng.permutation(topk[2])                                # order must not matter
    qm = W.main_query(wl, 0)
    dev = cache.device
    out = csa2.sparse_attn(cache, torch.from_numpy(topk).to(dev), qm.to(dev), wl.scale).float().cpu().numpy()
    for b, nb in enumerate(lengths):
        sel = np.unique(topk[b][topk[b] >= 0])
        codes, scales = U.oracle_kv_rows(wl, b, sel)
        full_codes = np.zeros((nb, 256), np.uint8)
        full_scales = np.zeros((nb, 32), np.uint8)
        full_codes[sel], full_scales[sel] = codes, scales
        ref = C.sparse_attention(qm[b].float().numpy(), full_codes, full_scales, topk[b], wl.scale)
        rel = U.assert_attention_close(out[b], ref, f"H={H} k={k} b={b}")
        print(f"H={H} k={k} b={b}: max rel err {rel:.2e}")


def test_sparse_attention_layers_with_their_own_topk(csa2):
    """One launch over layers with different Top-k equals one launch per layer."""
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=3)
    cache = U.build_cache(wl, csa2, lengths=[65536, 4000, 700])
    dev = cache.device
    rng = np.random.default_rng(11)
    tks, qs = [], []
    for layer in range(5):
        t = np.stack([np.sort(rng.choice(n, 512, replace=False)) for n in (65536, 4000, 700)]).astype(np.int32)
        t[2, 300:] = -1
        tks.append(torch.from_numpy(t).to(dev))
        qs.append(W.main_query(wl, layer).to(dev))
    ws = torch.empty(csa2.attn_workspace_bytes(5, 3, 64), dtype=torch.uint8, device=dev)
    multi = csa2.sparse_attn_layers(cache, tks, qs, wl.scale, workspace=ws)
    for layer in range(5):
        single = csa2.sparse_attn(cache, tks[layer], qs[layer], wl.scale)
        assert torch.equal(multi[layer], single), f"layer {layer}"
    assert csa2.get_error(cache)[0] == csa2.OK


def test_sparse_attention_layers_equal_single_layer_launches(csa2):
    """One launch over four layers sharing the Top-k (a Reindex layer and its
    Reuse layers) gives, per layer, exactly the single-layer launch's output."""
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=3, ctx=4000, heads=32)
    cache = U.build_cache(wl, csa2)
    dev = cache.device
    rng = np.random.default_rng(17)
    topk = torch.from_numpy(np.stack([np.sort(rng.choice(4000, 300, replace=False)) for _ in range(3)])
                            .astype(np.int32)).to(dev)
    qs = [W.main_query(wl, layer).to(dev) for layer in range(4)]
    multi = csa2.sparse_attn_layers(cache, topk, qs, wl.scale)
    for layer in range(4):
        single = csa2.sparse_attn(cache, topk, qs[layer], wl.scale)
        assert torch.equal(multi[layer], single), f"layer {layer}"
    assert csa2.get_error(cache)[0] == csa2.OK


@pytest.mark.parametrize("H,k,n_layers", [(64, 512, 4), (16, 300, 2), (32, 77, 1)])
def test_sparse_attention_workspace_exchange_is_bit_identical(csa2, H, k, n_layers):
    """The key splits merging through the caller's workspace (L2) give exactly
    the output of the merge through distributed shared memory; ragged Top-k
    with -1 padding, a query with no valid entry."""
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=3, ctx=5000, heads=H)
    cache = U.build_cache(wl, csa2)
    dev = cache.device
    rng = np.random.default_rng(23 + H)
    topk = np.stack([np.sort(rng.choice(5000, k, replace=False)) for _ in range(3)]).astype(np.int32)
    topk[1, k // 3:] = -1
    topk[2, :] = -1
    topk = torch.from_numpy(topk).to(dev)
    qs = [W.main_query(wl, layer).to(dev) for layer in range(n_layers)]
    ws = torch.full((csa2.attn_workspace_bytes(n_layers, 3, H),), 0xFF, dtype=torch.uint8, device=dev)
    via_smem = csa2.sparse_attn_layers(cache, topk, qs, wl.scale)
    via_ws = csa2.sparse_attn_layers(cache, topk, qs, wl.scale, workspace=ws)
    for layer in range(n_layers):
        assert torch.equal(via_ws[layer], via_smem[layer]), f"layer {layer}"
        assert torch.all(via_ws[layer][2] == 0), "a query with no valid entry attends to nothing"
    assert csa2.get_error(cache)[0] == csa2.OK


@pytest.mark.parametrize("nq", [8, 13])
def test_sparse_attention_key_splits(csa2, nq):
    """Launches of more queries take 2 (up to 12 queries) or 1 (more) CTAs per
    query instead of 4: parity with the oracle for every query, and the merge
    through the caller's workspace equals the merge through shared memory."""
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=3, ctx=5000, heads=64)
    cache = U.build_cache(wl, csa2)
    dev = cache.device
    rng = np.random.default_rng(31 + nq)
    q_req = (np.arange(nq) % 3).astype(np.int32)
    topk = np.stack([np.sort(rng.choice(5000, 512, replace=False)) for _ in range(nq)]).astype(np.int32)
    topk[1, 200:] = -1
    topk[nq - 1] = rng.permutation(topk[nq - 1])
    tq = torch.from_numpy(q_req).to(dev)
    tk = torch.from_numpy(topk).to(dev)
    qs = [W.main_query(wl, layer, rows=nq) for layer in range(2)]
    out = csa2.sparse_attn(cache, tk, qs[0].to(dev), wl.scale, q_req=tq).float().cpu().numpy()
    rows = {b: U.oracle_kv_rows(wl, b, np.arange(5000)) for b in range(3)}
    for i in range(nq):
        codes, scales = rows[int(q_req[i])]
        ref = C.sparse_attention(qs[0][i].float().numpy(), codes, scales, topk[i], wl.scale)
        U.assert_attention_close(out[i], ref, f"nq={nq} query {i}")
    ws = torch.full((csa2.attn_workspace_bytes(2, nq, 64),), 0xFF, dtype=torch.uint8, device=dev)
    via_smem = csa2.sparse_attn_layers(cache, tk, [q.to(dev) for q in qs], wl.scale, q_req=tq)
    via_ws = csa2.sparse_attn_layers(cache, tk, [q.to(dev) for q in qs], wl.scale, q_req=tq, workspace=ws)
    for layer in range(2):
        assert torch.equal(via_ws[layer], via_smem[layer]), f"layer {layer}"
    np.testing.assert_array_equal(via_smem[0].float().cpu().numpy(), out)
    assert csa2.get_error(cache)[0] == csa2.OK


def test_sparse_attention_empty_and_query_map(csa2):
    wl = W.scaled(W.WORKLOADS["full_4k_b1"], batch=2, heads=16, page_size=1024)
    cache = U.build_cache(wl, csa2, lengths=[2000, 3000])
    dev = cache.device
    rng = np.random.default_rng(5)
    nq = 6
    q_req = np.array([1, 0, 1, 1, 0, 0], np.int32)
    topk = np.full((nq, 64), -1, np.int32)
    for i in range(nq):
        if i != 3:   # query 3: no valid index -> zeros
            nb = [2000, 3000][q_req[i]]
            topk[i, :40] = rng.choice(nb, 40, replace=False)
    qm = W.main_query(wl, 0, rows=nq)
    out = csa2.sparse_attn(cache, torch.from_numpy(topk).to(dev), qm.to(dev), wl.scale,
                           q_req=torch.from_numpy(q_req).to(dev)).float().cpu().numpy()
    assert np.all(out[3] == 0)
    for i in range(nq):
        if i == 3:
            continue
        b = q_req[i]
        nb = [2000, 3000][b]
        codes, scales = U.oracle_kv_rows(wl, b, np.arange(nb))
        ref = C.sparse_attention(qm[i].float().numpy(), codes, scales, topk[i], wl.scale)
        U.assert_attention_close(out[i], ref, f"query {i}")


# ------------------------------------------------------------- error paths --

def test_device_bounds_are_reported_not_trapped(csa2):
    wl = W.scaled(W.WORKLOADS["full_4k_b1"], page_size=1024)
    cache = U.build_cache(wl, csa2, lengths=[4096])
    dev = cache.device
    # an index past the visible context
    topk = torch.tensor([[5, 4096 + 3, -1, 7]], dtype=torch.int32, device=dev)
    csa2.sparse_attn(cache, topk, W.main_query(wl, 0).to(dev), wl.scale)
    st, word = csa2.get_error(cache)
    assert st == csa2.ERR_DEVICE_BOUNDS and word[1] == 5 and word[3] == 4096 + 3
    # a corrupt page id in the page table
    cache.err_word.zero_()
    cache.page_table[0, 2] = 10_000
    q, w = W.index_query(wl, 0)
    csa2.index_full(cache, torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev))
    st, word = csa2.get_error(cache)
    assert st == csa2.ERR_DEVICE_BOUNDS and word[1] == 2
    # the context is still usable
    cache.page_table[0, 2] = 2
    cache.err_word.zero_()
    csa2.index_full(cache, torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev))
    assert csa2.get_error(cache)[0] == csa2.OK


@pytest.mark.parametrize("bad_len", [4096 + 1, -5])
def test_corrupt_length_is_reported_and_the_request_skipped(csa2, bad_len):
    """A ctx_len outside [0, capacity] must not truncate the request silently:
    every kernel that reads it records CSA2_ERR_DEVICE_BOUNDS (index = the
    length) and treats the request as empty, while the other requests of the
    call are computed normally."""
    wl = W.scaled(W.WORKLOADS["full_4k_b1"], page_size=1024, batch=2)
    cache = U.build_cache(wl, csa2, lengths=[4096, 4096])
    dev = cache.device
    q, w = W.index_query(wl, 0)
    tq, tw = torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev)
    good_bm = csa2.index_full(cache, tq, tw).clone()
    good_pool = csa2.pool_select(cache, good_bm, 64).clone()
    assert csa2.get_error(cache)[0] == csa2.OK
    cache.ctx_len[1] = bad_len

    def expect_bounds(kernel_id):
        st, word = csa2.get_error(cache)
        assert st == csa2.ERR_DEVICE_BOUNDS and word[1] == kernel_id and word[2] == 1 and word[3] == bad_len, word
        cache.err_word.zero_()

    bm = torch.full_like(good_bm, -7.0)
    csa2.index_full(cache, tq, tw, bm)
    expect_bounds(2)
    assert torch.equal(bm[0], good_bm[0]) and bool((bm[1] == -7.0).all())   # request 1 not scanned
    pool = csa2.pool_select(cache, good_bm, 64)
    expect_bounds(3)
    assert torch.equal(pool[0], good_pool[0]) and bool((pool[1] == -1).all())
    topk = csa2.reindex(cache, csa2.REINDEX, 512, good_pool, tq, tw)
    expect_bounds(4)
    assert bool((topk[1] == -1).all()) and bool((topk[0] >= 0).all())
    qm = W.main_query(wl, 0).to(dev)
    ids = torch.arange(512, dtype=torch.int32, device=dev).repeat(2, 1)
    out = csa2.sparse_attn(cache, ids, qm, wl.scale)
    expect_bounds(5)
    assert bool((out[1] == 0).all()) and bool((out[0] != 0).any())
    pos = torch.tensor([8000, 8100], dtype=torch.int32, device=dev)
    cache.ctx_len[0] = bad_len
    cache.ctx_len[1] = 4096
    tp = csa2.prefill_index(cache, 0, pos, tq, tw, k=64)
    st, word = csa2.get_error(cache)
    assert st == csa2.ERR_DEVICE_BOUNDS and word[1] == 6 and word[2] == 0 and word[3] == bad_len, word
    assert bool((tp == -1).all())
    # an out-of-range request index in the attention's query map
    cache.ctx_len[0] = 4096
    cache.err_word.zero_()
    out = csa2.sparse_attn(cache, ids, qm, wl.scale, q_req=torch.tensor([0, 9], dtype=torch.int32, device=dev))
    st, word = csa2.get_error(cache)
    assert st == csa2.ERR_DEVICE_BOUNDS and word[1] == 5 and word[2] == 9 and word[3] == -1, word
    assert bool((out[1] == 0).all())


def test_pipeline_wait_timeout_returns_status(csa2):
    """A zero wait bound makes the tensor-core pipeline give up at once: the
    kernel must record CSA2_ERR_TIMEOUT, drain and return (no hang, no trap)."""
    wl = W.scaled(W.WORKLOADS["full_4k_b1"], page_size=1024)
    cache = U.build_cache(wl, csa2, lengths=[4096])
    dev = cache.device
    q, w = W.index_query(wl, 0)
    tq, tw = torch.from_numpy(q).to(dev), torch.from_numpy(w).to(dev)
    try:
        csa2.set_wait_limit_ns(0)
        csa2.index_full(cache, tq, tw)
        st, word = csa2.get_error(cache)
    finally:
        csa2.set_wait_limit_ns(2_000_000_000)
    assert st in (csa2.ERR_TIMEOUT, csa2.OK)     # OK only if every wait happened to be ready
    cache.err_word.zero_()
    bm = csa2.index_full(cache, tq, tw)
    assert csa2.get_error(cache)[0] == csa2.OK
    codes, exp = U.oracle_request(wl, 0, 4096)
    s64 = C.indexer_scores(q[0], w[0], codes, exp)
    assert np.all(np.abs(bm[0, :512].cpu().numpy() - C.block_max(s64, 4096)) <= 1e-5 * C.block_max(s64, 4096))


# ------------------------------------------------------ sliding window (SWA) --

def test_swa_append_bitexact(csa2):
    rng = np.random.default_rng(61)
    B, Wn = 3, 96
    cache = _flat_cache(csa2, 256, batch=B, page_size=128)
    swa = csa2.SwaKV(cache, Wn)
    n = 250
    x = (rng.standard_normal((n, 512)) * np.exp(rng.normal(0, 3, (n, 1)))).astype(np.float32)
    x[5] = 0.0
    req = rng.integers(0, B, n).astype(np.int32)
    pos = rng.permutation(10_000)[:n].astype(np.int32)
    # one row per (request, slot): the last writer would otherwise be ambiguous
    _, keep = np.unique(req.astype(np.int64) * Wn + pos % Wn, return_index=True)
    keep = np.sort(keep)
    dev = cache.device
    csa2.swa_append(cache, swa, torch.from_numpy(x[keep]).to(dev), torch.from_numpy(pos[keep]).to(dev),
                    torch.from_numpy(req[keep]).to(dev))
    codes, exp = C.swa_quantize(x[keep])
    gc = swa.codes.cpu().numpy()[req[keep], pos[keep] % Wn]
    ge = swa.exp.cpu().numpy()[req[keep], pos[keep] % Wn]
    np.testing.assert_array_equal(ge, exp)
    np.testing.assert_array_equal(gc, codes)
    assert csa2.get_error(cache)[0] == csa2.OK


@pytest.mark.parametrize("H,k,window", [(64, 512, 128), (16, 100, 40), (32, 512, 1)])
def test_sparse_attention_swa_parity(csa2, H, k, window):
    """Top-k rows of the FP4 cache merged with the query's window of FP8 SWA
    rows, one softmax (the oracle's reading); windows that are full, cut at
    token 0, and wrapped around the ring."""
    rng = np.random.default_rng(70 + H + window)
    wl = W.scaled(W.WORKLOADS["group_64k_b8"], batch=3, ctx=3000, heads=H)
    cache = U.build_cache(wl, csa2)
    dev = cache.device
    swa = csa2.SwaKV(cache, window)
    q_pos = np.array([2999, window // 3, 5 * window + 7], dtype=np.int32)   # full, partial, wrapped
    rows = {}
    for b in range(3):
        # older tokens first (their slots collide with each other), then the
        # window's tokens, which overwrite them in a later, stream-ordered call
        p = int(q_pos[b])
        older = np.arange(max(0, p - 3 * window), max(0, p - window + 1))
        recent = np.arange(max(0, p - window + 1), p + 1)
        rows[b] = {}
        for toks in (older, recent):
            if len(toks) == 0:
                continue
            y = rng.standard_normal((len(toks), 512)).astype(np.float32)
            rows[b].update(zip(toks.tolist(), y))
            csa2.swa_append(cache, swa, torch.from_numpy(y).to(dev), torch.from_numpy(toks.astype(np.int32)).to(dev),
                            torch.full((len(toks),), b, dtype=torch.int32, device=dev))
    topk = np.stack([np.sort(rng.choice(3000, k, replace=False)) for _ in range(3)]).astype(np.int32)
    topk[1, k // 2:] = -1                                                    # a short Top-k
    qm = W.main_query(wl, 0)
    got = csa2.sparse_attn_swa(cache, torch.from_numpy(topk).to(dev), swa, torch.from_numpy(q_pos).to(dev),
                               qm.to(dev), wl.scale)
    for b in range(3):
        sel = topk[b][topk[b] >= 0]
        kvc, kvs = U.oracle_kv_rows(wl, b, sel)
        toks = C.swa_tokens(int(q_pos[b]), window)
        sc, se = C.swa_quantize(np.stack([rows[b][int(t)] for t in toks]))
        ref = C.sparse_attention_swa(qm[b].float().numpy(), kvc, kvs, np.arange(len(sel)), sc, se, wl.scale)
        U.assert_attention_close(got[b].float().cpu().numpy(), ref, f"swa attention b={b}")
    assert csa2.get_error(cache)[0] == csa2.OK
