"""Pins of the oracle's CSA2 step: closed forms and special cases of the score,
brute-force selection on tiny inputs, the invariants the pages fix
(hierarchical pool == flat Top-k while the context fits the pool; Reindex and
Full Top-k inside the pool; Reuse == the previous indices), and sparse
attention against torch's dense scaled-dot-product attention."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import csa2 as C
from oracle import formats as F


def _idx_rows(rng, n):
    k = rng.standard_normal((n, 128)).astype(np.float32)
    return F.quantize_indexer(k)


def _query(rng):
    return rng.standard_normal((32, 128)).astype(np.float32), rng.random(32).astype(np.float32)


# ------------------------------------------------------------------- score --

def test_score_reduces_to_plain_formula_when_quantisation_is_identity():
    """Rows already on the E4M3 grid with amax exactly 448 quantise to
    themselves with sigma = 1: the score is then the plain float64 formula
    sum_h w_h ReLU(q_h . k_t), evaluated here with torch (library)."""
    rng = np.random.default_rng(0)
    grid = F.e4m3_value(rng.integers(0, 127, (64, 128)) | (rng.integers(0, 2, (64, 128)) << 7))
    grid[:, 0] = 448.0
    k = grid[:40].astype(np.float32)
    q = grid[40:72 - 8].astype(np.float32)
    q = np.concatenate([q, grid[:8]]).astype(np.float32)
    w = rng.random(32).astype(np.float32)
    codes, byte = F.quantize_indexer(k)
    assert np.all(byte == 127)
    ours = C.indexer_scores(q, w, codes, byte)
    ref = torch.relu(torch.from_numpy(k).double() @ torch.from_numpy(q).double().T) @ torch.from_numpy(w).double()
    np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-15)


def test_score_one_hot_closed_form():
    """q = one-hot at (head h, dim d), w = e_h: s_t = ReLU(k~_{t,d}) * 448 * sigma^q
    with q's element quantised to 448."""
    rng = np.random.default_rng(1)
    codes, byte = _idx_rows(rng, 50)
    kd = F.dequantize_indexer(codes, byte)
    for h, d in [(0, 0), (7, 99), (31, 127)]:
        q = np.zeros((32, 128), np.float32)
        q[h, d] = 3.0                       # sigma^q = 2^-7, q^ = 384 -> q~ = 3
        w = np.zeros(32, np.float32)
        w[h] = 1.0
        np.testing.assert_array_equal(C.indexer_scores(q, w, codes, byte), np.maximum(kd[:, d], 0) * 3.0)


# ------------------------------------------------ score, FP4 indexer variant --

def _fp4_exact_rows(rng, n):
    """Rows whose every 16-element group is (E2M1 grid value) x s with the
    group's largest magnitude exactly 6 s and s an E4M3 value: the FP4 format
    holds them exactly."""
    grid = F.e2m1_value(rng.integers(0, 16, (n, 128)))
    grid = grid.reshape(n, 8, 16)
    grid[:, :, 0] = 6.0 * np.where(rng.random((n, 8)) < 0.5, -1.0, 1.0)
    s = F.e4m3_value(rng.integers(1, 127, (n, 8)))            # positive scales, subnormals included
    return (grid * s[..., None]).reshape(n, 128).astype(np.float32)


def test_fp4_score_reduces_to_plain_formula_on_exact_inputs():
    """Inputs the FP4 format holds exactly quantise to themselves, so the FP4
    score is the plain float64 sum_h w_h ReLU(q_h . k_t), evaluated here with
    torch (library); the stored codes dequantise to the inputs bit for bit."""
    rng = np.random.default_rng(11)
    k = _fp4_exact_rows(rng, 60)
    q = _fp4_exact_rows(rng, 32)
    w = rng.random(32).astype(np.float32)
    kp, ks = F.quantize_indexer_fp4(k)
    np.testing.assert_array_equal(F.dequantize_indexer_fp4(kp, ks), k.astype(np.float64))
    ours = C.indexer_scores_fp4(q, w, kp, ks)
    ref = torch.relu(torch.from_numpy(k).double() @ torch.from_numpy(q).double().T) @ torch.from_numpy(w).double()
    np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-15, atol=0)
    dots = k.astype(np.float64) @ q.astype(np.float64).T
    assert (dots < 0).mean() > 0.2                          # the ReLU drops a good share of the head terms


def test_fp4_indexer_format_is_the_main_kv_format():
    """The FP4 indexer row is the main-KV format on 128 elements: four indexer
    rows laid end to end quantise exactly like one 512-channel main-KV row
    (an independent implementation of the same rule)."""
    rng = np.random.default_rng(12)
    k = (rng.standard_normal((40, 128)) * np.exp(rng.normal(0, 2, (40, 1)))).astype(np.float32)
    k[3] = 0.0
    kp, ks = F.quantize_indexer_fp4(k)
    mp, ms = F.quantize_main_kv(k.reshape(10, 512))
    np.testing.assert_array_equal(kp.reshape(10, 256), mp)
    np.testing.assert_array_equal(ks.reshape(10, 32), ms)


def test_fp4_score_power_of_two_scaling_and_head_permutation():
    """Scaling the query by 2^j moves every E4M3 scale by j exponents and
    leaves the codes alone (inside the normal range), so scores scale by 2^j
    exactly; permuting the heads together with their weights changes nothing."""
    rng = np.random.default_rng(13)
    k = rng.standard_normal((50, 128)).astype(np.float32)
    q, w = _query(rng)
    kp, ks = F.quantize_indexer_fp4(k)
    base = C.indexer_scores_fp4(q, w, kp, ks)
    np.testing.assert_array_equal(C.indexer_scores_fp4(q * np.float32(4.0), w, kp, ks), base * 4.0)
    perm = rng.permutation(32)
    np.testing.assert_array_equal(C.indexer_scores_fp4(q[perm], w[perm], kp, ks), base)


def test_score_structure():
    rng = np.random.default_rng(2)
    codes, byte = _idx_rows(rng, 300)
    q, w = _query(rng)
    s = C.indexer_scores(q, w, codes, byte)
    assert np.all(s >= 0)
    # linear in w
    w2 = rng.random(32).astype(np.float32)
    np.testing.assert_allclose(C.indexer_scores(q, w + w2, codes, byte),
                               s + C.indexer_scores(q, w2, codes, byte), rtol=1e-6)
    # power-of-two scaling of q keeps the codes and scales the score
    np.testing.assert_allclose(C.indexer_scores(q * 4, w, codes, byte), 4 * s, rtol=1e-15)
    # ReLU: s(q) + s(-q) = sum_h w_h |q~_h . k~_t| (closed form of the two halves)
    qc, sq = C.quantize_index_query(q)
    kd = F.dequantize_indexer(codes, byte)
    absdot = np.abs(kd @ (F.e4m3_value(qc) * sq[:, None]).T) @ w.astype(np.float64)
    np.testing.assert_allclose(s + C.indexer_scores(-q, w, codes, byte), absdot, rtol=1e-12)
    # each row scored on its own: permuting rows permutes scores
    perm = rng.permutation(300)
    np.testing.assert_array_equal(C.indexer_scores(q, w, codes[perm], byte[perm]), s[perm])


def test_block_max_bruteforce():
    rng = np.random.default_rng(3)
    for n in [1, 7, 8, 9, 63, 64, 100]:
        s = rng.random(n + 5)
        bm = C.block_max(s, n)
        ref = [max(s[j * 8:min(j * 8 + 8, n)]) for j in range(-(-n // 8))]
        assert list(bm) == ref


# -------------------------------------------------------------- selections --

def _brute_topk(ids, scores, k):
    """Repeatedly take the best remaining candidate (highest score, then lowest id)."""
    left = list(zip(ids, scores))
    taken = []
    while left and len(taken) < k:
        best = max(left, key=lambda t: (t[1], -t[0]))
        taken.append(best[0])
        left.remove(best)
    return sorted(taken) + [-1] * (k - len(taken))


def test_topk_bruteforce_with_ties():
    rng = np.random.default_rng(4)
    for n, k in [(10, 3), (40, 16), (64, 64), (20, 30), (0, 4)]:
        ids = np.sort(rng.choice(1000, n, replace=False))
        scores = rng.integers(0, 6, n).astype(np.float64)      # many ties
        assert list(C.top_k_ascending(ids, scores, k)) == _brute_topk(list(ids), list(scores), k)
    # ties straddling the cut: equal scores everywhere, and a two-level case
    ids = np.arange(10) * 3
    assert list(C.top_k_ascending(ids, np.ones(10), 4)) == [0, 3, 6, 9]
    sc = np.array([1, 2, 2, 1, 2, 1, 2, 2, 1, 1], dtype=np.float64)
    assert list(C.top_k_ascending(ids, sc, 3)) == _brute_topk(list(ids), list(sc), 3) == [3, 6, 12]


def test_pool_bruteforce_tiny():
    rng = np.random.default_rng(5)
    s = rng.integers(0, 3, 64).astype(np.float64)           # block maxima tie across the cut
    bm = C.block_max(s, 64)
    pool = C.pool_select(bm, 4)
    blocks = sorted(range(8), key=lambda j: (-max(s[8 * j:8 * j + 8]), j))[:4]
    assert list(pool) == sorted(blocks)
    pos = C.pool_positions(pool, 64)
    assert list(pos) == [8 * j + i for j in sorted(blocks) for i in range(8)]


def test_pool_is_every_block_when_context_fits():
    rng = np.random.default_rng(6)
    for n in [1, 4095, 16384]:
        pool = C.pool_select(C.block_max(rng.random(n), n))
        nb = -(-n // 8)
        assert list(pool[:nb]) == list(range(nb)) and np.all(pool[nb:] == -1)


def test_hierarchical_equals_flat_up_to_pool_size():
    """ctx <= 16384: every block is in the pool, so the group with the pool
    selects exactly what it would select with no pool at all."""
    rng = np.random.default_rng(7)
    n = 16384
    codes, byte = _idx_rows(rng, n)
    qs, ws = zip(*[_query(rng) for _ in range(3)])
    modes = ("F", "Ri", "Ru")
    a = C.decode_group(modes, qs, ws, codes, byte, n, pool_blocks=2048)
    b = C.decode_group(modes, qs, ws, codes, byte, n, pool_blocks=None)
    for ta, tb in zip(a["topk"], b["topk"]):
        np.testing.assert_array_equal(ta, tb)


def test_group_invariants_with_pool():
    """Beyond the pool size: Full Top-k equals the flat Top-k (block max keeps
    every Top-512 position's block), Reindex Top-k lies inside the pool, Reuse
    repeats its predecessor."""
    rng = np.random.default_rng(8)
    n = 40000
    codes, byte = _idx_rows(rng, n)
    qs, ws = zip(*[_query(rng) for _ in range(6)])
    modes = ("F", "Ri", "Ri", "Ru", "Ru", "Ru")
    out = C.decode_group(modes, qs, ws, codes, byte, n, pool_blocks=256, k=64)
    pool_pos = set(C.pool_positions(out["pool"], n))
    flat = C.top_k_ascending(np.arange(n), out["scores"], 64)
    np.testing.assert_array_equal(out["topk"][0], flat)
    for t in out["topk"]:
        assert set(t[t >= 0]) <= pool_pos
    for l in (3, 4, 5):
        np.testing.assert_array_equal(out["topk"][l], out["topk"][2])
    # Reindex differs from a flat re-scan only through the pool restriction
    flat1 = C.top_k_ascending(np.arange(n), C.indexer_scores(qs[1], ws[1], codes, byte), 64)
    inside = np.isin(flat1, list(pool_pos))
    assert set(flat1[inside]) <= set(out["topk"][1])


def test_topk_pads_short_context():
    rng = np.random.default_rng(9)
    codes, byte = _idx_rows(rng, 100)
    q, w = _query(rng)
    t = C.decode_group(("F",), [q], [w], codes, byte, 100, pool_blocks=None)["topk"][0]
    assert list(t[:100]) == list(range(100)) and np.all(t[100:] == -1)


# --------------------------------------------------------------- attention --

def _kv(rng, n):
    x = (rng.standard_normal((n, 512)) * np.exp(0.5 * rng.standard_normal(512))).astype(np.float32)
    return F.quantize_main_kv(x)


def test_attention_dense_equivalence_vs_torch_sdpa():
    """ctx <= 512: Top-512 keeps every position, so sparse attention is dense
    attention over the whole context (torch SDPA in float64)."""
    rng = np.random.default_rng(10)
    n, H = 300, 16
    codes, scales = _kv(rng, n)
    q = torch.from_numpy(rng.standard_normal((H, 512)).astype(np.float32)).to(torch.bfloat16).double().numpy()
    idx = np.concatenate([rng.permutation(n), -np.ones(212, dtype=np.int64)])
    ours = C.sparse_attention(q, codes, scales, idx, 1 / np.sqrt(512))
    kv = torch.from_numpy(F.dequantize_main_kv(codes, scales))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], kv[None, None].expand(1, H, n, 512),
        kv[None, None].expand(1, H, n, 512), scale=1 / np.sqrt(512))[0, :, 0, :]
    np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(11)
    codes, scales = _kv(rng, 20)
    q = rng.standard_normal((4, 512))
    rows = F.dequantize_main_kv(codes, scales)
    one = C.sparse_attention(q, codes, scales, np.array([7, -1, -1]), 0.05)
    np.testing.assert_array_equal(one, np.broadcast_to(rows[7], (4, 512)))
    np.testing.assert_array_equal(C.sparse_attention(q, codes, scales, -np.ones(8, np.int64), 0.05), 0)
    # q = 0: uniform weights -> mean of the rows
    np.testing.assert_allclose(C.sparse_attention(np.zeros((2, 512)), codes, scales, np.arange(5), 1.0),
                               np.broadcast_to(rows[:5].mean(0), (2, 512)), rtol=1e-12)
    # order of the index list does not matter
    a = C.sparse_attention(q, codes, scales, np.array([1, 5, 9, 13]), 0.05)
    b = C.sparse_attention(q, codes, scales, np.array([13, 1, -1, 9, 5]), 0.05)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------------- prefill --

def test_prefill_visibility():
    # entry e covers tokens 2e, 2e+1 and is visible at token p iff 2e+1 <= p
    for p in range(0, 40):
        brute = sum(1 for e in range(100) if 2 * e + 1 <= p)
        assert C.prefill_visible(p) == brute
    assert C.prefill_visible(524288 - 8192) == 258048
    assert C.prefill_visible(524287) == 262144
    # other compression ratios: entry e covers tokens m*e .. m*e+m-1
    for m in (1, 3, 4):
        for p in range(-2, 30):
            brute = sum(1 for e in range(100) if all(t <= p for t in range(m * e, m * e + m)))
            assert C.prefill_visible(p, m) == brute


def test_prefill_topk_is_causal():
    rng = np.random.default_rng(12)
    codes, byte = _idx_rows(rng, 2000)
    q, w = _query(rng)
    t = C.prefill_topk(q, w, codes, byte, p=1500, k=64)
    assert t.max() < C.prefill_visible(1500)
    s = C.indexer_scores(q, w, codes[:750], byte[:750])
    np.testing.assert_array_equal(t, C.top_k_ascending(np.arange(750), s, 64))


def test_pages_constants_match_oracle(golden_dir):
    with open(os.path.join(golden_dir, "pages_constants.json")) as f:
        g = json.load(f)
    assert C.POOL_BLOCKS == g["pool_blocks"]["value"]
    assert C.BLOCK == g["block_positions"]["value"]
    assert C.POOL_BLOCKS * C.BLOCK == g["pool_positions"]["value"]
    assert C.TOPK == g["topk"]["value"]
    assert C.INDEX_HEADS == g["index_heads"]["value"]
    assert F.INDEXER_DIM == g["index_head_dim"]["value"]
    assert F.GROUP == g["scale_group_channels"]["value"]


# ----------------------------------------------------- sequence compressor --

def test_compress_tokens_is_the_exact_mean_rounded_once():
    # pinned against exact rational arithmetic: the mean of the m tokens as a
    # Fraction, rounded once to fp32
    from fractions import Fraction
    rng = np.random.default_rng(31)
    for m in (2, 4, 8):
        x = (rng.standard_normal((3 * m, 8)) * np.exp(rng.normal(0, 2, (3 * m, 8)))).astype(np.float32)
        got = C.compress_tokens(x, m)
        for i in range(3):
            for d in range(8):
                exact = sum(Fraction(float(x[m * i + j, d])) for j in range(m)) / m
                assert got[i, d] == np.float32(float(exact)), (m, i, d)
    x = rng.standard_normal((5, 16)).astype(np.float32)
    np.testing.assert_array_equal(C.compress_tokens(x, 1), x)            # m = 1: identity
    rep = np.repeat(x, 4, axis=0)
    np.testing.assert_array_equal(C.compress_tokens(rep, 4), x)          # identical tokens
    with pytest.raises(ValueError):
        C.compress_tokens(np.zeros((6, 4), np.float32), 3)


# ------------------------------------------------------- sliding window ------

def _swa_case(rng, n_main=40, n_win=9, H=4):
    x = (rng.standard_normal((n_main, 512)) * 2).astype(np.float32)
    codes, scales = F.quantize_main_kv(x)
    y = rng.standard_normal((n_win, 512)).astype(np.float32)
    sc, se = C.swa_quantize(y)
    q = rng.standard_normal((H, 512))
    return codes, scales, sc, se, q


def test_swa_window_tokens():
    np.testing.assert_array_equal(C.swa_tokens(10, 4), [7, 8, 9, 10])
    np.testing.assert_array_equal(C.swa_tokens(2, 8), [0, 1, 2])        # the window starts at token 0
    assert len(C.swa_tokens(1000, 128)) == 128


def test_swa_attention_is_the_softmax_merge_of_its_two_parts():
    # pinned by the identity of a softmax over a union of two key sets:
    # o = (L1 o1 + L2 o2) / (L1 + L2) with L_i = sum_j exp(logit_j) of part i,
    # where o1 is the (separately pinned) sparse attention over the Top-k rows
    # and o2 a plain softmax attention over the window rows
    rng = np.random.default_rng(8)
    codes, scales, sc, se, q = _swa_case(rng)
    idx = np.array([3, 17, -1, 25, 0, 39])
    scale = 0.04
    got = C.sparse_attention_swa(q, codes, scales, idx, sc, se, scale)
    k1 = F.dequantize_main_kv(codes[[3, 17, 25, 0, 39]], scales[[3, 17, 25, 0, 39]])
    k2 = F.e4m3_value(sc) * np.ldexp(1.0, se.astype(np.int64) - 127)[:, None]
    l1, l2 = q @ k1.T * scale, q @ k2.T * scale
    m = np.maximum(l1.max(1), l2.max(1))[:, None]
    L1, L2 = np.exp(l1 - m).sum(1)[:, None], np.exp(l2 - m).sum(1)[:, None]
    o1 = C.sparse_attention(q, codes, scales, idx, scale)
    o2 = (np.exp(l2 - m) @ k2) / L2
    np.testing.assert_allclose(got, (L1 * o1 + L2 * o2) / (L1 + L2), rtol=1e-12, atol=1e-12)
    # special cases: no window -> the sparse attention; no Top-k -> the window alone
    np.testing.assert_allclose(C.sparse_attention_swa(q, codes, scales, idx, sc[:0], se[:0], scale),
                               C.sparse_attention(q, codes, scales, idx, scale), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(C.sparse_attention_swa(q, codes, scales, np.array([-1]), sc, se, scale), o2,
                               rtol=1e-12, atol=1e-12)
    # one key in all: o = that key
    np.testing.assert_allclose(C.sparse_attention_swa(q, codes, scales, np.array([-1]), sc[:1], se[:1], scale),
                               np.repeat(k2[:1], len(q), 0), rtol=1e-14)


def test_swa_quantize_is_the_per_row_fp8_rule():
    # the same per-row power-of-two FP8 rule as the indexer rows, on 512-d rows:
    # every code decodes within half an E4M3 step of x / sigma, and sigma is the
    # smallest power of two with 448 * sigma >= max |row|
    rng = np.random.default_rng(3)
    y = (rng.standard_normal((20, 512)) * np.exp(rng.normal(0, 3, (20, 1)))).astype(np.float32)
    sc, se = C.swa_quantize(y)
    sigma = np.ldexp(1.0, se.astype(np.int64) - 127)
    amax = np.abs(y.astype(np.float64)).max(1)
    assert np.all(448 * sigma >= amax) and np.all(448 * sigma / 2 < amax)
    v = F.e4m3_value(sc)
    r = y / sigma[:, None]
    step = np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(r), 2.0 ** -6))).astype(np.int64) - 3)
    assert np.all(np.abs(v - r) <= step / 2 + 1e-12)


# ------------------------------------------------------- sharded pool merge --

@pytest.mark.parametrize("n,G,P", [(100000, 2, 2048), (100000, 3, 2048), (65536, 8, 512), (5000, 4, 2048),
                                   (1000, 5, 64), (64, 2, 4)])
def test_pool_merge_of_slices_equals_the_whole_pool(n, G, P):
    """The merged candidates of G consecutive slices give exactly the pool of
    the whole request (block maxima with many ties across slices), for even
    and uneven slices, and slices shorter than the pool."""
    rng = np.random.default_rng(n + G + P)
    nb = -(-n // 8)
    bm = np.round(rng.standard_normal(nb) * 3) / 3          # heavy ties
    bm[rng.choice(nb, nb // 10, replace=False)] = 1.0       # one big tie group spread over every slice
    cuts = np.sort(rng.choice(np.arange(1, nb), G - 1, replace=False)) if G > 1 else []
    bounds = [0, *cuts, nb]
    vals, ids = [], []
    for g in range(G):
        v, i = C.slice_candidates(bm[bounds[g]:bounds[g + 1]], bounds[g], P)
        vals.append(v)
        ids.append(i)
    np.testing.assert_array_equal(C.pool_merge(vals, ids, P), C.pool_select(bm, P))


def test_pool_merge_bruteforce_tiny():
    """Brute force: sort every (value, id) pair by value desc, id asc."""
    rng = np.random.default_rng(9)
    for _ in range(200):
        G = int(rng.integers(1, 4))
        P = int(rng.integers(1, 6))
        vals = [rng.integers(0, 3, P).astype(float) for _ in range(G)]
        ids = [rng.permutation(50)[:P] for _ in range(G)]
        for g in range(G):
            ids[g][rng.random(P) < 0.2] = -1
        pairs = sorted((-v, i) for g in range(G) for v, i in zip(vals[g], ids[g]) if i >= 0)
        want = sorted(i for _, i in pairs[:P])
        got = C.pool_merge(vals, ids, P)
        np.testing.assert_array_equal(got[:len(want)], want)
        assert np.all(got[len(want):] == -1)


def test_slice_candidates_carry_global_ids_and_values():
    bm = np.array([0.5, 3.0, 2.0, 3.0, -1.0])
    v, i = C.slice_candidates(bm, 1000, 3)
    np.testing.assert_array_equal(i, [1001, 1002, 1003])
    np.testing.assert_array_equal(v, [3.0, 2.0, 3.0])
    v, i = C.slice_candidates(bm[:2], 8, 4)
    np.testing.assert_array_equal(i, [8, 9, -1, -1])
