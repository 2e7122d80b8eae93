"""CSA2 decode step with the Hierarchical Sparse Indexer, in float64.

Test infrastructure: see the package docstring for who may import this.

What the pages fix, and the readings taken where they are silent:

* Layer modes [readance summary of the DeepSeek-V4.1-Flash report, section 4.2;
  4sapi blog, section 二 CSA2 (mode table)]: Full computes its own main KV and
  indexer K and picks its own Top-K; Reindex reuses that KV and indexer K but
  re-scores with its own indexer Q; Reuse takes main KV and Top-K indices as
  they are.
* Indexer shape [4sapi blog, section 四 Hierarchical Sparse Indexer]: 32 query
  heads of dim 128, Top-512 per query.
* Hierarchical pool [same section; alphalab analysis, section 2 CSA2]: the first
  Full layer scans the whole visible context and keeps 2048 blocks of 8
  positions (16,384 candidates); Reindex layers choose their Top-512 inside it.
* Score function (reading, unpinned against DeepSeek's model):
  s_t = sigma_t * sum_h w_h * ReLU(sigma^q_h * <q_h, k_t>) over FP8 codes.
* Block score (reading, unpinned): the max of the <= 8 visible scores of the
  block.  Ties in every selection go to the lower index (reading).
* Selections are returned sorted ascending, padded with -1.
* Attention (reading of "sparse attention over the gathered Top-K" with the
  512-d shared K=V latent): o_h = sum_i softmax_i(q_h . v_i * scale) v_i over the
  dequantised rows of the valid indices; no valid index gives o = 0.

Every inner product of two FP8 values is exact in float64 (each product has at
most 8 significant bits and every partial sum is a multiple of 2^-18 below
2^25), so the dot products below are exact whatever the summation order.
"""
from __future__ import annotations

import numpy as np

from .formats import (dequantize_indexer, dequantize_indexer_fp4, dequantize_main_kv, e4m3_value,
                      indexer_sigma, quantize_indexer, quantize_indexer_fp4)

INDEX_HEADS = 32
BLOCK = 8            # positions per pool block
POOL_BLOCKS = 2048   # blocks kept by the first Full layer
TOPK = 512


# ------------------------------------------------------------------ scores ---

def quantize_index_query(q):
    """Indexer query q[32,128] (fp32) -> (codes [32,128], sigma^q [32]) with the
    same per-row power-of-two FP8 rule as the cached indexer K."""
    codes, exp = quantize_indexer(q)
    return codes, indexer_sigma(exp)


def indexer_scores(q, w, ik_codes, ik_exp, chunk: int = 1 << 16) -> np.ndarray:
    """Full-mode score of every given row for one query.

    q: [32,128] fp32 indexer query; w: [32] head weights;
    ik_codes: [N,128] uint8 E4M3; ik_exp: [N] uint8 exponent bytes.
    Returns s[N] float64 with s_t = sigma_t * sum_h w_h ReLU(sigma^q_h <q^_h, k^_t>).
    """
    qc, sq = quantize_index_query(q)
    qv = e4m3_value(qc)                        # [32,128]
    w = np.asarray(w, dtype=np.float32).astype(np.float64)
    n = len(ik_codes)
    out = np.empty(n, dtype=np.float64)
    for a in range(0, n, chunk):
        kv = e4m3_value(ik_codes[a:a + chunk])     # [c,128]
        dots = kv @ qv.T                           # [c,32], exact
        relu = np.maximum(dots * sq, 0.0)
        out[a:a + chunk] = indexer_sigma(ik_exp[a:a + chunk]) * (relu @ w)
    return out


def indexer_scores_fp4(q, w, k_packed, k_scales) -> np.ndarray:
    """Full-mode score of every given row for one query, FP4 indexer variant
    (reading: q per head and k both in the FP4 format of
    formats.quantize_indexer_fp4; the pages give V4's indexer Q/K as FP4 but no
    score function).  s_t = sum_h w_h ReLU(<q~_h, k~_t>) with q~, k~ the
    dequantised values.  Each product of two dequantised values is a multiple
    of 2^-20 below 2^23, so every dot product is exact in float64.

    q: [32,128] fp32; w: [32]; k_packed: [N,64] uint8; k_scales: [N,8] uint8.
    """
    qc, qs = quantize_indexer_fp4(q)
    qv = dequantize_indexer_fp4(qc, qs)                      # [32,128]
    kv = dequantize_indexer_fp4(k_packed, k_scales)          # [N,128]
    w = np.asarray(w, dtype=np.float32).astype(np.float64)
    return np.maximum(kv @ qv.T, 0.0) @ w


def block_max(scores, n: int | None = None) -> np.ndarray:
    """m_j = max of the visible scores of block j (positions 8j..8j+7, < n)."""
    s = np.asarray(scores, dtype=np.float64)
    n = len(s) if n is None else n
    nb = -(-n // BLOCK)
    pad = np.full(nb * BLOCK, -np.inf)
    pad[:n] = s[:n]
    return pad.reshape(nb, BLOCK).max(axis=1)


# ------------------------------------------------------------- selections ---

def top_k_ascending(cand_ids, cand_scores, k: int) -> np.ndarray:
    """The k candidates with the largest score (ties: lower id first), returned
    sorted ascending and padded with -1 to length k."""
    cand_ids = np.asarray(cand_ids, dtype=np.int64)
    cand_scores = np.asarray(cand_scores, dtype=np.float64)
    order = np.lexsort((cand_ids, -cand_scores))   # by -score, then by id
    sel = np.sort(cand_ids[order[:k]])
    out = np.full(k, -1, dtype=np.int64)
    out[:len(sel)] = sel
    return out


def pool_select(blockmax, pool_blocks: int = POOL_BLOCKS) -> np.ndarray:
    """Top-`pool_blocks` block ids by block max, ascending, -1 padded.  With at
    most `pool_blocks` blocks the pool is every block."""
    m = np.asarray(blockmax, dtype=np.float64)
    return top_k_ascending(np.arange(len(m)), m, pool_blocks)


def slice_candidates(blockmax_slice, block_offset: int, pool_blocks: int = POOL_BLOCKS):
    """One context slice's candidates for a sharded pool: its own top
    `pool_blocks` blocks (pool_select over the slice's block maxima) as
    (block max, global block id) pairs, global id = local id + block_offset;
    empty entries have id -1 (value 0)."""
    m = np.asarray(blockmax_slice, dtype=np.float64)
    local = pool_select(m, pool_blocks)
    ok = local >= 0
    values = np.zeros(pool_blocks)
    values[ok] = m[local[ok]]
    return values, np.where(ok, local + block_offset, -1)


def pool_merge(cand_values, cand_ids, pool_blocks: int = POOL_BLOCKS) -> np.ndarray:
    """The pool of a request whose context is split into slices (one per
    device), from each slice's candidates (slice_candidates): the top
    `pool_blocks` of the union by block max, ties to the lower global block id,
    ascending, -1 padded.  A reading of the pages' remark that a 1M context may
    have to be sharded across machines (alphalab analysis, limits section):
    the merge is exact, because a block among the whole request's top
    pool_blocks has fewer than pool_blocks blocks ahead of it in the whole
    request, hence in its own slice, so its slice kept it."""
    v = np.concatenate([np.asarray(x, dtype=np.float64).reshape(-1) for x in cand_values])
    i = np.concatenate([np.asarray(x, dtype=np.int64).reshape(-1) for x in cand_ids])
    keep = i >= 0
    return top_k_ascending(i[keep], v[keep], pool_blocks)


def pool_positions(pool, n: int) -> np.ndarray:
    """Expand pool block ids into the visible positions they cover (ascending)."""
    pool = np.asarray(pool, dtype=np.int64)
    blocks = pool[pool >= 0]
    pos = (blocks[:, None] * BLOCK + np.arange(BLOCK)[None, :]).reshape(-1)
    return pos[pos < n]


def full_topk(scores, pool, n: int, k: int = TOPK) -> np.ndarray:
    """Full-mode Top-k: the best k of the Full scan's scores among the
    candidates (the pool's positions, or all n positions when pool is None)."""
    scores = np.asarray(scores, dtype=np.float64)
    cand = np.arange(n) if pool is None else pool_positions(pool, n)
    return top_k_ascending(cand, scores[cand], k)


def reindex_topk(q, w, ik_codes, ik_exp, pool, n: int, k: int = TOPK) -> np.ndarray:
    """Reindex-mode Top-k: re-score only the candidates (pool positions, or all
    n positions when pool is None) with this layer's own q, w."""
    cand = np.arange(n) if pool is None else pool_positions(pool, n)
    s = indexer_scores(q, w, ik_codes[cand], ik_exp[cand])
    return top_k_ascending(cand, s, k)


def reuse_topk(prev_topk) -> np.ndarray:
    """Reuse mode: the previous layer's Top-k indices, unchanged."""
    return np.array(prev_topk, copy=True)


# --------------------------------------------------------------- attention --

def sparse_attention(q_main, kv_codes, kv_scales, idx, scale: float) -> np.ndarray:
    """Sparse MQA attention for one query over the rows `idx` (-1 = skip).

    q_main: [H,512] (bf16 values); kv_codes/kv_scales: the whole request's main
    KV ([N,256] / [N,32]); K = V = the dequantised row.  Returns float64 [H,512].
    """
    q = np.asarray(q_main, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    idx = idx[idx >= 0]
    if len(idx) == 0:
        return np.zeros_like(q)
    rows = dequantize_main_kv(kv_codes[idx], kv_scales[idx])   # [n,512]
    logits = (q @ rows.T) * scale
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return p @ rows


# ------------------------------------------------------------ decode group ---

def decode_group(modes, q_idx, w_idx, ik_codes, ik_exp, n: int,
                 pool_blocks: int | None = POOL_BLOCKS, k: int = TOPK):
    """Index selection of one decode query through a CSA2 layer group.

    modes: sequence of "F", "Ri", "Ru" (the first must be "F");
    q_idx / w_idx: per-layer indexer query and head weights (ignored for "Ru");
    ik_codes / ik_exp: the request's cached indexer K for positions [0, n).
    pool_blocks None means no hierarchical pool (Top-k over the whole context).

    Returns dict(scores, blockmax, pool, topk=[per layer]).  The pool is built
    by the first Full layer; a later Full layer would start a new pool.
    """
    out = {"topk": []}
    pool = None
    prev = None
    for layer, mode in enumerate(modes):
        if mode == "F":
            s = indexer_scores(q_idx[layer], w_idx[layer], ik_codes[:n], ik_exp[:n])
            bm = block_max(s, n)
            pool = None if pool_blocks is None else pool_select(bm, pool_blocks)
            t = full_topk(s, pool, n, k)
            out.setdefault("scores", s)
            out.setdefault("blockmax", bm)
            out.setdefault("pool", pool)
        elif mode == "Ri":
            t = reindex_topk(q_idx[layer], w_idx[layer], ik_codes, ik_exp, pool, n, k)
        elif mode == "Ru":
            t = reuse_topk(prev)
        else:
            raise ValueError(f"unknown mode {mode!r}")
        out["topk"].append(t)
        prev = t
    return out


# ----------------------------------------------------------- causal prefill --

def prefill_visible(p: int, m: int = 2) -> int:
    """Entries visible to the query at token p when entry e covers the m tokens
    m*e .. m*e + m - 1 (m = 2 on the pages' compressed prefill): e is visible
    iff its last token is not after p, m*e + m - 1 <= p, i.e. floor((p + 1) / m).
    A negative p sees nothing."""
    return max(0, (p + 1) // m)


def prefill_topk(q, w, ik_codes, ik_exp, p: int, k: int = TOPK, m: int = 2) -> np.ndarray:
    """Top-k of one prefill query at token p over its visible entries (no pool)."""
    v = min(prefill_visible(p, m), len(ik_codes))
    s = indexer_scores(q, w, ik_codes[:v], ik_exp[:v])
    return top_k_ascending(np.arange(v), s, k)


# ------------------------------------------------------ sequence compressor --

COMPRESS_RATIOS = (1, 2, 4, 8)


def compress_tokens(x, m: int) -> np.ndarray:
    """Sequence compressor of the encoder groups [4sapi blog, section 三: the
    encoder's Full + 5 Reuse groups compress the sequence with m = 2].

    x: [n*m, d] fp32 token rows; returns [n, d] fp32 entries, entry i the mean of
    tokens m*i .. m*i + m - 1.  Reading (the pages name m only): a plain mean,
    summed in float64 in token order, scaled by 1/m and rounded once to fp32;
    m is a power of two up to 8, so the scaling is exact and the only rounding
    is the final one (the double sum of at most 8 fp32 values of similar size
    is exact).  The entries are then quantised on append like any cache row."""
    if m not in COMPRESS_RATIOS:
        raise ValueError(f"m must be one of {COMPRESS_RATIOS}")
    x = np.asarray(x, dtype=np.float32)
    if x.shape[0] % m:
        raise ValueError("the token count must be a multiple of m")
    g = x.reshape(x.shape[0] // m, m, x.shape[1]).astype(np.float64)
    acc = g[:, 0, :].copy()
    for j in range(1, m):
        acc += g[:, j, :]
    return (acc / m).astype(np.float32)


# ------------------------------------------------------- sliding window (SWA) --

def swa_tokens(p: int, window: int) -> np.ndarray:
    """Tokens of the local window of the query at token p: the last `window`
    tokens up to and including p (reading: the pages say every layer, Reuse
    layers included, keeps its own local SWA state [4sapi blog, section 二],
    but give no window size)."""
    return np.arange(max(0, p - window + 1), p + 1, dtype=np.int64)


def swa_quantize(x):
    """SWA KV rows x[..., 512] (fp32) -> FP8 E4M3 codes and one power-of-two
    scale byte per row.  The pages keep the precision-sensitive local SWA KV in
    FP8 [4sapi blog, section 五]; reading: the indexer's per-row rule."""
    return quantize_indexer(x)


def sparse_attention_swa(q_main, kv_codes, kv_scales, idx, swa_codes, swa_exp, scale: float) -> np.ndarray:
    """Sparse attention over the Top-k rows merged with the local window:
    reading (the pages state no merge rule) -- one softmax over the union of the
    dequantised Top-k rows (FP4 main KV, rows idx >= 0) and the window rows
    (FP8 SWA KV, swa_codes / swa_exp [n_window, 512] / [n_window]); K = V for
    both.  Returns float64 [H, 512]; no key at all gives o = 0."""
    q = np.asarray(q_main, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    idx = idx[idx >= 0]
    parts = []
    if len(idx):
        parts.append(dequantize_main_kv(kv_codes[idx], kv_scales[idx]))
    if len(swa_exp):
        parts.append(dequantize_indexer(swa_codes, swa_exp))
    if not parts:
        return np.zeros_like(q)
    rows = np.concatenate(parts)
    logits = (q @ rows.T) * scale
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return p @ rows
