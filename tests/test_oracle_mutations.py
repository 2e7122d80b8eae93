"""Each pin must catch a plausible mistake: plant one in the oracle (on the
CPU, via monkeypatch) and check that some pin fails."""
import numpy as np
import pytest

import oracle.csa2 as C
import oracle.formats as F
import tests.test_oracle_csa2 as PC
import tests.test_oracle_formats as PF


def _fails(fn, *args):
    with pytest.raises(Exception):
        fn(*args)


def test_mutation_ties_away_from_zero(monkeypatch, golden_dir):
    def bad(r, mant_bits, emin, vmax):
        r = np.asarray(r, dtype=np.float64)
        _, ex = np.frexp(r)
        e = np.maximum(ex - 1, emin)
        q = np.ldexp(1.0, e - mant_bits)
        return np.minimum(np.floor(r / q + 0.5) * q, vmax)
    monkeypatch.setattr(F, "_round_minifloat", bad)
    _fails(PF.test_fp4_hand_cases, golden_dir)
    _fails(PF.test_e4m3_encode_vs_torch_random_and_ties)
    _fails(PF.test_e2m1_encode_vs_bruteforce_and_library)


def test_mutation_subnormals_flushed(monkeypatch, golden_dir):
    orig = F._round_minifloat

    def bad(r, mant_bits, emin, vmax):
        v = orig(r, mant_bits, emin, vmax)
        return np.where(v < 2.0 ** emin, 0.0, v)
    monkeypatch.setattr(F, "_round_minifloat", bad)
    _fails(PF.test_indexer_hand_cases, golden_dir)
    _fails(PF.test_fp4_hand_cases, golden_dir)


def test_mutation_nibble_order(monkeypatch, golden_dir):
    orig = F.quantize_main_kv

    def bad(x):
        p, s = orig(x)
        return ((p >> 4) | (p << 4)).astype(np.uint8), s
    monkeypatch.setattr(F, "quantize_main_kv", bad)
    _fails(PF.test_fp4_hand_cases, golden_dir)
    _fails(PF.test_fp4_group_and_nibble_order)


def test_mutation_scale_rounds_up(monkeypatch, golden_dir):
    """A common alternative: ceil the scale so that nothing saturates."""
    def bad(x):
        x = np.asarray(x, dtype=np.float32).astype(np.float64)
        g = x.reshape(*x.shape[:-1], 32, 16)
        amax = np.abs(g).max(-1)
        sc = F.e4m3_encode(amax / 6.0)
        s = F.e4m3_value(sc)
        sc = np.where(s * 6 < amax, sc + 1, sc).astype(np.uint8)
        s = F.e4m3_value(sc)
        codes = F.e2m1_encode(g, s[..., None]).reshape(*x.shape[:-1], 512)
        return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8), sc
    monkeypatch.setattr(F, "quantize_main_kv", bad)
    _fails(PF.test_fp4_hand_cases, golden_dir)


def test_mutation_indexer_exponent_off_by_one(monkeypatch, golden_dir):
    orig = F.indexer_exponent
    monkeypatch.setattr(F, "indexer_exponent", lambda a: orig(a) + 1)
    _fails(PF.test_indexer_hand_cases, golden_dir)
    _fails(PF.test_indexer_exponent_is_minimal)


def _scores_with(dots_fn, relu=True, use_sigma_t=True):
    def scores(q, w, ik_codes, ik_exp, chunk=1 << 16):
        qc, sq = C.quantize_index_query(q)
        qv = F.e4m3_value(qc)
        kv = F.e4m3_value(ik_codes)
        d = dots_fn(kv, qv) * sq
        r = np.maximum(d, 0) if relu else d
        st = F.indexer_sigma(ik_exp) if use_sigma_t else 1.0
        return st * (r @ np.asarray(w, np.float64))
    return scores


def test_mutation_score_drops_relu(monkeypatch):
    monkeypatch.setattr(C, "indexer_scores", _scores_with(lambda k, q: k @ q.T, relu=False))
    _fails(PC.test_score_structure)
    _fails(PC.test_score_reduces_to_plain_formula_when_quantisation_is_identity)


def test_mutation_score_drops_key_scale(monkeypatch):
    monkeypatch.setattr(C, "indexer_scores", _scores_with(lambda k, q: k @ q.T, use_sigma_t=False))
    _fails(PC.test_score_one_hot_closed_form)


def test_mutation_score_wrong_head_weight_index(monkeypatch):
    def bad(q, w, c, e, chunk=1 << 16):
        return _scores_with(lambda k, qq: k @ qq.T)(q, np.asarray(w)[::-1], c, e)
    monkeypatch.setattr(C, "indexer_scores", bad)
    _fails(PC.test_score_one_hot_closed_form)


def test_mutation_topk_ties_to_higher_id(monkeypatch):
    def bad(ids, scores, k):
        ids = np.asarray(ids, np.int64)
        order = np.lexsort((-ids, -np.asarray(scores, np.float64)))
        sel = np.sort(ids[order[:k]])
        out = np.full(k, -1, np.int64)
        out[:len(sel)] = sel
        return out
    monkeypatch.setattr(C, "top_k_ascending", bad)
    _fails(PC.test_topk_bruteforce_with_ties)
    _fails(PC.test_pool_bruteforce_tiny)


def test_mutation_block_window_shifted(monkeypatch):
    orig = C.block_max
    monkeypatch.setattr(C, "block_max", lambda s, n=None: orig(np.roll(np.asarray(s), -1), n))
    _fails(PC.test_block_max_bruteforce)


def test_mutation_attention_missing_scale(monkeypatch):
    orig = C.sparse_attention
    monkeypatch.setattr(C, "sparse_attention", lambda q, c, s, i, scale: orig(q, c, s, i, 1.0))
    _fails(PC.test_attention_dense_equivalence_vs_torch_sdpa)


def test_mutation_attention_softmax_over_heads(monkeypatch):
    def bad(q_main, kv_codes, kv_scales, idx, scale):
        idx = np.asarray(idx)
        idx = idx[idx >= 0]
        rows = F.dequantize_main_kv(kv_codes[idx], kv_scales[idx])
        lg = (np.asarray(q_main, np.float64) @ rows.T) * scale
        p = np.exp(lg - lg.max(0, keepdims=True))
        p /= p.sum(0, keepdims=True)
        return p @ rows
    monkeypatch.setattr(C, "sparse_attention", bad)
    _fails(PC.test_attention_dense_equivalence_vs_torch_sdpa)


def test_mutation_prefill_off_by_one(monkeypatch):
    monkeypatch.setattr(C, "prefill_visible", lambda p, m=2: max(0, p // m))
    _fails(PC.test_prefill_visibility)


def test_mutation_compressor_drops_a_token(monkeypatch):
    def wrong(x, m):
        x = np.asarray(x, dtype=np.float32)
        g = x.reshape(x.shape[0] // m, m, x.shape[1]).astype(np.float64)
        return (g[:, : max(m - 1, 1), :].sum(axis=1) / m).astype(np.float32)
    monkeypatch.setattr(C, "compress_tokens", wrong)
    _fails(PC.test_compress_tokens_is_the_exact_mean_rounded_once)


def test_mutation_swa_merge_by_halves(monkeypatch):
    # a plausible wrong merge rule: the average of the two separate attentions
    def wrong(q_main, kv_codes, kv_scales, idx, swa_codes, swa_exp, scale):
        o1 = C.sparse_attention(q_main, kv_codes, kv_scales, idx, scale)
        k2 = F.e4m3_value(swa_codes) * np.ldexp(1.0, np.asarray(swa_exp, np.int64) - 127)[:, None]
        lg = np.asarray(q_main, np.float64) @ k2.T * scale
        p = np.exp(lg - lg.max(1, keepdims=True))
        return 0.5 * o1 + 0.5 * (p / p.sum(1, keepdims=True)) @ k2
    monkeypatch.setattr(C, "sparse_attention_swa", wrong)
    _fails(PC.test_swa_attention_is_the_softmax_merge_of_its_two_parts)


def test_mutation_fp4_indexer_nibble_order(monkeypatch):
    orig = F.quantize_indexer_fp4

    def bad(k):
        p, s = orig(k)
        return ((p >> 4) | (p << 4)).astype(np.uint8), s
    monkeypatch.setattr(F, "quantize_indexer_fp4", bad)
    monkeypatch.setattr(C, "quantize_indexer_fp4", bad)
    _fails(PC.test_fp4_indexer_format_is_the_main_kv_format)
    _fails(PC.test_fp4_score_reduces_to_plain_formula_on_exact_inputs)


def test_mutation_fp4_indexer_group_of_32(monkeypatch):
    def bad(k):
        x = np.asarray(k, dtype=np.float32).astype(np.float64)
        lead = x.shape[:-1]
        g = x.reshape(*lead, 4, 32)
        sc = F.e4m3_encode(np.abs(g).max(axis=-1) / 6.0)
        codes = F.e2m1_encode(g, F.e4m3_value(sc)[..., None]).reshape(*lead, 128)
        return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8), np.repeat(sc, 2, axis=-1).astype(np.uint8)
    monkeypatch.setattr(F, "quantize_indexer_fp4", bad)
    monkeypatch.setattr(C, "quantize_indexer_fp4", bad)
    _fails(PC.test_fp4_indexer_format_is_the_main_kv_format)
    _fails(PC.test_fp4_score_reduces_to_plain_formula_on_exact_inputs)


def test_mutation_fp4_score_drops_relu(monkeypatch):
    def bad(q, w, kp, ks):
        qv = F.dequantize_indexer_fp4(*F.quantize_indexer_fp4(q))
        kv = F.dequantize_indexer_fp4(kp, ks)
        return (kv @ qv.T) @ np.asarray(w, dtype=np.float64)
    monkeypatch.setattr(C, "indexer_scores_fp4", bad)
    _fails(PC.test_fp4_score_reduces_to_plain_formula_on_exact_inputs)


def test_mutation_slice_candidates_keep_local_ids(monkeypatch):
    """Forgetting the slice's block offset."""
    orig = C.slice_candidates
    monkeypatch.setattr(C, "slice_candidates", lambda m, off, P=C.POOL_BLOCKS: orig(m, 0, P))
    _fails(PC.test_pool_merge_of_slices_equals_the_whole_pool, 100000, 3, 2048)
    _fails(PC.test_slice_candidates_carry_global_ids_and_values)


def test_mutation_pool_merge_ties_to_higher_id(monkeypatch):
    def bad(vals, ids, P=C.POOL_BLOCKS):
        v = np.concatenate([np.asarray(x, dtype=np.float64).reshape(-1) for x in vals])
        i = np.concatenate([np.asarray(x, dtype=np.int64).reshape(-1) for x in ids])
        keep = i >= 0
        order = np.lexsort((-i[keep], -v[keep]))
        out = np.full(P, -1, np.int64)
        sel = np.sort(i[keep][order[:P]])
        out[:len(sel)] = sel
        return out
    monkeypatch.setattr(C, "pool_merge", bad)
    _fails(PC.test_pool_merge_of_slices_equals_the_whole_pool, 100000, 3, 2048)
    _fails(PC.test_pool_merge_bruteforce_tiny)


def test_mutation_pool_merge_drops_the_last_slice(monkeypatch):
    orig = C.pool_merge
    monkeypatch.setattr(C, "pool_merge", lambda vals, ids, P=C.POOL_BLOCKS: orig(vals[:-1], ids[:-1], P))
    _fails(PC.test_pool_merge_of_slices_equals_the_whole_pool, 100000, 3, 2048)
