"""Helpers of the GPU parity tests: fill a cache through the append kernel,
draw the oracle's view of the same inputs, and compare selections / outputs
under the parity rules.

Parity rules (from the benchmark spec of the path):
  * FP4/FP8 codes, scales and exponents: bit-exact.
  * Selections (pool blocks, Top-k positions): the GPU set may differ from the
    oracle's only at candidates whose float64 score lies within 1e-5 relative
    of the oracle's threshold (its k-th best value); a position whose block is
    in one pool and not the other (an allowed pool difference) is excused too.
  * Attention fed the same indices: per (query, head),
    |o_gpu - o64| <= 2e-3 * max|o64| + half a bf16 ulp of o64 (the output is
    bf16, whose own rounding is up to 2^-8 relative; the tolerance reading is
    "2e-3 of the largest output, on top of the output's rounding").
"""
from __future__ import annotations

import numpy as np
import torch

from kv_cache_decode_index_b200 import workloads as W

REL_TIE = 1e-5
ATTN_TOL = 2e-3


def build_cache(wl, csa2, append_last=False, lengths=None):
    """Cache for `wl`, filled through csa2_append_kv (see kv_cache_decode_index_b200.fill)."""
    from kv_cache_decode_index_b200.fill import build_cache as _build
    return _build(wl, csa2, append_last=append_last, lengths=lengths)


def oracle_request(wl, b, n=None):
    """The oracle's quantised cache rows of request b (positions [0, n))."""
    from oracle import formats as F
    n = int(W.ctx_lengths(wl)[b]) if n is None else n
    ik_codes, ik_exp = F.quantize_indexer(W.request_rows(wl, b, n, "ik"))
    return ik_codes, ik_exp


def oracle_kv_rows(wl, b, positions):
    from oracle import formats as F
    return F.quantize_main_kv(W.rows_at(wl, b, positions, "kv"))


def threshold(cand_scores, k):
    s = np.sort(np.asarray(cand_scores, dtype=np.float64))[::-1]
    return s[min(k, len(s)) - 1] if len(s) else 0.0


def assert_set_parity(gpu_ids, ora_ids, score_of, theta, excused=lambda t: False, what=""):
    g = set(int(x) for x in np.asarray(gpu_ids) if x >= 0)
    o = set(int(x) for x in np.asarray(ora_ids) if x >= 0)
    assert len(g) == len(o), f"{what}: {len(g)} selected vs oracle {len(o)}"
    tol = REL_TIE * max(abs(theta), 1e-30)
    bad = [t for t in g ^ o if abs(score_of(t) - theta) > tol and not excused(t)]
    assert not bad, f"{what}: {len(bad)} selections differ beyond the 1e-5 tie band, e.g. {bad[:5]} " \
                    f"(theta={theta!r}, scores={[score_of(t) for t in bad[:5]]})"
    return len(g ^ o)


def assert_sorted_padded(ids, what=""):
    ids = np.asarray(ids)
    v = ids[ids >= 0]
    assert np.all(np.diff(v) > 0), f"{what}: not strictly ascending"
    assert np.all(ids[len(v):] == -1), f"{what}: padding is not trailing -1"


def bf16_half_ulp(x):
    x = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(np.maximum(x, 1e-38))     # x = f * 2^e, f in [0.5, 1)
    return np.ldexp(1.0, e - 1 - 8)           # half of 2^(e-1-7)


def attention_errors(gpu_out, ora_out):
    """(raw, beyond_rounding) relative errors of a bf16 attention output, per
    (query, head) relative to max|o64| and maximised over the elements:
      raw             |o_gpu - o64| / max|o64|, which includes the bf16
                      rounding of the output itself (up to 2^-8 of an element);
      beyond_rounding (|o_gpu - o64| - half a bf16 ulp of o64) / max|o64|, the
                      error the kernel adds on top of that rounding: the figure
                      to read against the 2e-3 bound.
    A check against bf16(o64) instead would fail whenever the kernel's fp32
    result and o64 fall on opposite sides of a bf16 rounding boundary, which
    costs a whole ulp (up to 2^-7 of the largest output) for any error > 0."""
    g = np.asarray(gpu_out, dtype=np.float64)
    o = np.asarray(ora_out, dtype=np.float64)
    mx = np.maximum(np.abs(o).max(axis=-1, keepdims=True), 1e-30)
    err = np.abs(g - o)
    return float((err / mx).max()), float(max(0.0, ((err - bf16_half_ulp(o)) / mx).max()))


def assert_attention_close(gpu_out, ora_out, what=""):
    """gpu_out: bf16-valued float64 [H,512]; ora_out: float64 [H,512].
    Returns the raw max relative error (see attention_errors)."""
    g = np.asarray(gpu_out, dtype=np.float64)
    o = np.asarray(ora_out, dtype=np.float64)
    mx = np.abs(o).max(axis=1, keepdims=True)
    err = np.abs(g - o)
    allowed = ATTN_TOL * mx + bf16_half_ulp(o)
    worst = (err - allowed).max()
    raw, beyond = attention_errors(g, o)
    assert worst <= 0, f"{what}: attention error beyond tolerance by {worst:.3e} " \
                       f"(max rel {raw:.3e}, beyond the output's bf16 rounding {beyond:.3e})"
    return raw
