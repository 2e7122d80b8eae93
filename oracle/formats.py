"""FP4 (E2M1) and FP8 (E4M3) codecs and the two cache quantisers, in float64.

Test infrastructure: see the package docstring for who may import this.

Formats, as the pages state them:

* Main KV is stored as FP4 E2M1 codes with one E4M3 scale per 16 channels and
  no second-level (global) scale; the format reaches 6 x 448 = 2688
  [animattoys "DeepSeek發布新模型把KV緩存壓到原來的四分之一", section
  "把精度降到4比特"; 4sapi "DeepSeek V4.1 Flash CED/CSA2" blog, section 五 FP4 KV;
  alphalab "DeepSeek-V4.1-Flash 深度分析", section 3 FP4].
* The indexer K dtype is not given for V4.1 (the animattoys article says V4
  already kept indexer Q and K in FP4).  Reading taken here: FP8 E4M3 codes with
  one power-of-two scale per token (and per query head), the smallest power of
  two that brings the row's largest magnitude to <= 448.

Rounding reading (the pages are silent): round to nearest, ties to the even
code, saturate at the largest finite value, -0 stored as +0.  E2M1 and E4M3 are
both binary minifloats, so one textbook rounding routine serves both:
``_round_minifloat``.

Exactness notes (why float64 is enough to make every decision exactly):
* ``k / 2**e`` is a power-of-two scaling, exact.
* For the E4M3 scale of a 16-channel group the value rounded is amax/6 with amax
  an fp32 number (24 significant bits).  Every E4M3 midpoint times 6 has at most
  7 significant bits, so amax/6 is either exactly a midpoint or at least ~2^-24
  (relative) away from it; float64 division (error 2^-53) cannot flip the
  decision.  The same holds for |x|/s in the E2M1 step (x fp32, s <= 4 bits).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0   # 1.75 * 2**8, largest finite E4M3 (S.1111.110)
E2M1_MAX = 6.0     # 1.5 * 2**2, largest E2M1
MAIN_KV_DIM = 512
GROUP = 16         # channels per E4M3 scale
INDEXER_DIM = 128
INDEXER_EXP_BIAS = 127   # stored byte = e + 127, sigma = 2**e
INDEXER_EXP_MIN = -126   # clamp for all-zero or tiny rows


# ---------------------------------------------------------------- decoding ---

def e2m1_value(code) -> np.ndarray:
    """Value of a 4-bit E2M1 code: sign bit 3, 2 exponent bits (bias 1), 1
    mantissa bit; exponent field 0 is subnormal (m * 0.5).  No Inf/NaN."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 8, -1.0, 1.0)
    e = (c >> 1) & 3
    m = (c & 1).astype(np.float64)
    mag = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * np.exp2(e - 1.0))
    return sign * mag


def e4m3_value(code) -> np.ndarray:
    """Value of an 8-bit E4M3 code (OCP 'fn' variant): sign bit 7, 4 exponent
    bits (bias 7), 3 mantissa bits; exponent field 0 is subnormal (m * 2^-9);
    S.1111.111 is NaN; there is no infinity."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


# ---------------------------------------------------------------- rounding ---

def _round_minifloat(r, mant_bits: int, emin: int, vmax: float) -> np.ndarray:
    """Nearest value of a binary minifloat to r >= 0 (float64, taken as exact).

    The format has ``mant_bits`` fraction bits, smallest normal exponent
    ``emin`` (below it the spacing stays 2^(emin - mant_bits): subnormals) and
    saturates at ``vmax``.  Ties go to the even significand, which for these
    formats is the even code.
    """
    r = np.asarray(r, dtype=np.float64)
    _, ex = np.frexp(r)                       # r = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, emin)              # floor(log2 r), floored at emin
    quantum = np.ldexp(1.0, e - mant_bits)    # spacing of values in that binade
    n = np.rint(r / quantum)                  # exact scaling; rint = half-to-even
    return np.minimum(n * quantum, vmax)


def e4m3_round(r) -> np.ndarray:
    """Nearest E4M3 value to r >= 0, ties to even, saturating at 448."""
    return _round_minifloat(r, 3, -6, E4M3_MAX)


def e2m1_round(r) -> np.ndarray:
    """Nearest E2M1 value to r >= 0, ties to even, saturating at 6."""
    return _round_minifloat(r, 1, 0, E2M1_MAX)


def _e4m3_code_of_value(v) -> np.ndarray:
    """Code bits of a non-negative E4M3 value (inverse of e4m3_value)."""
    v = np.asarray(v, dtype=np.float64)
    _, ex = np.frexp(v)
    e = ex - 1
    normal = v >= 2.0 ** -6
    sub_code = np.rint(v * 2.0 ** 9)
    frac = np.where(normal, v / np.ldexp(1.0, np.where(normal, e, 0)), 1.0)
    norm_code = ((e + 7) << 3) + np.rint((frac - 1.0) * 8.0)
    return np.where(normal, norm_code, sub_code).astype(np.uint8)


def _e2m1_code_of_value(v) -> np.ndarray:
    """Code bits (0..7) of a non-negative E2M1 value."""
    v = np.asarray(v, dtype=np.float64)
    _, ex = np.frexp(v)
    e = ex - 1
    normal = v >= 1.0
    sub_code = np.rint(v * 2.0)
    frac = np.where(normal, v / np.ldexp(1.0, np.where(normal, e, 0)), 1.0)
    norm_code = ((e + 1) << 1) + np.rint((frac - 1.0) * 2.0)
    return np.where(normal, norm_code, sub_code).astype(np.uint8)


def e4m3_encode(r) -> np.ndarray:
    """E4M3 code of the real r (float64): nearest, ties to even, saturating,
    sign kept except that a result of magnitude 0 is stored as +0."""
    r = np.asarray(r, dtype=np.float64)
    mag = e4m3_round(np.abs(r))
    code = _e4m3_code_of_value(mag)
    neg = (r < 0) & (mag > 0)
    return np.where(neg, code | 0x80, code).astype(np.uint8)


def e2m1_encode(x, s) -> np.ndarray:
    """E2M1 code (0..15) of x under scale s: nearest grid value to |x|/s, ties
    to the even code, saturating at 6, sign kept, -0 stored as +0.  A zero
    scale gives code 0 for every channel."""
    x = np.asarray(x, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    safe = np.where(s > 0, s, 1.0)
    mag = np.where(s > 0, e2m1_round(np.abs(x) / safe), 0.0)
    code = _e2m1_code_of_value(mag)
    neg = (x < 0) & (mag > 0)
    return np.where(neg, code | 8, code).astype(np.uint8)


# ------------------------------------------------------------ main KV (FP4) --

def quantize_main_kv(x):
    """FP4 main-KV quantisation of rows x[..., 512] (fp32 values).

    Per group of 16 channels: s = E4M3(amax / 6), codes = E2M1(x / s).
    Returns (codes uint8 [..., 256], scales uint8 [..., 32]); code byte i holds
    channel 2i in its low nibble and channel 2i+1 in its high nibble.
    Pages: E2M1 with one E4M3 scale per 16 channels, no global scale
    [4sapi blog, section 五 FP4 KV; animattoys article, section "把精度降到4比特"].
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    assert x.shape[-1] == MAIN_KV_DIM
    lead = x.shape[:-1]
    g = x.reshape(*lead, MAIN_KV_DIM // GROUP, GROUP)
    amax = np.abs(g).max(axis=-1)
    scale_code = e4m3_encode(amax / 6.0)
    s = e4m3_value(scale_code)
    codes = e2m1_encode(g, s[..., None]).reshape(*lead, MAIN_KV_DIM)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, scale_code.astype(np.uint8)


def dequantize_main_kv(packed, scale_code) -> np.ndarray:
    """Rows [..., 512] in float64 from packed E2M1 codes and E4M3 scales."""
    packed = np.asarray(packed, dtype=np.uint8)
    lo = packed & 0xF
    hi = packed >> 4
    lead = packed.shape[:-1]
    codes = np.stack([lo, hi], axis=-1).reshape(*lead, MAIN_KV_DIM)
    vals = e2m1_value(codes).reshape(*lead, MAIN_KV_DIM // GROUP, GROUP)
    s = e4m3_value(scale_code)[..., None]
    return (vals * s).reshape(*lead, MAIN_KV_DIM)


# ------------------------------------------------ indexer K / Q (FP4 variant) -

def quantize_indexer_fp4(k):
    """FP4 indexer rows k[..., 128] (fp32 values) -> (packed E2M1 codes uint8
    [..., 64], E4M3 scales uint8 [..., 8]).

    The indexer variant the pages describe for V4, whose indexer Q and K were
    FP4 [animattoys article, section 把精度降到4比特].  Reading: the main-KV
    format applied to the 128-element row, one E4M3 scale per 16 elements,
    s = E4M3(amax / 6), codes = E2M1(x / s), byte i = element 2i (low nibble)
    and 2i + 1 (high nibble); no per-row or global scale.
    """
    x = np.asarray(k, dtype=np.float32).astype(np.float64)
    assert x.shape[-1] == INDEXER_DIM
    lead = x.shape[:-1]
    groups = x.reshape(*lead, INDEXER_DIM // GROUP, GROUP)
    scale_code = e4m3_encode(np.abs(groups).max(axis=-1) / 6.0)
    codes = e2m1_encode(groups, e4m3_value(scale_code)[..., None]).reshape(*lead, INDEXER_DIM)
    packed = codes[..., 0::2] | (codes[..., 1::2] << 4)
    return packed.astype(np.uint8), scale_code.astype(np.uint8)


def dequantize_indexer_fp4(packed, scale_code) -> np.ndarray:
    """FP4 indexer rows [..., 128] in float64 from packed codes and scales."""
    packed = np.asarray(packed, dtype=np.uint8)
    lead = packed.shape[:-1]
    codes = np.empty((*lead, INDEXER_DIM), dtype=np.uint8)
    codes[..., 0::2] = packed & 0xF
    codes[..., 1::2] = packed >> 4
    vals = e2m1_value(codes).reshape(*lead, INDEXER_DIM // GROUP, GROUP)
    return (vals * e4m3_value(scale_code)[..., None]).reshape(*lead, INDEXER_DIM)


# ------------------------------------------------------- indexer K / Q (FP8) -

def indexer_exponent(amax) -> np.ndarray:
    """Smallest integer e with 448 * 2^e >= amax, clamped below at -126
    (reading: per-row power-of-two scale; all-zero rows get -126)."""
    amax = np.asarray(amax, dtype=np.float64)
    with np.errstate(divide="ignore"):
        _, ex = np.frexp(amax / E4M3_MAX)     # estimate, within one of the answer
    e = ex.astype(np.int64)
    e = np.where(np.ldexp(E4M3_MAX, e - 1) >= amax, e - 1, e)
    e = np.where(np.ldexp(E4M3_MAX, e) < amax, e + 1, e)
    e = np.where(amax > 0, e, INDEXER_EXP_MIN)
    return np.maximum(e, INDEXER_EXP_MIN)


def _quantize_indexer_rows(k):
    k = np.asarray(k, dtype=np.float32).astype(np.float64)
    amax = np.abs(k).max(axis=-1)
    e = indexer_exponent(amax)
    codes = e4m3_encode(k / np.ldexp(1.0, e)[..., None])
    return codes.astype(np.uint8), (e + INDEXER_EXP_BIAS).astype(np.uint8)


def quantize_indexer(k, rows_per_chunk: int = 4096, threads: int = 8):
    """FP8 indexer rows k[..., 128] (fp32 values) -> (codes uint8 [..., 128],
    exponent byte uint8 [...]) with sigma = 2^(byte - 127) and
    codes = E4M3(k / sigma).  Used for the cached indexer K and, per head, for
    the indexer query.  Large inputs are processed in independent row chunks
    (each row is quantised on its own; chunking only bounds the temporaries)."""
    k = np.asarray(k, dtype=np.float32)
    if k.ndim != 2 or len(k) <= rows_per_chunk:
        return _quantize_indexer_rows(k)
    from concurrent.futures import ThreadPoolExecutor
    codes = np.empty(k.shape, dtype=np.uint8)
    exp = np.empty(k.shape[0], dtype=np.uint8)

    def one(a):
        codes[a:a + rows_per_chunk], exp[a:a + rows_per_chunk] = _quantize_indexer_rows(k[a:a + rows_per_chunk])

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(one, range(0, len(k), rows_per_chunk)))
    return codes, exp


def indexer_sigma(exp_byte) -> np.ndarray:
    """sigma = 2^(byte - 127) for stored exponent bytes."""
    return np.ldexp(1.0, np.asarray(exp_byte, dtype=np.int64) - INDEXER_EXP_BIAS)


def dequantize_indexer(codes, exp_byte) -> np.ndarray:
    """Indexer rows in float64: e4m3_value(codes) * sigma."""
    return e4m3_value(codes) * indexer_sigma(exp_byte)[..., None]
