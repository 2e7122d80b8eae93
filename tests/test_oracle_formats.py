"""Pins of the oracle's FP4 / FP8 codecs against things other than itself:
the pages' printed limits, library conversions (torch float8_e4m3fn,
ml_dtypes float4_e2m1fn), brute-force nearest-value search, and hand-worked
cases in tests/golden/."""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import formats as F


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ------------------------------------------------------------ decode tables --

def test_e2m1_grid_and_pages_max(golden_dir):
    pages = _golden(golden_dir, "pages_constants.json")
    mags = F.e2m1_value(np.arange(8))
    # OCP E2M1 grid; library decode of every code agrees
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(F.e2m1_value(np.arange(16)), lib)
    assert list(mags) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    # the pages: the format reaches 2688 = largest E2M1 x largest E4M3
    assert mags.max() * np.nanmax(F.e4m3_value(np.arange(128))) == pages["fp4_format_max"]["value"]


def test_e4m3_decode_exhaustive_vs_torch():
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.e4m3_value(np.arange(256))
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(lib))
    m = ~np.isnan(lib)
    np.testing.assert_array_equal(ours[m], lib[m])
    assert np.isnan(ours).sum() == 2                 # S.1111.111 only
    assert np.nanmax(ours) == F.E4M3_MAX == 448.0


# ----------------------------------------------------------------- encoders --

def _e4m3_midpoints():
    v = np.unique(np.abs(F.e4m3_value(np.arange(127))))
    return (v[:-1] + v[1:]) / 2


def test_e4m3_encode_vs_torch_random_and_ties():
    rng = np.random.default_rng(0)
    r = np.concatenate([
        rng.standard_normal(20000) * 10,
        rng.standard_normal(20000) * 1e-3,
        np.exp(rng.uniform(np.log(1e-4), np.log(460), 20000)) * rng.choice([-1, 1], 20000),
        _e4m3_midpoints(), -_e4m3_midpoints(),
        F.e4m3_value(np.arange(127)),
    ])
    r = r[(np.abs(r) < 464) & (r != 0)]       # torch gives NaN beyond 464 (no saturation)
    lib = torch.from_numpy(r).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = F.e4m3_encode(r)
    # torch keeps -0; the oracle stores +0 (reading): compare magnitudes there
    zero = F.e4m3_value(ours) == 0
    np.testing.assert_array_equal(ours[~zero], lib[~zero])
    np.testing.assert_array_equal(lib[zero] & 0x7F, 0)


def test_e4m3_saturates():
    np.testing.assert_array_equal(F.e4m3_encode([448, 463.9, 464, 470, 1e9, -1e9]),
                                  [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE])


def _e2m1_brute(x, s):
    """Nearest E2M1 grid value by exhaustive search; ties -> even code."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    out = []
    for xi, si in zip(np.ravel(x), np.ravel(s)):
        if si == 0:
            out.append(0)
            continue
        r = abs(float(xi)) / float(si)
        d = np.abs(grid - r)
        best = np.flatnonzero(d == d.min())
        c = int(best[0]) if len(best) == 1 else int(best[best % 2 == 0][0])
        if xi < 0 and c != 0:
            c |= 8
        out.append(c)
    return np.array(out, dtype=np.uint8).reshape(np.shape(x))


def test_e2m1_encode_vs_bruteforce_and_library():
    rng = np.random.default_rng(1)
    s = F.e4m3_value(rng.integers(1, 127, 4000))
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.0])
    x = np.concatenate([rng.standard_normal(4000) * 4 * s,
                        np.repeat(mids, 50) * np.resize(s, 450) * np.resize([1, -1], 450)])
    ss = np.concatenate([s, np.resize(s, 450)])
    x = x.astype(np.float32).astype(np.float64)
    ours = F.e2m1_encode(x, ss)
    np.testing.assert_array_equal(ours, _e2m1_brute(x, ss))
    # library (saturating RNE) on the same ratios; it keeps -0, we store +0
    lib = (x / ss).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    nz = F.e2m1_value(ours) != 0
    np.testing.assert_array_equal(ours[nz], lib[nz])


def test_fp4_hand_cases(golden_dir):
    cases = _golden(golden_dir, "fp4_hand_cases.json")["groups"]
    for c in cases:
        row = np.zeros(512, dtype=np.float32)
        row[:16] = c["x"]
        packed, sc = F.quantize_main_kv(row)
        assert sc[0] == c["scale_code"], c["why"]
        assert list(packed[:8]) == c["bytes"], c["why"]
        assert np.all(sc[1:] == 0) and np.all(packed[8:] == 0)
        deq = F.dequantize_main_kv(packed, sc)[:16]
        np.testing.assert_array_equal(deq, F.e2m1_value(c["codes"]) * F.e4m3_value(c["scale_code"]))


def test_fp4_group_and_nibble_order():
    # channel 2i -> low nibble, channel 2i+1 -> high nibble; group g -> scale g
    row = np.zeros(512, dtype=np.float32)
    row[16 * 5 + 2] = 6.0      # group 5, even channel
    row[16 * 5 + 3] = -3.0     # group 5, odd channel
    packed, sc = F.quantize_main_kv(row)
    assert sc[5] == 0x38 and np.count_nonzero(sc) == 1
    assert packed[(16 * 5 + 2) // 2] == (7 | (13 << 4))
    assert np.count_nonzero(packed) == 1


def test_fp4_roundtrip_error_bound():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((256, 512)) * np.exp(rng.standard_normal(512))).astype(np.float32)
    packed, sc = F.quantize_main_kv(x)
    deq = F.dequantize_main_kv(packed, sc)
    g = x.astype(np.float64).reshape(256, 32, 16)
    s = F.e4m3_value(sc)[..., None]
    err = np.abs(deq.reshape(256, 32, 16) - g)
    # within half the local E2M1 spacing (2 on [4,6], 1 on [2,4), 0.5 below), plus saturation
    spacing = np.where(np.abs(g) / s >= 4, 2.0, np.where(np.abs(g) / s >= 2, 1.0, 0.5)) * s
    over = np.maximum(np.abs(g) - 6 * s, 0)
    assert np.all(err <= spacing / 2 + over + 1e-300)
    # dequantised values hold <= 5 significant bits: exact in bfloat16
    assert np.array_equal(torch.from_numpy(deq).to(torch.bfloat16).double().numpy(), deq)


# ------------------------------------------------------------------ indexer --

def test_indexer_hand_cases(golden_dir):
    g = _golden(golden_dir, "fp8_indexer_hand_cases.json")
    for c in g["exponents"]:
        e = F.indexer_exponent(np.float32(c["amax"]))
        assert int(e) + 127 == c["byte"], c["why"]
    for c in g["rows"]:
        k = np.zeros(128, dtype=np.float32)
        k[:len(c["k_head"])] = c["k_head"]
        codes, byte = F.quantize_indexer(k)
        assert int(byte) == c["byte"], c["why"]
        assert list(codes[:len(c["codes_head"])]) == c["codes_head"], c["why"]


def test_indexer_exponent_is_minimal():
    rng = np.random.default_rng(3)
    amax = np.abs(rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    amax = np.concatenate([amax, (448.0 * np.exp2(np.arange(-20, 20))).astype(np.float32)])
    e = F.indexer_exponent(amax)
    a = amax.astype(np.float64)
    assert np.all(448.0 * np.exp2(e) >= a)
    assert np.all((448.0 * np.exp2(e - 1) < a) | (e == F.INDEXER_EXP_MIN))


def test_indexer_quantize_roundtrip():
    rng = np.random.default_rng(4)
    k = rng.standard_normal((1000, 128)).astype(np.float32)
    codes, byte = F.quantize_indexer(k)
    deq = F.dequantize_indexer(codes, byte)
    sig = F.indexer_sigma(byte)[:, None]
    assert np.abs(F.e4m3_value(codes)).max() <= 448
    # relative error of an E4M3 normal <= 2^-4; subnormal absolute <= 2^-10 sigma
    err = np.abs(deq - k)
    assert np.all(err <= np.maximum(np.abs(k) * 2.0 ** -4, 2.0 ** -10 * sig))
    # the largest element of each row lands in the top binade [256, 448]
    assert np.all(np.abs(F.e4m3_value(codes)).max(axis=1) >= 224)


def test_e4m3_scale_from_the_fp32_quotient_is_the_exact_code():
    """The kernels take a group's E4M3 scale as the round-to-nearest-even
    conversion of the fp32 quotient amax / 6 (one division, one conversion)
    instead of deciding against the exact quotient.  The two agree: every
    E4M3 midpoint times 6 is an fp32 value, so the fp32 quotient lies on the
    same side of every midpoint as the exact one.  Checked on the amax values
    closest to 6 x each midpoint (the only place a rounding could flip a
    decision), on 6 x each code value, and on random values over the whole
    range, against the oracle's exact rule."""
    vals = F.e4m3_value(np.arange(127))
    mids = (vals[:-1] + vals[1:]) / 2.0
    six = (6.0 * mids).astype(np.float32)
    near = [six, (6.0 * vals).astype(np.float32)]
    for k in range(1, 33):
        near.append((six.view(np.uint32) + k).view(np.float32))
        near.append((six.view(np.uint32) - k).view(np.float32))
    rng = np.random.default_rng(11)
    rand = [np.exp(rng.uniform(-35.0, 9.0, 200_000)).astype(np.float32),
            (rng.random(200_000) * 3000.0).astype(np.float32)]
    amax = np.abs(np.concatenate(near + rand))
    exact = F.e4m3_encode(amax.astype(np.float64) / 6.0)
    via_fp32 = F.e4m3_encode((amax / np.float32(6.0)).astype(np.float64))
    np.testing.assert_array_equal(via_fp32, exact)
