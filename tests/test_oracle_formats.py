"""Pins of the oracle's FP4 / FP8 formats and NVFP4 quantiser (CPU only).

The pins come from outside the oracle: the E2M1 table and the 6 x 448 range the
pages print (tests/golden), torch's own float8_e4m3fn conversion (a library
routine), exact rational arithmetic, and invariants of round-to-nearest.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _consts():
    return {r[0]: float(r[1]) for r in _golden("page_constants.txt")}


def test_e2m1_table_matches_golden():
    for code, val in _golden("e2m1_codes.txt"):
        v = oracle.e2m1_value(int(code))
        assert v == float(val) and np.signbit(v) == val.startswith("-"), (code, v, val)


def test_e4m3_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if np.isnan(ref[c]):
            assert np.isnan(v) and c in (0x7F, 0xFF)
        else:
            assert v == ref[c] and np.signbit(v) == np.signbit(ref[c]), c


def test_fp4_range_from_pages():
    c = _consts()
    assert oracle.e4m3_value(0x7E) == c["e4m3_max"]
    assert oracle.e2m1_value(7) == c["e2m1_max"]
    assert oracle.e2m1_value(7) * oracle.e4m3_value(0x7E) == c["fp4_max"]


def test_e4m3_encode_roundtrip_and_ties():
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    for c in range(0x7F):
        assert oracle.e4m3_encode(vals[c]) == c
    for c in range(0x7E):
        mid = (vals[c] + vals[c + 1]) / 2
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == even, c
    assert oracle.e4m3_encode(1e9) == 0x7E
    assert oracle.e4m3_encode(0.0) == 0


def test_e4m3_encode_matches_torch_rne():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(0, 460, 20000), np.exp(rng.uniform(-14, 6, 20000))]).astype(np.float32)
    x = x[x < 464.0]  # torch's conversion is round-to-nearest-even but not saturating above 464
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x])
    assert np.array_equal(got, ref)


def _exact_e4m3_nearest(fr):
    """Brute force over all finite non-negative E4M3 values in exact rationals."""
    if fr <= 0:
        return 0
    if fr >= 448:
        return 0x7E
    best, bd = None, None
    for c in range(0x7F):
        d = abs(Fraction(oracle.e4m3_value(c)) - fr)
        if bd is None or d < bd or (d == bd and c % 2 == 0):
            best, bd = c, d
    return best


def _exact_quant_group(xs):
    """Exact-rational NVFP4 quantisation of 16 floats: returns (codes, scale byte)."""
    amax = max(abs(float(v)) for v in xs)
    quot = np.float32(amax) / np.float32(6.0)
    sc = _exact_e4m3_nearest(Fraction(float(quot)))
    s = Fraction(oracle.e4m3_value(sc))
    grid = [Fraction(g) for g in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    codes = []
    for v in xs:
        if s == 0:
            codes.append(0)
            continue
        r = abs(Fraction(float(v))) / s
        ds = [abs(r - g) for g in grid]
        m = min(ds)
        cands = [i for i in range(8) if ds[i] == m]
        mag = cands[0] if len(cands) == 1 else [i for i in cands if i % 2 == 0][0]
        if r > 6:
            mag = 7
        codes.append(mag | (8 if np.signbit(v) else 0))
    return codes, sc


def _unpack(packed, ch):
    out = np.zeros((packed.shape[0], ch), np.int64)
    out[:, 0::2] = packed & 15
    out[:, 1::2] = packed >> 4
    return out


def test_quant_matches_exact_rational_bf16():
    rng = np.random.default_rng(2)
    x = torch.from_numpy(rng.standard_normal((64, 64)).astype(np.float32) * rng.choice(
        [1e-3, 0.1, 1.0, 30.0], (64, 1)).astype(np.float32)).to(torch.bfloat16)
    x[3, :16] = 0.0
    x[4, 16:32] = -0.0
    x[5, :] = torch.tensor([0.5, -0.5] * 32)  # many exact ties
    bits = x.view(torch.int16).numpy().view(np.uint16)
    packed, scales = oracle.quant_nvfp4(bits)
    codes = _unpack(packed, 64)
    xf = x.float().numpy()
    for r in range(64):
        for g in range(4):
            ec, es = _exact_quant_group(xf[r, 16 * g:16 * g + 16])
            assert scales[r, g] == es, (r, g)
            assert list(codes[r, 16 * g:16 * g + 16]) == ec, (r, g)


def test_quant_roundtrip_exact_grid_every_scale():
    """Pin (a): for every finite positive E4M3 scale s, a block whose entries are
    E2M1 grid values times s, with one entry at 6 s, quantises to exactly those
    codes and s, and dequantises to the inputs."""
    rng = np.random.default_rng(3)
    rows, want_codes, want_sc = [], [], []
    for sc in range(1, 0x7F):
        s = oracle.e4m3_value(sc)
        codes = rng.integers(0, 16, 16)
        codes[rng.integers(0, 16)] = 7 | (8 * rng.integers(0, 2))
        vals = [oracle.e2m1_value(int(c)) * s for c in codes]
        # zero magnitude keeps the sign bit only through -0.0
        rows.append(vals)
        want_codes.append(codes)
        want_sc.append(sc)
    x = np.array(rows, np.float32)
    assert np.array_equal(x.astype(np.float64), np.array(rows))  # exact in fp32
    packed, scales = oracle.quant_nvfp4(x)
    assert np.array_equal(scales[:, 0], np.array(want_sc, np.uint8))
    assert np.array_equal(_unpack(packed, 16), np.array(want_codes))
    deq = oracle.dequant_nvfp4(packed, scales)
    assert np.array_equal(deq, x.astype(np.float64))


def test_scale_rule_all_bf16_amax():
    """For every positive finite bf16 amax, the scale byte equals the exact
    nearest E4M3 of fp32(amax / 6) (the reading of the scale rule)."""
    allbits = np.arange(0x0001, 0x7F80, 37, dtype=np.uint16)  # stride keeps the test fast
    x = np.zeros((allbits.size, 16), np.uint16)
    x[:, 0] = allbits
    _, scales = oracle.quant_nvfp4(x)
    vals = torch.from_numpy(allbits.view(np.int16)).view(torch.bfloat16).float().numpy()
    for v, sc in zip(vals, scales[:, 0]):
        quot = np.float32(v) / np.float32(6.0)
        # bisection over the monotone E4M3 table instead of the brute force (same answer, faster)
        want = _exact_e4m3_nearest_fast(Fraction(float(quot)))
        assert sc == want, (v, sc, want)


_E4 = [Fraction(oracle.e4m3_value(c)) for c in range(0x7F)]


def _exact_e4m3_nearest_fast(fr):
    if fr <= 0:
        return 0
    if fr >= 448:
        return 0x7E
    lo = max(c for c in range(0x7F) if _E4[c] <= fr)
    if lo == 0x7E:
        return lo
    da, db = fr - _E4[lo], _E4[lo + 1] - fr
    if da != db:
        return lo if da < db else lo + 1
    return lo if lo % 2 == 0 else lo + 1


def test_quant_invariants_on_latents():
    """Rounding invariants: the amax element maps to magnitude 6 whenever the
    scale is normal; each dequantised value is within half a grid step of x;
    signs are kept; the latent bound of the pages keeps the scale unsaturated."""
    import synth
    x = synth.latent(7, 512)
    bits = synth.bf16_bits(x)
    packed, scales = oracle.quant_nvfp4(bits)
    deq = oracle.dequant_nvfp4(packed, scales)
    xf = x.float().numpy().astype(np.float64)
    codes = _unpack(packed, 512)
    s = np.array([[oracle.e4m3_value(int(b)) for b in row] for row in scales])
    assert s.max() < 448.0 and np.abs(xf).max() <= _consts()["latent_l2_bound"] + 0.1
    for r in range(0, 512, 7):
        for g in range(32):
            blk = slice(16 * g, 16 * g + 16)
            a = np.abs(xf[r, blk])
            j = int(np.argmax(a))
            if s[r, g] >= 2.0 ** -6:
                assert codes[r, 16 * g + j] & 7 == 7
            # local grid step at |x|/s is at most 2 (between 4 and 6): error <= s
            assert np.all(np.abs(deq[r, blk] - xf[r, blk]) <= s[r, g] * 1.0 + 0.0)
            nz = deq[r, blk] != 0
            assert np.all(np.sign(deq[r, blk][nz]) == np.sign(xf[r, blk][nz]))


def test_nibble_order():
    # channel 2j is the low nibble of byte j: +0.5 then -1.0 packs as 0xA1
    x = np.zeros((1, 16), np.float32)
    x[0, 0], x[0, 1], x[0, 2] = 0.5, -1.0, 6.0
    packed, scales = oracle.quant_nvfp4(x)
    assert oracle.e4m3_value(scales[0, 0]) == 1.0
    assert packed[0, 0] == 0xA1 and packed[0, 1] == 0x07
