"""Pins of the oracle's E4M3 encoder/decoder against things other than itself.

- the OCP format constants (tests/golden/e4m3_format.txt);
- torch's float8_e4m3fn cast (a library routine) for decoding and, inside the
  range where torch's cast is defined the same way (|v| <= 464), for encoding;
- two independent encoders (arithmetic vs nearest-by-search) over all 2^32
  float32 bit patterns;
- the round-to-nearest-even rule at every midpoint between adjacent codes.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_format.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        code, val = line.split()
        rows.append((int(code, 16), float(val)))
    return rows


def test_decode_golden_constants():
    for code, val in _golden():
        got = oracle.e4m3_decode(code)
        if math.isnan(val):
            assert math.isnan(got), hex(code)
        else:
            assert got == val, hex(code)
            assert math.copysign(1.0, got) == math.copysign(1.0, val), hex(code)


def test_decode_matches_torch_all_codes():
    table = oracle.e4m3_decode_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(table), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(table[fin], ref[fin])
    assert np.array_equal(np.signbit(table[fin]), np.signbit(ref[fin]))


def test_decode_structure():
    t = oracle.e4m3_decode_table()
    pos = t[:127]
    assert np.all(np.diff(pos) > 0), "codes 0x00..0x7E must be strictly increasing"
    assert np.array_equal(t[128:255], -pos)
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])
    assert pos[-1] == 448.0
    # every value times 2^9 is an integer (the grid the block-integer GEMM uses)
    assert np.all(np.floor(pos * 512) == pos * 512)


def test_encode_roundtrip_every_code():
    t = oracle.e4m3_decode_table()
    for c in range(256):
        if math.isnan(t[c]):
            continue
        assert oracle.e4m3_encode(t[c]) == c, hex(c)
        assert oracle.e4m3_encode_nearest(t[c]) == c, hex(c)


def test_encode_midpoints_ties_to_even():
    t = oracle.e4m3_decode_table()
    for c in range(126):
        lo, hi = t[c], t[c + 1]
        mid = (lo + hi) / 2          # exact in float32 (at most 5 significant bits)
        assert np.float32(mid) == mid
        even = c if c % 2 == 0 else c + 1
        for sgn, off in ((1.0, 0), (-1.0, 0x80)):
            v = np.float32(sgn * mid)
            assert oracle.e4m3_encode(v) == even + off, (c, mid)
            assert oracle.e4m3_encode_nearest(v) == even + off, (c, mid)
            above = np.nextafter(np.float32(mid), np.float32(np.inf)) * np.float32(sgn)
            below = np.nextafter(np.float32(mid), np.float32(0)) * np.float32(sgn)
            assert oracle.e4m3_encode(above) == c + 1 + off
            assert oracle.e4m3_encode(below) == c + off


def test_encode_saturation_and_specials():
    for v in (448.0, 449.0, 464.0, 480.0, 1e6, 3.0e38, np.inf):
        assert oracle.e4m3_encode(v) == 0x7E
        assert oracle.e4m3_encode(-v) == 0xFE
    assert oracle.e4m3_encode(np.nan) & 0x7F == 0x7F
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(-1e-30) == 0x80          # negative underflow keeps its sign
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00      # tie between 0 and 2^-9 -> even (0)
    assert oracle.e4m3_encode(np.nextafter(np.float32(2.0 ** -10), np.float32(1))) == 0x01
    assert oracle.e4m3_encode(15.5 * 2.0 ** -10) == 0x08  # 7.75*2^-9 -> 2^-6 across the binade edge


def _sample_patterns(rng, n_random):
    """Bit patterns clustered at every E4M3 rounding boundary plus random ones.

    An E4M3 midpoint has at most 5 significant bits, so in float32 its low 19
    bits are zero; the patterns with low bits in {0, 1, 2^19-1} cover each
    midpoint and its two float32 neighbours for every exponent and sign.
    """
    hi = np.arange(1 << 13, dtype=np.uint64) << np.uint64(19)
    pats = [hi, hi + 1, hi + np.uint64((1 << 19) - 1)]
    pats = np.concatenate(pats)
    pats = np.concatenate([pats, pats | np.uint64(1 << 31)])
    rnd = rng.integers(0, 1 << 32, size=n_random, dtype=np.uint64)
    return np.concatenate([pats, rnd]).astype(np.uint32)


def test_encode_matches_torch_where_defined():
    rng = np.random.default_rng(1234)
    pats = _sample_patterns(rng, 1 << 22)
    v = pats.view(np.float32)
    ok = np.isfinite(v) & (np.abs(v) <= 464.0)
    v = v[ok]
    mine = oracle.e4m3_encode_array(v)
    ref = torch.from_numpy(v.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(mine != ref)[0]
    assert bad.size == 0, (v[bad[:5]], mine[bad[:5]], ref[bad[:5]])


@pytest.mark.slow
def test_two_encoders_agree_on_all_fp32():
    step = 1 << 28
    total_bad = 0
    for start in range(0, 1 << 32, step):
        bad, first = oracle.sweep_encoders(start, step)
        assert bad == 0, "first mismatch at pattern 0x%08x" % first
        total_bad += bad
    assert total_bad == 0
