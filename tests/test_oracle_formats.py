"""Pins of the oracle's FP8 tables and encoders (CPU only).

The tables are checked against torch's float8_e4m3fn / float8_e4m3fnuz
decoding and the encoders against torch's round-to-nearest-even casts, which
are library routines independent of the oracle; plus the closed-form facts of
the formats from the E2B MI300X article's E4M3-vs-FNUZ tip, and an
exact-rational brute force.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "verify_stats.json")


def _torch_decode(dtype):
    return torch.arange(256, dtype=torch.uint8).view(dtype).to(torch.float64).numpy()


def test_tables_match_torch_decoding():
    for ours, dt in ((F.DEC_E4M3, torch.float8_e4m3fn), (F.DEC_E4M3FNUZ, torch.float8_e4m3fnuz)):
        ref = _torch_decode(dt)
        assert np.array_equal(np.isnan(ours), np.isnan(ref))
        m = ~np.isnan(ref)
        assert np.array_equal(ours[m], ref[m])


def test_format_facts_from_the_page():
    g = json.load(open(GOLDEN))["formats"]
    assert np.nanmax(F.DEC_E4M3) == g["e4m3_max"] == F.E4M3_MAX
    assert np.nanmax(F.DEC_E4M3FNUZ) == g["e4m3fnuz_max"] == F.E4M3FNUZ_MAX
    # 3 mantissa bits: 8 codes per binade in both formats
    assert F.DEC_E4M3[0x08] * 2 == F.DEC_E4M3[0x10]
    assert F.DEC_E4M3FNUZ[0x08] * 2 == F.DEC_E4M3FNUZ[0x10]
    # smallest subnormals and normals
    assert F.DEC_E4M3[1] == 2.0 ** -9 and F.DEC_E4M3[8] == 2.0 ** -6
    assert F.DEC_E4M3FNUZ[1] == 2.0 ** -10 and F.DEC_E4M3FNUZ[8] == 2.0 ** -7
    # no negative zero in FNUZ: exactly one zero code; E4M3 has +0 and -0
    assert np.sum(F.DEC_E4M3FNUZ == 0) == 1
    assert np.sum(F.DEC_E4M3 == 0) == 2
    # NaN codes
    assert [b for b in range(256) if np.isnan(F.DEC_E4M3[b])] == [0x7F, 0xFF]
    assert [b for b in range(256) if np.isnan(F.DEC_E4M3FNUZ[b])] == [0x80]


def test_fnuz_is_half_of_e4m3():
    for b in range(256):
        if b in (0x7F, 0xFF, 0x80):
            continue
        assert F.DEC_E4M3FNUZ[b] == F.DEC_E4M3[b] / 2


def _torch_cast(x, dtype):
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(dtype).view(torch.uint8).numpy().copy()
    t[t == 0x80] = 0  # canonical zero (torch keeps -0 for E4M3)
    return t


def _dense_fp32_sweep():
    """Every fp32 pattern within 4 ulp of every E4M3 value and midpoint, plus
    a coarse full-range sweep and random values."""
    mags = F.DEC_E4M3[:0x7F]
    pts = np.concatenate([mags, (mags[:-1] + mags[1:]) / 2, [448.0, 456.0, 463.9]])
    pts32 = pts.astype(np.float32)
    b = pts32.view(np.int32)
    offs = np.arange(-4, 5, dtype=np.int32)
    near = (b[:, None] + offs[None, :]).ravel()
    near = near[near >= 0].view(np.float32)
    coarse = (np.arange(0, 0x43E80000, 1 << 12, dtype=np.int64).astype(np.int32)).view(np.float32)
    rnd = np.random.default_rng(7).uniform(0, 464, 200_000).astype(np.float32)
    tiny = np.random.default_rng(8).uniform(0, 2.0 ** -8, 100_000).astype(np.float32)
    v = np.concatenate([near, coarse, rnd, tiny])
    v = v[(v < 464) & np.isfinite(v)]
    return np.concatenate([v, -v])


@pytest.mark.parametrize("fmt", ["e4m3", "e4m3fnuz"])
def test_encoder_matches_torch_rne_cast(fmt):
    v = _dense_fp32_sweep()
    if fmt == "e4m3":
        ours = F.enc_e4m3(v.astype(np.float64))
        ref = _torch_cast(v, torch.float8_e4m3fn)
    else:
        v = v[np.abs(v) < 248]  # torch's FNUZ cast overflows to NaN from 248 up
        ours = F.enc_e4m3fnuz(v.astype(np.float64))
        ref = _torch_cast(v, torch.float8_e4m3fnuz)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, (v[bad[:5]], ours[bad[:5]], ref[bad[:5]])


def test_encoder_saturation_nan_and_zero():
    big = np.array([448.0, 450, 464, 465, 1e4, 3.4e38, np.inf])
    assert np.all(F.enc_e4m3(big) == 0x7E)
    assert np.all(F.enc_e4m3(-big) == 0xFE)
    assert np.all(F.enc_e4m3fnuz(np.array([240.0, 241, 248, 1e4, np.inf])) == 0x7F)
    assert F.enc_e4m3(np.array([np.nan]))[0] == 0x7F
    assert F.enc_e4m3fnuz(np.array([np.nan]))[0] == 0x80
    # negative values that round to zero give the +0 code
    assert np.all(F.enc_e4m3(np.array([-0.0, -1e-30, -2.0 ** -10])) == 0)
    assert np.all(F.enc_e4m3fnuz(np.array([-0.0, -2.0 ** -11])) == 0)


def _exact_rne(x: Fraction, mags):
    a = abs(x)
    if a >= mags[-1]:
        code = len(mags) - 1
    else:
        best = None
        for c, m in enumerate(mags):
            d = abs(a - m)
            if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
                best = (d, c)
        code = best[1]
    if x < 0 and code != 0:
        code |= 0x80
    return code


def test_encoder_exact_rational_brute_force():
    mags = [Fraction(float(m)) for m in F.DEC_E4M3[:0x7F]]
    rng = np.random.default_rng(11)
    v = np.concatenate([
        rng.uniform(-460, 460, 3000),
        rng.uniform(-1, 1, 1000) * 2.0 ** -6,
        ((np.arange(-126, 127) + 0.5) * 2.0 ** -9),   # subnormal midpoints and beyond
    ]).astype(np.float32).astype(np.float64)
    ours = F.enc_e4m3(v)
    for x, c in zip(v, ours):
        assert c == _exact_rne(Fraction(x), mags), x


def test_every_midpoint_goes_to_the_even_code():
    mags = F.DEC_E4M3[:0x7F]
    mids = (mags[:-1] + mags[1:]) / 2
    codes = F.enc_e4m3(mids)
    assert np.all(codes % 2 == 0)
    assert np.all((codes == np.arange(126)) | (codes == np.arange(1, 127)))
