"""Pins of the oracle's scalar formats: OCP E4M3 encode/decode and bf16
rounding, checked against hand-worked values from the OFP8 specification and
against torch's own float8_e4m3fn / bfloat16 conversions (library routines
independent of the oracle)."""
import numpy as np
import pytest
import torch

from conftest import load_golden


def _f32(s):
    return np.float32(float(s))


def test_e4m3_hand_values(oracle_mod):
    fx = load_golden("e4m3_hand.json")
    vals = np.array([_f32(v) for v, _, _ in fx["values"]], np.float32)
    want = np.array([int(c, 16) for _, c, _ in fx["values"]], np.uint8)
    got = oracle_mod.e4m3_encode(vals)
    bad = [(fx["values"][i][0], hex(got[i]), fx["values"][i][1])
           for i in range(len(vals)) if got[i] != want[i]]
    assert not bad, bad


def _bits_range(lo, hi):
    return np.arange(lo, hi, dtype=np.uint64).astype(np.uint32)


def _torch_e4m3(v):
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@pytest.mark.parametrize("lo_exp,hi_exp", [(-13, -5), (6, 9)])
def test_e4m3_exhaustive_binades_vs_torch(oracle_mod, lo_exp, hi_exp):
    """Every binary32 in [2^lo, 2^hi) (capped at 448), both signs, against
    torch's float8_e4m3fn cast (round to nearest even).  The first range
    covers the subnormal/normal boundary of E4M3 and its flush to zero, the
    second the top binades up to the largest finite value."""
    lo = np.float32(2.0 ** lo_exp).view(np.uint32)
    hi = min(np.float32(2.0 ** hi_exp).view(np.uint32), np.float32(448.0).view(np.uint32) + 1)
    step = 1 << 24
    for start in range(int(lo), int(hi), step):
        bits = _bits_range(start, min(start + step, int(hi)))
        v = bits.view(np.float32)
        for sgn in (1, -1):
            vv = (v * np.float32(sgn)).astype(np.float32)
            got = oracle_mod.e4m3_encode(vv)
            want = _torch_e4m3(vv)
            if not np.array_equal(got, want):
                i = int(np.nonzero(got != want)[0][0])
                pytest.fail(f"v={vv[i]!r} oracle={got[i]:#04x} torch={want[i]:#04x}")


def test_e4m3_random_full_range_vs_torch(oracle_mod):
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2 ** 32, size=4_000_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    keep = np.isfinite(v) & (np.abs(v) <= 448.0)
    v = v[keep]
    assert np.array_equal(oracle_mod.e4m3_encode(v), _torch_e4m3(v))


def test_e4m3_saturation_region(oracle_mod):
    """Every finite |v| > 448 saturates to +-448 (0x7E / 0xFE)."""
    rng = np.random.default_rng(8)
    mag = np.exp(rng.uniform(np.log(448.0001), np.log(3e38), size=200_000)).astype(np.float32)
    mag = mag[mag > 448.0]
    assert np.all(oracle_mod.e4m3_encode(mag) == 0x7E)
    assert np.all(oracle_mod.e4m3_encode(-mag) == 0xFE)


def test_e4m3_decode_all_codes_vs_torch(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    got = oracle_mod.e4m3_decode(codes)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))
    # encode(decode(c)) == c for every non-NaN code
    assert np.array_equal(oracle_mod.e4m3_encode(got[~nan]), codes[~nan])


def test_bf16_rounding_vs_torch(oracle_mod):
    rng = np.random.default_rng(9)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        # exact ties: low 16 bits = 0x8000, both parities of the kept part
        (rng.integers(0x3f800000, 0x40000000, 2000).astype(np.uint32) & 0xffff0000 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 3.4e38, -3.4e38, 1e-40, -1e-40], np.float32),
    ])
    got = oracle_mod.float_to_bf16_bits(v)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
