"""Pins of the oracle's E4M3 codec (and its BF16 rounding) to facts fixed outside it.

Pins (P-E):
* the 256-code decode table equals torch's float8_e4m3fn decode (an independent
  library implementation), NaN exactly at 0x7F / 0xFF;
* the format facts printed in the P-cast paper (gist.science arXiv 2606.06521):
  3-bit mantissa (Problem statement), round-to-zero threshold 2^-10
  (Methodology), normal floor 2^-6 and largest finite 448 (Optimality of S=256,
  condition 3), 512 overflowing (lay explanation, S=512 "spills");
* encode(decode(c)) == c for every finite code;
* encode == torch's RNE cast over every FP32 bit pattern of 23 whole binades
  (2^-13 .. 2^9, both signs) where torch is defined (|x| <= 448);
* saturation (satfinite) above 448 and for infinities, NaN -> NaN;
* BF16 rounding against torch's float32 -> bfloat16 conversion.
"""
import json
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_format_facts.json")


def torch_decode_all():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_table_matches_library(oracle_mod):
    t = oracle_mod.e4m3_table()
    ref = torch_decode_all()
    nan_o = np.isnan(t)
    assert np.array_equal(nan_o, np.isnan(ref))
    assert set(np.flatnonzero(nan_o)) == {0x7F, 0xFF}
    assert np.array_equal(t[~nan_o], ref[~nan_o])


def test_format_facts_from_paper(oracle_mod):
    facts = json.load(open(GOLDEN))
    t = oracle_mod.e4m3_table()
    fin = t[np.isfinite(t)]
    assert fin.max() == facts["max_finite"]["value"]
    pos = fin[fin > 0]
    normals = pos[pos >= facts["normal_floor"]["value"]]
    # smallest normal value is 2^-6
    assert normals.min() == facts["normal_floor"]["value"]
    # 3-bit mantissa: 8 values per binade among normals
    binade = pos[(pos >= 1.0) & (pos < 2.0)]
    assert len(binade) == 2 ** facts["mantissa_bits"]["value"]
    # round-to-zero threshold: exactly 2^-10 -> 0, anything above -> smallest subnormal
    thr = np.float32(facts["round_to_zero_threshold"]["value"])
    above = np.nextafter(thr, np.float32(1))
    below = np.nextafter(thr, np.float32(0))
    enc = oracle_mod.e4m3_encode(np.array([thr, above, below], dtype=np.float32))
    assert list(enc) == [0x00, 0x01, 0x00]
    assert oracle_mod.e4m3_decode([0x01])[0] == 2.0 ** -9
    # S = 512 overflows the format: P = 1 would need 512 > 448, it saturates
    sat = oracle_mod.e4m3_encode(np.array([1.0], dtype=np.float32), S=facts["overflow_scale"]["value"])
    assert oracle_mod.e4m3_decode(sat)[0] == 448.0 != facts["overflow_scale"]["value"]


def test_encode_decode_round_trip(oracle_mod):
    t = oracle_mod.e4m3_table()
    codes = np.array([c for c in range(256) if np.isfinite(t[c])], dtype=np.uint8)
    assert len(codes) == 254
    vals = t[codes].astype(np.float32)
    assert np.array_equal(oracle_mod.e4m3_encode(vals), codes)


def test_encode_boundaries(oracle_mod):
    x = np.array([2.0 ** -6, 448.0, 464.0, 464.0001, 480.0, 1e30, np.inf, -np.inf, -448.0,
                  -1e-30, 0.0, -0.0, 1.0, 1.0625, 1.0625 + 1e-7, 1.1875], dtype=np.float32)
    got = oracle_mod.e4m3_encode(x)
    want = [0x08, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE,
            0x80, 0x00, 0x80, 0x38, 0x38, 0x39, 0x3A]
    # 1.0625 is the tie between 1.0 (m=0, even) and 1.125 (m=1): ties to even -> 1.0;
    # 1.1875 ties between 1.125 (m=1) and 1.25 (m=2): -> 1.25
    assert [int(c) for c in got] == want
    nan = oracle_mod.e4m3_encode(np.array([np.nan], dtype=np.float32))[0]
    assert (nan & 0x7F) == 0x7F


@pytest.mark.parametrize("sign", [0, 1])
def test_encode_matches_library_exhaustive_binades(oracle_mod, sign):
    # all FP32 patterns with exponent field 114 .. 136  (2^-13 <= |x| < 2^10)
    lo = (114 << 23) | (sign << 31)
    n = 23 << 23
    chunk = 1 << 25
    for start in range(lo, lo + n, chunk):
        m = min(chunk, lo + n - start)
        bits = np.arange(start, start + m, dtype=np.uint64).astype(np.uint32)
        x = bits.view(np.float32)
        ok = np.abs(x) <= 448.0
        got = oracle_mod.e4m3_encode_bits(start, m)
        ref = torch.from_numpy(x[ok]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(got[ok], ref), hex(start)
        # beyond 448 the oracle saturates
        assert np.all((got[~ok] & 0x7F) == 0x7E)


def test_scaled_encode_is_cast_of_fp32_product(oracle_mod):
    rng = np.random.default_rng(1)
    p = rng.random(1 << 20, dtype=np.float32) ** 8
    for S in (1.0, 16.0, 256.0, 448.0):
        prod = (np.float32(S) * p).astype(np.float32)
        ref = torch.from_numpy(prod).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(oracle_mod.e4m3_encode(p, S=S), ref)


def test_bf16_rounding_matches_library(oracle_mod):
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(20000) * 10.0 ** rng.uniform(-3, 3, 20000)).astype(np.float32)
    # include exact ties: 1 + 2^-8 (tie, even -> 1), 1 + 3*2^-8 (tie -> 1 + 2^-6)
    x = np.concatenate([x, np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8], dtype=np.float32)])
    got = oracle_mod.bf16_rne(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(got, ref)
    assert got[-2] == 1.0 and got[-1] == 1 + 2 ** -6
