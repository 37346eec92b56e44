"""Pins of the oracle's number formats (e4m3fn codec, bf16 rounding) against torch's library
casts, hand-derived points of the format definition and brute-force nearest searches."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def torch_e4m3_values():
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_all_codes_match_torch():
    ours, ref = O.e4m3_table(), torch_e4m3_values()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_decode_golden_points():
    with open(os.path.join(GOLDEN, "e4m3_points.json")) as f:
        pts = json.load(f)["points"]
    for p in pts:
        assert O.e4m3_table()[int(p["code"], 16)] == float.fromhex(p["value"]), p


def test_encode_roundtrips_every_finite_code():
    vals = O.e4m3_table()
    for code in range(256):
        if np.isnan(vals[code]):
            continue
        got = int(O.e4m3_encode(vals[code]))
        assert O.e4m3_table()[got] == vals[code] and (got & 0x80) == (code & 0x80), hex(code)


def _torch_cast(v):
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def test_encode_midpoints_ties_to_even():
    pos = np.sort(O.e4m3_table()[:0x7F])            # 0 .. 448
    mids = (pos[:-1] + pos[1:]) / 2.0               # every tie point, exactly representable
    mids = np.concatenate([mids, -mids])
    ours = O.e4m3_encode(mids)
    assert np.array_equal(ours, _torch_cast(mids))
    # ties go to the even mantissa
    assert np.all((ours & 1) == 0)


def test_encode_random_matches_torch_and_brute_force():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(0, 1, 20000),
                        rng.normal(0, 2.0 ** -7, 20000)]).astype(np.float32).astype(np.float64)
    ours = O.e4m3_encode(v)
    assert np.array_equal(ours, _torch_cast(v))
    # brute force: nearest finite value, ties to the even code
    table = O.e4m3_table()
    finite = np.array([c for c in range(128) if not np.isnan(table[c])])
    for x in v[:3000]:
        dist = np.abs(np.abs(x) - table[finite])
        best = finite[dist == dist.min()]
        c = best[best % 2 == 0][0] if len(best) > 1 else best[0]
        got = int(O.e4m3_encode(x))
        assert table[got & 0x7F] == table[c], (x, hex(got), hex(c))


def test_encode_saturates_and_nan():
    big = np.array([448.0, 448.5, 463.9, 464.0, 470.0, 1e6, np.inf])
    assert np.all(O.e4m3_encode(big) == 0x7E)
    assert np.all(O.e4m3_encode(-big) == 0xFE)
    assert int(O.e4m3_encode(np.nan)) == 0x7F
    # subnormal boundary and underflow to (signed) zero
    assert int(O.e4m3_encode(2.0 ** -10)) == 0x00          # tie between 0 and 2^-9 -> even (0)
    assert int(O.e4m3_encode(3 * 2.0 ** -11)) == 0x01
    assert int(O.e4m3_encode(-1e-9)) == 0x80


def test_bf16_round_brute_force_and_torch():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.normal(0, 3, 5000), rng.normal(0, 1e-3, 2000),
                        rng.uniform(-20, 20, 2000)])
    ours = O.bf16_round(v)
    # fp32-representable inputs: torch's fp32 -> bf16 cast is a single RNE rounding
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.bf16_round(v32.astype(np.float64)), ref)
    # brute force for the float64 inputs: nearest of the two bf16 neighbours, ties to even
    for x, got in zip(v[:2000], ours[:2000]):
        lo = np.float32(x).view(np.uint32) & np.uint32(0xFFFF0000)
        cands = []
        for b in (int(lo) - 0x10000, int(lo), int(lo) + 0x10000):
            val = float(np.uint32(b).view(np.float32))
            cands.append((abs(val - x), (b >> 16) & 1, b >> 16))
        best = min(cands)
        assert got == (best[2] & 0xFFFF), x
    # exact ties: 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> even (1.0)
    assert O.bf16_round(1.0 + 2.0 ** -8) == 0x3F80
    assert O.bf16_round(1.0 + 3 * 2.0 ** -8) == 0x3F82
