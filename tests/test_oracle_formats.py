"""Pins for the oracle's random numbers, number formats and rounding.

Independent references: PyTorch's CPU Philox engine and its bfloat16 /
float8_e4m3fn conversions (library routines), the OCP E2M1 value table,
brute-force nearest-value search, exact rational arithmetic, and
statistical unbiasedness over a million draws.
"""
import os
import subprocess
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as orc

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")


# ------------------------------------------------------------------ Philox

@pytest.fixture(scope="module")
def torch_philox(tmp_path_factory):
    import ctypes as ct
    out = str(tmp_path_factory.mktemp("philox") / "libtorch_philox_ref.so")
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    subprocess.run(["g++", "-O1", "-std=c++17", "-shared", "-fPIC", "-I", inc,
                    os.path.join(HERE, "torch_philox_ref.cpp"), "-o", out], check=True)
    lib = ct.CDLL(out)
    lib.torch_philox4x32_10.argtypes = [ct.c_void_p] * 3

    def call(ctr, key):
        c = np.ascontiguousarray(ctr, np.uint32)
        k = np.ascontiguousarray(key, np.uint32)
        o = np.zeros(4, np.uint32)
        lib.torch_philox4x32_10(c.ctypes.data, k.ctypes.data, o.ctypes.data)
        return o
    return call


def test_philox_matches_torch_engine(torch_philox):
    rng = np.random.default_rng(0)
    cases = [([0, 0, 0, 0], [0, 0]), ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2),
             ([1, 2, 3, 4], [5, 6])]
    cases += [(rng.integers(0, 2**32, 4, dtype=np.uint64), rng.integers(0, 2**32, 2, dtype=np.uint64))
              for _ in range(2000)]
    for ctr, key in cases:
        assert np.array_equal(orc.philox4x32_10(ctr, key), torch_philox(ctr, key)), (ctr, key)


# ------------------------------------------------------------------ decoding

def test_bf16_decode_all_codes():
    bits = np.arange(65536, dtype=np.uint32)
    ref = torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([orc.bf16_value(b) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_e4m3_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([orc.e4m3_value(c) for c in codes])
    nan = np.isnan(ref)
    assert nan.sum() == 2 and np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))
    assert np.nanmax(got) == 448.0 and orc.e4m3_value(1) == 2.0 ** -9


def load_e2m1_table():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_values.txt")) if l.strip() and l[0] != "#"]
    return {int(c): float(v) for c, v in rows}


def test_e2m1_decode_table():
    table = load_e2m1_table()
    assert len(table) == 16
    for c, v in table.items():
        got = orc.e2m1_value(c)
        assert got == v and np.signbit(got) == np.signbit(v), (c, got, v)


# ------------------------------------------------------- nearest rounding

def e4m3_sweep():
    pos = np.array(sorted({orc.e4m3_value(c) for c in range(0x7F)}))  # 0 .. 448
    mids = (pos[:-1] + pos[1:]) / 2
    vals = np.concatenate([pos, mids])
    f32 = vals.astype(np.float32)
    up = np.nextafter(f32, np.float32(np.inf))
    dn = np.nextafter(f32, np.float32(0))
    rng = np.random.default_rng(1)
    rnd = (rng.uniform(0, 448, 20000)).astype(np.float32)
    tiny = (rng.uniform(0, 2.0 ** -5, 5000)).astype(np.float32)
    allv = np.concatenate([f32, up, dn, rnd, tiny])
    allv = allv[np.abs(allv) <= 448]
    return np.concatenate([allv, -allv])


def test_e4m3_rne_matches_torch_in_range():
    v = e4m3_sweep()
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_rne(x) for x in v], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(v[i], got[i], ref[i]) for i in bad[:5]]


def test_e4m3_rne_saturates_and_nan():
    for v, c in [(448.0, 0x7E), (449.0, 0x7E), (463.99, 0x7E), (464.0, 0x7E), (1e6, 0x7E),
                 (np.inf, 0x7E), (-np.inf, 0xFE), (-500.0, 0xFE)]:
        assert orc.e4m3_rne(v) == c, v
    assert orc.e4m3_rne(np.nan) == 0x7F


def brute_nearest_even(v, values_by_code):
    """Nearest code to v by exhaustive search; ties to the even code."""
    best = None
    for c, val in values_by_code.items():
        d = abs(Fraction(float(v)) - Fraction(val))
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1]


def test_e2m1_rne_brute_force():
    table = load_e2m1_table()
    pos_codes = {c: v for c, v in table.items() if c < 8}
    mags = sorted(set(pos_codes.values()))
    mids = [(a + b) / 2 for a, b in zip(mags[:-1], mags[1:])]
    base = np.array(mags + mids + list(np.linspace(0, 6, 601)), np.float32)
    vals = np.concatenate([base, np.nextafter(base, np.float32(9)), np.nextafter(base, np.float32(-1))])
    vals = vals[(vals >= 0) & (vals <= 6)]
    for v in vals:
        want = brute_nearest_even(v, pos_codes)
        assert orc.e2m1_rne(v) == want, v
        if v > 0:
            assert orc.e2m1_rne(-v) == want | 8, -v
    for v in [6.0, 6.5, 7.0, 100.0, 1e30]:
        assert orc.e2m1_rne(v) == 7 and orc.e2m1_rne(-v) == 15


# ------------------------------------------------------ stochastic rounding

def bf16_neighbours(v):
    """(toward-zero, away-from-zero) bf16 neighbours of a finite fp32 v."""
    u = np.array([v], np.float32).view(np.uint32)[0]
    lo = (u >> 16) << 16
    hi = lo + (1 << 16)
    return (np.array([lo], np.uint32).view(np.float32)[0],
            np.array([hi], np.uint32).view(np.float32)[0])


def test_sr_bf16_picks_a_neighbour_and_keeps_representable():
    rng = np.random.default_rng(2)
    vals = np.concatenate([rng.normal(0, 1, 3000), rng.normal(0, 1e-30, 300),
                           rng.normal(0, 1e37, 300)]).astype(np.float32)
    rs = rng.integers(0, 2**32, vals.size, dtype=np.uint64)
    for v, r in zip(vals, rs):
        got = np.array([orc.sr_bf16(v, r) << 16], np.uint32).view(np.float32)[0]
        lo, hi = bf16_neighbours(v)
        assert got == lo or got == hi, (v, r, got, lo, hi)
    for b in rng.integers(0, 0x7F80, 500):
        v = np.array([int(b) << 16], np.uint32).view(np.float32)[0]
        for r in (0, 1, 2**31, 2**32 - 1):
            assert orc.sr_bf16(v, r) == b and orc.sr_bf16(-v, r) == (b | 0x8000)
    top = np.array([0x7F7FFFFF], np.uint32).view(np.float32)[0]
    assert orc.sr_bf16(top, 0) == 0x7F80            # rounds up into +inf
    assert orc.sr_bf16(np.float32(np.inf), 5) == 0x7F80
    assert orc.sr_bf16(np.float32(np.nan), 5) & 0x7FC0 == 0x7FC0


def e4m3_pairs():
    vals = sorted({orc.e4m3_value(c) for c in range(0x7F)})
    return list(zip(vals[:-1], vals[1:]))


def test_sr_e4m3_exact_rational_all_neighbour_pairs():
    """Every pair of adjacent non-negative e4m3 values, interior points and
    random words, against the rule in exact rationals:
    up iff r < floor((|v| - lo) / (hi - lo) * 2^32)."""
    rng = np.random.default_rng(3)
    code_of = {orc.e4m3_value(c): c for c in range(0x7F)}
    for lo, hi in e4m3_pairs():
        pts = np.float32(lo) + (np.float32(hi) - np.float32(lo)) * np.float32([0.03, 0.25, 0.5, 0.71, 0.97])
        for v in pts:
            fl = Fraction(float(v))
            assert Fraction(lo) < fl < Fraction(hi)
            F = int((fl - Fraction(lo)) / (Fraction(hi) - Fraction(lo)) * 2**32)
            for r in [0, F - 1, F, F + 1, 2**32 - 1] + list(rng.integers(0, 2**32, 4)):
                r = int(r)
                if not 0 <= r < 2**32:
                    continue
                want = code_of[hi] if r < F else code_of[lo]
                assert orc.sr_e4m3(v, r) == want, (v, r, F)
                assert orc.sr_e4m3(-v, r) == want | 0x80
    for c in range(0x7F):
        v = orc.e4m3_value(c)
        assert orc.sr_e4m3(v, 12345) == c
    assert orc.sr_e4m3(np.float32(460.0), 0) == 0x7E and orc.sr_e4m3(np.float32(-np.inf), 0) == 0xFE


@pytest.mark.parametrize("dtype", [orc.BF16, orc.E4M3])
def test_sr_unbiased_over_a_million_draws(dtype):
    """Mean of SR(v) over 10^6 Philox draws is within 5 sigma of v, and the
    fraction rounded up matches the position of v between its neighbours."""
    n = 1 << 20
    for v in [1.0 + 2.0 ** -9, 0.3, -2.7182817, 0.0137]:
        v32 = np.float32(v)
        arr = np.full(n, v32, np.float32)
        bits = orc.sr_head(dtype, 0x1234_5678_9ABC, 3, 1, 7, arr)
        if dtype == orc.BF16:
            vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            lo, hi = bf16_neighbours(v32)
        else:
            table = np.array([orc.e4m3_value(c) for c in range(256)])
            vals = table[bits]
            below = [x for x in table[:0x7F] if x <= abs(v32)]
            above = [x for x in table[:0x7F] if x > abs(v32)]
            lo, hi = np.sign(v32) * max(below), np.sign(v32) * min(above)
        assert set(np.unique(vals)) <= {float(lo), float(hi)}
        f = (float(v32) - float(lo)) / (float(hi) - float(lo))
        sigma = abs(float(hi) - float(lo)) * np.sqrt(f * (1 - f) / n)
        assert abs(vals.mean() - float(v32)) < 5 * sigma + 1e-300, (v, vals.mean(), sigma)
        p_up = np.mean(vals == float(hi))
        assert abs(p_up - f) < 5 * np.sqrt(f * (1 - f) / n)


def test_sr_counter_layout():
    """Element e of head h uses word e % 4 of Philox at (e/4, h, request,
    flush_count): two heads or two flushes draw different words."""
    v = np.full(64, np.float32(0.3), np.float32)
    a = orc.sr_head(orc.BF16, 99, 2, 0, 0, v)
    b = orc.sr_head(orc.BF16, 99, 2, 1, 0, v)
    c = orc.sr_head(orc.BF16, 99, 2, 0, 1, v)
    for e in range(64):
        w = orc.philox4x32_10([e // 4, 0, 2, 0], [99, 0])[e % 4]
        assert a[e] == orc.sr_bf16(v[e], w)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)


# ------------------------------------------------------------------- FP4

def load_fp4_blocks():
    out = []
    for line in open(os.path.join(GOLDEN, "fp4_blocks.txt")):
        if not line.strip() or line[0] == "#":
            continue
        vals, sc, codes = line.split("|")
        out.append((np.array(vals.split(), np.float32), int(sc, 16),
                    np.array([int(c, 16) for c in codes.split()], np.uint8)))
    return out


def test_fp4_hand_worked_blocks():
    blocks = load_fp4_blocks()
    assert len(blocks) == 7
    for vals, sc, codes in blocks:
        got_codes, got_sc = orc.fp4_quant16(vals)
        assert got_sc == sc and np.array_equal(got_codes, codes), (vals, hex(got_sc), got_codes)


def test_fp4_blocks_against_library_scale_and_brute_force_codes():
    """Scale = torch's float8_e4m3fn rounding of amax/6 (fp32); each code
    is the brute-force nearest e2m1 value (ties even) to v/s (fp32)."""
    table = load_e2m1_table()
    pos_codes = {c: v for c, v in table.items() if c < 8}
    rng = np.random.default_rng(4)
    for _ in range(300):
        vals = (rng.normal(0, 1, 16) * np.exp(rng.uniform(-6, 4))).astype(np.float32)
        codes, sc = orc.fp4_quant16(vals)
        amax = np.max(np.abs(vals))
        ref_sc = torch.tensor([amax / np.float32(6)], dtype=torch.float32).to(torch.float8_e4m3fn)
        assert sc == int(ref_sc.view(torch.uint8)[0])
        s = np.float32(orc.e4m3_value(sc))
        for i, v in enumerate(vals):
            c = (codes[i // 2] >> (4 * (i & 1))) & 15
            if s == 0:
                assert c == 0
                continue
            q = np.float32(v / s)
            mag = 7 if abs(q) >= 6 else brute_nearest_even(abs(q), pos_codes)
            assert c & 7 == mag and (c >> 3) == (1 if np.signbit(q) else 0), (v, s, c)
