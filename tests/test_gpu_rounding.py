"""Bit-exactness of the refresh's rounding functions on the GPU against the
oracle, given the same fp32 inputs, Philox key and counter (ReplaySSM
article s4: stochastic rounding of the update copy, FP4 output copy).
The device functions tested are the ones the refresh kernel calls."""
import numpy as np
import pytest
import torch

from hybrid_model_ssm_replay_b200 import rssm
from oracle import oracle as orc

pytestmark = pytest.mark.gpu

SEED, HEAD, REQ, FC = 0x0123_4567_89AB_CDEF, 5, 77, 3


@pytest.fixture(scope="module", autouse=True)
def _built():
    from hybrid_model_ssm_replay_b200 import build
    build.build()


def edge_values():
    e4 = np.array([orc.e4m3_value(c) for c in range(0x7F)], np.float64)
    mids = (e4[:-1] + e4[1:]) / 2
    base = np.concatenate([e4, mids]).astype(np.float32)
    near = np.concatenate([base, np.nextafter(base, np.float32(np.inf)), np.nextafter(base, np.float32(0))])
    special = np.array([0.0, 447.9, 448.0, 449.0, 463.9, 464.0, 480.0, 1e30, np.inf, 2.0 ** -9, 2.0 ** -10,
                        3 * 2.0 ** -11, 2.0 ** -126, 2.0 ** -149, 1e-40, 3.4e38,
                        np.float32(3.4028235e38), 1.0 + 2.0 ** -8, 1.0 + 2.0 ** -9], np.float32)
    v = np.concatenate([near, special])
    return np.concatenate([v, -v])


def random_values(n, seed=0):
    rng = np.random.default_rng(seed)
    mag = rng.normal(0, 1, n) * np.exp2(rng.uniform(-40, 40, n))
    return mag.astype(np.float32)


def test_philox_words():
    n = 1 << 16
    v = torch.zeros(n, device="cuda")
    got = rssm.rssm_round_test(4, v, SEED, HEAD, REQ, FC).cpu().numpy().view(np.uint32)
    key = [SEED & 0xFFFFFFFF, SEED >> 32]
    for e in list(range(64)) + list(range(n - 64, n)) + list(range(1000, n, 997)):
        assert got[e] == orc.philox4x32_10([e // 4, HEAD, REQ, FC], key)[e % 4], e


@pytest.mark.parametrize("op,dtype", [(0, orc.BF16), (1, orc.E4M3)])
def test_stochastic_rounding_bit_exact(op, dtype):
    v = np.concatenate([edge_values(), random_values(1 << 20)]).astype(np.float32)
    v = np.concatenate([v, np.full(7, np.nan, np.float32)])
    n = v.size - v.size % 16
    v = v[:n]
    got = rssm.rssm_round_test(op, torch.from_numpy(v).cuda(), SEED, HEAD, REQ, FC).cpu().numpy()
    ref = orc.sr_head(dtype, SEED, REQ, HEAD, FC, v)
    got = got.view(np.uint16) if op == 0 else got
    nan = np.isnan(v)
    assert np.array_equal(got[~nan], ref[~nan]), np.nonzero(got[~nan] != ref[~nan])[0][:10]
    if op == 0:
        assert np.all((got[nan] & 0x7FC0) == 0x7FC0)
    else:
        assert np.all((got[nan] & 0x7F) == 0x7F)


def test_e4m3_nearest_bit_exact():
    v = np.concatenate([edge_values(), random_values(1 << 17, 1) * np.float32(1e-6),
                        random_values(1 << 17, 2)]).astype(np.float32)
    v = np.concatenate([v, np.array([np.nan], np.float32)])
    got = rssm.rssm_round_test(2, torch.from_numpy(v).cuda()).cpu().numpy()
    ref = np.array([orc.e4m3_rne(x) for x in v], np.uint8)
    assert np.array_equal(got, ref), [(v[i], got[i], ref[i]) for i in np.nonzero(got != ref)[0][:10]]


def fp4_tie_blocks():
    """Blocks whose v/s lands exactly on e2m1 midpoints and saturation."""
    out = []
    scales = [orc.e4m3_value(c) for c in (0x08, 0x20, 0x38, 0x3A, 0x41, 0x5B, 0x70)]
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, 0.0]
    for s in scales:
        out.append(np.array(mids, np.float64) * s)
        out.append(np.array([6.0 * s] + [m * s for m in mids[:15]], np.float64))
    out.append(np.zeros(16))
    out.append(np.array([-0.0] * 16))
    out.append(np.full(16, 1e-30))
    out.append(np.array([7.125, 6.375, 1e-3] + [0.0] * 13))
    return np.concatenate(out).astype(np.float32)


def fp4_near_tie_blocks():
    """Blocks whose quotients v/s, or whose amax/6, lie a few ulps from a
    rounding boundary of e2m1 or e4m3 (where a bracketed quotient cannot
    decide the code and the exact division must)."""
    out = []
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    for sc in (0x01, 0x08, 0x20, 0x38, 0x3A, 0x41, 0x5B, 0x70, 0x7E):
        s = np.float32(orc.e4m3_value(sc))
        for k in (1, 2, 3):
            blk = [np.float32(6.0) * s]
            for m in mids:
                x = np.float32(m) * s
                up, dn = x, x
                for _ in range(k):
                    up, dn = np.nextafter(up, np.float32(np.inf)), np.nextafter(dn, np.float32(0))
                blk += [up, -dn]
            out.append(np.array(blk + [np.float32(0)], np.float32))
    # amax / 6 near the midpoint of two adjacent e4m3 values
    for sc in (0x02, 0x09, 0x21, 0x38, 0x3B, 0x55, 0x7C):
        m = np.float32((orc.e4m3_value(sc) + orc.e4m3_value(sc + 1)) / 2 * 6)
        for k in (-3, -1, 0, 1, 3):
            a = m
            for _ in range(abs(k)):
                a = np.nextafter(a, np.float32(np.inf) if k > 0 else np.float32(0))
            out.append(np.array([a] + [a * np.float32(f) for f in np.linspace(-0.9, 0.9, 15)], np.float32))
    return np.concatenate(out).astype(np.float32)


def test_fp4_block_copy_bit_exact():
    rng = np.random.default_rng(3)
    blocks = (rng.normal(0, 1, (1 << 16, 16)) * np.exp2(rng.uniform(-20, 10, (1 << 16, 1)))).astype(np.float32)
    v = np.concatenate([fp4_tie_blocks(), fp4_near_tie_blocks(), blocks.ravel()]).astype(np.float32)
    n = v.size
    got = rssm.rssm_round_test(3, torch.from_numpy(v).cuda()).cpu().numpy()
    codes, scales = orc.fp4_quant(v)
    assert np.array_equal(got[n // 2:], scales), "scales differ"
    bad = np.nonzero(got[: n // 2] != codes)[0]
    assert bad.size == 0, [(i, hex(got[i]), hex(codes[i]), v[2 * i:2 * i + 2]) for i in bad[:10]]


def test_fp4_read_path_decodes_exactly():
    """The FP4 decode of the replay and refresh kernels, applied to the
    kernels' own FP4 copy, gives exactly the oracle's dequantised values."""
    rng = np.random.default_rng(4)
    blocks = (rng.normal(0, 1, (1 << 14, 16)) * np.exp2(rng.uniform(-12, 8, (1 << 14, 1)))).astype(np.float32)
    v = np.concatenate([fp4_tie_blocks(), blocks.ravel()]).astype(np.float32)
    got = rssm.rssm_round_test(5, torch.from_numpy(v).cuda()).cpu().numpy()
    codes, scales = orc.fp4_quant(v)
    ref = orc.widen(orc.FP4, codes, scales)
    assert np.array_equal(got.astype(np.float64), ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))
