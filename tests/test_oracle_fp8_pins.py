"""Pins of the low-bit sparse-branch reading in oracle/sla_oracle_fp8.py.

The e4m3 rounding is checked against the format itself (every finite code is a fixed
point, halfway cases go to the even code, saturation, subnormal steps) and against
torch's own float8_e4m3fn conversion, and the decoder against every byte; the branch is
checked on inputs where quantisation is exact, where it must equal the full-precision
branch, and where one V block's P underflows in the units of the row's largest V scale.
"""

import math

import numpy as np
import pytest
import torch

from oracle import sla_oracle as so
from oracle import sla_oracle_fp8 as f8


def _e4m3_codes():
    """Every finite non-negative e4m3 value, from the format definition."""
    vals = []
    for E in range(16):
        for M in range(8):
            if E == 15 and M == 7:
                continue  # the NaN code
            vals.append(M * 2.0 ** -9 if E == 0 else (1 + M / 8) * 2.0 ** (E - 7))
    return np.array(sorted(set(vals)))


def test_codes_are_fixed_points_and_span_the_format():
    c = _e4m3_codes()
    assert c[0] == 0.0 and c[1] == 2.0 ** -9 and c[-1] == 448.0 and len(c) == 127
    np.testing.assert_array_equal(f8.e4m3_round(c), c)
    np.testing.assert_array_equal(f8.e4m3_round(-c), -c)


def test_halfway_cases_round_to_the_even_code():
    c = _e4m3_codes()
    mids = (c[:-1] + c[1:]) / 2
    r = f8.e4m3_round(mids)
    # the even code of each pair has an even mantissa (or is the power of two above it)
    lo, hi = c[:-1], c[1:]
    def even(v):
        if v == 0:
            return True
        if v < 2.0 ** -6:
            return round(v / 2.0 ** -9) % 2 == 0
        e = math.floor(math.log2(v))
        return round(v / 2.0 ** (e - 3)) % 2 == 0
    expect = np.array([a if even(a) else b for a, b in zip(lo, hi)])
    np.testing.assert_array_equal(r, expect)


def test_saturation_and_monotonicity():
    np.testing.assert_array_equal(f8.e4m3_round([449.0, 1e9, -500.0]), [448.0, 448.0, -448.0])
    x = np.linspace(-500, 500, 200001)
    assert np.all(np.diff(f8.e4m3_round(x)) >= 0)


def test_matches_torch_float8_e4m3fn_in_range():
    g = np.random.default_rng(0)
    x = np.concatenate([g.normal(0, 30, 20000), g.normal(0, 0.01, 20000), g.uniform(-448, 448, 20000)])
    ref = torch.from_numpy(x).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    # torch rounds the fp32 value; x is exactly representable in fp32 only after rounding, so
    # compare on fp32-rounded inputs
    x32 = x.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(f8.e4m3_round(x32), ref)


def test_nearest_code():
    g = np.random.default_rng(1)
    c = _e4m3_codes()
    allc = np.concatenate([-c[::-1], c])
    x = g.uniform(-448, 448, 5000)
    r = f8.e4m3_round(x)
    d = np.abs(allc[None, :] - x[:, None]).min(axis=1)
    np.testing.assert_allclose(np.abs(r - x), d, rtol=0, atol=1e-12)


@pytest.mark.parametrize("amax", [1e-3, 0.37, 1.0, 1.5, 127.9, 128.0, 200.0, 3e4])
def test_pow2_scale(amax):
    s = f8.pow2_scale(amax)
    assert math.frexp(s)[0] == 0.5  # a power of two
    assert 128.0 < amax / s <= 256.0


def test_fp8_branch_equals_exact_branch_when_quantisation_is_exact():
    g = np.random.default_rng(2)
    D, bk = 16, 8
    # values on the e4m3 grid after a power-of-two scale, and Q = 0 so every P is exactly 1;
    # the V blocks sit at different scales (2^0, 2^2, 2^-3), so P is rounded in units of the
    # largest and must stay exact
    k = f8.e4m3_round(g.normal(0, 20, (40, D))) / 64.0
    v = f8.e4m3_round(g.normal(0, 20, (40, D))) / 64.0
    v[16:24] *= 4.0
    v[32:40] /= 8.0
    q = np.zeros((8, D))
    crit = [0, 2, 4]
    o8, l8 = f8.sparse_branch_fp8(q, k, v, crit, bk)
    o, l = so.sparse_branch(q, k, v, crit, bk)
    np.testing.assert_allclose(o8, o, rtol=0, atol=1e-15)
    np.testing.assert_array_equal(l8, l)


def test_fp8_branch_rounds_p_after_the_v_scale_ratio():
    # Q = 0: every P is 1. Block 1's V scale is 2^-18 of block 0's, so its P in block 0's
    # units is 2^-18, below half the smallest e4m3 step (2^-9): it rounds to 0.
    # Block 1 then adds nothing to the numerator but its 8 keys still count in l.
    g = np.random.default_rng(5)
    D, bk = 16, 8
    k = g.normal(0, 1, (16, D))
    v = np.zeros((16, D))
    v[:8] = f8.e4m3_round(g.normal(0, 20, (8, D))) / 64.0
    v[8:] = v[:8] * 2.0 ** -18  # the same codes, 18 binades lower
    assert f8.pow2_scale(np.abs(v[8:]).max()) == f8.pow2_scale(np.abs(v[:8]).max()) * 2.0 ** -18
    q = np.zeros((4, D))
    o8, l8 = f8.sparse_branch_fp8(q, k, v, [0, 1], bk)
    np.testing.assert_array_equal(l8, np.full(4, 16.0))
    expect = np.broadcast_to(v[:8].sum(axis=0) / 16.0, (4, D))
    np.testing.assert_allclose(o8, expect, rtol=0, atol=1e-15)


def _two_block_row(t):
    # one query row q = e_0; block 0 keys are 0 (x = 0), block 1 keys are t e_0, so block 1's
    # x = t / sqrt(16) * log2(e). V: block 0 rows all v0, block 1 rows all v1, same amax.
    D, bk = 16, 8
    q = np.zeros((1, D))
    q[0, 0] = 1.0
    k = np.zeros((16, D))
    k[8:, 0] = t
    v0 = np.array([1.5, 0.5, -1.0, 0.25] * 4)
    v1 = np.array([-1.5, 1.0, 0.75, -0.125] * 4)
    v = np.concatenate([np.tile(v0, (8, 1)), np.tile(v1, (8, 1))])
    o8, _ = f8.sparse_branch_fp8(q, k, v, [0, 1], bk)
    return o8[0], v0, v1, t / 4.0 * math.log2(math.e)


def test_reference_stays_within_the_slack():
    # t = 6.5: x1 = 2.344 < 8, the reference stays at 0, block 1's P = 2^2.344 = 5.077 lies
    # in [4, 8) where e4m3 steps by 0.5, so it becomes 5 exactly; l keeps the unquantised
    # 8 (1 + 2^x1)
    o, v0, v1, x1 = _two_block_row(6.5)
    assert x1 < f8.P8_SLACK
    expect = (v0 + 5.0 * v1) / (1.0 + 2.0 ** x1)
    np.testing.assert_allclose(o, expect, rtol=0, atol=1e-12)


def test_reference_stays_for_a_growth_of_four_binades():
    # t = 12: x1 = 4.328 is inside the slack of 8, so block 1's P = 2^4.328 = 20.09 is rounded
    # at the old reference: in [16, 32) e4m3 steps by 2, so it becomes 20 (not saturated:
    # it is rounded at its own value, not scaled up)
    o, v0, v1, x1 = _two_block_row(12.0)
    assert 4 < x1 < f8.P8_SLACK
    np.testing.assert_allclose(o, (v0 + 20.0 * v1) / (1.0 + 2.0 ** x1), rtol=0, atol=1e-12)


def test_reference_moves_past_the_slack():
    # t = 24: x1 = 8.656 > 8, the reference moves to x1, both blocks' P are exactly 1 at
    # their own reference, and the result is the exact softmax
    o, v0, v1, x1 = _two_block_row(24.0)
    assert x1 > f8.P8_SLACK
    w0 = 2.0 ** -x1
    np.testing.assert_allclose(o, (w0 * v0 + v1) / (w0 + 1.0), rtol=0, atol=1e-12)


def test_decode_every_code():
    codes = np.arange(256, dtype=np.uint8)
    vals = f8.e4m3_decode(codes)
    nan = np.isnan(vals)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    fin = vals[~nan]
    # the finite codes are the format's values, each a fixed point of the rounding
    np.testing.assert_array_equal(np.unique(np.abs(fin)), _e4m3_codes())
    np.testing.assert_array_equal(f8.e4m3_round(fin), fin)
    # an independent decoder: torch's float8_e4m3fn reinterpretation of the same bytes
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(vals[~nan], ref[~nan])
    assert f8.e4m3_decode([0x7E])[0] == 448.0 and f8.e4m3_decode([0x01])[0] == 2.0 ** -9


def test_fp8_forward_close_to_full_precision():
    g = np.random.default_rng(3)
    B, H, N, D = 1, 1, 96, 16
    q, k, v = (g.normal(0, 1, (B, H, N, D)) for _ in range(3))
    alpha = g.uniform(0, 1, (H, D))
    o = so.forward(q, k, v, alpha, 16, 8, 0.3, 0.2)
    o8 = f8.forward_fp8(q, k, v, alpha, 16, 8, 0.3, 0.2)
    err = np.abs(o8 - o)
    assert err.max() < 0.1 and err.mean() < 0.02
    assert not np.array_equal(o8, o)


def test_quantize_blocks_scales_and_codes():
    g = np.random.default_rng(4)
    x = g.normal(0, 3, (70, 8))
    codes, scales = f8.quantize_blocks(x, 32)
    assert len(scales) == 3
    for bi, s in enumerate(scales):
        blk = slice(32 * bi, min(70, 32 * (bi + 1)))
        assert math.frexp(s)[0] == 0.5
        np.testing.assert_array_equal(f8.e4m3_round(codes[blk]), codes[blk])  # codes are e4m3 values
        assert np.abs(codes[blk]).max() <= 256.0
        # relative error of a normal e4m3 code is at most 2^-4
        big = np.abs(x[blk] / s) >= 2.0 ** -6
        assert np.all(np.abs(codes[blk][big] * s - x[blk][big]) <= 2.0 ** -4 * np.abs(x[blk][big]))


def test_slack_covers_float32_sized_score_errors():
    # Let the rounding see P with its log2 argument off by a relative 2e-6 (about what float32
    # scores give): every code that changes must be one the slack counts, so the output moves
    # by at most the slack.
    g = np.random.default_rng(6)
    D, bk = 32, 16
    q = g.normal(0, 1.0, (256, D))
    k = g.normal(0, 1.0, (256, D)) * np.repeat(2.0 ** g.integers(-1, 2, 16), 16)[:, None]
    v0 = g.normal(0, 1.0, (256, D)) * np.repeat(2.0 ** g.integers(-3, 2, 16), 16)[:, None]
    crit = list(range(0, 16, 2))
    for vscale in (1.0, 1000.0):  # V scales below and above 1
        v = v0 * vscale
        o, _, slack, near = f8.sparse_branch_fp8(q, k, v, crit, bk, with_slack=True)
        assert slack.max() > 0 and not near.any()
        moved = 0
        for d in (2e-6, -2e-6, 1e-6, -1e-6):
            od, _ = f8.sparse_branch_fp8(q, k, v, crit, bk, x_rel_perturb=d)
            diff = np.abs(od - o)
            assert np.all(diff <= slack * (1 + 1e-9) + 1e-13 * vscale)
            moved += int(np.count_nonzero(diff > 1e-13 * vscale))
        assert moved > 0  # some code did flip, so the check above was not vacuous
        # a perturbation a hundred times the window's size flips codes the slack does not count
        od, _ = f8.sparse_branch_fp8(q, k, v, crit, bk, x_rel_perturb=2e-4)
        assert np.any(np.abs(od - o) > slack * (1 + 1e-9) + 1e-13 * vscale)


def test_slack_is_zero_where_no_code_is_near_a_midpoint():
    # Q = 0: every P is a power of two, a code, far from any midpoint
    g = np.random.default_rng(7)
    k = g.normal(0, 1, (32, 16))
    v = g.normal(0, 1, (32, 16))
    _, _, slack, near = f8.sparse_branch_fp8(np.zeros((4, 16)), k, v, [0, 1, 3], 8, with_slack=True)
    assert not slack.any() and not near.any()
