"""Pins of the low-bit sparse-branch reading in oracle/sla_oracle_fp8.py.

The e4m3 rounding is checked against the format itself (every finite code is a fixed
point, halfway cases go to the even code, saturation, subnormal steps) and against
torch's own float8_e4m3fn conversion, and the decoder against every byte. The branch's
centre (P unrounded) must equal the full-precision branch when the operands already lie
on the scaled e4m3 grid. Its bound is derived by hand on two-block rows, and checked
against single-pass rounding schedules written here from the reading (the reference at
the row maximum, at the running maximum, moved only past a slack, held low, drawn at
random; the unit at the largest V scale or at each block's own): every schedule stays
inside the bound, and a key half a step from a code comes within 10% of it.
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


def _grid_inputs(g, n_blocks, bk, D, v_exps):
    """K, V whose blocks lie on the scaled e4m3 grid, V block j at scale 2^v_exps[j]."""
    k = f8.e4m3_round(g.normal(0, 20, (n_blocks * bk, D))) / 64.0
    v = f8.e4m3_round(g.normal(0, 20, (n_blocks * bk, D))) / 64.0
    for j, e in enumerate(v_exps):
        v[j * bk:(j + 1) * bk] *= 2.0 ** e
    return k, v


def test_centre_equals_exact_branch_on_the_grid():
    # Q, K, V already on the scaled e4m3 grid (V blocks at 2^0, 2^2, 2^-3): quantising them
    # changes nothing, and the centre (P unrounded) is the full-precision branch
    g = np.random.default_rng(2)
    D, bk = 16, 8
    k, v = _grid_inputs(g, 5, bk, D, [0, 0, 2, 0, -3])
    q = f8.e4m3_round(g.normal(0, 20, (8, D))) / 256.0
    crit = [0, 2, 4]
    o8, l8, bound = f8.sparse_branch_fp8(q, k, v, crit, bk)
    o, l = so.sparse_branch(q, k, v, crit, bk)
    np.testing.assert_allclose(o8, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l8, l, rtol=1e-13)
    assert np.all(bound > 0)


def test_centre_is_the_exact_branch_of_the_quantised_operands():
    # off-grid inputs: quantising Q (one query block), K and V (per KV block) with the
    # format's own rounding, then running the full-precision branch, gives the centre
    g = np.random.default_rng(12)
    D, bk = 16, 8
    q = g.normal(0, 1.3, (8, D))
    k = g.normal(0, 1.0, (48, D)) * np.repeat(2.0 ** g.integers(-2, 3, 6), bk)[:, None]
    v = g.normal(0, 1.0, (48, D)) * np.repeat(2.0 ** g.integers(-6, 3, 6), bk)[:, None]
    qc, qs = f8.quantize_blocks(q, q.shape[0])
    kc, ks = f8.quantize_blocks(k, bk)
    vc, vs = f8.quantize_blocks(v, bk)
    crit = [1, 2, 5]
    o, l = so.sparse_branch(qc * qs[0], kc * np.repeat(ks, bk)[:, None], vc * np.repeat(vs, bk)[:, None], crit, bk)
    o8, l8, _ = f8.sparse_branch_fp8(q, k, v, crit, bk)
    np.testing.assert_allclose(o8, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l8, l, rtol=1e-12)
    # and the quantisation does move it away from the unquantised branch
    assert np.abs(o8 - so.sparse_branch(q, k, v, crit, bk)[0]).max() > 1e-3


def _two_block_row(x1):
    # one query row q = e_0; block 0's keys are 0 (x = 0), block 1's are t e_0 with
    # t = 4 x1 ln 2, so block 1's x = t / sqrt(16) * log2(e) = x1. V: block 0's rows all
    # v0 (scale 2^-7), block 1's rows all v0 / 32 (scale 2^-12, the same codes).
    D, bk = 16, 8
    q = np.zeros((1, D))
    q[0, 0] = 1.0
    k = np.zeros((16, D))
    k[8:, 0] = 4.0 * x1 * math.log(2.0)
    v0 = np.array([1.5, 0.5, -1.0, 0.25] * 4)
    v = np.concatenate([np.tile(v0, (8, 1)), np.tile(v0 / 32.0, (8, 1))])
    return q, k, v, v0


def test_bound_by_hand_normal_terms_dominate():
    # x1 = 2: m = 2, P = 2^-2 on block 0 and 1 on block 1, l = 8 (0.25 + 1) = 10.
    # centre: (8 * 0.25 v0 + 8 * v0 / 32) / 10 = 0.225 v0.
    # per key: block 0 max(2^-4 * 2^-2, 2^-10 * 1) = 2^-6 times |v0|;
    #          block 1 max(2^-4 * 1, 2^-10 * 32) = 2^-4 times |v0| / 32;
    # bound = 8 (2^-6 + 2^-4 / 32) |v0| / 10 = 0.0140625 |v0|
    q, k, v, v0 = _two_block_row(2.0)
    # K's codes are exact only up to e4m3: take x1 from the quantised key
    o, l, bound = f8.sparse_branch_fp8(q, k, v, [0, 1], 8)
    kq = f8.e4m3_round(k[8, 0] / f8.pow2_scale(k[8, 0])) * f8.pow2_scale(k[8, 0])
    x1 = kq / 4.0 * math.log2(math.e)
    p0 = 2.0 ** -x1
    np.testing.assert_allclose(l, [8 * (p0 + 1.0)], rtol=1e-14)
    np.testing.assert_allclose(o[0], (8 * p0 * v0 + 8 * v0 / 32) / (8 * (p0 + 1.0)), rtol=1e-13)
    w0 = max(2.0 ** -4 * p0, 2.0 ** -10)
    w1 = max(2.0 ** -4, 2.0 ** -10 * 32)
    np.testing.assert_allclose(bound[0], 8 * (w0 + w1 / 32) * np.abs(v0) / (8 * (p0 + 1.0)), rtol=1e-13)
    # and with the exact x1 = 2 the numbers are the ones above
    assert abs(x1 - 2.0) < 0.05
    np.testing.assert_allclose(bound[0], 0.0140625 * np.abs(v0), rtol=0.05)


def test_bound_by_hand_subnormal_floor_dominates():
    # x1 = 8: block 0's P = 2^-8, whose relative half step 2^-12 lies below the floor 2^-10:
    # block 0 max(2^-4 * 2^-8, 2^-10) = 2^-10; block 1 max(2^-4, 2^-10 * 32) = 2^-4;
    # bound = 8 (2^-10 + 2^-4 / 32) |v0| / l = 0.0234375 |v0| / (8 (2^-8 + 1)) at x1 = 8
    q, k, v, v0 = _two_block_row(8.0)
    o, l, bound = f8.sparse_branch_fp8(q, k, v, [0, 1], 8)
    kq = f8.e4m3_round(k[8, 0] / f8.pow2_scale(k[8, 0])) * f8.pow2_scale(k[8, 0])
    x1 = kq / 4.0 * math.log2(math.e)
    p0 = 2.0 ** -x1
    assert 2.0 ** -4 * p0 < 2.0 ** -10
    np.testing.assert_allclose(bound[0], 8 * (2.0 ** -10 + 2.0 ** -4 / 32) * np.abs(v0) / (8 * (p0 + 1.0)),
                               rtol=1e-13)
    assert abs(x1 - 8.0) < 0.2


# ---------------------------------------------------------------- rounding schedules
# Each schedule rounds P the way some single-pass kernel might, from the reading alone:
# key n of block j is coded as e4m3(2^(x_n - r_n) sv_j / u) with r_n <= m and
# sv_j <= u <= s_max, and contributes code * 2^(r_n - m) * u / sv_j * vhat_n; l sums the
# unrounded P. Written here independently of the oracle's branch.


def _quantised_row_data(q_blk, k, v, crit, bk):
    D = k.shape[1]
    sq = f8.pow2_scale(float(np.abs(q_blk).max()))
    qh = f8.e4m3_round(q_blk / sq) * sq
    xs, vh, sv, blk = [], [], [], []
    for j in sorted(crit):
        kb, vb = k[j * bk:(j + 1) * bk], v[j * bk:(j + 1) * bk]
        sk, s_v = f8.pow2_scale(float(np.abs(kb).max())), f8.pow2_scale(float(np.abs(vb).max()))
        xs.append(qh @ (f8.e4m3_round(kb / sk) * sk).T * (math.log2(math.e) / math.sqrt(D)))
        vh.append(f8.e4m3_round(vb / s_v) * s_v)
        sv += [s_v] * kb.shape[0]
        blk += [j] * kb.shape[0]
    return np.concatenate(xs, axis=1), np.concatenate(vh), np.array(sv), np.array(blk)


def _schedule(q_blk, k, v, crit, bk, name, rng=None):
    x, vh, sv, blk = _quantised_row_data(q_blk, k, v, crit, bk)
    rows, n = x.shape
    m = x.max(axis=1)
    s_max = sv.max()
    out = np.zeros((rows, vh.shape[1]))
    for t in range(rows):
        xt = x[t]
        if name == "rowmax":
            r = np.full(n, m[t])
        elif name == "running":
            r = np.maximum.accumulate(xt)
        elif name.startswith("lazy"):
            slack = float(name[4:])
            r = np.empty(n)
            cur = None
            for j in np.unique(blk):
                sel = blk == j
                bm = xt[sel].max()
                if cur is None or bm > cur + slack:
                    cur = bm
                r[sel] = cur
        elif name == "low":
            r = np.maximum(np.full(n, m[t] - 7.9), xt - 7.9)
            r = np.minimum(r, m[t])
        elif name == "random":
            lo = np.maximum.accumulate(xt) - 8.0
            r = lo + rng.uniform(0, 1, n) * (m[t] - lo)
        else:
            raise ValueError(name)
        u = sv if name == "rowmax_perblock" else np.full(n, s_max)
        y = np.exp2(xt - r) * sv / u
        assert np.all(y <= 448.0)
        contrib = f8.e4m3_round(y) * np.exp2(r - m[t]) * u / sv
        out[t] = (contrib @ vh) / np.exp2(xt - m[t]).sum()
    return out


def _schedule_perblock_unit(q_blk, k, v, crit, bk):
    x, vh, sv, _ = _quantised_row_data(q_blk, k, v, crit, bk)
    m = x.max(axis=1, keepdims=True)
    y = np.exp2(x - m)  # u = sv_j: no V-scale ratio before rounding
    return (f8.e4m3_round(y) @ vh) / np.exp2(x - m).sum(axis=1, keepdims=True)


SCHEDULES = ["rowmax", "running", "lazy8", "lazy4", "lazy0", "low", "random"]


@pytest.mark.parametrize("vscale", [1.0, 1000.0, 1e-3])
def test_every_schedule_stays_inside_the_bound(vscale):
    g = np.random.default_rng(6)
    D, bk = 32, 16
    q = g.normal(0, 1.0, (64, D)) * 2.0
    k = g.normal(0, 1.0, (256, D)) * np.repeat(2.0 ** g.integers(-1, 2, 16), 16)[:, None]
    # V blocks 2^-12 .. 2^2 apart: small-scale blocks' codes fall into the subnormal range
    v = g.normal(0, 1.0, (256, D)) * np.repeat(2.0 ** g.integers(-12, 3, 16), 16)[:, None] * vscale
    crit = [0, 2, 3, 5, 8, 9, 12, 15]
    o, _, bound = f8.sparse_branch_fp8(q, k, v, crit, bk)
    used = 0.0
    for name in SCHEDULES:
        os_ = _schedule(q, k, v, crit, bk, name, rng=np.random.default_rng(1))
        d = np.abs(os_ - o)
        assert np.all(d <= bound * (1 + 1e-9) + 1e-15 * vscale), name
        assert np.any(d > 0), name  # the schedule did round something
        used = max(used, float((d / bound).max()))
    ob = _schedule_perblock_unit(q, k, v, crit, bk)
    assert np.all(np.abs(ob - o) <= bound * (1 + 1e-9) + 1e-15 * vscale)
    assert used > 0.05  # the bound is not vacuous on ordinary rows


def test_a_key_half_a_step_from_a_code_reaches_the_bound():
    # One critical block of 8 equal keys (every P = 1) with equal V rows, and a reference
    # log2(1.0625) below the row maximum: y = 2^(x - r) = 1.0625 lies on the midpoint between
    # the codes 1 and 1.125, so either neighbour is off by 2^-4 of y; carried back by
    # 2^(r - m) = 1/1.0625 that is 0.94 of the bound's 2^-4 per key.
    D, bk = 16, 8
    g = np.random.default_rng(9)
    k = np.tile(f8.e4m3_round(g.normal(0, 20, (1, D))) / 64.0, (bk, 1))
    v = np.tile(f8.e4m3_round(g.normal(0, 20, (1, D))) / 64.0, (bk, 1))  # equal rows: errors add up
    q = f8.e4m3_round(g.normal(0, 20, (2, D))) / 256.0
    o, l, bound = f8.sparse_branch_fp8(q, k, v, [0], bk)
    np.testing.assert_allclose(l, [8.0, 8.0], rtol=1e-14)
    x, vh, sv, _ = _quantised_row_data(q, k, v, [0], bk)
    m = x.max(axis=1)
    r = m - math.log2(1.0625)  # y = 1.0625 exactly up to rounding of the log
    y = np.exp2(x - r[:, None])
    assert np.allclose(y, 1.0625, rtol=1e-12)
    yq = f8.e4m3_round(y * (1 + 1e-12))  # just above the midpoint: 1.125; just below: 1.0
    yq_lo = f8.e4m3_round(y * (1 - 1e-12))
    for codes in (yq, yq_lo):
        os_ = ((codes * np.exp2(r - m)[:, None]) @ vh) / l[:, None]
        d = np.abs(os_ - o)
        assert np.all(d <= bound * (1 + 1e-9))
        assert np.all(d >= 0.9 * bound - 1e-15)


def test_subnormal_floor_is_reached_by_a_low_reference():
    # A key with P close to 2^-10 coded at its own value: y = P rounds to 0 or 2^-9, losing or
    # gaining about 2^-10 = the floor term; with u = s_max and a V block 2^-5 below the
    # largest, y = P / 32 is deeper in the subnormal range and the floor term grows by 32.
    D, bk = 16, 8
    q = np.zeros((1, D))
    q[0, 0] = 1.0
    k = np.zeros((16, D))
    # block 1's keys put x about 10 below block 0's (x = 0)
    k[8:, 0] = -40.0 * math.log(2.0)
    v = np.zeros((16, D))
    v[:8] = 1.0
    v[8:] = 1.0 / 32.0
    o, l, bound = f8.sparse_branch_fp8(q, k, v, [0, 1], bk)
    x, vh, sv, _ = _quantised_row_data(q, k, v, [0, 1], bk)
    p1 = 2.0 ** x[0, 8]
    assert 2.0 ** -11 < p1 < 2.0 ** -9
    # block 1's contribution to the bound: 8 * 2^-10 * 32 * (1/32) / l = 8 * 2^-10 / l
    block0 = 8 * 2.0 ** -4 * 1.0 / l[0]
    np.testing.assert_allclose(bound[0, 0], block0 + 8 * 2.0 ** -10 / l[0], rtol=1e-12)
