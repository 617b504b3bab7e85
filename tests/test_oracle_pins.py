"""Pins for the fp64 CPU oracle: worked examples, closed forms, limits, invariants, brute force.

Each test ties the oracle to something other than itself: hand-derived values
(tests/golden), library routines (torch SDPA, torch elu), an independent
token-level restatement on tiny inputs, or an identity the method must satisfy.
"""

import glob
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.sla_oracle import CRITICAL, MARGINAL, NEGLIGIBLE

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return scale * np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- counts


@pytest.mark.parametrize(
    "args, expected",
    [
        ((1024, 64, 64, 0.25, 0.25), (16, 16, 4, 4)),
        ((8192, 128, 64, 0.10, 0.40), (64, 128, 13, 51)),
        ((32760, 128, 64, 0.05, 0.10), (256, 512, 26, 51)),
        ((75600, 128, 64, 0.05, 0.15), (591, 1182, 60, 177)),
        ((32700, 128, 64, 0.05, 0.0), (256, 511, 26, 0)),
        ((32760, 128, 64, 1.0, 0.0), (256, 512, 512, 0)),
        ((32760, 128, 64, 0.0, 0.0), (256, 512, 0, 0)),
        ((32760, 128, 64, 0.01, 0.0), (256, 512, 6, 0)),
        ((32760, 128, 64, 0.025, 0.0), (256, 512, 13, 0)),
        ((130 * 64, 64, 64, 0.0, 0.1), (130, 130, 0, 13)),  # 0.1*130 must give 13, not 12
        ((1, 64, 64, 0.5, 0.5), (1, 1, 1, 0)),
    ],
)
def test_block_counts(args, expected):
    assert oracle.block_counts(*args) == expected


@pytest.mark.parametrize("bad", [(0, 64, 64, 0.1, 0.1), (64, 64, 64, 0.7, 0.4), (64, 64, 64, -0.1, 0.0)])
def test_block_counts_rejects(bad):
    with pytest.raises(ValueError):
        oracle.block_counts(*bad)


# ---------------------------------------------------------------- feature map and pooling


def test_phi_closed_form_and_library():
    assert oracle.phi(np.array([0.0]))[0] == 1.0
    assert oracle.phi(np.array([2.0]))[0] == 3.0
    assert abs(oracle.phi(np.array([-1.0]))[0] - math.exp(-1.0)) < 1e-16
    x = np.linspace(-30, 30, 2001)
    ref = torch.nn.functional.elu(torch.from_numpy(x)).numpy() + 1.0
    # elu(x) + 1 computed as (exp(x) - 1) + 1 loses the low bits of small values: absolute tolerance
    np.testing.assert_allclose(oracle.phi(x), ref, rtol=1e-15, atol=2.3e-16)
    assert np.all(oracle.phi(x) > 0)


def test_pool_mean_tail_closed_form():
    # x[n, d] = n + 100 d; block 4 over N = 10 -> blocks [0,4), [4,8), [8,10).
    n = np.arange(10)[:, None] + 100.0 * np.arange(3)[None, :]
    got = oracle.pool_mean(n, 4)
    assert got.shape == (3, 3)
    np.testing.assert_array_equal(got[:, 0], [1.5, 5.5, 8.5])
    np.testing.assert_array_equal(got[:, 2], [201.5, 205.5, 208.5])


# ---------------------------------------------------------------- router


def _brute_labels(S_row, kc, kn):
    order = sorted(range(len(S_row)), key=lambda j: (-S_row[j], j))
    lab = [MARGINAL] * len(S_row)
    for r, j in enumerate(order):
        if r < kc:
            lab[j] = CRITICAL
        elif r >= len(S_row) - kn:
            lab[j] = NEGLIGIBLE
    return lab


@pytest.mark.parametrize("seed", range(6))
def test_route_matches_bruteforce_sort(seed):
    rng = np.random.default_rng(seed)
    N, D, bq, bk = int(rng.integers(40, 200)), 8, 16, 8
    q = rng.standard_normal((1, 2, N, D))
    k = rng.standard_normal((1, 2, N, D))
    # duplicate a few K blocks so exact ties occur
    k[..., 8:16, :] = k[..., 0:8, :]
    kh, kl = [(0.25, 0.25), (0.1, 0.5), (0.5, 0.0), (0.0, 0.3), (1.0, 0.0), (0.33, 0.33)][seed]
    mask, S = oracle.route(q, k, bq, bk, kh, kl)
    Nq, Nk, kc, kn = oracle.block_counts(N, bq, bk, kh, kl)
    assert mask.shape == (1, 2, Nq, Nk)
    for h, i in itertools.product(range(2), range(Nq)):
        assert list(mask[0, h, i]) == _brute_labels(list(S[0, h, i]), kc, kn)
        assert np.count_nonzero(mask[0, h, i] == CRITICAL) == kc
        assert np.count_nonzero(mask[0, h, i] == NEGLIGIBLE) == kn


def test_route_exact_ties_prefer_lower_index():
    # All KV blocks identical -> every score in a row ties; lowest indices are
    # critical, highest negligible.
    D, bk = 4, 4
    blk = np.arange(16, dtype=float).reshape(4, 4) / 7.0
    k = np.tile(blk, (6, 1))[None, None]  # 6 identical blocks
    q = _rand((1, 1, 24, D), 3)
    mask, S = oracle.route(q, k, 8, bk, 2 / 6, 3 / 6)
    assert np.all(S[0, 0] == S[0, 0, :, :1])
    for row in mask[0, 0]:
        assert list(row) == [2, 2, 1, 0, 0, 0]


def test_compressed_probs_rows_and_order():
    S = oracle.compressed_scores(_rand((2, 3, 50, 8), 1), _rand((2, 3, 50, 8), 2), 10, 5)
    P = oracle.compressed_probs(S)
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-14)
    assert np.all(P > 0)
    # softmax is monotone: ranking on P equals ranking on S
    np.testing.assert_array_equal(np.argsort(-S, axis=-1, kind="stable"), np.argsort(-P, axis=-1, kind="stable"))


def test_route_permutation_within_block_invariant():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 1, 64, 8))
    k = rng.standard_normal((1, 1, 64, 8))
    perm = np.concatenate([b * 8 + rng.permutation(8) for b in range(8)])
    m1, _ = oracle.route(q, k, 16, 8, 0.25, 0.25)
    m2, _ = oracle.route(q[..., perm, :], k[..., perm, :], 16, 8, 0.25, 0.25)
    np.testing.assert_array_equal(m1, m2)


# ---------------------------------------------------------------- worked examples


@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(GOLDEN, "hand_example_*.json"))))
def test_golden_hand_examples(path):
    g = json.load(open(path))
    p = g["params"]
    q = np.array(g["q"], float)[None, None]
    k = np.array(g["k"], float)[None, None]
    v = np.array(g["v"], float)[None, None]
    a = np.array(g["alpha"], float)[None]
    O, parts = oracle.forward(q, k, v, a, p["block_q"], p["block_kv"], p["kh"], p["kl"], return_parts=True)
    np.testing.assert_array_equal(parts["mask"][0, 0], np.array(g["expected_mask"]))
    np.testing.assert_allclose(parts["O_s"][0, 0], g["expected_O_s"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(parts["O_l"][0, 0], g["expected_O_l"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(O[0, 0], g["expected_O"], rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- limits


@pytest.mark.parametrize("N, bq, bk", [(96, 32, 16), (100, 32, 16), (77, 16, 8)])
def test_all_critical_is_dense_softmax_attention(N, bq, bk):
    B, H, D = 2, 2, 16
    q, k, v = _rand((B, H, N, D), 11), _rand((B, H, N, D), 12), _rand((B, H, N, D), 13)
    alpha = np.random.default_rng(14).uniform(size=(H, D))
    O, parts = oracle.forward(q, k, v, alpha, bq, bk, kh=1.0, kl=0.0, return_parts=True)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()
    np.testing.assert_allclose(parts["O_s"], ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(parts["O_l"], 0.0)  # no marginal block
    np.testing.assert_allclose(O, alpha[None, :, None, :] * ref, rtol=1e-12, atol=1e-12)


def _token_linear_attention(q, k, v):
    """Linear attention through the explicit N x N kernel matrix (no per-block states)."""
    fq = np.where(q > 0, q + 1, np.exp(np.minimum(q, 0)))
    fk = np.where(k > 0, k + 1, np.exp(np.minimum(k, 0)))
    A = fq @ np.swapaxes(fk, -1, -2)  # [.., N, N]
    return (A @ v) / A.sum(-1, keepdims=True)


@pytest.mark.parametrize("N, bq, bk", [(96, 32, 16), (101, 32, 16)])
def test_no_critical_no_negligible_is_linear_attention(N, bq, bk):
    B, H, D = 1, 3, 8
    q, k, v = _rand((B, H, N, D), 21), _rand((B, H, N, D), 22), _rand((B, H, N, D), 23)
    alpha = np.random.default_rng(24).uniform(size=(H, D))
    O, parts = oracle.forward(q, k, v, alpha, bq, bk, kh=0.0, kl=0.0, return_parts=True)
    ref = _token_linear_attention(q, k, v)
    np.testing.assert_allclose(parts["O_l"], ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_array_equal(parts["O_s"], 0.0)
    np.testing.assert_allclose(O, (1 - alpha)[None, :, None, :] * ref, rtol=1e-11, atol=1e-12)


def test_alpha_one_and_zero_select_branches_and_blend_is_linear():
    B, H, N, D = 1, 2, 80, 8
    q, k, v = _rand((B, H, N, D), 31), _rand((B, H, N, D), 32), _rand((B, H, N, D), 33)
    one, zero = np.ones((H, D)), np.zeros((H, D))
    a = np.random.default_rng(34).uniform(size=(H, D))
    O1, p1 = oracle.forward(q, k, v, one, 16, 8, 0.3, 0.2, return_parts=True)
    O0 = oracle.forward(q, k, v, zero, 16, 8, 0.3, 0.2)
    Oa = oracle.forward(q, k, v, a, 16, 8, 0.3, 0.2)
    np.testing.assert_array_equal(O1, p1["O_s"])
    np.testing.assert_array_equal(O0, p1["O_l"])
    np.testing.assert_allclose(Oa, a[None, :, None] * O1 + (1 - a[None, :, None]) * O0, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- token-level brute force


def _bruteforce_token_level(q, k, v, alpha, mask, bq, bk):
    """Pure-Python loops over (query token, key token) with block labels expanded to tokens."""
    N, D = q.shape
    out = np.zeros((N, D))
    for t in range(N):
        i = t // bq
        ws, wl = [], []
        for n in range(N):
            lab = mask[i, n // bk]
            if lab == CRITICAL:
                ws.append((math.exp(sum(q[t, d] * k[n, d] for d in range(D)) / math.sqrt(D)), n))
            elif lab == MARGINAL:
                fq = [q[t, d] + 1 if q[t, d] > 0 else math.exp(q[t, d]) for d in range(D)]
                fk = [k[n, d] + 1 if k[n, d] > 0 else math.exp(k[n, d]) for d in range(D)]
                wl.append((sum(a * b for a, b in zip(fq, fk)), n))
        for d in range(D):
            os_ = sum(w * v[n, d] for w, n in ws) / sum(w for w, _ in ws) if ws else 0.0
            ol_ = sum(w * v[n, d] for w, n in wl) / sum(w for w, _ in wl) if wl else 0.0
            out[t, d] = alpha[d] * os_ + (1 - alpha[d]) * ol_
    return out


@pytest.mark.parametrize("seed, N, bq, bk", [(0, 24, 8, 4), (1, 23, 8, 4), (2, 30, 4, 8), (3, 17, 8, 8)])
def test_forward_matches_token_level_bruteforce(seed, N, bq, bk):
    rng = np.random.default_rng(seed)
    D = 3
    q, k, v = rng.standard_normal((N, D)), rng.standard_normal((N, D)), rng.standard_normal((N, D))
    alpha = rng.uniform(size=D)
    Nq, Nk = -(-N // bq), -(-N // bk)
    mask = rng.integers(0, 3, size=(Nq, Nk)).astype(np.int8)
    mask[0, :] = MARGINAL  # a row with no critical block
    mask[-1, :] = CRITICAL  # a row with no marginal block
    O = oracle.forward(q[None, None], k[None, None], v[None, None], alpha[None], bq, bk,
                       mask=mask[None, None])[0, 0]
    np.testing.assert_allclose(O, _bruteforce_token_level(q, k, v, alpha, mask, bq, bk), rtol=1e-12, atol=1e-12)


def test_kv_states_match_outer_product_loops():
    rng = np.random.default_rng(5)
    N, D, bk = 13, 3, 5
    k, v = rng.standard_normal((N, D)), rng.standard_normal((N, D))
    h, z = oracle.kv_states(k, v, bk)
    assert h.shape == (3, D, D) and z.shape == (3, D)
    for j in range(3):
        for a in range(D):
            for b in range(D):
                ref = sum((k[n, a] + 1 if k[n, a] > 0 else math.exp(k[n, a])) * v[n, b]
                          for n in range(j * bk, min(N, (j + 1) * bk)))
                assert abs(h[j, a, b] - ref) < 1e-13
            refz = sum((k[n, a] + 1 if k[n, a] > 0 else math.exp(k[n, a]))
                       for n in range(j * bk, min(N, (j + 1) * bk)))
            assert abs(z[j, a] - refz) < 1e-13


# ---------------------------------------------------------------- identities and invariants


def test_subtraction_identity_for_marginal_sums():
    # SPLA 2.2: the linear term over the unselected blocks equals the global one
    # minus the one over the selected blocks.
    rng = np.random.default_rng(9)
    Nk, D = 12, 4
    h, z = rng.standard_normal((Nk, D, D)), rng.standard_normal((Nk, D))
    rows = rng.integers(0, 3, size=(7, Nk)).astype(np.int8)
    Hs, Zs = oracle.marginal_sums(rows, h, z)
    for r in range(7):
        sel = rows[r] != MARGINAL
        np.testing.assert_allclose(Hs[r], h.sum(0) - h[sel].sum(0), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(Zs[r], z.sum(0) - z[sel].sum(0), rtol=1e-12, atol=1e-12)


def _case(seed, N=96, D=8, B=1, H=2):
    rng = np.random.default_rng(seed)
    q, k, v = rng.standard_normal((B, H, N, D)), rng.standard_normal((B, H, N, D)), rng.standard_normal((B, H, N, D))
    return q, k, v, rng.uniform(size=(H, D))


def test_negligible_blocks_are_skipped():
    q, k, v, a = _case(41)
    O, parts = oracle.forward(q, k, v, a, 16, 8, 0.25, 0.25, return_parts=True)
    mask = parts["mask"]
    for i in range(mask.shape[2]):
        # change V only inside the blocks that query block i labels negligible
        negl = np.nonzero(mask[0, 0, i] == NEGLIGIBLE)[0]
        assert len(negl) == 3
        v2 = v.copy()
        for j in negl:
            v2[0, 0, j * 8:(j + 1) * 8] += 100.0
        O2 = oracle.forward(q, k, v2, a, 16, 8, 0.25, 0.25)
        np.testing.assert_array_equal(O2[0, 0, i * 16:(i + 1) * 16], O[0, 0, i * 16:(i + 1) * 16])
        assert not np.allclose(O2[0, 0], O[0, 0])  # the change is visible elsewhere


def test_value_affine_equivariance_and_range():
    q, k, v, a = _case(42)
    O = oracle.forward(q, k, v, a, 16, 8, 0.25, 0.25)
    c, b = -2.5, np.arange(8) * 0.5
    O2 = oracle.forward(q, k, c * v + b, a, 16, 8, 0.25, 0.25)
    np.testing.assert_allclose(O2, c * O + b, rtol=1e-12, atol=1e-12)
    lo, hi = v.min(axis=2, keepdims=True), v.max(axis=2, keepdims=True)
    assert np.all(O >= lo - 1e-12) and np.all(O <= hi + 1e-12)


def test_permutation_within_kv_block_leaves_output_unchanged():
    q, k, v, a = _case(43)
    rng = np.random.default_rng(0)
    perm = np.concatenate([b * 8 + rng.permutation(8) for b in range(12)])
    O = oracle.forward(q, k, v, a, 16, 8, 0.25, 0.25)
    O2 = oracle.forward(q, k[..., perm, :], v[..., perm, :], a, 16, 8, 0.25, 0.25)
    np.testing.assert_allclose(O2, O, rtol=1e-12, atol=1e-12)


def test_normalisation_sums_positive_and_finite():
    q, k, v, a = _case(44, N=130)
    _, parts = oracle.forward(q, k, v, a, 16, 8, 0.3, 0.3, return_parts=True)
    ls, ld = parts["softmax_sum"], parts["linear_den"]
    assert np.all(np.isfinite(ls)) and np.all(ls >= 1.0)  # max-subtracted softmax row sums
    assert np.all(np.isfinite(ld)) and np.all(ld > 0.0)


def test_empty_branches_are_zero():
    q, k, v, a = _case(45)
    _, p0 = oracle.forward(q, k, v, a, 16, 8, 0.0, 0.5, return_parts=True)
    np.testing.assert_array_equal(p0["O_s"], 0.0)
    _, p1 = oracle.forward(q, k, v, a, 16, 8, 1.0, 0.0, return_parts=True)
    np.testing.assert_array_equal(p1["O_l"], 0.0)
    _, p2 = oracle.forward(q, k, v, a, 16, 8, 0.5, 0.5, return_parts=True)  # nothing marginal
    np.testing.assert_array_equal(p2["O_l"], 0.0)


def test_sampled_rows_equal_full_run():
    q, k, v, a = _case(46, N=100, B=2, H=2)
    O = oracle.forward(q, k, v, a, 16, 8, 0.25, 0.25)
    Os = oracle.forward(q, k, v, a, 16, 8, 0.25, 0.25, heads=[(1, 0)], query_blocks=[0, 6])
    np.testing.assert_array_equal(Os[1, 0, :16], O[1, 0, :16])
    np.testing.assert_array_equal(Os[1, 0, 96:], O[1, 0, 96:])
    assert np.isnan(Os[0, 0]).all() and np.isnan(Os[1, 0, 16:96]).all()
