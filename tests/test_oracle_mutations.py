"""Plant plausible mistakes in the oracle (CPU only) and check that a pin catches each one.

Every mutation is applied with monkeypatch to ``oracle.sla_oracle`` and undone
after the test; the pins themselves are the functions of test_oracle_pins.
"""

import glob
import math
import os

import numpy as np
import pytest

import oracle.sla_oracle as so
from tests import test_oracle_pins as pins

GOLDEN = sorted(glob.glob(os.path.join(os.path.dirname(__file__), "golden", "hand_example_*.json")))


def _patch(monkeypatch, name, fn):
    """Replace ``name`` both in the implementation module and in the package namespace."""
    import oracle

    monkeypatch.setattr(so, name, fn)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, fn)


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def _golden_any_fails():
    return any(_fails(pins.test_golden_hand_examples, p) for p in GOLDEN)


def test_mutation_phi_without_plus_one(monkeypatch):
    _patch(monkeypatch, "phi", lambda x: np.where(np.asarray(x) > 0, x, np.expm1(np.minimum(x, 0))) + 1e-3)
    assert _golden_any_fails()


def test_mutation_missing_score_scale(monkeypatch):
    orig = so.sparse_branch

    def unscaled(q_blk, k, v, crit, bk):
        return orig(q_blk * math.sqrt(k.shape[1]), k, v, crit, bk)

    _patch(monkeypatch, "sparse_branch", unscaled)
    assert _golden_any_fails()


def test_mutation_tie_break_reversed(monkeypatch):
    orig = so.route_from_scores

    def reversed_ties(S, kc, kn):
        return orig(S[..., ::-1], kc, kn)[..., ::-1]

    _patch(monkeypatch, "route_from_scores", reversed_ties)
    assert _fails(pins.test_route_exact_ties_prefer_lower_index)


def test_mutation_critical_count_rounded_down(monkeypatch):
    orig = so.block_counts

    def floor_counts(N, bq, bk, kh, kl):
        Nq, Nk, kc, kn = orig(N, bq, bk, kh, kl)
        return Nq, Nk, (int(round(kh * 1e6)) * Nk) // 1_000_000, kn

    _patch(monkeypatch, "block_counts", floor_counts)
    assert _fails(pins.test_block_counts, (32760, 128, 64, 0.05, 0.10), (256, 512, 26, 51))


def test_mutation_alpha_on_wrong_branch(monkeypatch):
    orig = so.forward

    def swapped(q, k, v, alpha, *a, **kw):
        return orig(q, k, v, 1.0 - so.as_f64(alpha), *a, **kw)

    _patch(monkeypatch, "forward", swapped)
    assert _golden_any_fails()


def test_mutation_transposed_state(monkeypatch):
    orig = so.kv_states

    def transposed(k, v, bk):
        h, z = orig(k, v, bk)
        return np.swapaxes(h, -1, -2), z

    _patch(monkeypatch, "kv_states", transposed)
    assert _fails(pins.test_forward_matches_token_level_bruteforce, 0, 24, 8, 4)


def test_mutation_negligible_counted_as_marginal(monkeypatch):
    def wrong_sums(rows, h, z):
        w = (rows != so.CRITICAL).astype(np.float64)
        Nk, D = z.shape
        return (w @ h.reshape(Nk, D * D)).reshape(-1, D, D), w @ z

    _patch(monkeypatch, "marginal_sums", wrong_sums)
    assert _golden_any_fails()


def test_mutation_pool_sum_instead_of_mean(monkeypatch):
    def pool_sum(x, block):
        N = x.shape[-2]
        return np.stack([x[..., s:min(N, s + block), :].sum(axis=-2) for s in range(0, N, block)], axis=-2)

    _patch(monkeypatch, "pool_mean", pool_sum)
    assert _fails(pins.test_pool_mean_tail_closed_form)


def test_mutation_softmax_over_all_keys(monkeypatch):
    # Not re-normalising over the critical set: the softmax runs over every key.
    orig = so.sparse_branch

    def all_keys(q_blk, k, v, crit, bk):
        every = list(range(-(-k.shape[0] // bk)))
        return orig(q_blk, k, v, every if len(crit) else crit, bk)

    _patch(monkeypatch, "sparse_branch", all_keys)
    assert _golden_any_fails()


# ---------------------------------------------------------------- the low-bit oracle

from oracle import sla_oracle_fp8 as f8  # noqa: E402
from tests import test_oracle_fp8_pins as pins8  # noqa: E402


def test_mutation_fp8_half_step_too_small(monkeypatch):
    monkeypatch.setattr(f8, "HALF_STEP_REL", 2.0 ** -5)  # a quarter step: rounding can exceed it
    assert _fails(pins8.test_a_key_half_a_step_from_a_code_reaches_the_bound)
    assert _fails(pins8.test_bound_by_hand_normal_terms_dominate)


def test_mutation_fp8_half_step_too_large(monkeypatch):
    monkeypatch.setattr(f8, "HALF_STEP_REL", 2.0 ** -3)  # a whole step: no rounding comes near it
    assert _fails(pins8.test_a_key_half_a_step_from_a_code_reaches_the_bound)


def test_mutation_fp8_subnormal_floor_dropped(monkeypatch):
    monkeypatch.setattr(f8, "HALF_STEP_ABS", 0.0)
    assert _fails(pins8.test_every_schedule_stays_inside_the_bound, 1.0)
    assert _fails(pins8.test_subnormal_floor_is_reached_by_a_low_reference)


def _branch_variant(drop_v_ratio=False, raw_q=False):
    """A copy of the low-bit branch with one planted mistake."""
    import math as _m

    def branch(q_blk, k, v, crit_blocks, block_kv):
        N, D = k.shape
        bq = q_blk.shape[0]
        if len(crit_blocks) == 0:
            return np.zeros((bq, D)), np.zeros(bq), np.zeros((bq, D))
        sq = f8.pow2_scale(float(np.abs(q_blk).max()))
        qh = q_blk if raw_q else f8.e4m3_round(q_blk / sq) * sq
        xs, vs, svs = [], [], []
        for j in sorted(int(j) for j in crit_blocks):
            a, e = j * block_kv, min(N, (j + 1) * block_kv)
            sk = f8.pow2_scale(float(np.abs(k[a:e]).max()))
            xs.append((qh @ (f8.e4m3_round(k[a:e] / sk) * sk).T) / _m.sqrt(D) * _m.log2(_m.e))
            sv = f8.pow2_scale(float(np.abs(v[a:e]).max()))
            vs.append(f8.e4m3_round(v[a:e] / sv) * sv)
            svs.append(np.full(e - a, sv))
        x, vh, sv = np.concatenate(xs, axis=1), np.concatenate(vs), np.concatenate(svs)
        p = np.exp2(x - x.max(axis=1, keepdims=True))
        l = p.sum(axis=1)
        ratio = np.ones_like(sv) if drop_v_ratio else sv.max() / sv
        w = np.maximum(f8.HALF_STEP_REL * p, f8.HALF_STEP_ABS * ratio[None, :])
        return (p @ vh) / l[:, None], l, (w @ np.abs(vh)) / l[:, None]

    return branch


def test_mutation_fp8_variant_harness_is_faithful(monkeypatch):
    # the unmutated copy passes the pins the mutations below are caught by
    monkeypatch.setattr(f8, "sparse_branch_fp8", _branch_variant())
    pins8.test_every_schedule_stays_inside_the_bound(1.0)
    pins8.test_subnormal_floor_is_reached_by_a_low_reference()
    pins8.test_centre_is_the_exact_branch_of_the_quantised_operands()


def test_mutation_fp8_v_scale_ratio_dropped_from_the_floor(monkeypatch):
    monkeypatch.setattr(f8, "sparse_branch_fp8", _branch_variant(drop_v_ratio=True))
    assert _fails(pins8.test_subnormal_floor_is_reached_by_a_low_reference)


def test_mutation_fp8_q_left_unquantised(monkeypatch):
    monkeypatch.setattr(f8, "sparse_branch_fp8", _branch_variant(raw_q=True))
    assert _fails(pins8.test_centre_is_the_exact_branch_of_the_quantised_operands)


def test_mutation_fp8_ties_away_from_zero(monkeypatch):
    def away(x):
        x = np.asarray(x, dtype=np.float64)
        ax = np.abs(x)
        _, ex = np.frexp(ax)
        q = np.exp2(np.maximum(ex - 1.0, -6.0) - 3.0)
        r = np.minimum(np.floor(ax / q + 0.5) * q, f8.E4M3_MAX)
        return np.where(x < 0, -r, r)

    monkeypatch.setattr(f8, "e4m3_round", away)
    assert _fails(pins8.test_halfway_cases_round_to_the_even_code)


# ---------------------------------------------------------------- the backward oracle

from oracle import sla_oracle_bwd as bw  # noqa: E402
from tests import test_oracle_bwd_pins as pinsb  # noqa: E402


def test_mutation_bwd_feature_map_derivative_dropped(monkeypatch):
    monkeypatch.setattr(bw, "dphi", lambda x: np.ones_like(np.asarray(x, dtype=np.float64)))
    assert _fails(pinsb.test_matches_central_differences, 0, 8)


def test_mutation_bwd_transposed_states(monkeypatch):
    orig = bw.kv_states

    def transposed(k, v, bk):
        h, z = orig(k, v, bk)
        return np.swapaxes(h, -1, -2), z

    monkeypatch.setattr(bw, "kv_states", transposed)
    assert _fails(pinsb.test_matches_central_differences, 0, 8)


# ---------------------------------------------------------------- the PISA oracle

import types  # noqa: E402

from tests import test_oracle_pisa_pins as pinsp  # noqa: E402


def _mutated_pisa(old, new):
    """A copy of oracle.sla_oracle_pisa with one source fragment replaced."""
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "sla_oracle_pisa.py")
    src = open(path).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle.sla_oracle_pisa_mutant")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), path, "exec"), mod.__dict__)
    return mod


FIRST_ORDER = "+ (qb * scale) @ Hbar * A.sum(axis=1, keepdims=True)"


@pytest.mark.parametrize("new", ["", "- (qb * scale) @ Hbar * A.sum(axis=1, keepdims=True)",
                                 "+ qb @ Hbar * A.sum(axis=1, keepdims=True)"],
                         ids=["dropped", "sign", "unscaled"])
def test_mutation_pisa_first_order_term(monkeypatch, new):
    monkeypatch.setattr(pinsp, "pisa", _mutated_pisa(FIRST_ORDER, new))
    assert _fails(pinsp.test_error_falls_as_the_square_of_the_key_spread)


def test_mutation_pisa_denominator_without_block_counts(monkeypatch):
    monkeypatch.setattr(pinsp, "pisa", _mutated_pisa("den = Pe.sum(axis=1) + A @ n[~crit]",
                                                     "den = Pe.sum(axis=1) + A.sum(axis=1)"))
    assert _fails(pinsp.test_blocks_of_equal_keys_make_the_expansion_exact, 1)


# ---------------------------------------------------------------- the second-order block score

from oracle import sla_oracle_route2 as r2  # noqa: E402
from tests import test_oracle_route2_pins as pinsr  # noqa: E402


def test_mutation_route2_quadratic_term_without_the_half(monkeypatch):
    orig = r2.block_variance
    monkeypatch.setattr(r2, "block_variance", lambda k, bk: 2.0 * orig(k, bk))
    assert _fails(pinsr.test_score_matches_the_exact_block_mean_to_fourth_order)


def test_mutation_route2_sample_variance(monkeypatch):
    def sample_var(k, bk):
        N = k.shape[-2]
        return np.stack([np.var(k[..., s:min(N, s + bk), :], axis=-2, ddof=1) for s in range(0, N, bk)], axis=-2)

    monkeypatch.setattr(r2, "block_variance", sample_var)
    assert _fails(pinsr.test_score_matches_the_exact_block_mean_to_fourth_order)


# ---------------------------------------------------------------- the dropped-linear-branch forward

def test_mutation_dropped_forward_renormalised(monkeypatch):
    # dividing by alpha's channel mean (renormalising what is left) must fail a pin
    from oracle import sla_oracle_salad as sd
    from tests import test_oracle_salad_pins as pins
    plain = sd.forward_dropped

    def renormalised(q, k, v, alpha, *args, **kw):
        a = np.asarray(alpha, dtype=np.float64)
        return plain(q, k, v, alpha, *args, **kw) / a.mean(axis=-1)[None, :, None, None]

    monkeypatch.setattr(sd, "forward_dropped", renormalised)
    with pytest.raises(AssertionError):
        pins.test_every_block_critical_is_alpha_times_dense_attention()
