"""GPU parity of the router and feature-map variants ("SPLA - Atención de Bloque Dispersa más
Lineal para el Modelado de Contexto Largo", §2.1 second-order block score, §2.3 exponential
feature map) and of SALAD's branch dropping ("SALAD: Achieve High-Sparsity Attention via
Efficient Linear Attention Tuning for Video Diffusion Transformer", §2) against their fp64
oracles, through the C ABI.

Labels must match the oracle's bit for bit except near ties (counted); the second-order
scores within 1e-12 relative; outputs within max-abs 2e-2 / mean-abs 2e-3 with the oracle's
labels passed in.
"""

import numpy as np
import pytest
import torch

from oracle import sla_oracle_expmap as xm
from oracle import sla_oracle_route2 as r2
from oracle import sla_oracle_salad as sd
from sparse_linear_attention_sla_b200 import binding
from sparse_linear_attention_sla_b200.workloads import WORKLOADS, make_inputs, random_inputs
from tests.parity_utils import assert_outputs_close, label_mismatches

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, N, D, bq, kh, kl
    (1, 2, 1024, 64, 64, 0.25, 0.25),
    (2, 2, 333, 128, 128, 0.2, 0.3),
    (1, 3, 4113, 128, 128, 0.1, 0.2),
    (1, 2, 1000, 128, 64, 0.0, 0.0),
]


def _second_order_parity(q, k, bq, kh, kl):
    mask, crit, S2 = binding.route_variant(q, k, bq, 64, kh, kl, block_score=1, want_scores=True, want_crit=True)
    B, H = q.shape[:2]
    p = binding.problem(*q.shape, bq, 64, kh, kl)
    _, Nk, kc, kn = binding.counts(p)
    gm, gs, gc = mask.cpu().numpy(), S2.cpu().numpy(), crit.cpu().numpy()
    om = gm.copy()
    total = excused = 0
    for b in range(B):
        for h in range(H):
            rm, S = r2.route_second_order(q[b, h].cpu(), k[b, h].cpu(), bq, 64, kh, kl)
            om[b, h] = rm
            rel = np.abs(gs[b, h] - S).max() / max(np.abs(S).max(), 1e-300)
            assert rel < 1e-12, f"second-order scores differ by {rel:.2e} (relative)"
            t, e = label_mismatches(gm[b, h], rm, S, kc, kn)
            total += t
            excused += e
            for i in range(gm.shape[2]):
                np.testing.assert_array_equal(gc[b, h, i], np.nonzero(gm[b, h, i] == 2)[0])
    assert total == excused, f"{total - excused} label mismatches outside near ties"
    if total:
        print(f"near-tie mismatches (excused): {total}")
    return torch.from_numpy(om).to(q.device), total


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_second_order_router_matches_oracle(cuda_device, case):
    B, H, N, D, bq, kh, kl = case
    q, k, _, _ = random_inputs(B, H, N, D, seed=5 * N + D, device=cuda_device)
    _second_order_parity(q, k, bq, kh, kl)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_exp_feature_map_matches_oracle(cuda_device, case):
    B, H, N, D, bq, kh, kl = case
    q, k, v, alpha = random_inputs(B, H, N, D, seed=3 * N + D, device=cuda_device)
    mask, _, _ = binding.route(q, k, bq, 64, kh, kl)
    out = binding.forward_variant(q, k, v, alpha, bq, 64, kh, kl, feature_map=1, mask=mask)
    ref = xm.forward_expmap(q.cpu(), k.cpu(), v.cpu(), alpha.cpu(), bq, 64, mask=mask.cpu().numpy())
    assert_outputs_close(out.float().cpu().numpy(), ref, f"exp feature map {case}")
    # the variant with feature_map = 0 is sla_forward itself
    o0 = binding.forward_variant(q, k, v, alpha, bq, 64, kh, kl, feature_map=0, mask=mask)
    assert torch.equal(o0, binding.forward(q, k, v, alpha, bq, 64, kh, kl, mask=mask))


def test_both_variants_on_the_wan13b_shape(cuda_device):
    """Second-order labels and the exponential feature map together on the Wan2.1-1.3B-shaped
    workload: router parity on every head, outputs on a sample of heads and query blocks."""
    w = WORKLOADS["wan13b_b1h12_n32760_d128"]
    q, k, v, alpha = (t.to(cuda_device) for t in make_inputs(w, device="cpu"))
    omask, nmis = _second_order_parity(q, k, w.block_q, w.kh, w.kl)
    out = binding.forward_variant(q, k, v, alpha, w.block_q, 64, w.kh, w.kl, feature_map=1, block_score=1)
    out_m = binding.forward_variant(q, k, v, alpha, w.block_q, 64, w.kh, w.kl, feature_map=1, mask=omask)
    if nmis == 0:
        assert torch.equal(out, out_m), "the variant's own router and its labels passed in disagree"
    qb = [0, 1, 100, 254, 255]
    for h in (0, 11):
        ref = xm.forward_expmap(q[:, h:h + 1].cpu(), k[:, h:h + 1].cpu(), v[:, h:h + 1].cpu(), alpha[h:h + 1].cpu(),
                                w.block_q, 64, mask=omask[:, h:h + 1].cpu().numpy())
        rows = np.concatenate([np.arange(i * w.block_q, min(w.N, (i + 1) * w.block_q)) for i in qb])
        assert_outputs_close(out_m[0, h, rows].float().cpu().numpy(), ref[0, 0, rows], f"wan13b both variants h{h}")


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_branch_dropping_matches_oracle(cuda_device, case):
    """s < tau_t: O = alpha O_s with the same labels; s >= tau_t: the SLA forward, bit for bit."""
    B, H, N, D, bq, kh, kl = case
    q, k, v, alpha = random_inputs(B, H, N, D, seed=7 * N + D, device=cuda_device)
    mask, _, _ = binding.route(q, k, bq, 64, kh, kl)
    ref = sd.forward_dropped(q.cpu(), k.cpu(), v.cpu(), alpha.cpu(), bq, 64, mask=mask.cpu().numpy())
    ws = binding.new_workspace(binding.problem(B, H, N, D, bq, 64, kh, kl), cuda_device)
    out_m = binding.forward_variant(q, k, v, alpha, bq, 64, kh, kl, mask=mask, ws=ws, linear_scale=0.1,
                                    drop_threshold=0.2)
    binding.check(ws)
    assert_outputs_close(out_m.float().cpu().numpy(), ref, f"linear branch dropped {case}")
    # the router path gives the same output on the same labels
    out_r = binding.forward_variant(q, k, v, alpha, bq, 64, kh, kl, ws=ws, linear_scale=0.1, drop_threshold=0.2)
    binding.check(ws)
    assert torch.equal(out_r, out_m)
    # kept (s >= tau_t): exactly sla_forward
    kept = binding.forward_variant(q, k, v, alpha, bq, 64, kh, kl, mask=mask, ws=ws, linear_scale=0.2,
                                   drop_threshold=0.2)
    assert torch.equal(kept, binding.forward(q, k, v, alpha, bq, 64, kh, kl, mask=mask))


def test_branch_dropping_with_second_order_labels(cuda_device):
    q, k, v, alpha = random_inputs(1, 2, 4113, 128, seed=41, device=cuda_device)
    omask, nmis = _second_order_parity(q, k, 128, 0.1, 0.2)
    out = binding.forward_variant(q, k, v, alpha, 128, 64, 0.1, 0.2, block_score=1, linear_scale=0.0,
                                  drop_threshold=0.5)
    out_m = binding.forward_variant(q, k, v, alpha, 128, 64, 0.1, 0.2, mask=omask, linear_scale=0.0,
                                    drop_threshold=0.5)
    if nmis == 0:
        assert torch.equal(out, out_m)
    ref = sd.forward_dropped(q.cpu(), k.cpu(), v.cpu(), alpha.cpu(), 128, 64, mask=omask.cpu().numpy())
    assert_outputs_close(out_m.float().cpu().numpy(), ref, "dropped, second-order labels")
