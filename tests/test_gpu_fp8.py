"""GPU parity of the low-bit (e4m3) sparse branch against the fp64 oracle of the same reading.

The K/V quantiser must match the oracle bit for bit (every code and every block exponent).
The fused forward is checked against the oracle's centre (P unrounded) with the oracle's
labels passed in: the reading leaves the rounding reference of P to the kernel, and the
oracle bounds, per output element, how far any admissible rounding can move the result.
The error beyond that bound must stay within max-abs 2e-2 and mean-abs 2e-3 times the
output's per-channel magnitude, max(1, max |O*|). The internal router must give the same
output whenever its labels equal the oracle's. Inputs are seeded; K and V blocks are
rescaled by powers of two, up and down, so that the per-block exponents (and the largest V
exponent a row's P is coded against) vary.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import sla_oracle_fp8 as f8
from sparse_linear_attention_sla_b200 import binding
from sparse_linear_attention_sla_b200.workloads import WORKLOADS, make_inputs, random_inputs
from tests.parity_utils import MAX_ABS, MEAN_ABS, output_errors

pytestmark = pytest.mark.gpu


def _rescale_blocks(x: torch.Tensor, seed: int, lo: int = -3, hi: int = 2) -> torch.Tensor:
    """x [B,H,N,D] with every 64-token block multiplied by 2^u, u uniform in [lo, hi]."""
    B, H, N, D = x.shape
    Nk = -(-N // 64)
    g = torch.Generator().manual_seed(seed)
    u = torch.randint(lo, hi + 1, (B, H, Nk), generator=g).to(torch.float32)
    f = torch.exp2(u).repeat_interleave(64, dim=-1)[..., :N, None]
    return (x.float().cpu() * f).to(torch.bfloat16)


def _assert_within_bound(got, ref, bound, what):
    """Error beyond the oracle's rounding bound, against the tolerances scaled by the output's
    per-channel magnitude, over the rows the oracle computed."""
    rows = ~np.isnan(ref[..., 0])
    g, r, bd = got[rows], ref[rows], bound[rows]
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    # per (b, h, channel) magnitude of the output over the computed rows, broadcast back
    absref = np.where(rows[..., None], np.abs(np.nan_to_num(ref)), 0.0)
    mag = np.maximum(1.0, absref.max(axis=-2, keepdims=True))
    scale = np.broadcast_to(mag, ref.shape)[rows]
    d = np.abs(g - r)
    excess = np.maximum(d - bd, 0.0) / scale
    mx, mean = float(excess.max()), float(excess.mean())
    used = f"{d.mean() / bd.mean():.3f} of it used on average" if bd.mean() > 0 else "no sparse branch"
    print(f"{what}: beyond-bound max {mx:.3e} mean {mean:.3e} (scaled); raw max-abs {d.max():.3e} "
          f"mean-abs {d.mean():.3e}; mean bound {bd.mean():.3e} ({used}); largest |O*| {float(mag.max()):.2f}")
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max {mx:.3e}, mean {mean:.3e} beyond the bound"
    return mx, mean


def _oracle_masks(q, k, bq, kh, kl):
    B, H = q.shape[:2]
    return np.stack([np.stack([oracle.route(q[b, h].cpu(), k[b, h].cpu(), bq, 64, kh, kl)[0] for h in range(H)])
                     for b in range(B)])


@pytest.mark.parametrize("N, D", [(1000, 128), (333, 64), (64, 128), (4096 + 17, 128)])
def test_quantize_kv_bit_exact(cuda_device, N, D):
    B, H = 1, 2
    g = torch.Generator().manual_seed(N + D)
    k = torch.randn(B, H, N, D, generator=g)
    v = 3.0 * torch.randn(B, H, N, D, generator=g)
    k = _rescale_blocks(k, N, -6, 6)
    v = _rescale_blocks(v, N + 1, -6, 6)
    if N >= 128:
        v[0, 0, 64:128] = 0                       # an all-zero block: exponent 0, codes 0
        k[0, 1, 64:128] = k[0, 1, 64:128] * 1e-37  # amax near 2^-120: the two-step power-of-two scaling
    k8, v8, kexp, vexp = binding.quantize_kv(k.to(cuda_device), v.to(cuda_device))
    for x, codes, exps in ((k, k8, kexp), (v, v8, vexp)):
        codes, exps = codes.cpu().numpy(), exps.cpu().numpy()
        for h in range(H):
            vals, scales = f8.quantize_blocks(x[0, h].double().numpy(), 64)
            np.testing.assert_array_equal(np.exp2(exps[0, h].astype(np.float64)), scales)
            np.testing.assert_array_equal(f8.e4m3_decode(codes[0, h]), vals)


@pytest.mark.parametrize("N", [1000, 4096 + 17])
def test_forward_fp8_codes_equal_quantiser(cuda_device, N):
    """The codes the low-bit forward leaves in its workspace are the standalone quantiser's, bit for bit."""
    B, H, D = 1, 2, 128
    q, k, v, alpha = random_inputs(B, H, N, D, seed=N, device="cpu")
    k = _rescale_blocks(k, N, -6, 6)
    v = _rescale_blocks(v, N + 1, -6, 6)
    q, k, v, alpha = (t.to(cuda_device) for t in (q, k, v, alpha))
    ws = binding.new_workspace(binding.problem(B, H, N, D, 128, 64, 0.25, 0.25), cuda_device, fp8=True)
    binding.forward_fp8(q, k, v, alpha, 128, 64, 0.25, 0.25, ws=ws)
    binding.check(ws)
    got = binding.lowbit_codes(ws, B, H, N, D)
    ref = binding.quantize_kv(k, v)
    for g, r in zip(got, ref):
        assert torch.equal(g.cpu(), r.cpu())


FP8_CASES = [
    # B, H, N, bq, kh, kl
    (1, 2, 1000, 128, 0.25, 0.25),
    (1, 2, 700, 64, 0.25, 0.25),
    (2, 1, 333, 128, 0.5, 0.2),
    (1, 3, 4113, 128, 0.1, 0.2),
    (1, 2, 1000, 128, 1.0, 0.0),   # every block critical: dense low-bit attention
    (1, 2, 1000, 128, 0.0, 0.5),   # empty sparse branch: the linear branch alone
    (1, 2, 1000, 128, 0.5, 0.5),   # empty linear branch
    (1, 1, 64, 128, 0.5, 0.0),     # a single KV block
]


@pytest.mark.parametrize("case", FP8_CASES, ids=lambda c: "x".join(map(str, c)))
def test_forward_fp8_matches_oracle(cuda_device, case):
    B, H, N, bq, kh, kl = case
    D = 128
    q, k, v, alpha = random_inputs(B, H, N, D, seed=7 * N + H, device="cpu")
    # K and V blocks rescaled up and down (V by 2^-3 .. 2^2): outputs reach |O| ~ 4 - 8, where the
    # tolerances scale with the output's magnitude
    k = _rescale_blocks(k, N)
    v = _rescale_blocks(v, N + 1, -3, 2)
    q, k, v, alpha = (t.to(cuda_device) for t in (q, k, v, alpha))
    omask = _oracle_masks(q, k, bq, kh, kl)
    ws = binding.new_workspace(binding.problem(B, H, N, D, bq, 64, kh, kl), cuda_device, fp8=True)
    out_m = binding.forward_fp8(q, k, v, alpha, bq, 64, kh, kl, mask=torch.from_numpy(omask).to(cuda_device), ws=ws)
    out = binding.forward_fp8(q, k, v, alpha, bq, 64, kh, kl, ws=ws)
    binding.check(ws)
    qc, kc_, vc, ac = (t.cpu() for t in (q, k, v, alpha))
    ref, bound = f8.forward_fp8(qc, kc_, vc, ac, bq, 64, mask=omask, with_bound=True)
    got = out_m.float().cpu().numpy()
    _assert_within_bound(got, ref, bound, f"low-bit, oracle labels {case}")
    gmask = binding.route(q, k, bq, 64, kh, kl)[0].cpu().numpy()
    if np.array_equal(gmask, omask):
        assert torch.equal(out, out_m), "router path and caller-mask path disagree on the same labels"
    # accuracy against full precision: no worse than the low-bit definition's own (its centre)
    # by more than the rounding of P the bound allows on average
    full = oracle.forward(qc, kc_, vc, ac, bq, 64, mask=omask)
    e_gpu = output_errors(got, full)[1]
    e_def = output_errors(ref, full)[1]
    assert e_gpu <= e_def + float(np.nanmean(bound)) + 1e-3, \
        f"mean-abs vs full precision {e_gpu:.3e}, definition {e_def:.3e}"


def _workload_fp8(w, device, heads, query_blocks=None):
    q, k, v, alpha = make_inputs(w, device="cpu")
    q, k, v, alpha = (t.to(device) for t in (q, k, v, alpha))
    B, H = w.B, w.H
    Nq = -(-w.N // w.block_q)
    Nk = -(-w.N // 64)
    om = np.zeros((B, H, Nq, Nk), dtype=np.int8)
    for b, h in heads:
        om[b, h] = oracle.route(q[b, h].cpu(), k[b, h].cpu(), w.block_q, 64, w.kh, w.kl)[0]
    gmask = binding.route(q, k, w.block_q, 64, w.kh, w.kl)[0]
    mask = gmask.cpu().numpy().copy()
    for b, h in heads:
        mask[b, h] = om[b, h]
    ws = binding.new_workspace(binding.problem(B, H, w.N, w.D, w.block_q, 64, w.kh, w.kl), device, fp8=True)
    out = binding.forward_fp8(q, k, v, alpha, w.block_q, 64, w.kh, w.kl, mask=torch.from_numpy(mask).to(device),
                              ws=ws)
    binding.check(ws)
    ref, bound = f8.forward_fp8(q.cpu(), k.cpu(), v.cpu(), alpha.cpu(), w.block_q, 64, mask=mask, heads=heads,
                                query_blocks=query_blocks, with_bound=True)
    _assert_within_bound(out.float().cpu().numpy(), ref, bound, w.name + " low-bit")


def test_fp8_field1d_b1h12_n8192_d128(cuda_device):
    _workload_fp8(WORKLOADS["field1d_b1h12_n8192_d128"], cuda_device, heads=[(0, 0), (0, 5), (0, 11)])


def test_fp8_wan13b_b1h12_n32760_d128_sampled(cuda_device):
    _workload_fp8(WORKLOADS["wan13b_b1h12_n32760_d128"], cuda_device, heads=[(0, 0), (0, 7)],
                  query_blocks=[0, 1, 100, 200, 254, 255])


def test_fp8_needs_d128(cuda_device):
    q, k, v, alpha = random_inputs(1, 1, 256, 64, seed=1, device=cuda_device)
    with pytest.raises(binding.SlaError, match="D=128"):
        binding.forward_fp8(q, k, v, alpha, 64, 64, 0.25, 0.25)
