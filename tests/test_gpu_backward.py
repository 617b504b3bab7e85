"""GPU parity of the backward pass (sla_backward) against the fp64 backward oracle.

The oracle (oracle/sla_oracle_bwd.py) is the exact derivative of the forward oracle with the
block labels held fixed, pinned on the CPU by central finite differences and by autograd of
dense and of linear attention. Here the kernels, given the oracle's labels, must match it:
the operands enter the tensor cores in bf16, so every gradient is compared at max-abs 2e-2
and mean-abs 2e-3 of its own scale (the largest |value| of that gradient, or 1).
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import sla_oracle_bwd as bw
from sparse_linear_attention_sla_b200 import binding
from sparse_linear_attention_sla_b200.workloads import WORKLOADS, make_inputs, random_inputs

pytestmark = pytest.mark.gpu


def _check(name, got, ref, rows=None):
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    if rows is not None:
        g, r = g[..., rows, :], r[..., rows, :]
    assert np.all(np.isfinite(g)), f"{name}: non-finite"
    scale = max(1.0, float(np.abs(r).max()))
    d = np.abs(g - r) / scale
    print(f"{name}: max-abs {d.max():.3e} mean-abs {d.mean():.3e} (of scale {scale:.3g})")
    assert d.max() <= 2e-2 and d.mean() <= 2e-3, f"{name}: max {d.max():.3e}, mean {d.mean():.3e}"


def _run(q, k, v, alpha, dO, bq, kh, kl):
    mask, _, _ = binding.route(q, k, bq, 64, kh, kl)
    dQ, dK, dV, da, ws = binding.backward(q, k, v, alpha, dO, bq, 64, kh, kl, mask=mask)
    binding.check(ws)
    return mask, dQ, dK, dV, da


CASES = [
    # B, H, N, kh, kl  (D = 128, block_q = 128)
    (1, 2, 1024, 0.25, 0.25),
    (2, 1, 333, 0.2, 0.3),
    (1, 2, 1000, 1.0, 0.0),   # every block critical: dense softmax attention
    (1, 2, 1000, 0.0, 0.0),   # every block marginal: linear attention
    (1, 1, 64, 0.5, 0.0),     # one KV block
    (1, 3, 4113, 0.1, 0.2),   # ragged tails
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_backward_matches_oracle(cuda_device, case):
    B, H, N, kh, kl = case
    D, bq = 128, 128
    q, k, v, alpha = random_inputs(B, H, N, D, seed=11 * N + H, device=cuda_device)
    g = torch.Generator(device=cuda_device).manual_seed(N)
    dO = torch.randn(B, H, N, D, generator=g, device=cuda_device).to(torch.bfloat16)
    mask, dQ, dK, dV, da = _run(q, k, v, alpha, dO, bq, kh, kl)
    rQ, rK, rV, ra = bw.backward(q.cpu(), k.cpu(), v.cpu(), alpha.cpu(), bq, 64, mask.cpu().numpy(), dO.cpu())
    _check("dQ", dQ.cpu(), rQ)
    _check("dK", dK.cpu(), rK)
    _check("dV", dV.cpu(), rV)
    _check("dalpha", da.cpu(), ra)


def test_backward_field1d_b1h12_n8192_d128(cuda_device):
    w = WORKLOADS["field1d_b1h12_n8192_d128"]
    q, k, v, alpha = (t.to(cuda_device) for t in make_inputs(w, device="cpu"))
    g = torch.Generator(device=cuda_device).manual_seed(8192)
    dO = torch.randn(q.shape, generator=g, device=cuda_device).to(torch.bfloat16)
    mask, dQ, dK, dV, da = _run(q, k, v, alpha, dO, w.block_q, w.kh, w.kl)
    m = mask.cpu().numpy()
    for h in (0, 5, 11):
        sl = slice(h, h + 1)
        rQ, rK, rV, ra = bw.backward(q[:, sl].cpu(), k[:, sl].cpu(), v[:, sl].cpu(), alpha[sl].cpu(), w.block_q, 64,
                                     m[:, sl], dO[:, sl].cpu())
        _check(f"dQ h{h}", dQ[:, sl].cpu(), rQ)
        _check(f"dK h{h}", dK[:, sl].cpu(), rK)
        _check(f"dV h{h}", dV[:, sl].cpu(), rV)


def test_backward_wan13b_sampled(cuda_device):
    """Wan2.1-1.3B shape: two heads checked in full against the oracle (its per-head cost
    is the full attention of that head)."""
    w = WORKLOADS["wan13b_b1h12_n32760_d128"]
    q, k, v, alpha = (t.to(cuda_device) for t in make_inputs(w, device="cpu"))
    g = torch.Generator(device=cuda_device).manual_seed(32760)
    dO = torch.randn(q.shape, generator=g, device=cuda_device).to(torch.bfloat16)
    mask, dQ, dK, dV, da = _run(q, k, v, alpha, dO, w.block_q, w.kh, w.kl)
    m = mask.cpu().numpy()
    for h in (0, 11):
        sl = slice(h, h + 1)
        rQ, rK, rV, ra = bw.backward(q[:, sl].cpu(), k[:, sl].cpu(), v[:, sl].cpu(), alpha[sl].cpu(), w.block_q, 64,
                                     m[:, sl], dO[:, sl].cpu())
        _check(f"dQ h{h}", dQ[:, sl].cpu(), rQ)
        _check(f"dK h{h}", dK[:, sl].cpu(), rK)
        _check(f"dV h{h}", dV[:, sl].cpu(), rV)


@pytest.mark.parametrize("case", [(1, 2, 1024, 0.25, 0.25), (1, 3, 4113, 0.1, 0.2)], ids=lambda c: "x".join(map(str, c)))
def test_backward_is_deterministic(cuda_device, case):
    """Every sum of the backward runs in a fixed order (no atomics): two calls agree bit for bit."""
    B, H, N, kh, kl = case
    q, k, v, alpha = random_inputs(B, H, N, 128, seed=N, device=cuda_device)
    g = torch.Generator(device=cuda_device).manual_seed(N + 1)
    dO = torch.randn(B, H, N, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    first = binding.backward(q, k, v, alpha, dO, 128, 64, kh, kl)
    second = binding.backward(q, k, v, alpha, dO, 128, 64, kh, kl)
    binding.check(first[4])
    binding.check(second[4])
    for name, a, b in zip(("dQ", "dK", "dV", "dalpha"), first[:4], second[:4]):
        assert torch.equal(a, b), f"{name} differs between two calls"


def test_backward_wan14b720p_sampled(cuda_device):
    """Wan2.1-14B 720p shape (B=2, H=40, N=75600): the backward over every head, two (batch,
    head) pairs checked in full against the oracle."""
    w = WORKLOADS["wan14b720p_b2h40_n75600_d128"]
    q, k, v, alpha = make_inputs(w, device=cuda_device)
    g = torch.Generator(device=cuda_device).manual_seed(75600)
    dO = torch.randn(q.shape, generator=g, device=cuda_device).to(torch.bfloat16)
    mask, dQ, dK, dV, da = _run(q, k, v, alpha, dO, w.block_q, w.kh, w.kl)
    m = mask.cpu().numpy()
    for b, h in ((0, 0), (1, 39)):
        bs, hs = slice(b, b + 1), slice(h, h + 1)
        rQ, rK, rV, ra = bw.backward(q[bs, hs].cpu(), k[bs, hs].cpu(), v[bs, hs].cpu(), alpha[hs].cpu(), w.block_q, 64,
                                     m[bs, hs], dO[bs, hs].cpu())
        _check(f"dQ b{b}h{h}", dQ[bs, hs].cpu(), rQ)
        _check(f"dK b{b}h{h}", dK[bs, hs].cpu(), rK)
        _check(f"dV b{b}h{h}", dV[bs, hs].cpu(), rV)


def test_backward_scores_far_above_the_first_block(cuda_device):
    """K blocks scaled geometrically from 1/4 to 16 along the sequence: most rows meet critical
    blocks scoring far above their first one, so pass 1's reference maximum (taken from a
    tile's first block) moves and its accumulator is rescaled; the gradients still match."""
    B, H, N, kh, kl = 1, 2, 4096 + 40, 0.5, 0.25
    q, k, v, alpha = random_inputs(B, H, N, 128, seed=17, device="cpu")
    f = torch.from_numpy(np.geomspace(0.25, 16.0, -(-N // 64))).repeat_interleave(64)[:N]
    k = (k.double() * f[None, None, :, None]).to(torch.bfloat16)
    q, k, v, alpha = (t.to(cuda_device) for t in (q, k, v, alpha))
    g = torch.Generator(device=cuda_device).manual_seed(N)
    dO = torch.randn(B, H, N, 128, generator=g, device=cuda_device).to(torch.bfloat16)
    mask, dQ, dK, dV, da = _run(q, k, v, alpha, dO, 128, kh, kl)
    rQ, rK, rV, ra = bw.backward(q.cpu(), k.cpu(), v.cpu(), alpha.cpu(), 128, 64, mask.cpu().numpy(), dO.cpu())
    _check("dQ", dQ.cpu(), rQ)
    _check("dK", dK.cpu(), rK)
    _check("dV", dV.cpu(), rV)
    _check("dalpha", da.cpu(), ra)
