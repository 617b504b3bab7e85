"""Seeded synthetic inputs for the sparse-plus-linear block attention forward.

This module only draws random tensors. It holds none of the attention
arithmetic (no pooling, no feature map, no softmax), so both the CUDA path and
the fp64 CPU oracle can take their inputs from it without sharing any of the
method's code.

The workloads stand in for the video-DiT self-attention the pages measure on
(Wan2.1-1.3B and Wan2.1-14B latents, "SLA: Beyond Sparsity in Diffusion
Transformers via Fine-Tunable Sparse-Linear Attention", Abstract; "SLA2:
Sparse-Linear Attention with Learnable Routing and QAT", §4). Real activations
are not available, so Q and K carry a smooth random field shared between them
(tokens that are close in the latent grid have similar queries and keys, which
is what makes block routing meaningful), V is white noise, and the per-head,
per-channel blend ratio alpha is uniform on (0, 1).

Recipe (all tensors generated in float32 on the requested device, then rounded
once, round-to-nearest-even, to bfloat16; alpha stays float32):

* ``iid``      : Q, K, V ~ N(0, 1).
* ``field1d``  : F = white noise along the token axis convolved with a Gaussian
                 of standard deviation ell/sqrt(2) (covariance ~ exp(-r^2 / 2 ell^2)),
                 scaled to unit variance per (b, h, channel); Q = F + N(0,1),
                 K = F + N(0,1); V ~ N(0,1).
* ``field3d``  : token n maps to (t, y, x) in t-major raster order over the
                 latent grid; F = white noise smoothed separably over (t, y, x)
                 with length scales (3, 6, 6) cells, unit variance per
                 (b, h, channel); Q = F + 0.5 N(0,1), K = F + 0.5 N(0,1);
                 V ~ N(0,1). A sequence shorter than the grid takes its first N
                 tokens.

Each tensor has its own torch.Generator seeded with
``1000 * config_id + 10 * tensor_id`` (tensor ids: field 1, Q noise 2,
K noise 3, V 4, alpha 5), so a workload is fully determined by its config id and
the device it is drawn on (CPU and CUDA generators give different streams).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, routing fractions and input recipe."""

    name: str
    config_id: int
    B: int
    H: int
    N: int
    D: int
    block_q: int
    block_kv: int
    kh: float
    kl: float
    kind: str  # "iid" | "field1d" | "field3d"
    grid: Optional[Tuple[int, int, int]] = None  # (T, Y, X) latent grid for field3d
    ell_1d: float = 256.0
    ell_3d: Tuple[float, float, float] = (3.0, 6.0, 6.0)
    noise_3d: float = 0.5

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workload families. Names say what the problem is; numbers are the sizes.
WORKLOADS = {
    "iid_b1h2_n1024_d64": Workload(
        "iid_b1h2_n1024_d64", 1, B=1, H=2, N=1024, D=64, block_q=64, block_kv=64,
        kh=0.25, kl=0.25, kind="iid"),
    "field1d_b1h12_n8192_d128": Workload(
        "field1d_b1h12_n8192_d128", 2, B=1, H=12, N=8192, D=128, block_q=128, block_kv=64,
        kh=0.10, kl=0.40, kind="field1d"),
    "wan13b_b1h12_n32760_d128": Workload(
        "wan13b_b1h12_n32760_d128", 3, B=1, H=12, N=32760, D=128, block_q=128, block_kv=64,
        kh=0.05, kl=0.10, kind="field3d", grid=(21, 30, 52)),
    "wan14b720p_b2h40_n75600_d128": Workload(
        "wan14b720p_b2h40_n75600_d128", 4, B=2, H=40, N=75600, D=128, block_q=128,
        block_kv=64, kh=0.05, kl=0.15, kind="field3d", grid=(21, 45, 80)),
}

# Sparsity sweep on the Wan2.1-1.3B-shaped grid: kl = 0 and these critical fractions.
SWEEP_KH = (0.0, 0.01, 0.025, 0.05, 0.10, 0.20, 1.0)


def sweep_workload(kh: float, N: int = 32760) -> Workload:
    """The sparsity-sweep problem at critical fraction ``kh`` (kl = 0)."""
    base = WORKLOADS["wan13b_b1h12_n32760_d128"]
    tag = f"sweep_n{N}_kh{kh:g}"
    return base.with_(name=tag, config_id=5, N=N, kh=kh, kl=0.0)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _unit_variance(f: torch.Tensor, token_dims: Sequence[int]) -> torch.Tensor:
    mean = f.mean(dim=tuple(token_dims), keepdim=True)
    std = f.std(dim=tuple(token_dims), keepdim=True)
    return (f - mean) / std


def _gaussian_smooth_fft(noise: torch.Tensor, dims: Sequence[int], sigmas: Sequence[float]) -> torch.Tensor:
    """Linear (zero-padded) convolution of ``noise`` with a separable Gaussian along ``dims``."""
    pads = [int(math.ceil(4.0 * s)) for s in sigmas]
    sizes = [noise.shape[d] + 2 * p for d, p in zip(dims, pads)]
    spec = torch.fft.rfftn(noise, s=sizes, dim=tuple(dims))
    # Multiply by the transfer function of each 1D Gaussian kernel (sampled on integers).
    for axis, (d, p, s, n) in enumerate(zip(dims, pads, sigmas, sizes)):
        taps = torch.arange(-p, p + 1, dtype=torch.float32, device=noise.device)
        kern = torch.exp(-0.5 * (taps / s) ** 2)
        kern = kern / kern.sum()
        full = torch.zeros(n, dtype=torch.float32, device=noise.device)
        full[: 2 * p + 1] = kern
        # Centre the kernel: shift by -p so that output index i sees input i - p .. i + p.
        full = torch.roll(full, -p)
        last = axis == len(dims) - 1
        tf = torch.fft.rfft(full) if last else torch.fft.fft(full)
        shape = [1] * spec.dim()
        shape[d] = tf.shape[0]
        spec = spec * tf.view(shape)
    out = torch.fft.irfftn(spec, s=sizes, dim=tuple(dims))
    index = [slice(None)] * out.dim()
    for d in dims:
        index[d] = slice(0, noise.shape[d])
    return out[tuple(index)].contiguous()


def make_inputs(w: Workload, device="cpu"):
    """Return (q, k, v, alpha) for workload ``w`` on ``device``.

    q, k, v: [B, H, N, D] bfloat16, contiguous (D fastest). alpha: [H, D] float32.
    """
    B, H, N, D = w.B, w.H, w.N, w.D
    base = 1000 * w.config_id
    f32 = torch.float32
    if w.kind == "iid":
        q = torch.randn(B, H, N, D, generator=_gen(device, base + 2), device=device, dtype=f32)
        k = torch.randn(B, H, N, D, generator=_gen(device, base + 3), device=device, dtype=f32)
    elif w.kind == "field1d":
        white = torch.randn(B, H, D, N, generator=_gen(device, base + 1), device=device, dtype=f32)
        field = _gaussian_smooth_fft(white, dims=[3], sigmas=[w.ell_1d / math.sqrt(2.0)])
        field = _unit_variance(field, token_dims=[3]).transpose(2, 3)  # [B,H,N,D]
        q = field + torch.randn(B, H, N, D, generator=_gen(device, base + 2), device=device, dtype=f32)
        k = field + torch.randn(B, H, N, D, generator=_gen(device, base + 3), device=device, dtype=f32)
        del white, field
    elif w.kind == "field3d":
        T, Y, X = w.grid
        assert N <= T * Y * X, "sequence longer than its latent grid"
        white = torch.randn(B, H, D, T, Y, X, generator=_gen(device, base + 1), device=device, dtype=f32)
        sig = [l / math.sqrt(2.0) for l in w.ell_3d]
        field = _gaussian_smooth_fft(white, dims=[3, 4, 5], sigmas=sig)
        del white
        field = _unit_variance(field, token_dims=[3, 4, 5])
        field = field.reshape(B, H, D, T * Y * X)[..., :N].transpose(2, 3)  # [B,H,N,D]
        s = w.noise_3d
        q = field + s * torch.randn(B, H, N, D, generator=_gen(device, base + 2), device=device, dtype=f32)
        k = field + s * torch.randn(B, H, N, D, generator=_gen(device, base + 3), device=device, dtype=f32)
        del field
    else:
        raise ValueError(f"unknown input kind {w.kind!r}")
    v = torch.randn(B, H, N, D, generator=_gen(device, base + 4), device=device, dtype=f32)
    alpha = torch.rand(H, D, generator=_gen(device, base + 5), device=device, dtype=f32)
    bf = torch.bfloat16
    return (q.to(bf).contiguous(), k.to(bf).contiguous(), v.to(bf).contiguous(), alpha.contiguous())


def random_inputs(B, H, N, D, seed, device="cpu", scale=1.0):
    """Small iid problems for unit tests: q, k, v ~ scale * N(0,1) in bf16, alpha ~ U(0,1)."""
    g = _gen(device, seed)
    q = (scale * torch.randn(B, H, N, D, generator=g, device=device)).to(torch.bfloat16)
    k = (scale * torch.randn(B, H, N, D, generator=g, device=device)).to(torch.bfloat16)
    v = torch.randn(B, H, N, D, generator=g, device=device).to(torch.bfloat16)
    alpha = torch.rand(H, D, generator=g, device=device)
    return q.contiguous(), k.contiguous(), v.contiguous(), alpha.contiguous()
