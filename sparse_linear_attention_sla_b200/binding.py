"""Python binding over the C ABI in include/sla.h (argument marshalling only).

Every step of the computation runs in libsla.so's CUDA kernels; this module
checks tensor shapes/dtypes, takes the current torch CUDA stream, allocates
outputs and workspaces with torch, and calls the library through ctypes. There
is no CPU path: without the built library, or without a CUDA device, every
call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsla.so")

SLA_OK = 0
_STATUS = {
    0: "SLA_OK", 1: "SLA_ERR_INVALID_ARG", 2: "SLA_ERR_UNSUPPORTED", 3: "SLA_ERR_WORKSPACE",
    4: "SLA_ERR_CUDA", 5: "SLA_ERR_TIMEOUT", 6: "SLA_ERR_BAD_MASK",
}

# Every symbol include/sla.h declares.
EXPORTS = ("sla_counts", "sla_workspace_size", "sla_route", "sla_kv_states", "sla_forward",
           "sla_forward_timed", "sla_check", "sla_last_error", "sla_version", "sla_route_noalloc",
           "sla_selftest_wait_timeout", "sla_workspace_size_fp8", "sla_forward_fp8", "sla_forward_fp8_timed",
           "sla_quantize_kv", "sla_aggregate_states", "sla_forward_launches", "sla_route_variant",
           "sla_forward_variant", "sla_workspace_size_backward", "sla_backward", "sla_workspace_size_pisa",
           "sla_forward_pisa", "sla_pisa_hbar", "sla_lowbit_codes")


class SlaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


class Variant(ctypes.Structure):
    """sla_variant: feature_map 0 (elu + 1) or 1 (exp); block_score 0 (first order) or 1 (second order);
    linear_scale, drop_threshold: the linear branch is dropped when linear_scale < drop_threshold."""
    _fields_ = [("feature_map", ctypes.c_int), ("block_score", ctypes.c_int), ("linear_scale", ctypes.c_float),
                ("drop_threshold", ctypes.c_float)]


class Problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("D", ctypes.c_int),
                ("block_q", ctypes.c_int), ("block_kv", ctypes.c_int),
                ("kh", ctypes.c_float), ("kl", ctypes.c_float)]


_lib = None
_lib_lock = threading.Lock()


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsla.so and declare its signatures. Raises if the library is missing."""
    global _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m sparse_linear_attention_sla_b200.build` "
                "(there is no CPU fallback)")
        lib = ctypes.CDLL(path)
        P = ctypes.POINTER(Problem)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        ip = ctypes.POINTER(ctypes.c_int)
        lib.sla_counts.argtypes = [P, ip, ip, ip, ip]
        lib.sla_workspace_size.argtypes = [P]
        lib.sla_workspace_size.restype = sz
        lib.sla_route.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.sla_kv_states.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
        lib.sla_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.sla_forward_timed.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp, ctypes.POINTER(ctypes.c_float)]
        lib.sla_check.argtypes = [vp, vp]
        lib.sla_workspace_size_fp8.argtypes = [P]
        lib.sla_workspace_size_fp8.restype = sz
        lib.sla_forward_fp8.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.sla_forward_fp8_timed.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp, ctypes.POINTER(ctypes.c_float)]
        lib.sla_quantize_kv.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
        lib.sla_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_uint, vp]
        lib.sla_selftest_wait_timeout.restype = ctypes.c_int
        lib.sla_aggregate_states.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.sla_workspace_size_backward.argtypes = [P]
        lib.sla_workspace_size_backward.restype = sz
        lib.sla_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.sla_workspace_size_pisa.argtypes = [P]
        lib.sla_workspace_size_pisa.restype = sz
        lib.sla_forward_pisa.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.sla_pisa_hbar.argtypes = [P, vp, vp, vp, vp, sz, vp]
        pp = ctypes.POINTER(ctypes.c_void_p)
        lib.sla_lowbit_codes.argtypes = [P, vp, sz, pp, pp, pp, pp]
        V = ctypes.POINTER(Variant)
        lib.sla_route_variant.argtypes = [P, V, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.sla_forward_variant.argtypes = [P, V, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.sla_forward_launches.argtypes = [P, ctypes.c_int, ctypes.c_int]
        lib.sla_forward_launches.restype = ctypes.c_int
        lib.sla_last_error.restype = ctypes.c_char_p
        lib.sla_version.restype = ctypes.c_char_p
        for name in ("sla_counts", "sla_route", "sla_kv_states", "sla_forward", "sla_forward_timed", "sla_check",
                     "sla_forward_fp8", "sla_forward_fp8_timed", "sla_quantize_kv", "sla_forward_pisa",
                     "sla_pisa_hbar", "sla_aggregate_states", "sla_backward", "sla_route_variant",
                     "sla_forward_variant", "sla_lowbit_codes"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
        return lib


def _raise(status: int):
    if status != SLA_OK:
        msg = load_library().sla_last_error().decode(errors="replace")
        raise SlaError(status, msg)


def problem(B, H, N, D, block_q, block_kv, kh=0.0, kl=0.0) -> Problem:
    return Problem(int(B), int(H), int(N), int(D), int(block_q), int(block_kv), float(kh), float(kl))


def counts(p: Problem) -> Tuple[int, int, int, int]:
    """(Nq, Nk, kc, kn) as the library computes them (host only)."""
    out = [ctypes.c_int(0) for _ in range(4)]
    _raise(load_library().sla_counts(ctypes.byref(p), *[ctypes.byref(o) for o in out]))
    return tuple(o.value for o in out)


def workspace_size(p: Problem) -> int:
    return int(load_library().sla_workspace_size(ctypes.byref(p)))


def workspace_size_fp8(p: Problem) -> int:
    return int(load_library().sla_workspace_size_fp8(ctypes.byref(p)))


def new_workspace(p: Problem, device, fp8: bool = False) -> torch.Tensor:
    """A zero-headed workspace for problem p on device (bytes, 256-byte aligned by the allocator);
    fp8=True sizes it for forward_fp8."""
    n = workspace_size_fp8(p) if fp8 else workspace_size(p)
    if n == 0:
        counts(p)  # raises with the library's message
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def _stream_handle(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check_act(name, t, B, H, N, D, device):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16 or tuple(t.shape) != (B, H, N, D) or not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous bf16 of shape {(B, H, N, D)}, got {t.dtype} {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def route(q, k, block_q, block_kv, kh, kl, want_scores=False, want_crit=False, ws=None):
    """Block labels [B,H,Nq,Nk] int8 (2 critical, 1 marginal, 0 negligible).

    Returns (mask, crit_idx or None, scores or None).
    """
    B, H, N, D = q.shape
    _check_act("q", q, B, H, N, D, q.device)
    _check_act("k", k, B, H, N, D, q.device)
    p = problem(B, H, N, D, block_q, block_kv, kh, kl)
    Nq, Nk, kc, _ = counts(p)
    dev = q.device
    mask = torch.empty(B, H, Nq, Nk, dtype=torch.int8, device=dev)
    crit = torch.empty(B, H, Nq, kc, dtype=torch.int32, device=dev) if want_crit else None
    scores = torch.empty(B, H, Nq, Nk, dtype=torch.float64, device=dev) if want_scores else None
    if ws is None:
        ws = new_workspace(p, dev)
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.sla_route(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(mask), _ptr(crit), _ptr(scores), _ptr(ws),
                           ctypes.c_size_t(ws.numel()), _stream_handle(dev))
    _raise(st)
    return mask, crit, scores


def kv_states(k, v, block_kv=64, ws=None):
    """Per-KV-block states h [B,H,Nk,D,D] and z [B,H,Nk,D], fp32."""
    B, H, N, D = k.shape
    _check_act("k", k, B, H, N, D, k.device)
    _check_act("v", v, B, H, N, D, k.device)
    p = problem(B, H, N, D, 128 if D == 128 else 64, block_kv)
    _, Nk, _, _ = counts(p)
    dev = k.device
    h = torch.empty(B, H, Nk, D, D, dtype=torch.float32, device=dev)
    z = torch.empty(B, H, Nk, D, dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.sla_kv_states(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(h), _ptr(z), _ptr(ws),
                               ctypes.c_size_t(ws.numel()), _stream_handle(dev))
    _raise(st)
    return h, z


def aggregate_states(k, v, mask, block_q, block_kv=64, ws=None):
    """Per-query-block sums of the marginal blocks' states: H [B,H,Nq,D,D] bf16, Z [B,H,Nq,D] fp32."""
    B, H, N, D = k.shape
    _check_act("k", k, B, H, N, D, k.device)
    _check_act("v", v, B, H, N, D, k.device)
    p = problem(B, H, N, D, block_q, block_kv)
    Nq, Nk, _, _ = counts(p)
    dev = k.device
    if mask.dtype != torch.int8 or tuple(mask.shape) != (B, H, Nq, Nk) or not mask.is_contiguous() \
            or mask.device != dev:
        raise ValueError(f"mask must be contiguous int8 [{B}, {H}, {Nq}, {Nk}] on {dev}")
    Hs = torch.empty(B, H, Nq, D, D, dtype=torch.bfloat16, device=dev)
    Zs = torch.empty(B, H, Nq, D, dtype=torch.float32, device=dev)
    if ws is None:
        ws = new_workspace(p, dev)
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.sla_aggregate_states(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(mask), _ptr(Hs), _ptr(Zs), _ptr(ws),
                                      ctypes.c_size_t(ws.numel()), _stream_handle(dev))
    _raise(st)
    return Hs, Zs, ws


def route_variant(q, k, block_q, block_kv, kh, kl, feature_map=0, block_score=0, want_scores=False,
                  want_crit=False, ws=None):
    """sla_route_variant: labels [B,H,Nq,Nk] int8 (and crit_idx, scores when asked)."""
    B, H, N, D = q.shape
    _check_act("q", q, B, H, N, D, q.device)
    _check_act("k", k, B, H, N, D, q.device)
    p = problem(B, H, N, D, block_q, block_kv, kh, kl)
    Nq, Nk, kc, _ = counts(p)
    dev = q.device
    mask = torch.empty(B, H, Nq, Nk, dtype=torch.int8, device=dev)
    crit = torch.empty(B, H, Nq, kc, dtype=torch.int32, device=dev) if want_crit else None
    scores = torch.empty(B, H, Nq, Nk, dtype=torch.float64, device=dev) if want_scores else None
    if ws is None:
        ws = new_workspace(p, dev)
    var = Variant(feature_map, block_score, 0.0, 0.0)
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.sla_route_variant(ctypes.byref(p), ctypes.byref(var), _ptr(q), _ptr(k), _ptr(mask), _ptr(crit),
                                   _ptr(scores), _ptr(ws), ctypes.c_size_t(ws.numel()), _stream_handle(dev))
    _raise(st)
    return mask, crit, scores


def forward_variant(q, k, v, alpha, block_q, block_kv, kh, kl, feature_map=0, block_score=0, mask=None, out=None,
                    ws=None, linear_scale=0.0, drop_threshold=0.0):
    """sla_forward_variant: O [B,H,N,D] bf16."""
    p, out, ws = _forward_args(q, k, v, alpha, block_q, block_kv, kh, kl, mask, out, ws)
    var = Variant(feature_map, block_score, float(linear_scale), float(drop_threshold))
    lib = load_library()
    dev = q.device
    with torch.cuda.device(dev):
        st = lib.sla_forward_variant(ctypes.byref(p), ctypes.byref(var), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                     _ptr(mask), _ptr(out), _ptr(ws), ctypes.c_size_t(ws.numel()),
                                     _stream_handle(dev))
    _raise(st)
    return out


def backward(q, k, v, alpha, dO, block_q=128, block_kv=64, kh=0.05, kl=0.10, mask=None, ws=None):
    """sla_backward: (dQ, dK, dV [B,H,N,D] fp32, dalpha [H,D] fp32) of sum(dO * O)."""
    B, H, N, D = q.shape
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v), ("dO", dO)):
        _check_act(name, t, B, H, N, D, dev)
    if alpha.dtype != torch.float32 or tuple(alpha.shape) != (H, D) or not alpha.is_contiguous():
        raise ValueError(f"alpha must be contiguous fp32 [{H}, {D}]")
    p = problem(B, H, N, D, block_q, block_kv, kh, kl)
    Nq, Nk, _, _ = counts(p)
    if mask is not None and (mask.dtype != torch.int8 or tuple(mask.shape) != (B, H, Nq, Nk)
                             or not mask.is_contiguous()):
        raise ValueError(f"mask must be contiguous int8 [{B}, {H}, {Nq}, {Nk}]")
    lib = load_library()
    if ws is None:
        n = lib.sla_workspace_size_backward(ctypes.byref(p))
        if n == 0:
            counts(p)
        ws = torch.empty(n, dtype=torch.uint8, device=dev)
        ws[:256].zero_()
    dQ, dK, dV = (torch.empty(B, H, N, D, dtype=torch.float32, device=dev) for _ in range(3))
    dalpha = torch.empty(H, D, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        st = lib.sla_backward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(mask), _ptr(dO),
                              _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dalpha), _ptr(ws), ctypes.c_size_t(ws.numel()),
                              _stream_handle(dev))
    _raise(st)
    return dQ, dK, dV, dalpha, ws


def lowbit_codes(ws: torch.Tensor, B, H, N, D, block_q=128, block_kv=64):
    """Copies of the e4m3 codes of K and V ([B,H,N,D] uint8) and block exponents ([B,H,Nk] int32)
    that the last forward_fp8 on workspace ws wrote."""
    p = problem(B, H, N, D, block_q, block_kv)
    _, Nk, _, _ = counts(p)
    ptrs = [ctypes.c_void_p() for _ in range(4)]
    _raise(load_library().sla_lowbit_codes(ctypes.byref(p), _ptr(ws), ctypes.c_size_t(ws.numel()),
                                           *[ctypes.byref(x) for x in ptrs]))
    base = ws.data_ptr()
    out = []
    for x, n, dt in ((ptrs[0], B * H * N * D, torch.uint8), (ptrs[1], B * H * N * D, torch.uint8),
                     (ptrs[2], B * H * Nk, torch.int32), (ptrs[3], B * H * Nk, torch.int32)):
        off = x.value - base
        nbytes = n * (4 if dt == torch.int32 else 1)
        out.append(ws[off:off + nbytes].view(dt).clone())
    return (out[0].view(B, H, N, D), out[1].view(B, H, N, D), out[2].view(B, H, Nk), out[3].view(B, H, Nk))


def new_workspace_pisa(p: Problem, device) -> torch.Tensor:
    """A zero-headed workspace of sla_workspace_size_pisa(p) bytes on device."""
    n = int(load_library().sla_workspace_size_pisa(ctypes.byref(p)))
    if n == 0:
        counts(p)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def forward_pisa(q, k, v, block_q=128, block_kv=64, kh=0.05, kl=0.10, labels=None, out=None, ws=None):
    """sla_forward_pisa: O [B,H,N,D] bf16. labels [B,H,Nq,Nk] int8 (2 = critical) or None (the router)."""
    B, H, N, D = q.shape
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_act(name, t, B, H, N, D, dev)
    p = problem(B, H, N, D, block_q, block_kv, kh, kl)
    Nq, Nk, _, _ = counts(p)
    if labels is not None and (labels.dtype != torch.int8 or tuple(labels.shape) != (B, H, Nq, Nk)
                               or not labels.is_contiguous() or labels.device != dev):
        raise ValueError(f"labels must be contiguous int8 [{B}, {H}, {Nq}, {Nk}] on {dev}")
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = new_workspace_pisa(p, dev)
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.sla_forward_pisa(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(labels), _ptr(out), _ptr(ws),
                                  ctypes.c_size_t(ws.numel()), _stream_handle(dev))
    _raise(st)
    return out


def pisa_hbar(k, v, block_kv=64, ws=None):
    """sla_pisa_hbar: Hbar [B,H,D,D] fp32, the mean over KV blocks of (K_j - kbar_j)^T V_j."""
    B, H, N, D = k.shape
    dev = k.device
    for name, t in (("k", k), ("v", v)):
        _check_act(name, t, B, H, N, D, dev)
    p = problem(B, H, N, D, 128, block_kv)
    if ws is None:
        ws = new_workspace_pisa(p, dev)
    out = torch.empty(B, H, D, D, dtype=torch.float32, device=dev)
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.sla_pisa_hbar(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(out), _ptr(ws), ctypes.c_size_t(ws.numel()),
                               _stream_handle(dev))
    _raise(st)
    return out


def forward_launches(p, with_mask=False, low_bit=False) -> int:
    """Kernel launches one sla_forward (or sla_forward_fp8) call enqueues for problem p."""
    n = load_library().sla_forward_launches(ctypes.byref(p), int(bool(with_mask)), int(bool(low_bit)))
    if n < 0:
        raise SlaError(1, "invalid problem")
    return n


def _forward_args(q, k, v, alpha, block_q, block_kv, kh, kl, mask, out, ws, fp8=False):
    B, H, N, D = q.shape
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_act(name, t, B, H, N, D, dev)
    if alpha.dtype != torch.float32 or tuple(alpha.shape) != (H, D) or not alpha.is_contiguous() or alpha.device != dev:
        raise ValueError(f"alpha must be contiguous fp32 [{H}, {D}] on {dev}")
    p = problem(B, H, N, D, block_q, block_kv, kh, kl)
    Nq, Nk, _, _ = counts(p)
    if mask is not None:
        if mask.dtype != torch.int8 or tuple(mask.shape) != (B, H, Nq, Nk) or not mask.is_contiguous() \
                or mask.device != dev:
            raise ValueError(f"mask must be contiguous int8 [{B}, {H}, {Nq}, {Nk}] on {dev}")
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_act("out", out, B, H, N, D, dev)
    if ws is None:
        ws = new_workspace(p, dev, fp8)
    return p, out, ws


def forward(q, k, v, alpha, block_q=128, block_kv=64, kh=0.05, kl=0.10, mask=None, out=None, ws=None):
    """Fused SLA forward: O = alpha * O_s + (1 - alpha) * O_l, bf16 [B,H,N,D]."""
    p, out, ws = _forward_args(q, k, v, alpha, block_q, block_kv, kh, kl, mask, out, ws)
    lib = load_library()
    with torch.cuda.device(q.device):
        st = lib.sla_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(mask), _ptr(out),
                             _ptr(ws), ctypes.c_size_t(ws.numel()), _stream_handle(q.device))
    _raise(st)
    return out


def forward_timed(q, k, v, alpha, block_q=128, block_kv=64, kh=0.05, kl=0.10, mask=None, out=None, ws=None):
    """forward() plus per-stage device milliseconds (precompute, route, aggregate, attention).

    Synchronises the current stream."""
    p, out, ws = _forward_args(q, k, v, alpha, block_q, block_kv, kh, kl, mask, out, ws)
    ms = (ctypes.c_float * 4)()
    lib = load_library()
    with torch.cuda.device(q.device):
        st = lib.sla_forward_timed(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(mask), _ptr(out),
                                   _ptr(ws), ctypes.c_size_t(ws.numel()), _stream_handle(q.device), ms)
    _raise(st)
    return out, [float(x) for x in ms]


def forward_fp8(q, k, v, alpha, block_q=128, block_kv=64, kh=0.05, kl=0.10, mask=None, out=None, ws=None):
    """forward() with the low-bit (e4m3) sparse branch (include/sla.h states the reading); D = 128."""
    p, out, ws = _forward_args(q, k, v, alpha, block_q, block_kv, kh, kl, mask, out, ws, fp8=True)
    lib = load_library()
    with torch.cuda.device(q.device):
        st = lib.sla_forward_fp8(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(mask), _ptr(out),
                                 _ptr(ws), ctypes.c_size_t(ws.numel()), _stream_handle(q.device))
    _raise(st)
    return out


def forward_fp8_timed(q, k, v, alpha, block_q=128, block_kv=64, kh=0.05, kl=0.10, mask=None, out=None, ws=None):
    """forward_fp8() plus per-stage device milliseconds (precompute, route, aggregate, quantise,
    attention). Synchronises the current stream."""
    p, out, ws = _forward_args(q, k, v, alpha, block_q, block_kv, kh, kl, mask, out, ws, fp8=True)
    ms = (ctypes.c_float * 5)()
    lib = load_library()
    with torch.cuda.device(q.device):
        st = lib.sla_forward_fp8_timed(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(mask),
                                       _ptr(out), _ptr(ws), ctypes.c_size_t(ws.numel()), _stream_handle(q.device), ms)
    _raise(st)
    return out, [float(x) for x in ms]


def quantize_kv(k, v, block_kv=64):
    """e4m3 codes of K and V ([B,H,N,D] uint8) and their per-KV-block scale exponents
    ([B,H,Nk] int32): code * 2^exp approximates the input."""
    B, H, N, D = k.shape
    _check_act("k", k, B, H, N, D, k.device)
    _check_act("v", v, B, H, N, D, k.device)
    p = problem(B, H, N, D, 128 if D == 128 else 64, block_kv)
    _, Nk, _, _ = counts(p)
    dev = k.device
    k8 = torch.empty(B, H, N, D, dtype=torch.uint8, device=dev)
    v8 = torch.empty(B, H, N, D, dtype=torch.uint8, device=dev)
    kexp = torch.empty(B, H, Nk, dtype=torch.int32, device=dev)
    vexp = torch.empty(B, H, Nk, dtype=torch.int32, device=dev)
    lib = load_library()
    with torch.cuda.device(dev):
        st = lib.sla_quantize_kv(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(k8), _ptr(v8), _ptr(kexp), _ptr(vexp),
                                 _stream_handle(dev))
    _raise(st)
    return k8, v8, kexp, vexp


def check(ws: torch.Tensor):
    """Synchronise and raise if a kernel recorded a device-side error in ws."""
    lib = load_library()
    with torch.cuda.device(ws.device):
        _raise(lib.sla_check(_ptr(ws), _stream_handle(ws.device)))


def selftest_wait_timeout(ws: torch.Tensor, limit_us: int = 50000):
    """Enqueue the device self-test of the bounded-wait path (see include/sla.h); a
    following check(ws) raises SlaError with status SLA_ERR_TIMEOUT."""
    lib = load_library()
    with torch.cuda.device(ws.device):
        _raise(lib.sla_selftest_wait_timeout(_ptr(ws), ctypes.c_size_t(ws.numel()), ctypes.c_uint(int(limit_us)),
                                             _stream_handle(ws.device)))


def version() -> str:
    return load_library().sla_version().decode()
