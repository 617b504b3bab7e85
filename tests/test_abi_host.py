"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/sla.h declares, and its host logic (counts, argument
checks, workspace sizing) behaves as documented."""

import ctypes
import os
import re

import pytest

import oracle
from sparse_linear_attention_sla_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def _declared_symbols():
    names = set()
    for path in os.listdir(os.path.join(ROOT, "include")):
        if path.endswith(".h"):
            text = open(os.path.join(ROOT, "include", path)).read()
            names |= set(re.findall(r"^\s*(?:sla_status|size_t|int|const char\*)\s+(sla_\w+)\s*\(", text, re.M))
    return names


def test_header_declares_the_binding_exports():
    assert _declared_symbols() == set(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert lib.sla_version().decode().startswith("sla-b200")


@pytest.mark.parametrize("shape", [
    (1, 2, 1024, 64, 64, 64, 0.25, 0.25),
    (1, 12, 8192, 128, 128, 64, 0.10, 0.40),
    (1, 12, 32760, 128, 128, 64, 0.05, 0.10),
    (2, 40, 75600, 128, 128, 64, 0.05, 0.15),
    (1, 12, 32700, 128, 128, 64, 0.05, 0.0),
    (1, 12, 32760, 128, 128, 64, 1.0, 0.0),
    (1, 1, 130 * 64, 64, 64, 64, 0.0, 0.1),
    (1, 1, 1, 64, 64, 64, 0.5, 0.5),
    (3, 5, 777, 128, 64, 64, 0.33, 0.33),
])
def test_counts_match_oracle(lib, shape):
    B, H, N, D, bq, bk, kh, kl = shape
    p = binding.problem(B, H, N, D, bq, bk, kh, kl)
    # kh, kl pass through a C float: compare with the oracle at the same float value
    f32 = lambda x: ctypes.c_float(x).value
    assert binding.counts(p) == oracle.block_counts(N, bq, bk, f32(kh), f32(kl))
    assert binding.workspace_size(p) > 0


@pytest.mark.parametrize("bad, status", [
    ((1, 1, 64, 96, 64, 64, 0.1, 0.1), 2),     # D unsupported
    ((1, 1, 64, 64, 32, 64, 0.1, 0.1), 2),     # block_q unsupported
    ((1, 1, 64, 64, 64, 128, 0.1, 0.1), 2),    # block_kv unsupported
    ((0, 1, 64, 64, 64, 64, 0.1, 0.1), 1),     # B < 1
    ((1, 1, 0, 64, 64, 64, 0.1, 0.1), 1),      # N < 1
    ((1, 1, 64, 64, 64, 64, 0.7, 0.4), 1),     # kh + kl > 1
    ((1, 1, 64, 64, 64, 64, -0.1, 0.0), 1),    # kh < 0
    ((1, 1, 64, 64, 64, 64, float("nan"), 0.0), 1),
    ((1, 1, 64 * 20000, 64, 64, 64, 0.1, 0.1), 2),  # too many KV blocks
])
def test_invalid_problems_rejected_on_host(lib, bad, status):
    p = binding.problem(*bad)
    with pytest.raises(binding.SlaError) as e:
        binding.counts(p)
    assert e.value.status == status
    assert binding.workspace_size(p) == 0
    assert lib.sla_last_error().decode()


def test_entry_points_reject_bad_pointers_before_any_launch(lib):
    p = binding.problem(1, 1, 128, 64, 64, 64, 0.25, 0.25)
    null = ctypes.c_void_p(0)
    # NULL / misaligned pointers and missing workspace are host-side errors (no CUDA call made)
    assert lib.sla_forward(ctypes.byref(p), null, null, null, null, null, null, null, 0, null) == 1
    assert lib.sla_route(ctypes.byref(p), null, null, null, null, null, null, 0, null) == 1
    assert lib.sla_kv_states(ctypes.byref(p), null, null, null, null, null, 0, null) == 1
    fake = ctypes.c_void_p(1 << 20)  # aligned but never dereferenced on the host
    assert lib.sla_forward(ctypes.byref(p), fake, fake, fake, fake, null, ctypes.c_void_p(2 << 20), null, 0, null) == 3
    assert lib.sla_forward(ctypes.byref(p), fake, fake, fake, fake, null, fake, ctypes.c_void_p(4 << 20), 0, null) == 1
    small = binding.workspace_size(p) - 1
    assert lib.sla_forward(ctypes.byref(p), fake, fake, fake, fake, null, ctypes.c_void_p(2 << 20),
                           ctypes.c_void_p(8 << 20), small, null) == 3
    assert lib.sla_check(null, null) == 3


def test_low_bit_entry_points_host_checks(lib):
    B, H, N, D = 1, 2, 1000, 128
    p = binding.problem(B, H, N, D, 128, 64, 0.25, 0.25)
    _, Nk, _, _ = binding.counts(p)
    base, full = binding.workspace_size(p), binding.workspace_size_fp8(p)
    # the low-bit workspace adds the e4m3 codes of K and V and their block exponents
    extra = full - base
    assert 2 * B * H * N * D + 2 * B * H * Nk * 4 <= extra <= 2 * B * H * N * D + 2 * B * H * Nk * 4 + 4 * 256
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)
    out = ctypes.c_void_p(8 << 20)
    ws = ctypes.c_void_p(16 << 20)
    # a workspace sized for sla_forward is too small for sla_forward_fp8
    assert lib.sla_forward_fp8(ctypes.byref(p), fake, fake, fake, fake, null, out, ws, base, null) == 3
    assert lib.sla_forward_fp8(ctypes.byref(p), null, fake, fake, fake, null, out, ws, full, null) == 1
    assert lib.sla_forward_fp8_timed(ctypes.byref(p), fake, fake, fake, fake, null, out, ws, full, null, None) == 1
    # the low-bit branch needs D = 128
    p64 = binding.problem(1, 1, 256, 64, 64, 64, 0.25, 0.25)
    assert lib.sla_forward_fp8(ctypes.byref(p64), fake, fake, fake, fake, null, out, ws,
                               binding.workspace_size_fp8(p64), null) == 2
    assert "D=128" in lib.sla_last_error().decode()
    # the quantiser: NULL and misaligned outputs
    assert lib.sla_quantize_kv(ctypes.byref(p), null, fake, fake, fake, fake, fake, null) == 1
    assert lib.sla_quantize_kv(ctypes.byref(p), fake, fake, ctypes.c_void_p((1 << 20) + 4), fake, fake, fake,
                               null) == 1
    assert lib.sla_quantize_kv(ctypes.byref(p), fake, fake, fake, fake, ctypes.c_void_p((1 << 20) + 2), fake,
                               null) == 1
    assert binding.workspace_size_fp8(binding.problem(1, 1, 64, 96, 64, 64, 0.1, 0.1)) == 0


def _noalloc(lib):
    fn = lib.sla_route_noalloc
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(binding.Problem), vp, vp, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    return fn


def test_route_noalloc_host_checks(lib):
    """sla_route_noalloc's argument errors and its size refusal return before any CUDA call."""
    fn = _noalloc(lib)
    p = binding.problem(1, 2, 1000, 128, 128, 64, 0.1, 0.2)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced on the host
    assert fn(ctypes.byref(p), null, fake, fake, null, null, null) == 1           # q NULL
    assert fn(ctypes.byref(p), fake, ctypes.c_void_p((1 << 20) + 8), fake, null, null, null) == 1  # k misaligned
    assert fn(ctypes.byref(p), fake, fake, null, null, null, null) == 1           # mask_out NULL
    assert "mask_out" in lib.sla_last_error().decode()
    assert fn(ctypes.byref(p), fake, fake, fake, ctypes.c_void_p((1 << 20) + 2), null, null) == 1  # crit misaligned
    assert fn(ctypes.byref(p), fake, fake, fake, null, ctypes.c_void_p((1 << 20) + 4), null) == 1  # scores misaligned
    for bad, status in [((1, 1, 64, 96, 64, 64, 0.1, 0.1), 2), ((1, 1, 0, 64, 64, 64, 0.1, 0.1), 1),
                        ((1, 1, 64, 64, 64, 64, 0.7, 0.4), 1)]:
        assert fn(ctypes.byref(binding.problem(*bad)), fake, fake, fake, null, null, null) == status


def test_route_noalloc_refuses_oversize_problem(lib):
    fn = _noalloc(lib)
    # 16 heads of N = 131072 need ~200 MB of scratch without caller outputs: refused on the host.
    p = binding.problem(1, 16, 131072, 128, 128, 64, 0.05, 0.1)
    fake = ctypes.c_void_p(1 << 20)
    null = ctypes.c_void_p(0)
    assert fn(ctypes.byref(p), fake, fake, fake, null, null, null) == 3
    assert "maximum" in lib.sla_last_error().decode()
    # the same problem with both outputs given by the caller still needs more than the array holds
    assert fn(ctypes.byref(p), fake, fake, fake, fake, ctypes.c_void_p(2 << 20), null) == 3


def test_forward_launch_counts(lib):
    """One launch per stage: precompute, labels (the router's scores and selection, or the
    caller mask's lists), aggregation, attention, and the K/V quantiser for the low-bit call."""
    p = binding.problem(1, 12, 32760, 128, 128, 64, 0.05, 0.1)
    assert binding.forward_launches(p) == 5
    assert binding.forward_launches(p, with_mask=True) == 4
    assert binding.forward_launches(p, low_bit=True) == 6
    assert binding.forward_launches(binding.problem(2, 40, 75600, 128, 128, 64, 0.05, 0.15)) == 5
    assert lib.sla_forward_launches(ctypes.byref(binding.problem(1, 1, 64, 96, 64, 64, 0.1, 0.1)), 0, 0) == -1


def test_aggregate_states_host_checks(lib):
    p = binding.problem(1, 1, 128, 64, 64, 64, 0.25, 0.25)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(16 << 20)
    size = binding.workspace_size(p)
    assert lib.sla_aggregate_states(ctypes.byref(p), fake, fake, null, fake, fake, ws, size, null) == 1  # no mask
    assert lib.sla_aggregate_states(ctypes.byref(p), fake, fake, fake, ctypes.c_void_p((1 << 20) + 8), fake, ws,
                                    size, null) == 1  # H_out misaligned
    assert lib.sla_aggregate_states(ctypes.byref(p), fake, fake, fake, fake, fake, ws, size - 1, null) == 3


def test_variant_entry_points_reject_bad_variants(lib):
    p = binding.problem(1, 1, 128, 64, 64, 64, 0.25, 0.25)
    fake = ctypes.c_void_p(1 << 20)
    null = ctypes.c_void_p(0)
    ws = ctypes.c_void_p(16 << 20)
    size = binding.workspace_size(p)
    for bad in (binding.Variant(2, 0), binding.Variant(0, -1)):
        assert lib.sla_route_variant(ctypes.byref(p), ctypes.byref(bad), fake, fake, fake, null, null, ws, size,
                                     null) == 1
        assert lib.sla_forward_variant(ctypes.byref(p), ctypes.byref(bad), fake, fake, fake, fake, null,
                                       ctypes.c_void_p(8 << 20), ws, size, null) == 1
    assert lib.sla_route_variant(ctypes.byref(p), None, fake, fake, fake, null, null, ws, size, null) == 1
    nan_scale = binding.Variant(0, 0, float("nan"), 0.5)
    assert lib.sla_forward_variant(ctypes.byref(p), ctypes.byref(nan_scale), fake, fake, fake, fake, null,
                                   ctypes.c_void_p(8 << 20), ws, size, null) == 1
    assert "finite" in lib.sla_last_error().decode()


def test_backward_host_checks(lib):
    p = binding.problem(1, 1, 256, 128, 128, 64, 0.25, 0.25)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(32 << 20)
    size = lib.sla_workspace_size_backward(ctypes.byref(p))
    assert size > binding.workspace_size(p)
    # only calls the host rejects before any CUDA call (unsupported shape, NULL pointer, small workspace)
    args = [fake, fake, fake, fake, null, fake, fake, fake, fake, fake]
    p64 = binding.problem(1, 1, 256, 64, 64, 64, 0.25, 0.25)
    assert lib.sla_backward(ctypes.byref(p64), *args, ws, size, null) == 2
    pbq = binding.problem(1, 1, 256, 128, 64, 64, 0.25, 0.25)
    assert lib.sla_backward(ctypes.byref(pbq), *args, ws, size, null) == 2
    assert lib.sla_backward(ctypes.byref(p), null, *args[1:], ws, size, null) == 1
    assert lib.sla_backward(ctypes.byref(p), *args, ws, size - 1, null) == 3


def test_pisa_host_checks(lib):
    p = binding.problem(1, 2, 1000, 128, 128, 64, 0.25, 0.25)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(64 << 20)
    size = lib.sla_workspace_size_pisa(ctypes.byref(p))
    # the forward's workspace plus centroid keys and values, per-part first-order sums and Hbar
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    BH, Nk, D = 2, 16, 128
    parts = min(Nk, max(1, 148 // BH))
    assert size == binding.workspace_size(p) + 2 * a256(BH * Nk * D * 2) + a256(BH * parts * D * D * 4) + \
        a256(BH * D * D * 2)
    out = ctypes.c_void_p(8 << 20)
    assert lib.sla_forward_pisa(ctypes.byref(p), null, fake, fake, null, out, ws, size, null) == 1
    assert lib.sla_forward_pisa(ctypes.byref(p), fake, fake, fake, null, fake, ws, size, null) == 1  # out aliases q
    assert lib.sla_forward_pisa(ctypes.byref(p), fake, fake, fake, null, out, ws, size - 1, null) == 3
    assert lib.sla_pisa_hbar(ctypes.byref(p), fake, fake, null, ws, size, null) == 1
    assert lib.sla_pisa_hbar(ctypes.byref(p), fake, fake, out, ws, size - 1, null) == 3
    bad = binding.problem(1, 2, 1000, 96, 128, 64, 0.25, 0.25)
    assert lib.sla_workspace_size_pisa(ctypes.byref(bad)) == 0
    assert lib.sla_forward_pisa(ctypes.byref(bad), fake, fake, fake, null, out, ws, size, null) == 2
