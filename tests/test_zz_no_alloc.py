"""sla_route_noalloc: the router for callers that cannot allocate device memory.

Some callers may not call cudaMalloc or hand the library a workspace (a plugin
inside a runtime that owns all device memory, a loop with a fixed memory
budget). sla_route_noalloc keeps its scratch in an array compiled into the
library instead. These tests call it through the C ABI and check that it gives
exactly what sla_route (with a caller workspace) gives, on consecutive calls
that reuse the shared scratch, including rows long enough that the fp64 scores
are kept in that scratch. The host-side refusals (bad arguments, a problem too
large for the scratch) are checked without a GPU in test_abi_host.py.

This file is named to be collected last: it passes on its own in a fresh
process and after the rest of the GPU suite.
"""

import ctypes

import numpy as np
import pytest
import torch

from sparse_linear_attention_sla_b200 import binding
from sparse_linear_attention_sla_b200.workloads import random_inputs

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    lib = binding.load_library()
    fn = lib.sla_route_noalloc
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(binding.Problem), vp, vp, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    return lib, fn


def _call_noalloc(q, k, bq, kh, kl, want_crit, want_scores):
    lib, fn = _noalloc_fn()
    B, H, N, D = q.shape
    p = binding.problem(B, H, N, D, bq, 64, kh, kl)
    Nq, Nk, kc, _ = binding.counts(p)
    mask = torch.full((B, H, Nq, Nk), -1, dtype=torch.int8, device=q.device)
    crit = torch.full((B, H, Nq, kc), -1, dtype=torch.int32, device=q.device) if want_crit else None
    scores = torch.full((B, H, Nq, Nk), np.nan, dtype=torch.float64, device=q.device) if want_scores else None
    stream = ctypes.c_void_p(torch.cuda.current_stream(q.device).cuda_stream)
    st = fn(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
            ctypes.c_void_p(mask.data_ptr()), ctypes.c_void_p(crit.data_ptr() if crit is not None else 0),
            ctypes.c_void_p(scores.data_ptr() if scores is not None else 0), stream)
    assert st == 0, lib.sla_last_error().decode()
    torch.cuda.synchronize(q.device)
    return mask, crit, scores


# (B, H, N, D, block_q, kh, kl): two different problems back to back share the scratch.
PROBLEMS = [(1, 3, 4113, 128, 128, 0.1, 0.2), (2, 2, 1000, 64, 64, 0.25, 0.25)]


@pytest.mark.parametrize("want_crit, want_scores", [(True, True), (False, False), (True, False), (False, True)])
def test_noalloc_router_matches_workspace_router(cuda_device, want_crit, want_scores):
    for rep in range(2):  # two calls in a row per problem, alternating problems
        for case in PROBLEMS:
            B, H, N, D, bq, kh, kl = case
            q, k, _, _ = random_inputs(B, H, N, D, seed=31 + rep + N, device=cuda_device)
            ref_mask, ref_crit, ref_scores = binding.route(q, k, bq, 64, kh, kl, want_scores=True, want_crit=True)
            mask, crit, scores = _call_noalloc(q, k, bq, kh, kl, want_crit, want_scores)
            # labels and index lists are integers: bit-exact; scores: same kernels, same order
            assert torch.equal(mask, ref_mask)
            if want_crit:
                assert torch.equal(crit, ref_crit)
            if want_scores:
                np.testing.assert_allclose(scores.cpu().numpy(), ref_scores.cpu().numpy(), rtol=1e-12, atol=0)


@pytest.mark.parametrize("want_crit, want_scores", [(False, False), (True, True)])
def test_noalloc_router_long_rows(cuda_device, want_crit, want_scores):
    """Rows of more than 2048 KV blocks: with scores_out NULL the fp64 scores live in the
    static scratch (about 27 MiB here with the critical lists), else in the caller's buffer."""
    B, H, N, D, bq, kh, kl = 1, 1, 2050 * 64, 64, 128, 0.03, 0.05
    q, k, _, _ = random_inputs(B, H, N, D, seed=2050, device=cuda_device)
    ref_mask, ref_crit, ref_scores = binding.route(q, k, bq, 64, kh, kl, want_scores=True, want_crit=True)
    for _ in range(2):
        mask, crit, scores = _call_noalloc(q, k, bq, kh, kl, want_crit, want_scores)
        assert torch.equal(mask, ref_mask)
        if want_crit:
            assert torch.equal(crit, ref_crit)
        if want_scores:
            np.testing.assert_allclose(scores.cpu().numpy(), ref_scores.cpu().numpy(), rtol=1e-12, atol=0)
