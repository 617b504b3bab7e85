"""The device-side failure path: a bounded wait that runs out is reported, not hung on.

Every wait in the library's kernels is bounded; when one runs out the kernel records
SLA_ERR_TIMEOUT in the workspace's error word, returns, and sla_check reports it. The
self-test entry point runs that path on purpose with a short limit: one thread waits on
an mbarrier nothing arrives on. No fault, trap or hang is involved, and the context stays
usable: the forward that follows must still match the oracle.
"""

import time

import numpy as np
import pytest
import torch

import oracle
from sparse_linear_attention_sla_b200 import binding
from sparse_linear_attention_sla_b200.workloads import random_inputs
from tests.parity_utils import assert_outputs_close

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives(cuda_device):
    B, H, N, D, bq, kh, kl = 1, 2, 700, 128, 128, 0.25, 0.25
    ws = binding.new_workspace(binding.problem(B, H, N, D, bq, 64, kh, kl), cuda_device)
    binding.check(ws)  # clean to begin with
    t0 = time.perf_counter()
    binding.selftest_wait_timeout(ws, limit_us=50000)
    with pytest.raises(binding.SlaError) as e:
        binding.check(ws)
    waited = time.perf_counter() - t0
    assert e.value.status == 5, str(e.value)
    assert 0.04 <= waited < 5.0, f"the 50 ms wait took {waited:.3f} s"
    binding.check(ws)  # the error word was cleared
    # the context is still usable: a forward right after matches the oracle
    q, k, v, alpha = random_inputs(B, H, N, D, seed=77, device=cuda_device)
    mask, _, _ = binding.route(q, k, bq, 64, kh, kl)
    out = binding.forward(q, k, v, alpha, bq, 64, kh, kl, mask=mask, ws=ws)
    binding.check(ws)
    ref = oracle.forward(q.cpu(), k.cpu(), v.cpu(), alpha.cpu(), bq, 64, kh, kl, mask=mask.cpu().numpy())
    assert_outputs_close(out.float().cpu().numpy(), np.asarray(ref), "forward after a reported timeout")


def test_selftest_rejects_bad_arguments(cuda_device):
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(binding.SlaError) as e:
        binding.selftest_wait_timeout(ws, limit_us=0)
    assert e.value.status == 1
    with pytest.raises(binding.SlaError) as e:
        binding.selftest_wait_timeout(ws[:128], limit_us=10)
    assert e.value.status == 3
    binding.check(ws)
