"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Every input is seeded; the oracle sees exactly the bf16 tensors the kernels
see. Labels must match bit for bit except near ties (counted and reported);
outputs must match within max-abs 2e-2 and mean-abs 2e-3.
"""

import numpy as np
import pytest
import torch

import oracle
from sparse_linear_attention_sla_b200 import binding
from sparse_linear_attention_sla_b200.workloads import (SWEEP_KH, WORKLOADS, make_inputs, random_inputs,
                                                        sweep_workload)
from tests.parity_utils import assert_outputs_close, label_mismatches

pytestmark = pytest.mark.gpu


def _to_cpu(*ts):
    return [t.detach().cpu() for t in ts]


def _route_parity(q, k, bq, kh, kl, heads=None):
    """GPU router vs oracle on the given heads: labels (near-tie rule), scores, crit lists.

    Returns (gpu_mask, oracle_mask, mismatches). oracle_mask holds the oracle's
    labels on the checked heads and the GPU's labels elsewhere.
    """
    mask, crit, scores = binding.route(q, k, bq, 64, kh, kl, want_scores=True, want_crit=True)
    B, H, N, D = q.shape
    p = binding.problem(B, H, N, D, bq, 64, kh, kl)
    Nq, Nk, kc, kn = binding.counts(p)
    heads = heads or [(b, h) for b in range(B) for h in range(H)]
    gm, gs, gc = mask.cpu().numpy(), scores.cpu().numpy(), crit.cpu().numpy()
    om = gm.copy()
    worst_rel = 0.0
    total = excused = 0
    for b, h in heads:
        rm, S = oracle.route(q[b, h].cpu(), k[b, h].cpu(), bq, 64, kh, kl)
        om[b, h] = rm
        rel = np.abs(gs[b, h] - S).max() / max(np.abs(S).max(), 1e-300)
        worst_rel = max(worst_rel, rel)
        t, e = label_mismatches(gm[b, h], rm, S, kc, kn)
        total += t
        excused += e
        # the critical list is the ascending index list of the GPU's own critical labels
        for i in range(Nq):
            np.testing.assert_array_equal(gc[b, h, i], np.nonzero(gm[b, h, i] == 2)[0])
        assert np.all((gm[b, h] == 2).sum(-1) == kc) and np.all((gm[b, h] == 0).sum(-1) == kn)
    assert worst_rel < 1e-12, f"scores differ from the oracle by {worst_rel:.2e} (relative)"
    assert total == excused, f"{total - excused} label mismatches outside near ties ({total} total)"
    if total:
        print(f"near-tie label mismatches (excused): {total}")
    return mask, torch.from_numpy(om).to(q.device), total


def _oracle_rows(q, k, v, alpha, bq, mask, heads, query_blocks=None):
    """Oracle output for the sampled heads (NaN elsewhere), one head at a time."""
    B, H, N, D = q.shape
    ref = np.full((B, H, N, D), np.nan)
    m = mask.cpu().numpy()
    for b, h in heads:
        o = oracle.forward(q[b, h][None, None].cpu(), k[b, h][None, None].cpu(), v[b, h][None, None].cpu(),
                           alpha[h][None].cpu(), bq, 64, mask=m[b, h][None, None], query_blocks=query_blocks)
        ref[b, h] = o[0, 0]
    return ref


CASES = [
    # B, H, N, D, bq, kh, kl
    (1, 2, 1024, 64, 64, 0.25, 0.25),
    (1, 1, 200, 64, 64, 0.3, 0.2),
    (2, 2, 333, 128, 128, 0.2, 0.3),
    (1, 3, 4113, 128, 128, 0.1, 0.2),
    (1, 2, 700, 128, 64, 0.25, 0.25),
    (1, 2, 129, 64, 128, 0.5, 0.25),
    (1, 2, 1000, 128, 128, 1.0, 0.0),   # every block critical: dense softmax attention
    (1, 2, 1000, 128, 128, 0.0, 0.0),   # no critical, no negligible: pure linear attention
    (1, 2, 1000, 128, 128, 0.0, 0.5),   # empty sparse branch
    (1, 2, 1000, 128, 128, 0.5, 0.5),   # empty linear branch
    (1, 1, 64, 128, 128, 0.5, 0.0),     # a single KV block
    (1, 1, 1, 64, 64, 1.0, 0.0),        # a single token
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_forward_matches_oracle(cuda_device, case):
    B, H, N, D, bq, kh, kl = case
    q, k, v, alpha = random_inputs(B, H, N, D, seed=sum(case[:5]), device=cuda_device)
    gmask, omask, nmis = _route_parity(q, k, bq, kh, kl)
    ws = binding.new_workspace(binding.problem(B, H, N, D, bq, 64, kh, kl), cuda_device)
    out = binding.forward(q, k, v, alpha, bq, 64, kh, kl, ws=ws)          # internal router
    out_m = binding.forward(q, k, v, alpha, bq, 64, kh, kl, mask=omask, ws=ws)  # oracle's labels
    binding.check(ws)
    heads = [(b, h) for b in range(B) for h in range(H)]
    ref = _oracle_rows(q, k, v, alpha, bq, omask, heads)
    assert_outputs_close(out_m.float().cpu().numpy(), ref, f"oracle labels {case}")
    if nmis == 0:
        assert torch.equal(out, out_m), "router path and caller-mask path disagree on the same labels"


def test_kv_states_match_oracle(cuda_device):
    for (B, H, N, D) in [(1, 2, 1024, 64), (1, 2, 333, 128), (2, 1, 4096 + 7, 128)]:
        q, k, v, _ = random_inputs(B, H, N, D, seed=N, device=cuda_device)
        h, z = binding.kv_states(k, v)
        kc_, vc = _to_cpu(k, v)
        rh, rz = oracle.kv_states(kc_, vc, 64)
        # phi(k) enters the tensor core in bf16 (relative rounding 2^-8) with fp32 accumulation
        scale_h = np.abs(rh).max()
        assert np.abs(h.cpu().numpy() - rh).max() <= 8e-3 * scale_h
        np.testing.assert_allclose(z.cpu().numpy(), rz, rtol=1e-5, atol=1e-4)


def _workload_parity(w, device, heads=None, query_blocks=None, gen_device="cpu"):
    q, k, v, alpha = make_inputs(w, device=gen_device)
    q, k, v, alpha = (t.to(device) for t in (q, k, v, alpha))
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    gmask, omask, nmis = _route_parity(q, k, w.block_q, w.kh, w.kl, heads=heads)
    ws = binding.new_workspace(binding.problem(w.B, w.H, w.N, w.D, w.block_q, 64, w.kh, w.kl), device)
    out = binding.forward(q, k, v, alpha, w.block_q, 64, w.kh, w.kl, ws=ws)
    out_m = binding.forward(q, k, v, alpha, w.block_q, 64, w.kh, w.kl, mask=omask, ws=ws)
    binding.check(ws)
    ref = _oracle_rows(q, k, v, alpha, w.block_q, omask, heads, query_blocks)
    err = assert_outputs_close(out_m.float().cpu().numpy(), ref, w.name)
    if nmis == 0:
        assert torch.equal(out, out_m)
    print(f"{w.name}: max-abs {err[0]:.3e} mean-abs {err[1]:.3e} near-tie mismatches {nmis}")
    return err, nmis


def test_iid_b1h2_n1024_d64(cuda_device):
    _workload_parity(WORKLOADS["iid_b1h2_n1024_d64"], cuda_device)


def test_field1d_b1h12_n8192_d128(cuda_device):
    _workload_parity(WORKLOADS["field1d_b1h12_n8192_d128"], cuda_device)


def test_wan13b_b1h12_n32760_d128(cuda_device):
    _workload_parity(WORKLOADS["wan13b_b1h12_n32760_d128"], cuda_device)


def test_wan14b720p_sampled(cuda_device):
    w = WORKLOADS["wan14b720p_b2h40_n75600_d128"]
    Nq = -(-w.N // w.block_q)
    rng = np.random.default_rng(4)
    heads = [(0, 0), (1, 39)] + [(int(rng.integers(2)), int(rng.integers(40))) for _ in range(2)]
    qbs = sorted({0, Nq - 1, *[int(x) for x in rng.integers(1, Nq - 1, size=6)]})
    _workload_parity(w, cuda_device, heads=heads, query_blocks=qbs, gen_device=cuda_device)


@pytest.mark.parametrize("kh", [kh for kh in SWEEP_KH if kh < 1.0])
def test_sparsity_sweep_full(cuda_device, kh):
    """Every head and every query block of the sweep point, router parity on every head."""
    _workload_parity(sweep_workload(kh), cuda_device)


def test_sparsity_sweep_dense_sampled(cuda_device):
    """kh = 100% (every block critical: alpha times dense softmax attention): router on every head, outputs
    on a seeded sample of heads and query blocks (the full fp64 run is ~6.6 TFLOP)."""
    w = sweep_workload(1.0)
    rng = np.random.default_rng(100)
    heads = [(0, 0), (0, 11)] + [(0, int(h)) for h in rng.choice(np.arange(1, 11), size=2, replace=False)]
    Nq = -(-w.N // w.block_q)
    qbs = sorted({0, 1, Nq - 1, *[int(x) for x in rng.integers(2, Nq - 1, size=5)]})
    _workload_parity(w, cuda_device, heads=heads, query_blocks=qbs)


def test_sparsity_sweep_tail_n32700(cuda_device):
    """The sweep's ragged case (N = 32700: 60-token last query and KV blocks), in full."""
    _workload_parity(sweep_workload(0.05, N=32700), cuda_device)


def _scale_blocks(k, factors):
    """K with its 64-key block j multiplied by factors[j] (fp64, then back to bf16)."""
    N = k.shape[2]
    f = torch.as_tensor(factors, dtype=torch.float64).repeat_interleave(64)[:N]
    return (k.double() * f[None, None, :, None]).to(torch.bfloat16)


def _reference_moves(q, k, crit_mask, bq, log2_margin):
    """Rows whose largest score over their later critical blocks exceeds the largest score of
    their first critical block by more than log2_margin (log2 units), counted over every head."""
    B, H, N, D = q.shape
    scale = np.log2(np.e) / np.sqrt(D)
    moved = 0
    for b in range(B):
        for h in range(H):
            S = (q[b, h].double() @ k[b, h].double().T).cpu().numpy() * scale
            for i in range(crit_mask.shape[2]):
                blocks = np.nonzero(crit_mask[b, h, i] == 2)[0]
                if len(blocks) < 2:
                    continue
                rows = S[i * bq:min(N, (i + 1) * bq)]
                first = rows[:, blocks[0] * 64:min(N, blocks[0] * 64 + 64)].max(axis=1)
                later = np.concatenate([rows[:, j * 64:min(N, j * 64 + 64)] for j in blocks[1:]], axis=1).max(axis=1)
                moved += int((later - first > log2_margin).sum())
    return moved


@pytest.mark.parametrize("shape", ["rising", "steps", "falling", "rising_d64"])
def test_scores_far_above_the_first_block(cuda_device, shape):
    """K blocks scaled so that a row's later critical blocks mostly score far above (rising, steps)
    or far below (falling) its first one. The softmax's reference maximum is taken from a tile's
    first block and must move (rescaling O_s and the normaliser) whenever a block's exponentials
    would pass 2^20; far below it they only shrink. Both against the oracle."""
    B, H, N, D, bq, kh, kl = 1, 2, 4096 + 40, 128, 128, 0.5, 0.25
    if shape == "rising_d64":  # D = 64 with 64-row query blocks
        D, bq = 64, 64
    q, k, v, alpha = random_inputs(B, H, N, D, seed={"rising": 5, "steps": 6, "falling": 7, "rising_d64": 8}[shape],
                                   device="cpu")
    nb = -(-N // 64)
    if shape.startswith("rising"):
        f = np.geomspace(0.25, 16.0, nb)
    elif shape == "steps":
        f = 0.5 * 2.0 ** (np.arange(nb) % 5)
    else:
        f = np.geomspace(16.0, 0.25, nb)
    k = _scale_blocks(k, f)
    q, k, v, alpha = (t.to(cuda_device) for t in (q, k, v, alpha))
    gmask, omask, nmis = _route_parity(q, k, bq, kh, kl)
    moved = _reference_moves(q, k, omask.cpu().numpy(), bq, 21.0)
    if shape != "falling":  # (falling: a few hundred rows still meet a larger block later)
        assert moved > 1000, f"only {moved} rows move their reference"
    out_m = binding.forward(q, k, v, alpha, bq, 64, kh, kl, mask=omask)
    ref = _oracle_rows(q, k, v, alpha, bq, omask, [(0, 0), (0, 1)])
    assert_outputs_close(out_m.float().cpu().numpy(), ref, f"block scales {shape}")
    o2 = binding.forward(q, k, v, alpha, bq, 64, kh, kl, mask=omask)
    assert torch.equal(out_m, o2)
    assert torch.isfinite(out_m.float()).all()


def test_output_invariants(cuda_device):
    q, k, v, alpha = random_inputs(1, 2, 2000, 128, seed=9, device=cuda_device)
    o1 = binding.forward(q, k, v, alpha, 128, 64, 0.2, 0.2)
    o2 = binding.forward(q, k, v, alpha, 128, 64, 0.2, 0.2)
    assert torch.equal(o1, o2), "forward is not deterministic"
    vf = v.float()
    lo, hi = vf.amin(dim=2, keepdim=True), vf.amax(dim=2, keepdim=True)
    o = o1.float()
    slack = 1e-2 * (hi - lo)
    assert bool(((o >= lo - slack) & (o <= hi + slack)).all()), "output outside the per-channel V range"
    # V -> 2 V + 1 gives O -> 2 O + 1 (both branches are normalised averages of V rows)
    o3 = binding.forward(q, k, (2 * vf + 1).to(torch.bfloat16), alpha, 128, 64, 0.2, 0.2).float()
    assert (o3 - (2 * o + 1)).abs().max().item() < 6e-2


def test_bad_caller_mask_is_reported(cuda_device):
    q, k, v, alpha = random_inputs(1, 1, 256, 64, seed=3, device=cuda_device)
    mask = torch.ones(1, 1, 4, 4, dtype=torch.int8, device=cuda_device)
    mask[0, 0, 1, 2] = 3
    ws = binding.new_workspace(binding.problem(1, 1, 256, 64, 64, 64), cuda_device)
    binding.forward(q, k, v, alpha, 64, 64, 0.0, 0.0, mask=mask, ws=ws)
    with pytest.raises(binding.SlaError) as e:
        binding.check(ws)
    assert e.value.status == 6
    binding.check(ws)  # the error word was cleared


def _clustered_keys(N, D, seed):
    """Inputs whose compressed scores tie in fp32 but not in fp64.

    Every KV block is the same random block except in one channel d*, where the
    block's first token carries a perturbation delta_j (exactly representable in
    bf16) and the rest are zero; every query token has 1.0 in channel d*. So
    S_j = S_base + delta_j / (64 sqrt(D)). A quarter of the blocks get large
    positive deltas, a quarter large negative ones, and half get deltas of
    m * 2^-30 with m in [-40, 40) (many exact repeats): their scores agree to
    ~1e-12, far below fp32 resolution, so the labels inside that cluster are
    decided by fp64 scores and then by index.
    """
    g = torch.Generator().manual_seed(seed)
    Nk = N // 64
    dstar = 5
    base = torch.randn(64, D, generator=g)
    base[:, dstar] = 0.0
    k = base.repeat(Nk, 1)
    m_small = torch.randint(-40, 40, (Nk,), generator=g).double()
    m_big = torch.randint(1, 120, (Nk,), generator=g).double()
    j = torch.arange(Nk)
    delta = torch.where(j % 2 == 0, m_small * 2.0 ** -30,
                        torch.where(j % 4 == 1, m_big * 2.0 ** -4, -m_big * 2.0 ** -4))
    k[j * 64, dstar] = delta.float()
    q = torch.randn(N, D, generator=g)
    q[:, dstar] = 1.0
    v = torch.randn(N, D, generator=g)
    kb = k.to(torch.bfloat16)
    assert torch.equal(kb[j * 64, dstar].double(), delta), "perturbations must be exact in bf16"
    return q.to(torch.bfloat16), kb, v.to(torch.bfloat16)


@pytest.mark.parametrize("N, D, bq, kh, kl", [(32768, 128, 128, 0.5, 0.375), (8192, 64, 64, 0.375, 0.375),
                                              (32768, 128, 128, 0.3, 0.45)])
def test_router_resolves_fp32_ties_in_fp64(cuda_device, N, D, bq, kh, kl):
    """Labels inside a cluster of scores that fp32 cannot tell apart match the oracle exactly."""
    q, k, v = _clustered_keys(N, D, seed=N + D)
    rm, S = oracle.route(q, k, bq, 64, kh, kl)
    Nk = N // 64
    # the construction is meaningful: the boundaries fall inside the cluster, where fp32 ties
    s32 = S.astype(np.float32)
    clustered = np.arange(Nk) % 2 == 0
    assert np.all(s32[:, clustered] == s32[:, clustered][:, :1]) or np.ptp(s32[:, clustered], axis=1).max() <= \
        4 * np.spacing(np.abs(s32).max())
    assert np.all((rm[:, clustered] == 2).any(-1)) and np.all((rm[:, clustered] == 1).any(-1))
    qd, kd = q[None, None].to(cuda_device), k[None, None].to(cuda_device)
    mask, crit, _ = binding.route(qd, kd, bq, 64, kh, kl, want_scores=True, want_crit=True)
    gm = mask[0, 0].cpu().numpy()
    assert np.array_equal(gm, rm), f"{int((gm != rm).sum())} labels differ inside an fp32 tie cluster"
    gc = crit[0, 0].cpu().numpy()
    for i in range(gm.shape[0]):
        np.testing.assert_array_equal(gc[i], np.nonzero(rm[i] == 2)[0])
    # the fused forward's own router gives the same labels (through the forward output)
    alpha = torch.rand(1, D, generator=torch.Generator().manual_seed(1)).to(cuda_device)
    vd = v[None, None].to(cuda_device)
    o_int = binding.forward(qd, kd, vd, alpha, bq, 64, kh, kl)
    o_ext = binding.forward(qd, kd, vd, alpha, bq, 64, kh, kl, mask=torch.from_numpy(rm)[None, None].to(cuda_device))
    assert torch.equal(o_int, o_ext)


def test_long_rows_use_the_fp64_selection(cuda_device):
    """Rows of more than 2048 KV blocks take the fp64 score and selection kernels."""
    B, H, N, D, bq, kh, kl = 1, 1, 2049 * 64 + 17, 64, 128, 0.02, 0.05
    q, k, v, alpha = random_inputs(B, H, N, D, seed=2049, device=cuda_device)
    p = binding.problem(B, H, N, D, bq, 64, kh, kl)
    Nq, Nk, kc, kn = binding.counts(p)
    assert Nk > 2048
    mask, _, _ = _route_parity(q, k, bq, kh, kl)
    # the fused forward's own router gives the same labels (through the output), and a
    # sample of query blocks matches the oracle
    ws = binding.new_workspace(p, cuda_device)
    out_int = binding.forward(q, k, v, alpha, bq, 64, kh, kl, ws=ws)
    out_ext = binding.forward(q, k, v, alpha, bq, 64, kh, kl, mask=mask, ws=ws)
    binding.check(ws)
    assert torch.equal(out_int, out_ext)
    qb = [0, 1, Nq // 2, Nq - 1]
    ref = _oracle_rows(q, k, v, alpha, bq, mask, [(0, 0)], query_blocks=qb)
    assert_outputs_close(out_ext.float().cpu().numpy(), ref, "long rows")


@pytest.mark.parametrize("B, H, N, D, bq, kh, kl", [(1, 2, 1000, 128, 128, 0.2, 0.3), (2, 1, 333, 64, 64, 0.25, 0.25),
                                                     (1, 3, 4113, 128, 128, 0.0, 0.0)])
def test_aggregate_states_match_oracle(cuda_device, B, H, N, D, bq, kh, kl):
    """H_i, Z_i after the aggregation against the oracle's sums over the marginal blocks.

    Bound per entry: phi(k) enters the tensor core in bf16, h_j and z_j are stored in bf16 and
    H_i is rounded to bf16 (three roundings, each at most 2^-8 relative: bf16 carries 8
    significant bits); the sums accumulate in fp32. So |H - H_ref| <= 3 * 2^-8 * sum over
    marginal j of (phi(K_j)^T |V_j|) and |Z - Z_ref| <= 2^-8 * Z_ref (phi > 0), plus fp32
    slack."""
    q, k, v, _ = random_inputs(B, H, N, D, seed=N + D, device=cuda_device)
    mask, _, _ = binding.route(q, k, bq, 64, kh, kl)
    Hs, Zs, ws = binding.aggregate_states(k, v, mask, bq)
    binding.check(ws)
    kc_, vc = _to_cpu(k, v)
    h, z = oracle.kv_states(kc_, vc, 64)
    h_abs, _ = oracle.kv_states(kc_, vc.abs(), 64)
    m = mask.cpu().numpy()
    Hg, Zg = Hs.float().cpu().numpy(), Zs.cpu().numpy()
    for b in range(B):
        for hh in range(H):
            Hr, Zr = oracle.marginal_sums(m[b, hh], h[b, hh], z[b, hh])
            Ha, _ = oracle.marginal_sums(m[b, hh], h_abs[b, hh], z[b, hh])
            tol_h = 3 * 2.0 ** -8 * Ha + 1e-6 * (Ha.max() + 1)
            assert np.all(np.abs(Hg[b, hh] - Hr) <= tol_h), float((np.abs(Hg[b, hh] - Hr) - tol_h).max())
            np.testing.assert_allclose(Zg[b, hh], Zr, rtol=2.0 ** -8 + 1e-6, atol=1e-5)
    if kh == 0 and kl == 0:  # every block marginal: H_i is the sum over all blocks for every row
        assert np.allclose(Hg[0, 0, 0], Hg[0, 0, -1]) and np.allclose(Zg[0, 0, 0], Zg[0, 0, -1])


def test_alpha_at_zero_and_one(cuda_device):
    """Channels with alpha exactly 0 (linear branch only) and 1 (sparse branch only) next to
    ordinary ones: the fused blend floors alpha at 2^-24, which stays within the tolerances."""
    B, H, N, D, bq, kh, kl = 1, 2, 1000, 128, 128, 0.25, 0.25
    q, k, v, alpha = random_inputs(B, H, N, D, seed=77, device=cuda_device)
    alpha[:, 0::4] = 0.0
    alpha[:, 1::4] = 1.0
    gmask, omask, nmis = _route_parity(q, k, bq, kh, kl)
    out = binding.forward(q, k, v, alpha, bq, 64, kh, kl, mask=omask)
    ref = _oracle_rows(q, k, v, alpha, bq, omask, [(0, 0), (0, 1)])
    assert_outputs_close(out.float().cpu().numpy(), ref, "alpha in {0, 1}")
