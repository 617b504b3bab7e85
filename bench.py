#!/usr/bin/env python
"""Benchmark of the fused SLA forward (sla_forward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step is one sla_forward call (router, KV states, aggregation, fused
attention) over one batch of seeded synthetic inputs already resident in HBM.
L2 is flushed (512 MiB write, untimed) before every call; each call is timed
with CUDA events on the launching stream. Rank 0 prints one JSON line.

With --gpus N > 1 (launched by torch.distributed.run) every rank runs its own
replica of the workload on its own GPU (the heads of a batch are independent
problems, so there is no data-path collective); the step time is the maximum
over ranks and the value counts the work of all ranks ("scaling": "weak").

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0
only), one head of the workload per step.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "effective attention TFLOPS and ms/call at 1 B200; fraction of roofline"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "wan13b_b1h12_n32760_d128"
FLUSH_BYTES = 512 << 20


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the low-bit (e4m3) sparse-branch measurement")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward measurement")
    ap.add_argument("--no-pisa", action="store_true", help="skip the PISA variant measurement")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the router / feature-map / branch-dropping variant measurements")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration table (the other workloads, the kh sweep and its tail)")
    ap.add_argument("--config-steps", type=int, default=10, help="timed calls per configuration of that table")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle baseline sample")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    return args


# ---------------------------------------------------------------- peaks and work accounting


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def dense_equivalent_flops(w):
    return 4.0 * w.B * w.H * float(w.N) ** 2 * w.D


def algorithmic_work(w, mask):
    """Algorithmic FLOPs and bytes of one forward (no recomputation or padding credited).

    mask: [B,H,Nq,Nk] int8 labels actually used. Sparse FLOPs count the valid
    query rows and keys of every critical (query block, KV block) pair.
    """
    import torch

    B, H, N, D = w.B, w.H, w.N, w.D
    BH = B * H
    Nq, Nk = mask.shape[-2], mask.shape[-1]
    qsize = torch.clamp(N - torch.arange(Nq, device=mask.device) * w.block_q, max=w.block_q).double()
    ksize = torch.clamp(N - torch.arange(Nk, device=mask.device) * w.block_kv, max=w.block_kv).double()
    crit = (mask == 2).double().reshape(BH, Nq, Nk)
    pairs = torch.einsum("i,bij,j->", qsize, crit, ksize).item()
    marg = (mask == 1).sum(-1).double().reshape(BH, Nq)
    nonmarg = Nk - marg
    f_sparse = 4.0 * D * pairs
    f_states = 2.0 * N * D * D * BH
    f_apply = 2.0 * N * D * D * BH
    f_agg = float(torch.minimum(marg, nonmarg).sum().item()) * D * D
    f_router = 2.0 * (N * D + Nq * Nk * D) * BH
    f_elem = 3.0 * N * D * BH
    f_alg = f_sparse + f_states + f_apply + f_agg + f_router + f_elem
    bytes_alg = 8.0 * N * D * BH + Nq * Nk * BH + H * D * 4
    # backward with the labels fixed: five products per critical pair (S recomputed, dP, dV, dQ,
    # dK), four D x D products per row in the linear branch (G H^T, u^T G, phi(K) dh, V dh^T),
    # the transposed aggregation, and the row terms
    f_bwd = 2.5 * f_sparse + 4.0 * N * D * D * BH + f_agg + 8.0 * N * D * BH
    # PISA with the same critical sets: the critical pairs, two D-products per row and
    # non-critical block (its centroid's score and value sum), the first-order term per row, and
    # the centred first-order matrices of the blocks
    noncrit = (Nk - (mask == 2).sum(-1)).double().reshape(BH, Nq)
    f_pisa = f_sparse + 4.0 * D * float(torch.einsum("i,bi->", qsize, noncrit).item()) + \
        2.0 * N * D * D * BH + 2.0 * N * D * D * BH
    return {"flops": f_alg, "bytes": bytes_alg, "f_sparse": f_sparse, "f_attn_kernel": f_sparse + f_apply,
            "f_states": f_states, "f_agg": f_agg, "f_router": f_router, "f_bwd": f_bwd, "f_pisa": f_pisa}


def max_over_ranks(x, dist=None, device="cpu"):
    """Largest value of x over all ranks (x itself without a process group)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world, flops_per_rank, ms_step):
    """Aggregate throughput of `world` replicas that each did flops_per_rank in ms_step (the slowest rank)."""
    return world * flops_per_rank / (ms_step * 1e-3) / 1e12


# sources each attention kernel is built from (its recorded traffic is void once one changes)
KERNEL_SOURCES = {
    "attn_kernel": ("attention.cuh", "softmax_block.cuh", "sm100.cuh"),
    "attn_fp8_kernel": ("attention_fp8.cuh", "fp8.cuh", "attention.cuh", "softmax_block.cuh", "sm100.cuh"),
}


def kernel_source_sha(kernel="attn_kernel"):
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "sparse_linear_attention_sla_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, kernel="attn_kernel"):
    """DRAM bytes per launch of an attention kernel from the committed ncu summary, if still current."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("source_sha") != kernel_source_sha(kernel) or t.get("workload") != workload:
        return None
    return float(t["dram_bytes_per_launch"])


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock, power and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="sla_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                                 "hw_slowdown": parts[5], "hw_thermal_slowdown": parts[6],
                                 "sw_thermal_slowdown": parts[7], "sw_power_cap": parts[8]})
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r["power"] > 250.0] or rows
        reasons = sorted({k for r in loaded for k in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                                          "sw_power_cap") if r[k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r["power"] for r in rows)}


# ---------------------------------------------------------------- CPU oracle baseline


def cpu_oracle_sample(w, target_s, max_heads=None):
    """Time the fp64 oracle (as it stands) on whole heads of w until ~target_s seconds have passed.

    Returns (effective TFLOP/s, seconds, heads, threads)."""
    import torch

    import oracle
    from sparse_linear_attention_sla_b200.workloads import make_inputs

    try:
        import threadpoolctl

        threads = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()) or 1
    except Exception:  # noqa: BLE001 - thread count is informational
        threads = os.cpu_count() or 1
    q, k, v, alpha = make_inputs(w, device="cpu")
    per_head = 4.0 * float(w.N) ** 2 * w.D
    done, spent = 0, 0.0
    limit = max_heads or w.B * w.H
    for bh in range(limit):
        b, h = divmod(bh, w.H)
        t0 = time.perf_counter()
        oracle.forward(q[b, h][None, None], k[b, h][None, None], v[b, h][None, None], alpha[h][None],
                       w.block_q, w.block_kv, w.kh, w.kl)
        spent += time.perf_counter() - t0
        done += 1
        if spent >= target_s:
            break
    del torch
    return per_head * done / spent / 1e12, spent, done, threads


# ---------------------------------------------------------------- the other configurations


def config_table_workloads():
    """The workloads measured beside the headline one: the 1D-field and Wan2.1-14B 720p
    shapes, every point of the kh sweep on the Wan2.1-1.3B grid (kh = 100% is the dense
    reference) and the sweep's ragged N = 32700 case."""
    from sparse_linear_attention_sla_b200.workloads import SWEEP_KH, WORKLOADS, sweep_workload

    ws = [WORKLOADS["field1d_b1h12_n8192_d128"], WORKLOADS["wan14b720p_b2h40_n75600_d128"]]
    # the ragged case is timed next to its full-length counterpart (kh = 5%), before the
    # heavier sweep points, so that both run under the same clocks
    ws += [sweep_workload(kh) for kh in SWEEP_KH if kh <= 0.05]
    ws.append(sweep_workload(0.05, N=32700))
    ws += [sweep_workload(kh) for kh in SWEEP_KH if kh > 0.05]
    return ws


def measure_config(w, dev, flush, stream, steps, warmup, peaks):
    """ms per sla_forward call (L2 flushed before each, CUDA events on the launching stream),
    per-stage times, the whole-path roofline fraction and the attention kernel's fraction."""
    import torch

    from sparse_linear_attention_sla_b200 import binding
    from sparse_linear_attention_sla_b200.workloads import make_inputs

    q, k, v, alpha = make_inputs(w, device=dev)
    p = binding.problem(w.B, w.H, w.N, w.D, w.block_q, w.block_kv, w.kh, w.kl)
    ws = binding.new_workspace(p, dev)
    out = torch.empty_like(q)
    times, stages = [], []
    for it in range(warmup + steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        binding.forward(q, k, v, alpha, w.block_q, w.block_kv, w.kh, w.kl, out=out, ws=ws)
        e1.record(stream)
        e1.synchronize()
        if it >= warmup:
            times.append(e0.elapsed_time(e1))
    for _ in range(steps):
        flush.zero_()
        _, st = binding.forward_timed(q, k, v, alpha, w.block_q, w.block_kv, w.kh, w.kl, out=out, ws=ws)
        stages.append(st)
    binding.check(ws)
    mask, _, _ = binding.route(q, k, w.block_q, w.block_kv, w.kh, w.kl)
    work = algorithmic_work(w, mask)
    del mask, q, k, v, out, ws
    ms = statistics.median(times)
    st = [statistics.median(x[i] for x in stages) for i in range(4)]
    t_roof = max(work["flops"] / (peaks["bf16_tflops"] * 1e12), work["bytes"] / (peaks["hbm_gbs"] * 1e9))
    attn_tf = work["f_attn_kernel"] / (st[3] * 1e-3) / 1e12
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "kh": w.kh, "kl": w.kl,
            "ms_per_call": round(ms, 4), "ms_p10_p90": [round(float(x), 4) for x in
                                                       (sorted(times)[len(times) // 10], sorted(times)[-1 - len(times) // 10])],
            "effective_tflops": round(dense_equivalent_flops(w) / (ms * 1e-3) / 1e12, 2),
            "executed_tflops": round(work["flops"] / (ms * 1e-3) / 1e12, 2),
            "stage_ms": {"precompute": round(st[0], 4), "route": round(st[1], 4), "aggregate": round(st[2], 4),
                         "attention": round(st[3], 4)},
            "path_roofline": {"t_roof_us": round(t_roof * 1e6, 2), "frac": round(t_roof / (ms * 1e-3), 4),
                              "bound": "tensor" if work["flops"] / (peaks["bf16_tflops"] * 1e12) >=
                              work["bytes"] / (peaks["hbm_gbs"] * 1e9) else "hbm"},
            "attn_kernel": {"achieved_tflops": round(attn_tf, 2), "frac": round(attn_tf / peaks["bf16_tflops"], 4)},
            "timed_calls": steps}


# ---------------------------------------------------------------- our arm


def run_ours(args):
    import torch
    import torch.distributed as dist

    from sparse_linear_attention_sla_b200 import binding
    from sparse_linear_attention_sla_b200.workloads import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def rank_max(x):
        return max_over_ranks(x, dist if world > 1 else None, dev)

    w = WORKLOADS[args.workload]
    q, k, v, alpha = make_inputs(w, device=dev)
    p = binding.problem(w.B, w.H, w.N, w.D, w.block_q, w.block_kv, w.kh, w.kl)
    ws = binding.new_workspace(p, dev)
    out = torch.empty_like(q)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        # one sla_forward call, L2 flushed first (untimed), timed with events on the launching stream
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        binding.forward(q, k, v, alpha, w.block_q, w.block_kv, w.kh, w.kl, out=out, ws=ws)
        e1.record(stream)
        return e0, e1

    def step_staged():
        # the same call through sla_forward_timed: per-stage device times (events between stages)
        flush.zero_()
        _, stages = binding.forward_timed(q, k, v, alpha, w.block_q, w.block_kv, w.kh, w.kl, out=out, ws=ws)
        return stages

    for _ in range(args.warmup):
        step()
        step_staged()
    torch.cuda.synchronize(dev)
    binding.check(ws)

    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        wall0 = time.perf_counter()
        events = [step() for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - wall0
        stage_sum = [0.0] * 4
        for _ in range(args.steps):
            stage_sum = [a + b for a, b in zip(stage_sum, step_staged())]
        torch.cuda.synchronize(dev)
    barrier()
    binding.check(ws)
    clock_info = clocks.summary()

    ms_local = sum(e0.elapsed_time(e1) for e0, e1 in events) / len(events)
    ms_step = rank_max(ms_local)
    stage_ms = [s / args.steps for s in stage_sum]
    attn_ms = rank_max(stage_ms[3])

    # labels actually used, for the work accounting
    mask, _, _ = binding.route(q, k, w.block_q, w.block_kv, w.kh, w.kl)
    work = algorithmic_work(w, mask)
    del mask
    peaks = measured_peaks()
    eff_flops = dense_equivalent_flops(w)
    value = whole_job_tflops(world, eff_flops, ms_step)

    # dominant kernel: the fused attention (stage 3)
    achieved = work["f_attn_kernel"] / (attn_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": f"attn_kernel<{w.D}>", "achieved": round(achieved, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json)" if peaks["source"] == "measured"
                else "fallback 1590 TFLOP/s", "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                "kernel_ms": round(attn_ms, 4), "kernel_flops_per_launch": work["f_attn_kernel"],
                "traffic": recorded_traffic(w.name)}
    t_roof = max(work["flops"] / (peaks["bf16_tflops"] * 1e12), work["bytes"] / (peaks["hbm_gbs"] * 1e9))
    path_roofline = {"t_roof_us": round(t_roof * 1e6, 2), "t_us": round(ms_step * 1e3, 2),
                     "frac": round(t_roof / (ms_step * 1e-3), 4), "flops_alg": work["flops"],
                     "bytes_alg": work["bytes"], "executed_tflops": round(work["flops"] / (ms_step * 1e-3) / 1e12, 2)}

    # End to end through the public call with host buffers (copies inside the timed region).
    # The heads are split into groups; the host-to-device copy of group g+1, the forward of
    # group g and the device-to-host copy of group g-1 run on three streams and overlap
    # (PCIe is full duplex). Each group is one sla_forward call on a contiguous head range. Only
    # the last group's forward and copy out are exposed, so the last group is a single head
    # and the others take about a third of the heads each (measured at B=1 H=12: groups of
    # 4, 4, 3, 1 heads 6.16 ms; 3, 3, 3, 3 6.52 ms; twelve of 1 6.60 ms).
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ha = alpha.cpu().pin_memory()
        hout = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        dq, dk, dv, da = (torch.empty_like(t) for t in (q, k, v, alpha))
        h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        # groups of (batch, head range); every group is contiguous in the [B, H, N, D] layout
        per = max(1, (w.H - 1) // 3 + ((w.H - 1) % 3 > 0))
        groups = [(b, h0, min(w.H - 1, h0 + per)) for b in range(w.B) for h0 in range(0, w.H - 1, per)]
        groups = [g for g in groups if g[2] > g[1]]
        groups += [(b, w.H - 1, w.H) for b in range(w.B)]
        groups.sort()

        def e2e_step():
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            h2d_stream.wait_event(e0)
            d2h_stream.wait_event(e0)
            with torch.cuda.stream(h2d_stream):
                da.copy_(ha, non_blocking=True)
            done_in, done_fwd = [], []
            for (b, h0, h1) in groups:
                with torch.cuda.stream(h2d_stream):
                    for dst, src in ((dq, hq), (dk, hk), (dv, hv)):
                        dst[b, h0:h1].copy_(src[b, h0:h1], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(h2d_stream)
                    done_in.append(ev)
            for gi, (b, h0, h1) in enumerate(groups):
                stream.wait_event(done_in[gi])
                binding.forward(dq[b:b + 1, h0:h1], dk[b:b + 1, h0:h1], dv[b:b + 1, h0:h1], da[h0:h1],
                                w.block_q, w.block_kv, w.kh, w.kl, out=out[b:b + 1, h0:h1], ws=ws)
                ev = torch.cuda.Event()
                ev.record(stream)
                done_fwd.append(ev)
                d2h_stream.wait_event(ev)
                with torch.cuda.stream(d2h_stream):
                    hout[b, h0:h1].copy_(out[b, h0:h1], non_blocking=True)
            stream.wait_stream(d2h_stream)
            e1.record(stream)
            e1.synchronize()
            return e0.elapsed_time(e1)

        for _ in range(args.warmup):
            e2e_step()
        barrier()
        ms_e2e = rank_max(sum(e2e_step() for _ in range(args.steps)) / args.steps)
        barrier()
        torch.cuda.synchronize(dev)
        assert torch.equal(hout, out.cpu()), "e2e output differs from the device-resident forward"
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, ha))
        e2e = {"value": round(whole_job_tflops(world, eff_flops, ms_e2e), 3), "unit": UNIT,
               "ms_per_step": round(ms_e2e, 4), "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": hout.numel() * hout.element_size(),
               "pipeline": f"{len(groups)} head groups of {[g[2] - g[1] for g in groups]} heads; H2D, sla_forward "
                           "and D2H on three overlapping streams"}
        del hq, hk, hv, ha, hout, dq, dk, dv, da
        binding.check(ws)

    # the same kernel at kh = 100%: dense-attention reference on the same inputs
    dense = None
    if not args.no_dense:
        wd = w.with_(kh=1.0, kl=0.0)
        pd = binding.problem(w.B, w.H, w.N, w.D, w.block_q, w.block_kv, 1.0, 0.0)
        wsd = binding.new_workspace(pd, dev)
        times, attn_d = [], []
        for it in range(3 + 5):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            _, st_d = binding.forward_timed(q, k, v, alpha, w.block_q, w.block_kv, 1.0, 0.0, out=out, ws=wsd)
            e1.record(stream)
            e1.synchronize()
            if it >= 3:
                times.append(e0.elapsed_time(e1))
                attn_d.append(st_d[3])
        binding.check(wsd)
        ms_d = rank_max(sum(times) / len(times))
        dense = {"workload": wd.name + "_kh1", "ms_per_call": round(ms_d, 4),
                 "effective_tflops": round(eff_flops / (ms_d * 1e-3) / 1e12, 2),
                 "attn_kernel_ms": round(sum(attn_d) / len(attn_d), 4),
                 "speedup_of_sparse_over_dense": round(ms_d / ms_step, 3)}
        del wsd

    # the low-bit sparse branch (SLA2 §2.C) on the same inputs: sla_forward_fp8, L2 flushed,
    # events on the launching stream; the attention kernel against the e4m3 tensor peak
    # (twice the measured bf16 peak, the nominal dense fp8 : bf16 ratio)
    low = None
    if not args.no_fp8 and w.D == 128:
        wsf = binding.new_workspace(p, dev, fp8=True)
        times, stages_f = [], []
        n_f = min(args.steps, 20)
        for it in range(3 + n_f):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            binding.forward_fp8(q, k, v, alpha, w.block_q, w.block_kv, w.kh, w.kl, out=out, ws=wsf)
            e1.record(stream)
            e1.synchronize()
            if it >= 3:
                times.append(e0.elapsed_time(e1))
        for it in range(n_f):
            flush.zero_()
            _, st_f = binding.forward_fp8_timed(q, k, v, alpha, w.block_q, w.block_kv, w.kh, w.kl, out=out, ws=wsf)
            stages_f.append(st_f)
        binding.check(wsf)
        ms_f = rank_max(sum(times) / len(times))
        st_f = [sum(x[i] for x in stages_f) / len(stages_f) for i in range(5)]
        attn_f = rank_max(st_f[4])
        fp8_peak = 2.0 * peaks["bf16_tflops"]
        ach_f = work["f_attn_kernel"] / (attn_f * 1e-3) / 1e12
        low = {"call": "sla_forward_fp8", "ms_per_call": round(ms_f, 4),
               "effective_tflops": round(eff_flops / (ms_f * 1e-3) / 1e12, 2),
               "speedup_over_bf16": round(ms_step / ms_f, 3),
               "stage_ms": {"precompute": round(st_f[0], 4), "route": round(st_f[1], 4),
                            "aggregate": round(st_f[2], 4), "quantise_kv": round(st_f[3], 4),
                            "attention": round(st_f[4], 4)},
               "roofline": {"bound": "tensor", "kernel": "attn_fp8_kernel", "achieved": round(ach_f, 2),
                            "peak": round(fp8_peak, 1), "unit": "TFLOP/s", "frac": round(ach_f / fp8_peak, 4),
                            "peak_source": "2 x measured bf16 burst (nominal e4m3 : bf16 dense ratio)",
                            "kernel_ms": round(attn_f, 4),
                            "traffic": recorded_traffic(w.name, "attn_fp8_kernel")},
               "timed_calls": n_f}
        del wsf

    # the backward (dQ, dK, dV, dalpha with the forward's labels held fixed), same timing rules
    bwd = None
    if not args.no_bwd and w.D == 128 and w.block_q == 128:
        mask_b = binding.route(q, k, w.block_q, w.block_kv, w.kh, w.kl)[0]
        g = torch.Generator(device=dev).manual_seed(1234)
        dO = torch.randn(q.shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
        wsb, times = None, []
        n_b = min(args.steps, 10)
        for it in range(3 + n_b):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            _, _, _, _, wsb = binding.backward(q, k, v, alpha, dO, w.block_q, w.block_kv, w.kh, w.kl, mask=mask_b,
                                               ws=wsb)
            e1.record(stream)
            e1.synchronize()
            if it >= 3:
                times.append(e0.elapsed_time(e1))
        binding.check(wsb)
        ms_b = rank_max(sum(times) / len(times))
        f_b = work["f_bwd"]
        ach_b = f_b / (ms_b * 1e-3) / 1e12
        bwd = {"call": "sla_backward", "ms_per_call": round(ms_b, 4), "algorithmic_tflop": round(f_b / 1e12, 4),
               "achieved_tflops": round(ach_b, 2), "frac_of_bf16_peak": round(ach_b / peaks["bf16_tflops"], 4),
               "peak_source": "measured bf16 burst", "labels": "the router's, held fixed", "dO": "seeded normal",
               "timed_calls": n_b, "ratio_to_forward": round(ms_b / ms_step, 3)}
        del wsb, dO

    # the PISA variant with the router's critical sets, same timing rules
    pisa = None
    if not args.no_pisa:
        wsp = binding.new_workspace_pisa(p, dev)
        times = []
        n_p = min(args.steps, 20)
        for it in range(3 + n_p):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            binding.forward_pisa(q, k, v, w.block_q, w.block_kv, w.kh, w.kl, out=out, ws=wsp)
            e1.record(stream)
            e1.synchronize()
            if it >= 3:
                times.append(e0.elapsed_time(e1))
        binding.check(wsp)
        ms_p = rank_max(sum(times) / len(times))
        ach_p = work["f_pisa"] / (ms_p * 1e-3) / 1e12
        pisa = {"call": "sla_forward_pisa", "ms_per_call": round(ms_p, 4),
                "algorithmic_tflop": round(work["f_pisa"] / 1e12, 4), "achieved_tflops": round(ach_p, 2),
                "frac_of_bf16_peak": round(ach_p / peaks["bf16_tflops"], 4), "labels": "the router's",
                "timed_calls": n_p, "ratio_to_sla_forward": round(ms_p / ms_step, 3)}
        del wsp

    # the SPLA / SALAD variants of the forward on the same inputs, same timing rules
    variants = None
    if not args.no_variants:
        variants = {}
        for name, kw in (("exp_feature_map", {"feature_map": 1}), ("second_order_router", {"block_score": 1}),
                         ("linear_branch_dropped", {"linear_scale": 0.0, "drop_threshold": 0.5})):
            times = []
            n_v = min(args.steps, 20)
            for it in range(3 + n_v):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                binding.forward_variant(q, k, v, alpha, w.block_q, w.block_kv, w.kh, w.kl, out=out, ws=ws, **kw)
                e1.record(stream)
                e1.synchronize()
                if it >= 3:
                    times.append(e0.elapsed_time(e1))
            binding.check(ws)
            ms_v = rank_max(sum(times) / len(times))
            variants[name] = {"call": "sla_forward_variant", "args": kw, "ms_per_call": round(ms_v, 4),
                              "effective_tflops": round(eff_flops / (ms_v * 1e-3) / 1e12, 2),
                              "ratio_to_sla_forward": round(ms_v / ms_step, 3), "timed_calls": n_v}

    # the other configurations: one table, same timing rules (c3 stays the headline value)
    configs = None
    if not args.no_configs:
        configs = [measure_config(wc, dev, flush, stream, args.config_steps, 3, peaks)
                   for wc in config_table_workloads()]
        torch.cuda.empty_cache()

    cpu = None
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        tf, spent, heads, threads = cpu_oracle_sample(w, args.cpu_seconds)
        cpu = {"value": round(tf, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
               "cores_meaning": "threads of numpy's BLAS pool, which runs the oracle's matrix products; "
                                "its Python loops over blocks run on one of them",
               "sample": f"fp64 oracle on {heads} of {w.B * w.H} heads of {w.name} (all {math.ceil(w.N / w.block_q)} "
                         f"query blocks each: router, states, both branches), {spent:.1f} s"}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "block_q": w.block_q,
                   "block_kv": w.block_kv, "kh": w.kh, "kl": w.kl, "inputs": w.kind,
                   "l2": "flushed before every call (512 MiB write, untimed)",
                   "parallelism": "one replica per GPU" if world > 1 else "single GPU"},
        "stage_ms": {"precompute": round(stage_ms[0], 4), "route": round(stage_ms[1], 4),
                     "aggregate": round(stage_ms[2], 4), "attention": round(stage_ms[3], 4),
                     "sum": round(sum(stage_ms), 4),
                     "how": "sla_forward_timed after the timed loop: events between the stages of the same "
                            "launches sla_forward makes"},
        "roofline": roofline, "path_roofline": path_roofline,
        "clocks": clock_info, "e2e": e2e, "gpu_launches": binding.forward_launches(p) * args.steps,
        "dense_reference": dense, "low_bit": low, "backward": bwd, "pisa": pisa, "variants": variants, "configs": configs, "cpu_baseline": cpu,
        "wall_s_timed": round(wall, 3),
    }
    print(json.dumps(line), flush=True)
    return line


# ---------------------------------------------------------------- reference arm (the oracle)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    import torch

    import oracle
    from sparse_linear_attention_sla_b200.workloads import WORKLOADS, make_inputs

    try:
        import threadpoolctl

        threads = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()) or 1
    except Exception:  # noqa: BLE001
        threads = os.cpu_count() or 1
    w = WORKLOADS[args.workload]
    q, k, v, alpha = make_inputs(w, device="cpu")
    per_head = 4.0 * float(w.N) ** 2 * w.D

    def one(step):
        bh = step % (w.B * w.H)
        b, h = divmod(bh, w.H)
        t0 = time.perf_counter()
        oracle.forward(q[b, h][None, None], k[b, h][None, None], v[b, h][None, None], alpha[h][None],
                       w.block_q, w.block_kv, w.kh, w.kl)
        return time.perf_counter() - t0

    for s in range(args.warmup):
        one(s)
    times = [one(args.warmup + s) for s in range(args.steps)]
    sec = sum(times) / len(times)
    value = per_head / sec / 1e12
    del torch
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "block_q": w.block_q,
                   "block_kv": w.block_kv, "kh": w.kh, "kl": w.kl, "inputs": w.kind,
                   "step": "one head, all query blocks"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "cores_meaning": "threads of numpy's BLAS pool, which runs the oracle's matrix products; "
                                          "its Python loops over blocks run on one of them",
                         "sample": f"one of {w.B * w.H} heads of {w.name} per step (router, states, both branches)"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return line


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
