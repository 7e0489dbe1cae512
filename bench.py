"""Benchmark of the block-sparse prefill hot path (plan + prefill) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole path over one attention layer of synthetic
input: stage 1 (pooling, scoring, thresholding, CSR) and stage 2 (sparse
attention with mean correction).  The default workload is the 128K-token
Qwen3-4B-shaped layer (32 query / 8 kv heads, head dim 128, block 128,
tau 0.05, low-rank + needle generator).

Prints one JSON line.  `value` is dense-equivalent TFLOP/s of the whole layer
(2*d*Hq*sum L(L+1) per step, divided by the max over ranks of the device
time), inputs resident in HBM.  On N GPUs the layer is split by kv-head: rank
r runs its contiguous share of the kv-heads (and their query heads) in place
in the full-layer tensors (strong scaling, no collective on the data path);
torch.distributed only provides the barrier and the max over ranks.

The line also carries the FP8-e4m3 leg (plan + online quantisation + e4m3
prefill on the same layer) and the dense baseline (the same kernels with
tau = 0), each timed the same way.

--impl reference runs the float64 CPU oracle on a bounded sample of the same
workload (rank 0 only) and prints the same metric for it.
--sweep prints one line per cell of the L x tau sweep (BF16 and FP8) instead.
--correction-curve prints the mean-correction overhead and error vs tau at 64K.
--density prints attention time against density on the 128K topics layers.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_long_fp2_b200 import synth  # noqa: E402

METRIC = "ms/layer & dense-equiv TFLOPS at 128K prefill; tensor-pipe % of B200 peak"
UNIT = "dense-equiv TFLOP/s"


def dense_equiv_flop(wl) -> float:
    """Causal attention FLOP of the dense layer: 2 * d * Hq * sum L (L + 1)."""
    return float(sum(2.0 * wl.d * wl.Hq * L * (L + 1) for L in wl.seqlens))


def kept_tile_flop(wl) -> float:
    """Tensor-core FLOP of one kept (row, key block) pair: QK^T + PV for the
    G heads x B tokens of the row = 4 * d * G * B^2."""
    G = wl.Hq // wl.Hkv
    return 4.0 * wl.d * G * wl.B * wl.B


def plan_launches(wl, tau=None) -> int:
    """Kernels fp2_plan launches: pool, meta, threshold (which also takes the
    e4m3 means' chunk maxima) and CSR (which also writes their codes); with
    tau > 0 the scorer, and the separate norms kernel when the G query heads of
    a kv-head do not fall into one pooling CTA (1024 columns)."""
    tau = wl.tau if tau is None else tau
    G = wl.Hq // wl.Hkv
    return 4 + (1 if tau > 0 else 0) + (1 if tau > 0 and 1024 % (G * wl.d) != 0 else 0)


def rank_slice(wl, world: int, rank: int):
    """The kv-heads a rank runs: the layer split over the ranks by kv-head
    (each kv-head with its G query heads is planned and attended on its own,
    so the ranks exchange nothing on the data path).  Returns (first kv-head,
    kv-heads)."""
    from block_sparse_long_fp2_b200.binding import kv_head_slice
    return kv_head_slice(wl.Hkv, world, rank)


def max_over_ranks(values, world: int, device):
    """Element-wise maximum of per-rank values (device times) over all ranks."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_value(flop: float, ms: float) -> float:
    """Throughput of the whole job: the layer's work (all ranks' slices
    together) over the slowest rank's time."""
    return flop / (ms * 1e-3) / 1e12


def attn_traffic(workload: str, dtype: str):
    """DRAM bytes per launch of the attention kernel on this workload, from the
    committed single-pass ncu capture (profiles/k_attn_traffic.json), or None
    when the kernel source changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "k_attn_traffic.json")) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, "block_sparse_long_fp2_b200", "csrc", "fp2_attn.cu")
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
        if rec.get("source_sha256") != digest or rec.get("workload") != workload:
            return None
        return rec.get(dtype)
    except Exception:
        return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16": p["bf16_tflops"],
                "bf16_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.f = None

    def __enter__(self):
        try:
            self.f = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.f is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.f.seek(0)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from block_sparse_long_fp2_b200 import binding as fb
    from block_sparse_long_fp2_b200 import build as fbuild

    fbuild.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = synth.workloads()[args.workload]
    x = synth.generate(wl)
    h0, hn = rank_slice(wl, world, rank)   # this rank's kv-heads of the layer
    G = wl.Hq // wl.Hkv
    slice_kw = {"kv_head_begin": h0, "num_kv_heads_total": wl.Hkv}
    stream = torch.cuda.current_stream()

    def dev_bf16(a):
        return torch.from_numpy(a).to(torch.bfloat16).to(dev)

    q = dev_bf16(x["q"])
    if wl.page_size:
        k, v = dev_bf16(x["k_pool"]), dev_bf16(x["v_pool"])
        pt = torch.from_numpy(x["page_table"]).to(dev)
    else:
        k, v = dev_bf16(x["k"]), dev_bf16(x["v"])
        pt = None
    cu = torch.from_numpy(x["cu_seqlens"]).to(dev)
    prob = fb.Problem(wl.seqlens, cu, G * hn, hn, wl.d, wl.B, wl.tau,
                      page_size=wl.page_size, page_table=pt,
                      num_pages=int(x["k_pool"].shape[0]) if wl.page_size else 0, **slice_kw)
    lay, plan, ws = fb.allocate(prob, dev)
    o = torch.empty((wl.T, wl.Hq, wl.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.Hq, wl.T), dtype=torch.float32, device=dev)
    in_bytes = (q.numel() + k.numel() + v.numel()) * 2          # the layer's Q, K, V
    slice_bytes = in_bytes * hn // wl.Hkv                          # this rank's heads of them

    def step():
        fb.fp2_plan(prob, q, k, v, plan, ws, stream)
        fb.fp2_prefill(prob, plan, q, k, v, o, lse, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rc, st = fb.fp2_status_check(plan, stream)
    if rc != 0:
        raise RuntimeError(f"device status {st:#x} ({fb.strerror(rc)})")
    nnz = int(fb.PlanView(plan, lay, hn, wl.d).row_ptr[-1].item())

    # timed region: K steps, per-stage events on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                      int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])) as clk:
        t0.record(stream)
        for s in range(args.steps):
            ev[s][0].record(stream)
            fb.fp2_plan(prob, q, k, v, plan, ws, stream)
            ev[s][1].record(stream)
            fb.fp2_prefill(prob, plan, q, k, v, o, lse, stream=stream)
            ev[s][2].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = t0.elapsed_time(t1)
    plan_ms = [e[0].elapsed_time(e[1]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    # plan: pool, meta, [norms, score], threshold, csr; prefill: attn
    # (+ the split merge when the schedule splits rows)
    launches_per_step = plan_launches(wl) + 1 + (1 if lay.num_split_slots > 0 else 0)

    # dense baseline: the same kernels on the same inputs with tau = 0 (every
    # causally visible block kept, no pseudo tiles)
    dense = None
    if not args.no_dense and wl.tau > 0:
        prob0 = fb.Problem(wl.seqlens, cu, G * hn, hn, wl.d, wl.B, 0.0,
                           page_size=wl.page_size, page_table=pt,
                           num_pages=int(x["k_pool"].shape[0]) if wl.page_size else 0, **slice_kw)
        lay0, plan0, ws0 = fb.allocate(prob0, dev)

        def step0(evs=None):
            if evs is not None:
                evs[0].record(stream)
            fb.fp2_plan(prob0, q, k, v, plan0, ws0, stream)
            if evs is not None:
                evs[1].record(stream)
            fb.fp2_prefill(prob0, plan0, q, k, v, o, lse, stream=stream)
            if evs is not None:
                evs[2].record(stream)

        for _ in range(args.warmup):
            step0()
        torch.cuda.synchronize()
        rc, st = fb.fp2_status_check(plan0, stream)
        if rc != 0:
            raise RuntimeError(f"device status {st:#x} ({fb.strerror(rc)})")
        nnz0 = int(fb.PlanView(plan0, lay0, hn, wl.d).row_ptr[-1].item())
        ev0 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        d0 = torch.cuda.Event(enable_timing=True)
        d1 = torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for s_ in range(args.steps):
            step0(ev0[s_])
        d1.record(stream)
        torch.cuda.synchronize()
        ms0 = max_over_ranks([d0.elapsed_time(d1)], world, dev)[0] / args.steps
        attn0 = statistics.mean(e[1].elapsed_time(e[2]) for e in ev0)
        plan0_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev0)
        ach0 = nnz0 * kept_tile_flop(wl) / (attn0 * 1e-3) / 1e12
        dense = {"tau": 0.0, "ms_per_layer": round(ms0, 4), "ms_plan": round(plan0_ms, 4),
                 "ms_attention": round(attn0, 4), "nnz": nnz0,
                 "value": round(whole_job_value(dense_equiv_flop(wl), ms0), 2),
                 "unit": UNIT,
                 "roofline": {"bound": "tensor", "achieved": round(ach0, 1),
                              "peak": peaks()["bf16_sustained"], "unit": "TFLOP/s",
                              "frac": round(ach0 / peaks()["bf16_sustained"], 4)},
                 "gpu_launches": (plan_launches(wl, 0.0) + 1
                                  + (1 if lay0.num_split_slots > 0 else 0)) * args.steps}
        del plan0, ws0

    # FP8-e4m3 leg: plan (bf16) + direct online quantisation of Q, K, V + e4m3 prefill
    fp8 = None
    if not args.no_fp8 and wl.d == 128:
        NB = int(lay.num_blocks)
        q8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
        k8 = torch.empty(k.shape, dtype=torch.uint8, device=dev)
        v8 = torch.empty(v.shape, dtype=torch.uint8, device=dev)
        qs = torch.empty((NB, G * hn), dtype=torch.float32, device=dev)
        ks = torch.empty((NB, hn), dtype=torch.float32, device=dev)
        vs = torch.empty((NB, hn), dtype=torch.float32, device=dev)

        def step8(evs=None):
            if evs is not None:
                evs[0].record(stream)
            fb.fp2_plan(prob, q, k, v, plan, ws, stream)
            fb.fp2_quantize_fp8_qkv(prob, plan, q, k, v, q8, k8, v8, qs, ks, vs, stream)
            if evs is not None:
                evs[1].record(stream)
            fb.fp2_prefill(prob, plan, q8, k8, v8, o, lse, q_scale=qs, k_scale=ks, v_scale=vs,
                           dtype=fb.FP2_DTYPE_E4M3, stream=stream)
            if evs is not None:
                evs[2].record(stream)

        for _ in range(args.warmup):
            step8()
        torch.cuda.synchronize()
        rc, st = fb.fp2_status_check(plan, stream)
        if rc != 0:
            raise RuntimeError(f"device status {st:#x} ({fb.strerror(rc)})")
        ev8 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for s_ in range(args.steps):
            step8(ev8[s_])
        f1.record(stream)
        torch.cuda.synchronize()
        ms8 = max_over_ranks([f0.elapsed_time(f1)], world, dev)[0] / args.steps
        attn8 = statistics.mean(e[1].elapsed_time(e[2]) for e in ev8)
        pre8 = statistics.mean(e[0].elapsed_time(e[1]) for e in ev8)
        ach8 = nnz * kept_tile_flop(wl) / (attn8 * 1e-3) / 1e12
        fp8 = {"ms_per_layer": round(ms8, 4), "ms_plan_and_quantize": round(pre8, 4),
               "ms_attention": round(attn8, 4),
               "value": round(whole_job_value(dense_equiv_flop(wl), ms8), 2),
               "unit": UNIT, "dtype": "e4m3",
               "roofline": {"bound": "tensor", "achieved": round(ach8, 1),
                            "peak": round(2 * peaks()["bf16_sustained"], 1), "unit": "TFLOP/s",
                            "frac": round(ach8 / (2 * peaks()["bf16_sustained"]), 4),
                            "traffic": attn_traffic(wl.name, "fp8"),
                            "peak_kind": "e4m3 = 2 x measured bf16 sustained (nominal ratio)"},
               "gpu_launches": (launches_per_step + 1 + 1) * args.steps}

    # end to end through the C ABI with host buffers (pinned), copies inside
    qh = torch.from_numpy(x["q"]).to(torch.bfloat16).pin_memory()
    kh = (torch.from_numpy(x["k_pool"] if wl.page_size else x["k"]).to(torch.bfloat16)
          .pin_memory())
    vh = (torch.from_numpy(x["v_pool"] if wl.page_size else x["v"]).to(torch.bfloat16)
          .pin_memory())
    oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    lh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_steps = args.steps
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        q.copy_(qh, non_blocking=True)
        k.copy_(kh, non_blocking=True)
        v.copy_(vh, non_blocking=True)
        step()
        oh.copy_(o, non_blocking=True)
        lh.copy_(lse, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    # max over ranks
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world, dev)
    ms_step = total_ms / args.steps
    flop = dense_equiv_flop(wl)
    value = whole_job_value(flop, ms_step)
    pk = peaks()
    attn_avg = statistics.mean(attn_ms)
    plan_avg = statistics.mean(plan_ms)
    executed = nnz * kept_tile_flop(wl)
    achieved = executed / (attn_avg * 1e-3) / 1e12
    R = int(lay.num_rows)
    density = nnz / float(lay.nnz_cap)
    plan_bytes = slice_bytes + int(lay.num_blocks) * hn * wl.d * (4 + 4 + 2 + 2)
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded low-rank + needles generator; no model weights)",
        "config": {"workload": wl.name, "seqlens": wl.seqlens, "Hq": wl.Hq, "Hkv": wl.Hkv,
                   "head_dim": wl.d, "block": wl.B, "tau": wl.tau, "paged": bool(wl.page_size),
                   "parallelism": f"kv-head split of one layer x{world}",
                   "kv_heads_per_rank": [list(rank_slice(wl, world, r_)) for r_ in range(world)],
                   "l2": "inputs (%.2f GB) larger than L2 (126 MB), no flush" % (in_bytes / 1e9)},
        "ms_per_layer": round(ms_step, 4), "ms_plan": round(plan_avg, 4),
        "ms_attention": round(attn_avg, 4), "density": round(density, 5), "nnz": nnz,
        "dense_equiv_tflop": round(flop / 1e12, 3),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1),
                     "peak": pk["bf16_sustained"], "unit": "TFLOP/s",
                     "frac": round(achieved / pk["bf16_sustained"], 4),
                     "traffic": attn_traffic(wl.name, "bf16"),
                     "traffic_unit": "DRAM bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                     "kernel": "k_attn (sparse attention + correction)",
                     "peak_kind": f"bf16 sustained ({pk['source']})",
                     "frac_of_burst_peak": round(achieved / pk["bf16"], 4)},
        "planning": {"achieved_gbs": round(plan_bytes / (plan_avg * 1e-3) / 1e9, 1),
                     "peak_gbs": pk["hbm_gbs"],
                     "frac": round(plan_bytes / (plan_avg * 1e-3) / 1e9 / pk["hbm_gbs"], 4)},
        "e2e": {"value": round(whole_job_value(flop, e2e_ms), 2), "unit": UNIT,
                "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps,
                "how": "torch copy_ of pinned host Q/K/V into the device tensors, fp2_plan + "
                       "fp2_prefill through the C ABI, copy_ of O and LSE back, per step",
                "h2d_bytes_per_step": int(in_bytes),
                "d2h_bytes_per_step": int(o.numel() * 2 + lse.numel() * 4)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "fp8": fp8,
        "dense": dense,
        "sparse_speedup_vs_dense": (round(dense["ms_per_layer"] / ms_step, 3) if dense else None),
        "rows": R, "G": G,
    }
    return out, x


def oracle_sample(wl, x, budget_s: float = 20.0):
    """Times the oracle on a bounded sample of the workload: block means of
    the whole layer plus scoring and attention of a few query blocks per
    kv-head, reported as dense-equivalent FLOP of the sampled rows / s."""
    import oracle
    t_start = time.perf_counter()
    nb = [(L + wl.B - 1) // wl.B for L in wl.seqlens]
    s_last = int(np.argmax(wl.seqlens))
    rng = np.random.default_rng(0)
    cand = sorted(rng.choice(np.arange(nb[s_last]), size=min(nb[s_last], 64), replace=False),
                  reverse=True)
    q, k, v = x["q"], x.get("k"), x.get("v")
    if wl.page_size:
        k = oracle.gather_paged(x["k_pool"], x["page_table"], wl.seqlens, wl.page_size)
        v = oracle.gather_paged(x["v_pool"], x["page_table"], wl.seqlens, wl.page_size)
    sample = [(s_last, int(i)) for i in cand]
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau, rows=sample)
    rows, flop = [], 0.0
    for (s_, i) in sample:
        oracle.attend_rows(q, k, v, pl, [(s_, i)])
        rows.append((s_, i))
        n_i = min(wl.B, wl.seqlens[s_] - i * wl.B)
        p0 = i * wl.B
        flop += 2.0 * 2.0 * wl.d * wl.Hq * sum(p0 + u + 1 for u in range(n_i))
        if time.perf_counter() - t_start > budget_s:
            break
    el = time.perf_counter() - t_start
    return flop / el / 1e12, el, rows


def run_reference(args, rank, world):
    if rank != 0:
        return None
    os.environ.setdefault("OMP_NUM_THREADS", str(len(os.sched_getaffinity(0))))
    wl = synth.workloads()[args.workload]
    x = synth.generate(wl)
    cores = len(os.sched_getaffinity(0))
    per_step = []
    rows = []
    budget = max(5.0, 120.0 / max(1, args.steps + args.warmup))
    for s in range(args.warmup + args.steps):
        val, el, rows = oracle_sample(wl, x, budget)
        if s >= args.warmup:
            per_step.append((val, el))
    value = statistics.mean(v for v, _ in per_step)
    ms = statistics.mean(e for _, e in per_step) * 1e3
    sample = (f"block means of the full layer + scoring and attention of {len(rows)} "
              f"query blocks (all kv-heads) of the {wl.seqlens[0]}-token layer, float64 NumPy")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "seqlens": wl.seqlens, "Hq": wl.Hq, "Hkv": wl.Hkv,
                       "head_dim": wl.d, "block": wl.B, "tau": wl.tau},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_correction_curve(args):
    """Mean-correction overhead and accuracy at 64K (one 32 q / 8 kv-head, d 128,
    B 128 layer; N(0,1) and low-rank generators): for each tau, attention time
    with and without the correction (BF16 and FP8-e4m3) and the rel-L2 distance
    of O to the dense (tau = 0) output of the same kernels, with and without it.
    One JSON line per (generator, tau) on stdout (not the benchmark line)."""
    import torch
    from block_sparse_long_fp2_b200 import binding as fb
    from block_sparse_long_fp2_b200 import build as fbuild

    fbuild.build()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    L, taus = 65536, [0.05, 0.1, 0.2, 0.4]
    for gen in ("normal", "lowrank"):
        wl = synth.small_workload([L], 32, 8, 128, 128, 0.0, seed=2024, generator=gen)
        x = synth.generate(wl)
        q = torch.from_numpy(x["q"]).to(torch.bfloat16).to(dev)
        k = torch.from_numpy(x["k"]).to(torch.bfloat16).to(dev)
        v = torch.from_numpy(x["v"]).to(torch.bfloat16).to(dev)
        cu = torch.from_numpy(x["cu_seqlens"]).to(dev)
        o = torch.empty((wl.T, wl.Hq, wl.d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((wl.Hq, wl.T), dtype=torch.float32, device=dev)

        def plan_for(tau):
            prob = fb.Problem(wl.seqlens, cu, wl.Hq, wl.Hkv, wl.d, wl.B, tau)
            lay, plan, ws = fb.allocate(prob, dev)
            fb.fp2_plan(prob, q, k, v, plan, ws, stream)
            return prob, lay, plan

        def quantised(prob, plan, NB):
            out = []
            for which, src, H in ((0, q, wl.Hq), (1, k, wl.Hkv), (2, v, wl.Hkv)):
                c = torch.empty(src.shape, dtype=torch.uint8, device=dev)
                sc = torch.empty((NB, H), dtype=torch.float32, device=dev)
                fb.fp2_quantize_fp8(prob, plan, src, which, c, sc, stream)
                out.append((c, sc))
            return out

        def timed(fn):
            for _ in range(args.warmup):
                fn()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / args.steps

        prob0, lay0, plan0 = plan_for(0.0)
        q80 = quantised(prob0, plan0, int(lay0.num_blocks))
        fb.fp2_prefill(prob0, plan0, q, k, v, o, lse, stream=stream)
        dense16 = o.float().clone()
        fb.fp2_prefill(prob0, plan0, q80[0][0], q80[1][0], q80[2][0], o, lse, q_scale=q80[0][1],
                       k_scale=q80[1][1], v_scale=q80[2][1], dtype=fb.FP2_DTYPE_E4M3, stream=stream)
        dense8 = o.float().clone()
        del plan0
        for tau in taus:
            prob, lay, plan = plan_for(tau)
            q8 = quantised(prob, plan, int(lay.num_blocks))
            nnz = int(fb.PlanView(plan, lay, wl.Hkv, wl.d).row_ptr[-1].item())
            row = {"generator": gen, "L": L, "tau": tau, "density": round(nnz / float(lay.nnz_cap), 4)}
            for tag, dense in (("bf16", dense16), ("fp8", dense8)):
                for corr in (True, False):
                    flags = 0 if corr else fb.FP2_NO_CORRECTION
                    if tag == "bf16":
                        def fn():
                            fb.fp2_prefill(prob, plan, q, k, v, o, lse, flags=flags, stream=stream)
                    else:
                        def fn():
                            fb.fp2_prefill(prob, plan, q8[0][0], q8[1][0], q8[2][0], o, lse,
                                           q_scale=q8[0][1], k_scale=q8[1][1], v_scale=q8[2][1],
                                           dtype=fb.FP2_DTYPE_E4M3, flags=flags, stream=stream)
                    ms = timed(fn)
                    rc, st = fb.fp2_status_check(plan, stream)
                    if rc != 0:
                        raise RuntimeError(f"device status {st:#x}")
                    err = float((o.float() - dense).norm() / dense.norm())
                    key = f"{tag}_{'corr' if corr else 'nocorr'}"
                    row[key] = {"ms_attention": round(ms, 4), "rel_l2_to_dense": round(err, 5)}
                row[f"{tag}_correction_overhead"] = round(
                    row[f"{tag}_corr"]["ms_attention"] / row[f"{tag}_nocorr"]["ms_attention"] - 1.0, 4)
            print(json.dumps(row), flush=True)
            del plan, q8
            torch.cuda.empty_cache()


def run_sweep(args):
    """Throughput of every cell of the dense-vs-sparse sweep (32 q / 8 kv heads,
    d 128, block 128, L in 4K..128K, tau in {0, 0.05, 0.2}), BF16 and FP8-e4m3,
    one JSON line per cell on stdout (not the benchmark line)."""
    import torch
    from block_sparse_long_fp2_b200 import binding as fb
    from block_sparse_long_fp2_b200 import build as fbuild

    fbuild.build()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    pk = peaks()
    names = sorted((n for n in synth.workloads() if n.startswith("sweep_")),
                   key=lambda n: (synth.workloads()[n].T, synth.workloads()[n].tau))
    for name in names:
        wl = synth.workloads()[name]
        x = synth.generate(wl)
        q = torch.from_numpy(x["q"]).to(torch.bfloat16).to(dev)
        k = torch.from_numpy(x["k"]).to(torch.bfloat16).to(dev)
        v = torch.from_numpy(x["v"]).to(torch.bfloat16).to(dev)
        cu = torch.from_numpy(x["cu_seqlens"]).to(dev)
        prob = fb.Problem(wl.seqlens, cu, wl.Hq, wl.Hkv, wl.d, wl.B, wl.tau)
        lay, plan, ws = fb.allocate(prob, dev)
        o = torch.empty((wl.T, wl.Hq, wl.d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((wl.Hq, wl.T), dtype=torch.float32, device=dev)
        NB = int(lay.num_blocks)
        q8, k8, v8 = (torch.empty(t.shape, dtype=torch.uint8, device=dev) for t in (q, k, v))
        qs = torch.empty((NB, wl.Hq), dtype=torch.float32, device=dev)
        ks = torch.empty((NB, wl.Hkv), dtype=torch.float32, device=dev)
        vs = torch.empty((NB, wl.Hkv), dtype=torch.float32, device=dev)

        def bf16_step(ev):
            ev[0].record(stream)
            fb.fp2_plan(prob, q, k, v, plan, ws, stream)
            ev[1].record(stream)
            fb.fp2_prefill(prob, plan, q, k, v, o, lse, stream=stream)
            ev[2].record(stream)

        def fp8_step(ev):
            ev[0].record(stream)
            fb.fp2_plan(prob, q, k, v, plan, ws, stream)
            fb.fp2_quantize_fp8_qkv(prob, plan, q, k, v, q8, k8, v8, qs, ks, vs, stream)
            ev[1].record(stream)
            fb.fp2_prefill(prob, plan, q8, k8, v8, o, lse, q_scale=qs, k_scale=ks, v_scale=vs,
                           dtype=fb.FP2_DTYPE_E4M3, stream=stream)
            ev[2].record(stream)

        row = {"workload": name, "L": wl.seqlens[0], "tau": wl.tau}
        for tag, fn in (("bf16", bf16_step), ("fp8", fp8_step)):
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
                   for _ in range(args.warmup + args.steps)]
            for e in evs:
                fn(e)
            torch.cuda.synchronize()
            rc, st = fb.fp2_status_check(plan, stream)
            if rc != 0:
                raise RuntimeError(f"{name}: device status {st:#x}")
            tim = evs[args.warmup:]
            ms = statistics.median(e[0].elapsed_time(e[2]) for e in tim)
            att = statistics.median(e[1].elapsed_time(e[2]) for e in tim)
            nnz = int(fb.PlanView(plan, lay, wl.Hkv, wl.d).row_ptr[-1].item())
            peak = pk["bf16_sustained"] * (2 if tag == "fp8" else 1)
            row[tag] = {"ms_per_layer": round(ms, 4), "ms_attention": round(att, 4),
                        "dense_equiv_tflops": round(dense_equiv_flop(wl) / (ms * 1e-3) / 1e12, 1),
                        "tensor_frac": round(nnz * kept_tile_flop(wl) / (att * 1e-3) / 1e12 / peak,
                                             4)}
            row["density"] = round(nnz / float(lay.nnz_cap), 4)
        print(json.dumps(row), flush=True)
        del q, k, v, o, lse, plan, ws, q8, k8, v8
        torch.cuda.empty_cache()


def pseudo_tiles(kept_mask: np.ndarray, wl) -> int:
    """Pseudo tiles the attention kernel runs: per row (s, g, i), the groups of
    B consecutive blocks below i holding at least one skipped block."""
    B = wl.B
    n, r = 0, 0
    for _g in range(wl.Hkv):
        for L in wl.seqlens:
            nb = (L + B - 1) // B
            for i in range(nb):
                words = kept_mask[r]
                bits = np.unpackbits(words.view(np.uint8), bitorder="little")[:i]
                skipped = np.flatnonzero(bits == 0)
                n += len(np.unique(skipped // B))
                r += 1
    return n


def run_density(args):
    """Attention time against density on the 128K layer shape with block-level
    topics (about 5, 10 and 20 % of the blocks kept; the pages' real prompts
    keep 4.6-9.4 % at 64K-128K, Table 3), BF16: ms, executed-block tensor
    fraction, and the time the dense (tau = 0) run of the same inputs predicts
    when time is proportional to the tiles executed (kept blocks + pseudo
    tiles of the correction) -- Figure 5's "tracks the theoretical bound".
    One JSON line per density on stdout (not the benchmark line)."""
    import torch
    from block_sparse_long_fp2_b200 import binding as fb
    from block_sparse_long_fp2_b200 import build as fbuild

    fbuild.build()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    pk = peaks()
    names = [n for n in synth.workloads() if n.startswith("topics_128k_")]
    for name in names:
        wl = synth.workloads()[name]
        x = synth.generate(wl)
        q = torch.from_numpy(x["q"]).to(torch.bfloat16).to(dev)
        k = torch.from_numpy(x["k"]).to(torch.bfloat16).to(dev)
        v = torch.from_numpy(x["v"]).to(torch.bfloat16).to(dev)
        del x
        cu = torch.tensor(np.concatenate([[0], np.cumsum(wl.seqlens)]).astype(np.int32), device=dev)
        o = torch.empty((wl.T, wl.Hq, wl.d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((wl.Hq, wl.T), dtype=torch.float32, device=dev)
        row = {"workload": name, "L": wl.seqlens[0], "tau": wl.tau}
        for tag, tau in (("sparse", wl.tau), ("dense", 0.0)):
            prob = fb.Problem(wl.seqlens, cu, wl.Hq, wl.Hkv, wl.d, wl.B, tau)
            lay, plan, ws = fb.allocate(prob, dev)
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
                   for _ in range(args.warmup + args.steps)]
            for e in evs:
                e[0].record(stream)
                fb.fp2_plan(prob, q, k, v, plan, ws, stream)
                e[1].record(stream)
                fb.fp2_prefill(prob, plan, q, k, v, o, lse, stream=stream)
                e[2].record(stream)
            torch.cuda.synchronize()
            rc, st = fb.fp2_status_check(plan, stream)
            if rc != 0:
                raise RuntimeError(f"{name}: device status {st:#x}")
            tim = evs[args.warmup:]
            view = fb.PlanView(plan, lay, wl.Hkv, wl.d)
            nnz = int(view.row_ptr[-1].item())
            att = statistics.median(e[1].elapsed_time(e[2]) for e in tim)
            ent = {"ms_per_layer": round(statistics.median(e[0].elapsed_time(e[2]) for e in tim), 4),
                   "ms_plan": round(statistics.median(e[0].elapsed_time(e[1]) for e in tim), 4),
                   "ms_attention": round(att, 4), "nnz": nnz,
                   "density": round(nnz / float(lay.nnz_cap), 4),
                   "tensor_frac": round(nnz * kept_tile_flop(wl) / (att * 1e-3) / 1e12
                                        / pk["bf16_sustained"], 4)}
            if tag == "sparse":
                ent["pseudo_tiles"] = pseudo_tiles(view.kept_mask.cpu().numpy(), wl)
            row[tag] = ent
            del plan, ws
        sp, dn = row["sparse"], row["dense"]
        per_tile = dn["ms_attention"] / dn["nnz"]
        pred = per_tile * (sp["nnz"] + sp["pseudo_tiles"])
        row["predicted_ms_attention"] = round(pred, 4)
        row["actual_over_predicted"] = round(sp["ms_attention"] / pred, 4)
        row["speedup_vs_dense"] = round(dn["ms_per_layer"] / sp["ms_per_layer"], 3)
        print(json.dumps(row), flush=True)
        del q, k, v, o, lse
        torch.cuda.empty_cache()


def chunk_dense_equiv_flop(wl, q_lens) -> float:
    """Causal attention FLOP of the chunk's queries over all earlier keys:
    4 * d * Hq * sum over query positions p of (p + 1)."""
    tot = 0.0
    for L, Q in zip(wl.seqlens, q_lens):
        off = L - Q
        tot += (L * (L + 1) - off * (off + 1)) / 2.0
    return 4.0 * wl.d * wl.Hq * tot


def run_chunked(args):
    """Chunked prefill (Table 6's serving mode): the last C tokens of the 128K
    layer as new queries over all 131072 keys, C in {8K, 16K}; plan + BF16
    attention, one JSON line per chunk size on stdout (not the benchmark line)."""
    import torch
    from block_sparse_long_fp2_b200 import binding as fb
    from block_sparse_long_fp2_b200 import build as fbuild

    fbuild.build()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    pk = peaks()
    wl = synth.workloads()[args.workload]
    x = synth.generate(wl)
    k = torch.from_numpy(x["k"]).to(torch.bfloat16).to(dev)
    v = torch.from_numpy(x["v"]).to(torch.bfloat16).to(dev)
    cu = torch.from_numpy(x["cu_seqlens"]).to(dev)
    for C in (8192, 16384):
        q_lens = [min(C, L) for L in wl.seqlens]
        parts, t0 = [], 0
        for L, Q in zip(wl.seqlens, q_lens):
            parts.append(x["q"][t0 + L - Q:t0 + L])
            t0 += L
        q = torch.from_numpy(np.concatenate(parts, axis=0)).to(torch.bfloat16).to(dev)
        cu_q = torch.from_numpy(np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)).to(dev)
        prob = fb.Problem(wl.seqlens, cu, wl.Hq, wl.Hkv, wl.d, wl.B, wl.tau, q_seqlens=q_lens,
                          cu_q_seqlens=cu_q)
        lay, plan, ws = fb.allocate(prob, dev)
        Tq = sum(q_lens)
        o = torch.empty((Tq, wl.Hq, wl.d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((wl.Hq, Tq), dtype=torch.float32, device=dev)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
               for _ in range(args.warmup + args.steps)]
        for e in evs:
            e[0].record(stream)
            fb.fp2_plan(prob, q, k, v, plan, ws, stream)
            e[1].record(stream)
            fb.fp2_prefill(prob, plan, q, k, v, o, lse, stream=stream)
            e[2].record(stream)
        torch.cuda.synchronize()
        rc, st = fb.fp2_status_check(plan, stream)
        if rc != 0:
            raise RuntimeError(f"chunk {C}: device status {st:#x}")
        tim = evs[args.warmup:]
        ms = statistics.median(e[0].elapsed_time(e[2]) for e in tim)
        plan_ms = statistics.median(e[0].elapsed_time(e[1]) for e in tim)
        att = statistics.median(e[1].elapsed_time(e[2]) for e in tim)
        nnz = int(fb.PlanView(plan, lay, wl.Hkv, wl.d).row_ptr[-1].item())
        vis = sum((L + wl.B - 1) // wl.B * ((L + wl.B - 1) // wl.B + 1) // 2
                  - ((L - Q) // wl.B) * ((L - Q) // wl.B + 1) // 2
                  for L, Q in zip(wl.seqlens, q_lens)) * wl.Hkv
        print(json.dumps({
            "workload": f"{wl.name}_chunk{C // 1024}k", "kv_tokens": wl.T, "q_tokens": Tq,
            "tau": wl.tau, "ms": round(ms, 4), "ms_plan": round(plan_ms, 4),
            "ms_attention": round(att, 4), "density": round(nnz / vis, 4),
            "dense_equiv_tflops": round(chunk_dense_equiv_flop(wl, q_lens) / (ms * 1e-3) / 1e12, 1),
            "tensor_frac": round(nnz * kept_tile_flop(wl) / (att * 1e-3) / 1e12 / pk["bf16_sustained"], 4),
        }), flush=True)
        del q, o, lse, plan, ws
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="qwen_128k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8-e4m3 leg")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense tau = 0 leg")
    ap.add_argument("--sweep", action="store_true",
                    help="one line per L x tau cell of the dense-vs-sparse sweep instead")
    ap.add_argument("--correction-curve", action="store_true",
                    help="mean-correction overhead and error vs tau at 64K instead")
    ap.add_argument("--density", action="store_true",
                    help="attention time against density on the 128K topics layers")
    ap.add_argument("--chunked", action="store_true",
                    help="chunked prefill of the last 8K / 16K tokens of the layer instead")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.sweep:
        run_sweep(args)
        return
    if args.chunked:
        run_chunked(args)
        return
    if args.correction_curve:
        run_correction_curve(args)
        return
    if args.density:
        run_density(args)
        return

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    out, x = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        wl = synth.workloads()[args.workload]
        val, el, rows = oracle_sample(wl, x, 20.0)
        out["cpu_baseline"] = {
            "value": val, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"block means of the whole layer + scoring/attention of {len(rows)} query "
                      f"blocks (all kv-heads), {el:.1f} s"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
