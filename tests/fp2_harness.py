"""Test harness: runs the CUDA path through the C ABI and compares it with
the float64 oracle on the same seeded inputs.

Tolerances (from the problem statement of the method):
  * kept block lists: bit-exact, except blocks whose oracle score lies within
    1e-5 relative of the row threshold (counted and reported);
  * O: rel-L2 = |O - O*|_2 / |O*|_2 <= 1e-2 (BF16);
  * LSE: max |LSE - LSE*| <= 1e-3.
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

import oracle
from block_sparse_long_fp2_b200 import binding as fb
from block_sparse_long_fp2_b200 import synth

REL_L2_BF16 = 1e-2
LSE_ABS = 1e-3
BAND = 1e-5


def to_bf16_device(x: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).cuda()


class GpuRun:
    """Uploads a workload's inputs and runs plan (+ prefill) on the GPU."""

    def __init__(self, wl: synth.Workload, x: Dict[str, object], paged: Optional[bool] = None):
        import torch
        self.wl = wl
        self.x = x
        self.paged = bool(wl.page_size) if paged is None else paged
        self.q = to_bf16_device(x["q"])
        self.cu = torch.from_numpy(np.asarray(x["cu_seqlens"], dtype=np.int32)).cuda()
        if self.paged:
            self.k = to_bf16_device(x["k_pool"])
            self.v = to_bf16_device(x["v_pool"])
            self.pt = torch.from_numpy(np.ascontiguousarray(x["page_table"])).cuda()
            self.prob = fb.Problem(wl.seqlens, self.cu, wl.Hq, wl.Hkv, wl.d, wl.B, wl.tau,
                                   page_size=64, page_table=self.pt,
                                   num_pages=int(x["k_pool"].shape[0]))
        else:
            self.k = to_bf16_device(x["k"])
            self.v = to_bf16_device(x["v"])
            self.pt = None
            self.prob = fb.Problem(wl.seqlens, self.cu, wl.Hq, wl.Hkv, wl.d, wl.B, wl.tau)
        self.lay, self.plan_buf, self.ws = fb.allocate(self.prob)
        self.view = fb.PlanView(self.plan_buf, self.lay, wl.Hkv, wl.d)

    def plan(self):
        fb.fp2_plan(self.prob, self.q, self.k, self.v, self.plan_buf, self.ws)
        return self

    def prefill(self, flags: int = 0):
        import torch
        T = self.wl.T
        self.o = torch.full((T, self.wl.Hq, self.wl.d), float("nan"), dtype=torch.bfloat16,
                            device="cuda")
        self.lse = torch.full((self.wl.Hq, T), float("nan"), dtype=torch.float32, device="cuda")
        fb.fp2_prefill(self.prob, self.plan_buf, self.q, self.k, self.v, self.o, self.lse,
                       flags=flags)
        return self

    def status(self):
        return fb.fp2_status_check(self.plan_buf)

    def kept_lists(self) -> Dict[int, List[int]]:
        rp = self.view.row_ptr.cpu().numpy()
        ci = self.view.col_idx.cpu().numpy()
        return {r: ci[rp[r]:rp[r + 1]].tolist() for r in range(len(rp) - 1)}

    def outputs(self):
        return self.o.float().cpu().numpy(), self.lse.cpu().numpy()


def oracle_inputs(x: Dict[str, object], wl: synth.Workload):
    """Contiguous K/V for the oracle (its own paged gather when paged)."""
    if wl.page_size:
        k = oracle.gather_paged(x["k_pool"], x["page_table"], wl.seqlens, wl.page_size)
        v = oracle.gather_paged(x["v_pool"], x["page_table"], wl.seqlens, wl.page_size)
        return x["q"], k, v
    return x["q"], x["k"], x["v"]


def compare_plan(pl: Dict[str, object], gpu_kept: Dict[int, List[int]],
                 rows: Optional[Sequence[int]] = None) -> Dict[str, object]:
    """Compares kept lists row by row; differences are allowed only for blocks
    within the 1e-5 relative band of the threshold."""
    R = len(pl["kept"])
    rows = range(R) if rows is None else rows
    outside, band_blocks, diffs = 0, 0, []
    min_gap = math.inf
    for r in rows:
        ref = set(int(j) for j in pl["kept"][r])
        got = set(gpu_kept[r])
        sc = pl["scores"][r]
        t = pl["thresh"][r]
        if t is not None:
            band = {j for j in range(len(sc)) if abs(sc[j] - t) <= BAND * abs(t)}
            band_blocks += len(band)
        else:
            band = set()
        for j in ref ^ got:
            if j in band:
                continue
            outside += 1
            gap = abs(sc[j] - t) / max(abs(t), 1e-300) if t is not None else math.inf
            min_gap = min(min_gap, gap)
            diffs.append((r, j))
        if list(sorted(got)) != gpu_kept[r]:
            outside += 1
            diffs.append((r, "not ascending"))
    return {"outside_band": outside, "band_blocks": band_blocks, "min_gap": min_gap,
            "diffs": diffs[:20]}


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def token_rows(wl: synth.Workload, rows_si: Sequence[tuple]) -> np.ndarray:
    """Token indices covered by the given (s, i) query blocks."""
    cu = np.concatenate([[0], np.cumsum(wl.seqlens)])
    out = []
    for s, i in rows_si:
        lo = cu[s] + i * wl.B
        hi = cu[s] + min((i + 1) * wl.B, wl.seqlens[s])
        out.append(np.arange(lo, hi))
    return np.concatenate(out)


def sample_rows(wl: synth.Workload, per_seq: int, seed: int) -> List[tuple]:
    rows = []
    for s, L in enumerate(wl.seqlens):
        nb = (L + wl.B - 1) // wl.B
        rows += [(s, i) for i in synth.sample_qblocks(nb, per_seq, seed + s)]
    return rows


def csr_rows(wl: synth.Workload, rows_si: Sequence[tuple]) -> List[int]:
    nb = [(L + wl.B - 1) // wl.B for L in wl.seqlens]
    cu_b = np.concatenate([[0], np.cumsum(nb)])
    NB = int(cu_b[-1])
    return [g * NB + int(cu_b[s]) + i for g in range(wl.Hkv) for (s, i) in rows_si]


def attend_rows_mt(q, k, v, pl, rows_si, correction=True, kept_override=None, workers=None):
    """oracle.attend_rows over the query blocks rows_si, one call per block,
    the calls spread over the host's cores by threads (NumPy releases the GIL
    inside its matrix products and element-wise loops; BLAS is held to one
    thread per call so the threads do not oversubscribe).  The oracle is
    unchanged: every (s, i) block is computed on its own, so splitting the
    list does not change any value.  Returns what attend_rows returns for the
    whole list, in its order."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    from threadpoolctl import threadpool_limits
    rows_si = list(rows_si)
    if not rows_si:
        return oracle.attend_rows(q, k, v, pl, rows_si, correction, kept_override)
    workers = workers or len(os.sched_getaffinity(0))
    order = sorted(range(len(rows_si)), key=lambda n: -rows_si[n][1])   # longest rows first

    def one(n):
        return n, oracle.attend_rows(q, k, v, pl, [rows_si[n]], correction=correction,
                                     kept_override=kept_override)

    with threadpool_limits(1), ThreadPoolExecutor(max_workers=workers) as ex:
        res = dict(ex.map(one, order))
    parts = [res[n] for n in range(len(rows_si))]
    return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts], axis=0),
            np.concatenate([p[2] for p in parts], axis=1))


def check_attention(wl, x, run: GpuRun, pl, rows_si=None, correction=True):
    """O / LSE of the GPU against the oracle on the given query blocks, with
    the oracle using the GPU's block lists where the two differ inside the
    threshold band (so both attend over the same blocks)."""
    q, k, v = oracle_inputs(x, wl)
    gk = run.kept_lists()
    nb = [(L + wl.B - 1) // wl.B for L in wl.seqlens]
    cu_b = np.concatenate([[0], np.cumsum(nb)])
    NB = int(cu_b[-1])
    if rows_si is None:
        rows_si = [(s, i) for s in range(len(wl.seqlens)) for i in range(nb[s])]
    override = {}
    for (s, i) in rows_si:
        for g in range(wl.Hkv):
            r = g * NB + int(cu_b[s]) + i
            if list(pl["kept"][r]) != gk[r]:
                override[(s, g, i)] = gk[r]
    toks, O_ref, L_ref = attend_rows_mt(q, k, v, pl, rows_si, correction=correction,
                                        kept_override=override)
    O, LSE = run.outputs()
    assert np.array_equal(toks, token_rows(wl, rows_si))
    e_o = rel_l2(O[toks], O_ref)
    e_l = float(np.max(np.abs(LSE[:, toks] - L_ref)))
    return {"rel_l2": e_o, "lse_max_abs": e_l, "n_override": len(override),
            "finite": bool(np.isfinite(O[toks]).all() and np.isfinite(LSE[:, toks]).all())}


REL_L2_FP8 = 5e-2


def fp8_prefill(wl: synth.Workload, run: GpuRun):
    """Quantises q, k, v on the GPU (fp2_quantize_fp8_qkv) and runs the e4m3
    prefill on run's plan; returns (O, LSE) as float32 host arrays."""
    import torch
    NB = int(run.lay.num_blocks)
    out = {}
    for which, src, H in [(0, run.q, wl.Hq), (1, run.k, wl.Hkv), (2, run.v, wl.Hkv)]:
        codes = torch.zeros(src.shape, dtype=torch.uint8, device="cuda")
        scales = torch.zeros((NB, H), dtype=torch.float32, device="cuda")
        out[which] = (codes, scales)
    fb.fp2_quantize_fp8_qkv(run.prob, run.plan_buf, run.q, run.k, run.v, out[0][0], out[1][0],
                            out[2][0], out[0][1], out[1][1], out[2][1])
    o = torch.full((wl.T, wl.Hq, wl.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((wl.Hq, wl.T), float("nan"), dtype=torch.float32, device="cuda")
    fb.fp2_prefill(run.prob, run.plan_buf, out[0][0], out[1][0], out[2][0], o, lse,
                   q_scale=out[0][1], k_scale=out[1][1], v_scale=out[2][1],
                   dtype=fb.FP2_DTYPE_E4M3)
    res = (o.float().cpu().numpy(), lse.cpu().numpy())
    del out, o, lse
    return res


def dequantised_operands(wl: synth.Workload, q, k, v, rows_si):
    """The FP8 path's inputs as its definition gives them: Q, K and V after
    direct online quantisation (per (block, head) scale = absmax / 448,
    e4m3 round-to-nearest-even, saturating) and dequantisation, from the
    oracle's quantiser -- K and V whole, Q only on the query blocks rows_si
    (zeros elsewhere).  The block means stay the plan's float64 means: how
    the kernel carries them into its e4m3 products is its own business and
    part of its error.  Scales are per (block, head), so each block is
    quantised on its own as a one-block sequence (same codes, less memory)."""
    cu = np.concatenate([[0], np.cumsum(wl.seqlens)])

    def dq_block(a, lo, hi, out):
        c, sc = oracle.quantize_e4m3(np.asarray(a[lo:hi]), [hi - lo], wl.B)
        out[lo:hi] = oracle.dequantize_e4m3(c, sc, [hi - lo], wl.B)

    q_dq = np.zeros(np.shape(q))
    k_dq = np.empty(np.shape(k))
    v_dq = np.empty(np.shape(v))
    for s, L in enumerate(wl.seqlens):
        for i in range((L + wl.B - 1) // wl.B):
            lo, hi = cu[s] + i * wl.B, cu[s] + min((i + 1) * wl.B, L)
            dq_block(k, lo, hi, k_dq)
            dq_block(v, lo, hi, v_dq)
    for s, i in rows_si:
        lo, hi = cu[s] + i * wl.B, cu[s] + min((i + 1) * wl.B, wl.seqlens[s])
        dq_block(q, lo, hi, q_dq)
    return q_dq, k_dq, v_dq


# Regression guard for the distance of the FP8 output to the plain oracle
# (bf16 inputs, no quantisation).  e4m3 rounding of Q, K and V alone moves O
# by 4e-2 (N(0,1) inputs) to 7e-2 (low-rank generator) rel-L2 in the float64
# oracle itself (tests/test_oracle.py), and e4m3 P in the P.V product adds
# about 3e-2; the stated 5e-2 is checked against the oracle on the
# quantised inputs (REL_L2_FP8 above).
REL_L2_FP8_PLAIN_GUARD = 0.15


def check_fp8(wl, x, run: GpuRun, pl, rows_si, O8, L8):
    """FP8 O / LSE against the oracle on the quantised inputs (Q, K, V through
    the direct online quantisation, then float64 arithmetic with the plan's
    float64 block means) and against the plain bf16-input oracle (the
    accuracy cost of e4m3).  The GPU's block lists are used where they differ
    inside the threshold band."""
    q, k, v = oracle_inputs(x, wl)
    gk = run.kept_lists()
    nb = [(L + wl.B - 1) // wl.B for L in wl.seqlens]
    cu_b = np.concatenate([[0], np.cumsum(nb)])
    NB = int(cu_b[-1])
    override = {}
    for (s, i) in rows_si:
        for g in range(wl.Hkv):
            r = g * NB + int(cu_b[s]) + i
            if list(pl["kept"][r]) != gk[r]:
                override[(s, g, i)] = gk[r]
    q_dq, k_dq, v_dq = dequantised_operands(wl, q, k, v, rows_si)
    toks, O_dq, L_dq = attend_rows_mt(q_dq, k_dq, v_dq, pl, rows_si, kept_override=override)
    del q_dq, k_dq, v_dq
    _, O_ref, L_ref = attend_rows_mt(q, k, v, pl, rows_si, kept_override=override)
    assert np.array_equal(toks, token_rows(wl, rows_si))
    return {"rel_l2_dq": rel_l2(O8[toks], O_dq), "rel_l2_plain": rel_l2(O8[toks], O_ref),
            "lse_dq": float(np.max(np.abs(L8[:, toks] - L_dq))),
            "lse_plain": float(np.max(np.abs(L8[:, toks] - L_ref))),
            "finite": bool(np.isfinite(O8[toks]).all() and np.isfinite(L8[:, toks]).all())}


def assert_fp8(res):
    """The FP8 tolerances: O rel-L2 <= 5e-2 and LSE <= 1e-3 against the oracle
    on the quantised inputs; the distance to the plain oracle under its guard."""
    assert res["finite"], res
    assert res["rel_l2_dq"] <= REL_L2_FP8, res
    assert res["lse_dq"] <= LSE_ABS, res
    assert res["rel_l2_plain"] <= REL_L2_FP8_PLAIN_GUARD, res
