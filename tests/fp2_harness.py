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
    toks, O_ref, L_ref = oracle.attend_rows(q, k, v, pl, rows_si, correction=correction,
                                            kept_override=override)
    O, LSE = run.outputs()
    assert np.array_equal(toks, token_rows(wl, rows_si))
    e_o = rel_l2(O[toks], O_ref)
    e_l = float(np.max(np.abs(LSE[:, toks] - L_ref)))
    return {"rel_l2": e_o, "lse_max_abs": e_l, "n_override": len(override),
            "finite": bool(np.isfinite(O[toks]).all() and np.isfinite(LSE[:, toks]).all())}
