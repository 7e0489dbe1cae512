"""GPU parity over the dense-vs-sparse sweep: one 32 q / 8 kv-head, head dim
128, block 128 layer at L in {4K, 8K, 16K, 32K, 64K, 128K} x tau in {0 (dense),
0.05, 0.2}, BF16 and FP8-e4m3, low-rank generator, and the FP8-e4m3 run of the
128K needles layer.

Each cell is checked on a seeded sample of 16 query blocks (always the first
and the last) across every kv-head and query head: block lists, and O / LSE.
FP8 is checked against the oracle on the quantised inputs (direct online
quantisation of Q, K, V; float64 block means) and its distance to the plain
oracle is held under a regression guard.
"""

import numpy as np
import pytest

import oracle
from block_sparse_long_fp2_b200 import binding as fb
from block_sparse_long_fp2_b200 import synth

from fp2_harness import (LSE_ABS, REL_L2_BF16, GpuRun, assert_fp8, check_attention, check_fp8,
                         compare_plan, csr_rows, fp8_prefill, oracle_inputs, sample_rows)

pytestmark = pytest.mark.gpu

SWEEP = sorted((n for n in synth.workloads() if n.startswith("sweep_")),
               key=lambda n: synth.workloads()[n].T)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_fp2_b200 import build
    build.build()
    fb.lib()


def _cell(name, fp8=True):
    import torch
    wl = synth.workloads()[name]
    x = synth.generate(wl)
    run = GpuRun(wl, x).plan().prefill()
    assert run.status() == (fb.FP2_OK, 0)
    q, k, v = oracle_inputs(x, wl)
    rows_plan = sample_rows(wl, 16, seed=21)
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau, rows=rows_plan)
    res = compare_plan(pl, run.kept_lists(), rows=csr_rows(wl, rows_plan))
    assert res["outside_band"] == 0, res
    rows_o = rows_plan
    att = check_attention(wl, x, run, pl, rows_si=rows_o)
    out = {"plan": res, "bf16": att}
    if fp8:
        O8, L8 = fp8_prefill(wl, run)
        assert run.status() == (fb.FP2_OK, 0)
        out["fp8"] = check_fp8(wl, x, run, pl, rows_o, O8, L8)
    print(name, {k_: v_ for k_, v_ in out.items() if k_ != "plan"})
    del run
    torch.cuda.empty_cache()
    return out


@pytest.mark.parametrize("name", SWEEP)
def test_sweep_cell(name):
    res = _cell(name)
    bf = res["bf16"]
    assert bf["finite"] and bf["rel_l2"] <= REL_L2_BF16 and bf["lse_max_abs"] <= LSE_ABS, bf
    assert_fp8(res["fp8"])
