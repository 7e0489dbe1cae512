"""GPU parity in the low-density regime the method targets.

The 128K-token layer shape (32 q / 8 kv heads, d 128, block 128, tau 0.5) on
the block-level "topics" generator keeps about 5, 10 and 20 % of the blocks
(Table 3 reports 4.6-9.4 % at 64K-128K on real prompts), so most of each row
runs through the mean-correction path.  On a seeded sample of 64 query blocks
(always the first and the last) across every kv-head and query head: block
lists bit-exact outside the threshold band, O / LSE within the BF16
tolerances, and FP8 against the oracle on the quantised inputs.
"""

import numpy as np
import pytest

import oracle
from block_sparse_long_fp2_b200 import binding as fb
from block_sparse_long_fp2_b200 import synth

from fp2_harness import (LSE_ABS, REL_L2_BF16, GpuRun, assert_fp8, check_attention, check_fp8,
                         compare_plan, csr_rows, fp8_prefill, sample_rows)

pytestmark = pytest.mark.gpu

# workload -> the density it is built for (kept / visible blocks)
POINTS = {"topics_128k_5pct": 0.05, "topics_128k_10pct": 0.10, "topics_128k_20pct": 0.20}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_fp2_b200 import build
    build.build()
    fb.lib()


@pytest.mark.parametrize("name", sorted(POINTS))
def test_low_density_layer(name):
    import torch
    wl = synth.workloads()[name]
    x = synth.generate(wl)
    run = GpuRun(wl, x).plan().prefill()
    assert run.status() == (fb.FP2_OK, 0)
    nnz = int(run.view.row_ptr[-1].item())
    density = nnz / float(run.lay.nnz_cap)
    # forced sink and diagonal blocks add about 2 / (i + 1) per row
    assert POINTS[name] * 0.8 <= density <= POINTS[name] * 1.3, density
    q, k, v = x["q"], x["k"], x["v"]
    rows_si = sample_rows(wl, 64, seed=31)
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau, rows=rows_si)
    res = compare_plan(pl, run.kept_lists(), rows=csr_rows(wl, rows_si))
    assert res["outside_band"] == 0, res
    att = check_attention(wl, x, run, pl, rows_si=rows_si)
    O8, L8 = fp8_prefill(wl, run)
    assert run.status() == (fb.FP2_OK, 0)
    f8 = check_fp8(wl, x, run, pl, rows_si, O8, L8)
    print(name, "density", round(density, 4), "bf16", att, "fp8", f8)
    assert att["finite"] and att["rel_l2"] <= REL_L2_BF16 and att["lse_max_abs"] <= LSE_ABS, att
    assert_fp8(f8)
    del run
    torch.cuda.empty_cache()
