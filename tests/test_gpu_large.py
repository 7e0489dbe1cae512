"""GPU parity at full workload sizes, in the configuration bench.py times.

The float64 oracle cannot run these layers whole, so it checks a seeded
sample: block lists (and K/V block means) for 64 query blocks per sequence
across every kv-head, and O / LSE for 8 query blocks per sequence across
every query head and token.  Samples always hold the first and last block.
"""

import numpy as np
import pytest

import oracle
from block_sparse_long_fp2_b200 import binding as fb
from block_sparse_long_fp2_b200 import synth

from fp2_harness import (LSE_ABS, REL_L2_BF16, GpuRun, check_attention, compare_plan, csr_rows,
                         oracle_inputs, sample_rows)

pytestmark = pytest.mark.gpu

_CACHE = {}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_fp2_b200 import build
    build.build()
    fb.lib()
    yield
    _CACHE.clear()


def _run(name):
    if name not in _CACHE:
        _CACHE.clear()
        wl = synth.workloads()[name]
        x = synth.generate(wl)
        run = GpuRun(wl, x).plan().prefill()
        assert run.status() == (fb.FP2_OK, 0)
        q, k, v = oracle_inputs(x, wl)
        _CACHE[name] = (wl, x, run, (q, k, v))
    return _CACHE[name]


@pytest.mark.parametrize("name", ["llama_32k", "qwen_128k", "paged_mix"])
def test_block_lists_on_sampled_rows(name):
    wl, x, run, (q, k, v) = _run(name)
    rows_si = sample_rows(wl, 64, seed=7)
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau, rows=rows_si)
    rows = csr_rows(wl, rows_si)
    res = compare_plan(pl, run.kept_lists(), rows=rows)
    assert res["outside_band"] == 0, res
    # block means of K and V for every block
    assert np.allclose(run.view.kbar.cpu().numpy(), pl["kbar"], rtol=2e-7, atol=1e-7)
    assert np.allclose(run.view.vbar.cpu().numpy(), pl["vbar"], rtol=2e-7, atol=1e-7)
    # the density the bench reports is the CSR's
    nnz = int(run.view.row_ptr[-1].item())
    assert 0 < nnz <= run.lay.nnz_cap


@pytest.mark.parametrize("name", ["llama_32k", "qwen_128k", "paged_mix"])
def test_attention_on_sampled_rows(name):
    wl, x, run, (q, k, v) = _run(name)
    rows_si = sample_rows(wl, 8, seed=11)
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau, rows=rows_si)
    res = check_attention(wl, x, run, pl, rows_si=rows_si)
    assert res["finite"], res
    assert res["rel_l2"] <= REL_L2_BF16, res
    assert res["lse_max_abs"] <= LSE_ABS, res
