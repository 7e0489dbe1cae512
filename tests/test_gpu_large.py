"""GPU parity at full workload sizes, in the configuration bench.py times.

The float64 oracle cannot run these layers whole, so it checks a seeded
sample of 64 query blocks per sequence (fewer when the sequence is shorter),
always holding the first and the last block, across every kv-head and every
query head of each: block lists and K/V block means, and O / LSE for BF16
and for FP8-e4m3 (direct online quantisation of Q, K and V, then the e4m3
prefill).  The oracle's rows run on the host's cores in threads.
"""

import numpy as np
import pytest

import oracle
from block_sparse_long_fp2_b200 import binding as fb
from block_sparse_long_fp2_b200 import synth

from fp2_harness import (LSE_ABS, REL_L2_BF16, GpuRun, assert_fp8, check_attention, check_fp8,
                         compare_plan, csr_rows, fp8_prefill, oracle_inputs, sample_rows)

pytestmark = pytest.mark.gpu

SAMPLE = 64   # query blocks per sequence, every kv-head and query head of each

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
        import torch
        torch.cuda.empty_cache()
        wl = synth.workloads()[name]
        x = synth.generate(wl)
        run = GpuRun(wl, x).plan().prefill()
        assert run.status() == (fb.FP2_OK, 0)
        q, k, v = oracle_inputs(x, wl)
        rows_si = sample_rows(wl, SAMPLE, seed=7)
        pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau, rows=rows_si)
        _CACHE[name] = (wl, x, run, (q, k, v), rows_si, pl)
    return _CACHE[name]


NAMES = ["llama_32k", "qwen_128k", "paged_mix"]


@pytest.mark.parametrize("name", NAMES)
def test_block_lists_on_sampled_rows(name):
    wl, x, run, (q, k, v), rows_si, pl = _run(name)
    res = compare_plan(pl, run.kept_lists(), rows=csr_rows(wl, rows_si))
    assert res["outside_band"] == 0, res
    # block means of K and V for every block
    assert np.allclose(run.view.kbar.cpu().numpy(), pl["kbar"], rtol=2e-7, atol=1e-7)
    assert np.allclose(run.view.vbar.cpu().numpy(), pl["vbar"], rtol=2e-7, atol=1e-7)
    # the density the bench reports is the CSR's
    nnz = int(run.view.row_ptr[-1].item())
    assert 0 < nnz <= run.lay.nnz_cap


@pytest.mark.parametrize("name", NAMES)
def test_attention_on_sampled_rows(name):
    wl, x, run, (q, k, v), rows_si, pl = _run(name)
    res = check_attention(wl, x, run, pl, rows_si=rows_si)
    print(name, "bf16", len(rows_si), "query blocks", res)
    assert res["finite"], res
    assert res["rel_l2"] <= REL_L2_BF16, res
    assert res["lse_max_abs"] <= LSE_ABS, res


@pytest.mark.parametrize("name", NAMES)
def test_fp8_attention_on_sampled_rows(name):
    wl, x, run, (q, k, v), rows_si, pl = _run(name)
    O8, L8 = fp8_prefill(wl, run)
    assert run.status() == (fb.FP2_OK, 0)
    res = check_fp8(wl, x, run, pl, rows_si, O8, L8)
    print(name, "fp8", len(rows_si), "query blocks", res)
    assert_fp8(res)
