"""The debug build (libfp2_debug.so, compiled with FP2_DEBUG) on the small
parity cases.

compute-sanitizer is closed on this machine; its stand-in is a build whose index
checks -- schedule entries, CSR column ids, page-table indices, pseudo-tile
block coordinates, O / LSE / split-scratch rows, score and CSR writes -- record
FP2_STATUS_BOUNDS in the plan's status word (and clamp or skip the access)
instead of reading or writing out of range.  Every small case, BF16 and FP8,
contiguous and paged, split and unsplit, must run through it with a clean
status and give exactly the regular build's block lists, O and LSE (the
checks do not change the arithmetic).
"""

import numpy as np
import pytest

from block_sparse_long_fp2_b200 import binding as fb

from fp2_harness import GpuRun, fp8_prefill
from test_gpu_parity import SMALL, _case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_fp2_b200 import build
    build.build()
    fb.lib()
    yield
    fb.use_debug_library(False)


def _run(wl, x):
    run = GpuRun(wl, x).plan().prefill()
    status = run.status()
    out = {"kept": run.kept_lists(), "bf16": run.outputs()}
    if wl.d == 128:
        out["fp8"] = fp8_prefill(wl, run)
        status = (status, run.status())
    return status, out


@pytest.mark.parametrize("name", sorted(SMALL))
def test_debug_build_is_clean_and_equal(name):
    wl, x = _case(name)
    fb.use_debug_library(False)
    st_ref, ref = _run(wl, x)
    fb.use_debug_library(True)
    try:
        st_dbg, dbg = _run(wl, x)
    finally:
        fb.use_debug_library(False)
    assert st_dbg == st_ref, (st_dbg, st_ref)      # FP2_OK and no FP2_STATUS_BOUNDS
    assert dbg["kept"] == ref["kept"]
    for key in ("bf16", "fp8"):
        if key in ref:
            for a, b in zip(dbg[key], ref[key]):
                assert np.array_equal(a, b, equal_nan=True), key
