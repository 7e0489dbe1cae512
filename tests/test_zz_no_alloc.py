"""fp2_plan_static: planning without a caller workspace.

Some callers cannot allocate device memory for fp2_plan's workspace (a
serving process whose KV-cache pool already holds the device memory, or a
host that only receives device pointers from another runtime).  They call
fp2_plan_static, which keeps its scratch in a fixed array inside the
library.  Its results must equal fp2_plan's, call after call.

This file is collected last on purpose (a failure here stops a -x run only
after every other test has run).
"""

import numpy as np
import pytest

from block_sparse_long_fp2_b200 import binding as fb
from block_sparse_long_fp2_b200 import build as fbuild
from block_sparse_long_fp2_b200 import synth


def _lib():
    fbuild.build()
    return fb.lib()


def test_rejects_problems_beyond_the_fixed_scratch():
    _lib()
    # a 128K-token layer needs far more scratch than the fixed array holds
    p = fb.Problem([131072], 0x1000, 32, 8, 128, 128, 0.05)
    lay = fb.fp2_plan_sizes(p)
    assert lay.workspace_bytes > fb.FP2_STATIC_WORKSPACE_BYTES
    rc = fb.lib().fp2_plan_static(p.ref, 0x10000, 0x10000, 0x10000, 0x100000, lay.plan_bytes, None)
    assert rc == fb.FP2_ERR_CAPACITY


def test_documented_shape_fits_the_fixed_scratch():
    _lib()
    # the header names one 32K-token layer (32 q / 8 kv heads, d 128, B 128)
    # as fitting the fixed array, and a 64K-token one as not
    for L, fits in ((32768, True), (65536, False)):
        p = fb.Problem([L], 0x1000, 32, 8, 128, 128, 0.1)
        assert (fb.fp2_plan_sizes(p).workspace_bytes <= fb.FP2_STATIC_WORKSPACE_BYTES) == fits, L


def test_binding_constant_matches_the_header():
    import os
    import re
    hdr = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fp2.h")
    m = re.search(r"#define FP2_STATIC_WORKSPACE_BYTES \(\(size_t\)(\d+) << (\d+)\)", open(hdr).read())
    assert m and int(m.group(1)) << int(m.group(2)) == fb.FP2_STATIC_WORKSPACE_BYTES


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["ragged_d128", "pr1_ref_1k", "paged"])
def test_static_plan_equals_workspace_plan_twice(case):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _lib()
    from fp2_harness import LSE_ABS, REL_L2_BF16, GpuRun, rel_l2

    if case == "pr1_ref_1k":
        wl = synth.workloads()["pr1_ref_1k"]
    elif case == "paged":
        wl = synth.small_workload([1500, 640, 97], 8, 2, 128, 128, 0.1, seed=311, page_size=64,
                                  pool_pages=60)
    else:
        wl = synth.small_workload([700, 333, 1100], 8, 2, 128, 128, 0.1, seed=312)
    x = synth.generate(wl)
    ref = GpuRun(wl, x).plan().prefill()
    assert ref.status() == (fb.FP2_OK, 0)
    assert ref.lay.workspace_bytes <= fb.FP2_STATIC_WORKSPACE_BYTES
    O_ref, L_ref = ref.outputs()
    kept_ref = ref.kept_lists()

    run = GpuRun(wl, x)
    for _ in range(2):                           # two calls in a row share the array
        run.plan_buf.fill_(0xAB)
        fb.fp2_plan_static(run.prob, run.q, run.k, run.v, run.plan_buf)
        run.prefill()
        assert run.status() == (fb.FP2_OK, 0)
        assert run.kept_lists() == kept_ref
        assert np.array_equal(run.view.kbar.cpu().numpy(), ref.view.kbar.cpu().numpy())
        assert np.array_equal(run.view.vbar.cpu().numpy(), ref.view.vbar.cpu().numpy())
        O, L = run.outputs()
        assert rel_l2(O, O_ref) <= REL_L2_BF16
        assert np.max(np.abs(L - L_ref)) <= LSE_ABS
