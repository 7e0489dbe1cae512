"""A layer split by kv-head, run in place: the multi-GPU split of one layer.

Each kv-head and its G query heads are planned and attended on their own, so
running kv-heads [h0, h0 + n) of a layer through kv_head_begin /
num_kv_heads_total (every tensor keeps all of the layer's heads) must give
exactly the full layer's results for those heads: the same block lists and
K/V block means, and -- when neither run splits rows -- the same O and LSE
bit for bit (the same kernels do the same arithmetic on the same tiles).  The
halves run one after the other on one GPU, each writing only its own heads of
the shared O / LSE tensors.  FP8: quantisation of a slice writes the slice's
codes (bit-exact with the full layer's) and its own scales.
"""

import numpy as np
import pytest

from block_sparse_long_fp2_b200 import binding as fb
from block_sparse_long_fp2_b200 import synth

from fp2_harness import GpuRun, to_bf16_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_fp2_b200 import build
    build.build()
    fb.lib()


CASES = {
    # name: (seqlens, Hq, Hkv, d, B, tau, page_size, pool_pages, slices)
    "two_halves": ([1500, 700, 2100], 16, 4, 128, 128, 0.1, 0, 0, [(0, 2), (2, 2)]),
    "uneven_paged": ([1000, 333], 24, 3, 64, 64, 0.2, 64, 40, [(0, 2), (2, 1)]),
    "llama_32k_quarters": ([32768], 32, 8, 128, 128, 0.1, 0, 0, [(0, 2), (2, 2), (4, 2), (6, 2)]),
}


def _slice_problem(run, wl, h0, n):
    G = wl.Hq // wl.Hkv
    kw = {"kv_head_begin": h0, "num_kv_heads_total": wl.Hkv}
    if run.paged:
        return fb.Problem(wl.seqlens, run.cu, G * n, n, wl.d, wl.B, wl.tau, page_size=64,
                          page_table=run.pt, num_pages=int(run.x["k_pool"].shape[0]), **kw)
    return fb.Problem(wl.seqlens, run.cu, G * n, n, wl.d, wl.B, wl.tau, **kw)


@pytest.mark.parametrize("name", sorted(CASES))
def test_head_slices_equal_the_full_layer(name):
    import torch
    seqlens, Hq, Hkv, d, B, tau, page, pool, slices = CASES[name]
    if name == "llama_32k_quarters":
        wl = synth.workloads()["llama_32k"]
    else:
        wl = synth.small_workload(seqlens, Hq, Hkv, d, B, tau, seed=900 + len(name),
                                  page_size=page, pool_pages=pool)
    x = synth.generate(wl)
    full = GpuRun(wl, x).plan().prefill()
    assert full.status() == (fb.FP2_OK, 0)
    kept_full = full.kept_lists()
    O_full, L_full = full.outputs()
    NB = int(full.lay.num_blocks)
    G = wl.Hq // wl.Hkv
    o = torch.full_like(full.o, float("nan"))
    lse = torch.full_like(full.lse, float("nan"))
    any_split = full.lay.num_split_slots > 0
    for (h0, n) in slices:
        prob = _slice_problem(full, wl, h0, n)
        lay, plan, ws = fb.allocate(prob)
        fb.fp2_plan(prob, full.q, full.k, full.v, plan, ws)
        fb.fp2_prefill(prob, plan, full.q, full.k, full.v, o, lse)
        assert fb.fp2_status_check(plan) == (fb.FP2_OK, 0)
        any_split = any_split or lay.num_split_slots > 0
        view = fb.PlanView(plan, lay, n, wl.d)
        rp = view.row_ptr.cpu().numpy()
        ci = view.col_idx.cpu().numpy()
        for gl in range(n):
            for b in range(NB):
                r = gl * NB + b
                assert ci[rp[r]:rp[r + 1]].tolist() == kept_full[(h0 + gl) * NB + b], (h0, gl, b)
        assert torch.equal(view.kbar, full.view.kbar[:, h0:h0 + n])
        assert torch.equal(view.vbar, full.view.vbar[:, h0:h0 + n])
        # FP8: quantising the slice gives the full layer's codes for its heads
        for which, src, H, hs in ((0, full.q, G * n, G * h0), (1, full.k, n, h0)):
            codes = torch.zeros(src.shape, dtype=torch.uint8, device="cuda")
            scales = torch.zeros((NB, H), dtype=torch.float32, device="cuda")
            fb.fp2_quantize_fp8(prob, plan, src, which, codes, scales)
            codes_f = torch.zeros_like(codes)
            scales_f = torch.zeros((NB, src.shape[-2]), dtype=torch.float32, device="cuda")
            fb.fp2_quantize_fp8(full.prob, full.plan_buf, src, which, codes_f, scales_f)
            assert torch.equal(scales, scales_f[:, hs:hs + H])
            # (the head axis is the second-to-last one, contiguous or paged)
            assert torch.equal(codes[..., hs:hs + H, :], codes_f[..., hs:hs + H, :])
            assert int(codes[..., :hs, :].count_nonzero()) == 0   # other heads untouched
        del plan, ws
    O, L = o.float().cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(O).all() and np.isfinite(L).all()   # every head written once
    if not any_split:
        assert np.array_equal(O, O_full) and np.array_equal(L, L_full)
    else:
        # splits decided per run (the layer's share per CTA differs): merged by
        # log-sum-exp, equal up to rounding
        assert np.max(np.abs(L - L_full)) <= 1e-4
        assert np.linalg.norm(O - O_full) <= 1e-3 * np.linalg.norm(O_full)
