"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Block lists must match bit-exactly outside the 1e-5 threshold band; O within
rel-L2 1e-2 and LSE within 1e-3 (BF16).  Small cases are checked on every
row; they span several tiles, ragged tails, one and several query-tile
pairs per row, several pseudo tiles per row, varlen and paged layouts.
"""

import numpy as np
import pytest

import oracle
from block_sparse_long_fp2_b200 import binding as fb
from block_sparse_long_fp2_b200 import synth

from fp2_harness import (LSE_ABS, REL_L2_BF16, REL_L2_FP8, REL_L2_FP8_PLAIN_GUARD, GpuRun,
                         check_attention, compare_plan, oracle_inputs)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_fp2_b200 import build
    build.build()
    fb.lib()


SMALL = {
    # name: (seqlens, Hq, Hkv, d, B, tau, generator, needles, page_size, pool_pages)
    "pr1_ref_1k": ([1024], 4, 1, 64, 64, 0.3, "needles", 8, 0, 0),
    "ragged_d128": ([700, 333, 1100], 8, 2, 128, 128, 0.1, "lowrank", 0, 0, 0),
    "one_tile_G2_B64": ([513], 2, 1, 64, 64, 0.05, "lowrank", 0, 0, 0),
    "one_tile_G1_B128": ([640, 200], 4, 4, 128, 128, 0.3, "lowrank", 0, 0, 0),
    "G8_d64_B128_tau1": ([900], 16, 2, 64, 128, 1.0, "lowrank", 0, 0, 0),
    "G3_odd_tiles": ([1000, 129], 6, 2, 64, 128, 0.2, "lowrank", 0, 0, 0),
    "B64_d128": ([777], 8, 2, 128, 64, 0.1, "lowrank", 0, 0, 0),
    "dense_tau0": ([1000, 300], 8, 2, 128, 128, 0.0, "lowrank", 0, 0, 0),
    "paged_mix_small": ([1500, 640, 97], 8, 2, 128, 128, 0.1, "lowrank", 0, 64, 60),
    "two_pseudo_tiles": ([9000], 2, 1, 64, 64, 0.2, "lowrank", 0, 0, 0),
    # degenerate lengths: one token, two tokens, a block plus one, a partial block
    "tiny_lengths": ([1, 2, 129, 3, 130], 8, 2, 128, 128, 0.5, "normal", 0, 0, 0),
    "tiny_paged": ([1, 65, 64], 8, 2, 128, 128, 0.5, "normal", 0, 64, 8),
    # one kv-head with long rows: the rows are cut into count-balanced splits
    "split_long_rows": ([4096], 2, 1, 64, 64, 0.2, "lowrank", 0, 0, 0),
    "split_d128_paged": ([3000, 700], 2, 1, 128, 64, 0.1, "normal", 0, 64, 70),
}


def _case(name, seed_base=500):
    seqlens, Hq, Hkv, d, B, tau, gen, nn, page, pool = SMALL[name]
    wl = synth.small_workload(seqlens, Hq, Hkv, d, B, tau, seed=seed_base + sorted(SMALL).index(name),
                              generator=gen, n_needles=nn, page_size=page, pool_pages=pool)
    if name == "pr1_ref_1k":
        wl = synth.workloads()["pr1_ref_1k"]
    return wl, synth.generate(wl)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_plan_matches_oracle(name):
    wl, x = _case(name)
    run = GpuRun(wl, x).plan()
    rc, st = run.status()
    assert rc == fb.FP2_OK and st == 0
    q, k, v = oracle_inputs(x, wl)
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau)
    res = compare_plan(pl, run.kept_lists())
    assert res["outside_band"] == 0, res
    # the CSR is exactly the kept lists: row_ptr consistent, nnz <= cap
    rp = run.view.row_ptr.cpu().numpy()
    assert rp[0] == 0 and np.all(np.diff(rp) >= 1) and rp[-1] <= run.lay.nnz_cap
    # block means of K and V (fp32 of the exact means)
    kb = run.view.kbar.cpu().numpy()
    vb = run.view.vbar.cpu().numpy()
    assert np.allclose(kb, pl["kbar"], rtol=2e-7, atol=1e-7)
    assert np.allclose(vb, pl["vbar"], rtol=2e-7, atol=1e-7)
    kb16 = run.view.kbar_bf16.float().cpu().numpy()
    assert np.allclose(kb16, pl["kbar"], rtol=2 ** -8, atol=1e-6)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_prefill_matches_oracle(name):
    wl, x = _case(name)
    run = GpuRun(wl, x).plan().prefill()
    rc, st = run.status()
    assert rc == fb.FP2_OK and st == 0
    q, k, v = oracle_inputs(x, wl)
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau)
    res = check_attention(wl, x, run, pl)
    assert res["finite"], res
    assert res["rel_l2"] <= REL_L2_BF16, res
    assert res["lse_max_abs"] <= LSE_ABS, res


def test_no_correction_flag_drops_the_surrogate():
    # N(0, 1) inputs keep the logits O(1), so the skipped mass is visible
    wl = synth.small_workload([700, 333, 1100], 8, 2, 128, 128, 0.3, seed=91, generator="normal")
    x = synth.generate(wl)
    run = GpuRun(wl, x).plan().prefill(flags=fb.FP2_NO_CORRECTION)
    q, k, v = oracle_inputs(x, wl)
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau)
    res = check_attention(wl, x, run, pl, correction=False)
    assert res["rel_l2"] <= REL_L2_BF16 and res["lse_max_abs"] <= LSE_ABS, res
    # and the corrected run is measurably different (something was skipped)
    run2 = GpuRun(wl, x).plan().prefill()
    assert len(run2.kept_lists()[0]) >= 1
    assert float((run2.lse - run.lse).abs().max()) > 1e-2


@pytest.mark.parametrize("flags", [0, fb.FP2_NO_CORRECTION])
def test_split_rows_with_empty_splits_match_oracle(flags):
    # One 4096-token sequence with 2/1 heads and B = 64 gives 64 rows of one
    # query tile for 148 SMs, so the long rows are cut into count-balanced
    # splits (row 63 into 9) merged by log-sum-exp.  At tau = 1 a row keeps 2
    # or 3 blocks (plus one pseudo tile with the correction), so most of its
    # splits have no tile at all.
    wl = synth.small_workload([4096], 2, 1, 64, 64, 1.0, seed=98, generator="normal")
    x = synth.generate(wl)
    run = GpuRun(wl, x).plan()
    assert run.lay.num_split_slots > 0 and run.lay.num_work_items > 64
    run.prefill(flags=flags)
    rc, st = run.status()
    assert rc == fb.FP2_OK and st == 0
    q, k, v = oracle_inputs(x, wl)
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau)
    assert len(run.kept_lists()[63]) + 1 < 9   # fewer tiles than splits
    res = check_attention(wl, x, run, pl, correction=flags == 0)
    assert res["finite"] and res["rel_l2"] <= REL_L2_BF16 and res["lse_max_abs"] <= LSE_ABS, res


def test_dense_tau0_equals_brute_force_dense():
    wl, x = _case("dense_tau0")
    run = GpuRun(wl, x).plan().prefill()
    O, LSE = run.outputs()
    Od, Ld = oracle.dense_attention(x["q"], x["k"], x["v"], wl.seqlens)
    from fp2_harness import rel_l2
    assert rel_l2(O, Od) <= REL_L2_BF16
    assert np.max(np.abs(LSE - Ld)) <= LSE_ABS


def test_paged_layout_is_bit_identical_to_contiguous():
    # equal-length batch, shuffled pages vs the packed contiguous layout
    seqlens = [1536, 1536, 1536]
    wl = synth.small_workload(seqlens, 8, 2, 128, 128, 0.1, seed=77, page_size=64, pool_pages=90)
    x = synth.generate(wl)
    a = GpuRun(wl, x, paged=True).plan().prefill()
    b = GpuRun(wl, x, paged=False).plan().prefill()
    assert a.kept_lists() == b.kept_lists()
    Oa, La = a.outputs()
    Ob, Lb = b.outputs()
    assert np.array_equal(Oa, Ob) and np.array_equal(La, Lb)


def test_repeat_calls_are_deterministic():
    wl, x = _case("ragged_d128")
    run = GpuRun(wl, x).plan().prefill()
    O1, L1 = run.outputs()
    run.plan().prefill()
    O2, L2 = run.outputs()
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


@pytest.mark.parametrize("edit", ["empty_sequence", "total_mismatch", "nonzero_start"])
def test_device_check_bad_cu_seqlens_does_no_work(edit):
    # cu_seqlens whose sizes disagree with the host seqlens: every kernel
    # returns without touching memory and the status word says why.  (A
    # permutation of lengths that keeps every total is consistent, and is
    # simply the problem the device was given.)
    import torch
    wl, x = _case("ragged_d128")
    run = GpuRun(wl, x)
    if edit == "empty_sequence":
        run.cu[2] = run.cu[1]
    elif edit == "total_mismatch":
        run.cu[3] += 1
    else:
        run.cu[0] = 1
    run.plan().prefill()
    rc, st = run.status()
    assert rc == fb.FP2_ERR_DEVICE_CHECK and st & fb.FP2_STATUS_BAD_SEQLENS
    assert torch.isnan(run.o.float()).all()   # prefill did not write


def test_device_check_bad_page_id_is_recorded():
    wl, x = _case("paged_mix_small")
    x = dict(x)
    pt = x["page_table"].copy()
    pt[1, 3] = 10_000                # out of the pool
    x["page_table"] = pt
    run = GpuRun(wl, x).plan().prefill()
    rc, st = run.status()
    assert rc == fb.FP2_ERR_DEVICE_CHECK and st & fb.FP2_STATUS_BAD_PAGE
    # a fresh, valid plan on the same context works again
    wl2, x2 = _case("paged_mix_small")
    run2 = GpuRun(wl2, x2).plan().prefill()
    assert run2.status() == (fb.FP2_OK, 0)


def test_quantize_fp8_matches_oracle_codes():
    import torch
    wl, x = _case("ragged_d128")
    run = GpuRun(wl, x).plan()
    NB = int(run.lay.num_blocks)
    for which, name, H in [(0, "q", wl.Hq), (1, "k", wl.Hkv), (2, "v", wl.Hkv)]:
        src = {0: run.q, 1: run.k, 2: run.v}[which]
        codes = torch.zeros(src.shape, dtype=torch.uint8, device="cuda")
        scales = torch.zeros((NB, H), dtype=torch.float32, device="cuda")
        fb.fp2_quantize_fp8(run.prob, run.plan_buf, src, which, codes, scales)
        got = codes.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()
        ref, ref_s = oracle.quantize_e4m3(x[name], wl.seqlens, wl.B)
        assert np.array_equal(scales.cpu().numpy().astype(np.float64), ref_s)
        assert np.array_equal(got, ref)
    # the one-launch form gives the same codes and scales
    outs = [(torch.zeros(t.shape, dtype=torch.uint8, device="cuda"),
             torch.zeros((NB, t.shape[1]), dtype=torch.float32, device="cuda"))
            for t in (run.q, run.k, run.v)]
    fb.fp2_quantize_fp8_qkv(run.prob, run.plan_buf, run.q, run.k, run.v, outs[0][0], outs[1][0],
                            outs[2][0], outs[0][1], outs[1][1], outs[2][1])
    for which, name in ((0, "q"), (1, "k"), (2, "v")):
        ref, ref_s = oracle.quantize_e4m3(x[name], wl.seqlens, wl.B)
        got = outs[which][0].view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()
        assert np.array_equal(got, ref)
        assert np.array_equal(outs[which][1].cpu().numpy().astype(np.float64), ref_s)


def test_bounded_wait_times_out_and_context_survives():
    # Fault injection on the host side of the contract: a flag makes the
    # producer never load Q, so the MMA warp's first wait can never complete.
    # Every wait is bounded (~1 s): the kernel must record FP2_STATUS_TIMEOUT,
    # drain its in-flight copies, free tensor memory and return, leaving the
    # context usable for the next call.
    import time
    wl, x = _case("pr1_ref_1k")
    run = GpuRun(wl, x).plan()
    t0 = time.time()
    run.prefill(flags=fb.FP2_DEBUG_DROP_Q_LOAD)
    rc, st = run.status()
    assert rc == fb.FP2_ERR_TIMEOUT and st & fb.FP2_STATUS_TIMEOUT
    assert time.time() - t0 < 30
    run.plan().prefill()
    assert run.status() == (fb.FP2_OK, 0)
    q, k, v = oracle_inputs(x, wl)
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau)
    res = check_attention(wl, x, run, pl)
    assert res["rel_l2"] <= REL_L2_BF16 and res["lse_max_abs"] <= LSE_ABS, res


@pytest.mark.parametrize("pos", [2 * 128 + 40, 5 * 128 + 100, 3 * 128 + 5])
def test_row_maximum_jump_inside_a_tile(pos):
    # One key far larger than every other, in the middle of a later block:
    # rows whose score jumps by far more than the exp2 headroom must move
    # their reference inside the tile (rescaling O, l and the P columns
    # already written for that tile) and still match the oracle.
    wl = synth.small_workload([1100, 900], 8, 2, 128, 128, 0.0, seed=123, generator="normal")
    x = synth.generate(wl)
    x = dict(x)
    k = x["k"].copy()
    k[pos, 0, :] *= 100.0
    x["k"] = synth.bf16_round(k)
    run = GpuRun(wl, x).plan().prefill()
    assert run.status() == (fb.FP2_OK, 0)
    q, kk, v = oracle_inputs(x, wl)
    pl = oracle.plan(q, kk, v, wl.seqlens, wl.B, wl.tau)
    res = check_attention(wl, x, run, pl)
    assert res["finite"], res
    assert res["rel_l2"] <= REL_L2_BF16 and res["lse_max_abs"] <= LSE_ABS, res


@pytest.mark.parametrize("name", ["ragged_d128", "two_pseudo_tiles", "paged_mix_small"])
def test_mean_codes_for_the_fp8_correction(name):
    # e4m3 block means of the FP8 correction, as the header defines them: one
    # scale per chunk of B blocks of a sequence and kv-head, absmax / 448 of
    # the chunk's fp32 means; V means in one e4m3 term (within e4m3's 2^-4
    # relative rounding), K means in two (hi + lo, within 2^-8 relative), both
    # down to the subnormal quantum 2^-9 of the scale
    import torch
    wl, x = _case(name)
    run = GpuRun(wl, x).plan()
    L = run.lay
    NB, Hkv, d, B = int(L.num_blocks), wl.Hkv, wl.d, wl.B
    buf = run.plan_buf

    def arr(off, n, dt):
        return buf[off:off + n * torch.tensor([], dtype=dt).element_size()].view(dt)

    kb = run.view.kbar.cpu().numpy().astype(np.float64)
    vb = run.view.vbar.cpu().numpy().astype(np.float64)
    e4 = torch.float8_e4m3fn
    hi_k = arr(L.off_kbar_e4m3, NB * Hkv * d, e4).float().cpu().numpy().reshape(NB, Hkv, d)
    lo_k = arr(L.off_kbar_e4m3_lo, NB * Hkv * d, e4).float().cpu().numpy().reshape(NB, Hkv, d)
    hi_v = arr(L.off_vbar_e4m3, NB * Hkv * d, e4).float().cpu().numpy().reshape(NB, Hkv, d)
    sk = arr(L.off_kbar_scale, NB * Hkv, torch.float32).cpu().numpy().reshape(NB, Hkv)
    sv = arr(L.off_vbar_scale, NB * Hkv, torch.float32).cpu().numpy().reshape(NB, Hkv)
    b0 = 0
    for Ls in wl.seqlens:
        nb = (Ls + B - 1) // B
        for c0 in range(0, nb, B):
            lo, hi = b0 + c0, b0 + min(c0 + B, nb)
            for g in range(Hkv):
                for mean, scale, approx, rel in ((kb, sk, hi_k + lo_k, 2.0 ** -8),
                                                 (vb, sv, hi_v, 2.0 ** -4)):
                    amax = np.float32(np.abs(mean[lo:hi, g].astype(np.float32)).max())
                    want = amax / np.float32(448.0) if amax > 0 else np.float32(1.0)
                    assert scale[lo, g] == want, (lo, g, scale[lo, g], want)
                    err = np.abs(approx[lo:hi, g] * float(scale[lo, g]) - mean[lo:hi, g])
                    bound = rel * np.abs(mean[lo:hi, g]) + 2.0 ** -10 * float(scale[lo, g])
                    assert np.all(err <= bound * 1.0001), (lo, g, float((err / bound).max()))
        b0 += nb


def _fp8_run(wl, x, run):
    """Quantise q, k, v on the GPU and run the e4m3 prefill; returns the codes,
    scales and outputs."""
    import torch
    NB = int(run.lay.num_blocks)
    out = {}
    for which, src, H in [(0, run.q, wl.Hq), (1, run.k, wl.Hkv), (2, run.v, wl.Hkv)]:
        codes = torch.zeros(src.shape, dtype=torch.uint8, device="cuda")
        scales = torch.zeros((NB, H), dtype=torch.float32, device="cuda")
        fb.fp2_quantize_fp8(run.prob, run.plan_buf, src, which, codes, scales)
        out[which] = (codes, scales)
    o = torch.full((wl.T, wl.Hq, wl.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((wl.Hq, wl.T), float("nan"), dtype=torch.float32, device="cuda")
    fb.fp2_prefill(run.prob, run.plan_buf, out[0][0], out[1][0], out[2][0], o, lse,
                   q_scale=out[0][1], k_scale=out[1][1], v_scale=out[2][1],
                   dtype=fb.FP2_DTYPE_E4M3)
    return o.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("name,gen", [("ragged_d128", "normal"), ("ragged_d128", "lowrank"),
                                      ("B64_d128", "normal"), ("paged_mix_small", "normal"),
                                      ("split_d128_paged", "normal")])
def test_fp8_prefill(name, gen):
    from fp2_harness import rel_l2, token_rows
    seqlens, Hq, Hkv, d, B, tau, _, nn, page, pool = SMALL[name]
    wl = synth.small_workload(seqlens, Hq, Hkv, d, B, tau, seed=700 + len(name), generator=gen,
                              page_size=page, pool_pages=pool)
    x = synth.generate(wl)
    run = GpuRun(wl, x).plan()
    O8, L8 = _fp8_run(wl, x, run)
    assert run.status() == (fb.FP2_OK, 0)
    q, k, v = oracle_inputs(x, wl)
    pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau)
    # the oracle on the quantised inputs (direct online quantisation of Q, K, V;
    # float64 block means of the plan) and on the plain bf16 inputs
    dq = [oracle.dequantize_e4m3(*oracle.quantize_e4m3(a, wl.seqlens, wl.B), wl.seqlens, wl.B)
          for a in (q, k, v)]
    rows = [(s, i) for s in range(len(wl.seqlens)) for i in range((wl.seqlens[s] + B - 1) // B)]
    toks, O_dq, L_dq = oracle.attend_rows(dq[0], dq[1], dq[2], pl, rows)
    _, O_ref, L_ref = oracle.attend_rows(q, k, v, pl, rows)
    assert np.isfinite(O8[toks]).all() and np.isfinite(L8[:, toks]).all()
    e_dq = rel_l2(O8[toks], O_dq)
    e_ref = rel_l2(O8[toks], O_ref)
    l_dq = float(np.max(np.abs(L8[:, toks] - L_dq)))
    print(f"fp8 {name}/{gen}: rel-L2 vs quantised-input oracle {e_dq:.3e}, vs plain {e_ref:.3e}, "
          f"LSE vs quantised-input oracle {l_dq:.3e}")
    assert l_dq <= LSE_ABS
    assert e_dq <= REL_L2_FP8
    assert e_ref <= REL_L2_FP8_PLAIN_GUARD


@pytest.mark.parametrize("name", ["ragged_d128", "paged_mix_small", "B64_d128"])
def test_plan_from_fp8_kv_cache(name):
    # An FP8 KV cache: K and V quantised on the GPU (codes bit-exact with the
    # oracle's quantiser, see test_quantize_fp8_matches_oracle_codes), then
    # planned from the codes and scales; the oracle plans the dequantised cache.
    import torch
    from fp2_harness import dequantised_operands
    wl, x = _case(name)
    run = GpuRun(wl, x).plan()
    NB = int(run.lay.num_blocks)
    kv8 = []
    for which, src in ((1, run.k), (2, run.v)):
        codes = torch.zeros(src.shape, dtype=torch.uint8, device="cuda")
        scales = torch.zeros((NB, wl.Hkv), dtype=torch.float32, device="cuda")
        fb.fp2_quantize_fp8(run.prob, run.plan_buf, src, which, codes, scales)
        kv8.append((codes, scales))
    lay, plan8, ws8 = fb.allocate(run.prob)
    fb.fp2_plan_kv8(run.prob, run.q, kv8[0][0], kv8[1][0], kv8[0][1], kv8[1][1], plan8, ws8)
    rc, st = fb.fp2_status_check(plan8)
    assert (rc, st) == (fb.FP2_OK, 0)
    view = fb.PlanView(plan8, lay, wl.Hkv, wl.d)
    q, k, v = oracle_inputs(x, wl)
    _, k_dq, v_dq = dequantised_operands(wl, q, k, v, [])
    pl = oracle.plan(q, k_dq, v_dq, wl.seqlens, wl.B, wl.tau)
    rp = view.row_ptr.cpu().numpy()
    ci = view.col_idx.cpu().numpy()
    kept = {r: ci[rp[r]:rp[r + 1]].tolist() for r in range(len(rp) - 1)}
    res = compare_plan(pl, kept)
    assert res["outside_band"] == 0, res
    assert np.allclose(view.kbar.cpu().numpy(), pl["kbar"], rtol=2e-7, atol=1e-7)
    assert np.allclose(view.vbar.cpu().numpy(), pl["vbar"], rtol=2e-7, atol=1e-7)
