"""Pins for the float64 oracle (CPU only).

Each test fixes the oracle to something other than itself: closed forms,
a hand-worked example, brute force on tiny inputs, invariants the method
implies, and a library routine where one computes the same thing.
"""

import math
import os

import numpy as np
import pytest

import oracle
from block_sparse_long_fp2_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_inputs(seqlens, Hq, Hkv, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    T = sum(seqlens)
    q = rng.standard_normal((T, Hq, d)) * scale
    k = rng.standard_normal((T, Hkv, d)) * scale
    v = rng.standard_normal((T, Hkv, d))
    return q, k, v


# ---------------------------------------------------------------------------
# block means
# ---------------------------------------------------------------------------

def test_block_means_partial_block_uses_own_count():
    # seq of 5 tokens, B=2: blocks {0,1}, {2,3}, {4}; x_t = t
    x = np.arange(5, dtype=np.float64).reshape(5, 1, 1)
    m, n = oracle.block_means(x, [5], 2)
    assert n.tolist() == [2, 2, 1]
    assert m[:, 0, 0].tolist() == [0.5, 2.5, 4.0]


def test_block_means_varlen_and_constant_blocks():
    seqlens = [3, 7]
    x = np.zeros((10, 2, 4))
    x[:3] = 1.0
    x[3:] = -2.0
    m, n = oracle.block_means(x, seqlens, 4)
    assert n.tolist() == [3, 4, 3]
    assert np.all(m[0] == 1.0) and np.all(m[1:] == -2.0)


def test_block_means_b1_is_identity():
    q, _, _ = _rand_inputs([6, 3], 2, 1, 5, seed=1)
    m, n = oracle.block_means(q, [6, 3], 1)
    assert np.array_equal(m, q) and np.all(n == 1)


# ---------------------------------------------------------------------------
# scores and selection
# ---------------------------------------------------------------------------

def test_block_scores_match_hand_loops():
    rng = np.random.default_rng(3)
    G, d, nb = 3, 5, 6
    qbar_i = rng.standard_normal((G, d))
    kbar = rng.standard_normal((nb, d))
    i = 4
    sc = oracle.block_scores(qbar_i, kbar, i)
    assert sc.shape == (i + 1,)
    for j in range(i + 1):
        best = -np.inf
        for h in range(G):
            acc = 0.0
            for e in range(d):
                acc += qbar_i[h, e] * kbar[j, e]
            best = max(best, acc / math.sqrt(d))
        assert abs(sc[j] - best) < 1e-12


def test_one_hot_head_decides_the_max():
    d = 4
    qbar = np.zeros((2, d))
    qbar[1, 0] = 10.0           # only head 1 aligns with block 2's key mean
    kbar = np.zeros((3, d))
    kbar[2, 0] = 1.0
    kbar[1, 1] = 1.0
    sc = oracle.block_scores(qbar, kbar, 2)
    assert sc[2] == pytest.approx(10.0 / 2.0) and sc[1] == 0.0


def test_select_tau0_keeps_all_and_tau1_keeps_forced_and_argmax():
    sc = np.array([-1.0, 0.3, 2.0, 0.7, -0.5])
    assert oracle.select_blocks(sc, 0.0).tolist() == [0, 1, 2, 3, 4]
    assert oracle.select_blocks(sc, 1.0).tolist() == [0, 2, 4]
    assert oracle.select_blocks(sc, 0.3).tolist() == [0, 2, 3, 4]   # 0.7 >= 0.6 kept, 0.3 < 0.6
    # ties at the threshold are kept
    assert oracle.select_blocks(np.array([0.0, 1.0, 0.5, 0.0]), 0.5).tolist() == [0, 1, 2, 3]
    # negative maximum: the literal rule, forced blocks still kept
    sc_neg = np.array([-3.0, -1.0, -2.0, -4.0])
    # m = -1, threshold -0.5: no score reaches it, only the forced blocks remain
    assert oracle.select_blocks(sc_neg, 0.5).tolist() == [0, 3]
    assert oracle.select_blocks(sc_neg, 1.0).tolist() == [0, 1, 3]   # -1 >= -1


def test_plan_csr_consistent_and_nested_in_tau():
    wl = synth.small_workload([300, 129], 4, 2, 16, 32, 0.1, seed=11)
    x = synth.generate(wl)
    dens = []
    prev = None
    for tau in [1.0, 0.5, 0.3, 0.2, 0.1, 0.05, 0.02, 0.0]:
        pl = oracle.plan(x["q"], x["k"], x["v"], wl.seqlens, wl.B, tau)
        rp, ci = pl["row_ptr"], pl["col_idx"]
        R = len(pl["kept"])
        assert rp[0] == 0 and rp[-1] == len(ci)
        for r in range(R):
            assert np.array_equal(ci[rp[r]:rp[r + 1]], pl["kept"][r])
            kept = pl["kept"][r]
            assert np.all(np.diff(kept) > 0)
            i = len(pl["scores"][r]) - 1
            assert kept[0] == 0 and kept[-1] == i
            if prev is not None:          # kept sets are nested as tau falls
                assert set(prev["kept"][r].tolist()) <= set(kept.tolist())
        dens.append(len(ci))
        prev = pl
    assert all(a <= b for a, b in zip(dens, dens[1:]))
    nb = [(L + wl.B - 1) // wl.B for L in wl.seqlens]
    assert dens[-1] == wl.Hkv * sum(n * (n + 1) // 2 for n in nb)


def test_plan_row_order_is_kv_head_major():
    wl = synth.small_workload([200, 90], 4, 2, 8, 32, 0.2, seed=5)
    x = synth.generate(wl)
    pl = oracle.plan(x["q"], x["k"], x["v"], wl.seqlens, wl.B, wl.tau)
    NB = 7 + 3
    assert len(pl["kept"]) == 2 * NB
    # row of (s=1, g=1, i=2) is g*NB + (blocks before s) + i
    r = 1 * NB + 7 + 2
    assert len(pl["scores"][r]) == 3
    qbar, _ = oracle.block_means(x["q"], wl.seqlens, wl.B)
    kbar, _ = oracle.block_means(x["k"], wl.seqlens, wl.B)
    expect = (qbar[9, 2:4] @ kbar[7:10, 1].T).max(axis=0) / math.sqrt(8)
    assert np.allclose(pl["scores"][r], expect, rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seqlens,Hq,Hkv,d,B", [([37], 2, 1, 8, 8), ([20, 33, 5], 4, 2, 6, 4),
                                                 ([64], 8, 8, 4, 16), ([17, 9], 3, 1, 5, 8)])
def test_tau0_equals_brute_force_dense(seqlens, Hq, Hkv, d, B):
    q, k, v = _rand_inputs(seqlens, Hq, Hkv, d, seed=sum(seqlens) + Hq, scale=1.5)
    pl = oracle.plan(q, k, v, seqlens, B, 0.0)
    O, L = oracle.attend(q, k, v, pl)
    Od, Ld = oracle.dense_attention(q, k, v, seqlens)
    assert np.max(np.abs(O - Od)) <= 1e-12
    assert np.max(np.abs(L - Ld)) <= 1e-12


def test_dense_attention_closed_forms():
    # L=1: output is the single value, LSE is the single logit
    q = np.array([[[2.0, 0.0]]])
    k = np.array([[[1.5, 7.0]]])
    v = np.array([[[3.0, -1.0]]])
    O, L = oracle.dense_attention(q, k, v, [1])
    assert np.allclose(O[0, 0], [3.0, -1.0]) and L[0, 0] == pytest.approx(3.0 / math.sqrt(2))
    # all logits zero: O_t = mean of v_0..v_t and LSE_t = ln(t+1)
    T = 6
    q = np.zeros((T, 1, 3))
    k = np.random.default_rng(0).standard_normal((T, 1, 3))
    v = np.random.default_rng(1).standard_normal((T, 1, 3))
    O, L = oracle.dense_attention(q, k, v, [T])
    for t in range(T):
        assert np.allclose(O[t, 0], v[:t + 1, 0].mean(axis=0), atol=1e-14)
        assert L[0, t] == pytest.approx(math.log(t + 1), abs=1e-14)


def test_dense_attention_explicit_loops():
    seqlens = [5, 4]
    q, k, v = _rand_inputs(seqlens, 4, 2, 3, seed=9)
    O, L = oracle.dense_attention(q, k, v, seqlens)
    t0 = 0
    for Ls in seqlens:
        for h in range(4):
            g = h // 2
            for a in range(Ls):
                w = [math.exp(float(q[t0 + a, h] @ k[t0 + b, g]) / math.sqrt(3)) for b in range(a + 1)]
                den = sum(w)
                num = sum(wi * v[t0 + b, g] for b, wi in enumerate(w))
                assert np.allclose(O[t0 + a, h], num / den, atol=1e-13)
                assert L[h, t0 + a] == pytest.approx(math.log(den), abs=1e-13)
        t0 += Ls


def _golden_hand_example():
    rows = {}
    with open(os.path.join(GOLDEN, "identical_keys_hand_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            t, o, lse = line.split()
            rows[int(t)] = (float(o), float(lse))
    return rows


@pytest.mark.parametrize("tau", [1.0, 0.5, 0.05])
def test_hand_example_identical_keys(tau):
    q = np.array([0, 0, 0, 0, -1, -1], dtype=np.float64).reshape(6, 1, 1)
    k = np.array([0, 0, 1, 1, 0, 0], dtype=np.float64).reshape(6, 1, 1)
    v = np.array([0, 0, 2, 4, 0, 0], dtype=np.float64).reshape(6, 1, 1)
    pl = oracle.plan(q, k, v, [6], 2, tau)
    assert pl["kept"][2].tolist() == [0, 2]          # block 1 skipped
    assert pl["scores"][2].tolist() == [0.0, -1.0, 0.0]
    O, L = oracle.attend(q, k, v, pl)
    for t, (o, lse) in _golden_hand_example().items():
        assert O[t, 0, 0] == pytest.approx(o, abs=1e-11)
        assert L[0, t] == pytest.approx(lse, abs=1e-11)
    Od, Ld = oracle.dense_attention(q, k, v, [6])
    assert np.allclose(O, Od, atol=1e-14) and np.allclose(L, Ld, atol=1e-14)
    # without the correction the skipped mass is simply lost
    O0, L0 = oracle.attend(q, k, v, pl, correction=False)
    assert O0[5, 0, 0] == 0.0 and L0[0, 5] == pytest.approx(math.log(4.0))


@pytest.mark.parametrize("tau", [1.0, 0.3, 0.1])
def test_identical_key_blocks_make_correction_exact(tau):
    seqlens, Hq, Hkv, d, B = [48, 29], 4, 2, 8, 8
    rng = np.random.default_rng(21)
    T = sum(seqlens)
    q = rng.standard_normal((T, Hq, d))
    k = np.empty((T, Hkv, d))
    t0 = 0
    for L in seqlens:              # every block's keys are one repeated vector
        for i in range(0, L, B):
            k[t0 + i:t0 + min(i + B, L)] = rng.standard_normal((1, Hkv, d)) * 1.5
        t0 += L
    v = rng.standard_normal((T, Hkv, d))
    pl = oracle.plan(q, k, v, seqlens, B, tau)
    assert len(pl["col_idx"]) < Hkv * (21 + 10)   # something was skipped
    O, L = oracle.attend(q, k, v, pl)
    Od, Ld = oracle.dense_attention(q, k, v, seqlens)
    assert np.max(np.abs(O - Od)) <= 1e-12 and np.max(np.abs(L - Ld)) <= 1e-12
    # and the uncorrected output is measurably different
    O0, _ = oracle.attend(q, k, v, pl, correction=False)
    assert np.max(np.abs(O0 - Od)) > 1e-3


def test_block_size_one_is_dense_for_any_tau():
    seqlens = [13, 6]
    q, k, v = _rand_inputs(seqlens, 2, 1, 4, seed=4, scale=2.0)
    Od, Ld = oracle.dense_attention(q, k, v, seqlens)
    for tau in [1.0, 0.5, 0.1]:
        pl = oracle.plan(q, k, v, seqlens, 1, tau)
        O, L = oracle.attend(q, k, v, pl)
        assert np.max(np.abs(O - Od)) <= 1e-12 and np.max(np.abs(L - Ld)) <= 1e-12


def test_constant_v_gives_constant_output():
    seqlens = [70]
    q, k, _ = _rand_inputs(seqlens, 4, 2, 6, seed=8, scale=2.0)
    v = np.broadcast_to(np.array([1.25, -3.0, 0.5, 0.0, 2.0, 7.0]), (70, 2, 6)).copy()
    for tau in [1.0, 0.2]:
        pl = oracle.plan(q, k, v, seqlens, 8, tau)
        O, _ = oracle.attend(q, k, v, pl)
        assert np.max(np.abs(O - v[0, 0])) <= 1e-12


def test_lse_rises_monotonically_as_tau_falls():
    wl = synth.small_workload([256, 160], 4, 2, 16, 16, 0.1, seed=31, generator="lowrank")
    x = synth.generate(wl)
    Od, Ld = oracle.dense_attention(x["q"], x["k"], x["v"], wl.seqlens)
    prev = None
    skipped_any = False
    for tau in [1.0, 0.5, 0.3, 0.2, 0.1, 0.05, 0.02, 0.0]:
        pl = oracle.plan(x["q"], x["k"], x["v"], wl.seqlens, wl.B, tau)
        _, L = oracle.attend(x["q"], x["k"], x["v"], pl)
        if prev is not None:
            assert np.all(L >= prev - 1e-12)
            skipped_any |= bool(np.any(L > prev + 1e-9))
        prev = L
    assert skipped_any
    assert np.max(np.abs(prev - Ld)) <= 1e-12


def test_correction_lse_lies_between_uncorrected_and_dense():
    # Jensen: a skipped block's tokens contribute sum_t e^{q.k_t} >= n e^{q.Kbar},
    # so the pseudo-token (Figure 4) adds a lower bound of the skipped mass:
    # LSE without correction <= LSE with correction <= dense LSE, row by row,
    # for every tau; the first inequality is strict where a block is skipped.
    wl = synth.small_workload([768, 320], 4, 2, 32, 32, 0.1, seed=37, generator="normal")
    x = synth.generate(wl)
    _, Ld = oracle.dense_attention(x["q"], x["k"], x["v"], wl.seqlens)
    strict = False
    for tau in [0.05, 0.2, 0.5, 1.0]:
        pl = oracle.plan(x["q"], x["k"], x["v"], wl.seqlens, wl.B, tau)
        _, L1 = oracle.attend(x["q"], x["k"], x["v"], pl, correction=True)
        _, L0 = oracle.attend(x["q"], x["k"], x["v"], pl, correction=False)
        assert np.all(L0 <= L1 + 1e-12)
        assert np.all(L1 <= Ld + 1e-12)
        strict |= bool(np.any(L1 > L0 + 1e-6))
    assert strict


def test_gqa_grouping_matches_replicated_heads():
    seqlens = [40]
    q, k, v = _rand_inputs(seqlens, 4, 2, 6, seed=12, scale=1.5)
    pl = oracle.plan(q, k, v, seqlens, 8, 0.3)
    O, L = oracle.attend(q, k, v, pl)
    # G=1 per head on one-head problems built by hand from kv-head h // 2
    for h in range(4):
        qh = q[:, h:h + 1, :]
        kh = k[:, h // 2:h // 2 + 1, :]
        vh = v[:, h // 2:h // 2 + 1, :]
        # same selection: the group shares one kept list, so pass it through
        over = {(0, 0, i): pl["kept"][(h // 2) * 5 + i] for i in range(5)}
        pl1 = oracle.plan(qh, kh, vh, seqlens, 8, 0.3)
        O1, L1 = oracle.attend(qh, kh, vh, pl1, kept_override=over)
        assert np.max(np.abs(O1[:, 0] - O[:, h])) <= 1e-13
        assert np.max(np.abs(L1[0] - L[h])) <= 1e-13


def test_rows_subset_matches_full():
    wl = synth.small_workload([200, 77], 4, 1, 8, 16, 0.2, seed=17)
    x = synth.generate(wl)
    pl = oracle.plan(x["q"], x["k"], x["v"], wl.seqlens, wl.B, wl.tau)
    O, L = oracle.attend(x["q"], x["k"], x["v"], pl)
    Os, Ls = oracle.attend(x["q"], x["k"], x["v"], pl, rows=[(0, 3), (1, 4)])
    assert np.array_equal(Os[48:64], O[48:64]) and np.array_equal(Ls[:, 200 + 64:277], L[:, 264:277])
    assert np.isnan(Os[0, 0, 0])
    toks, Or, Lr = oracle.attend_rows(x["q"], x["k"], x["v"], pl, [(1, 4), (0, 3)])
    assert toks.tolist() == list(range(264, 277)) + list(range(48, 64))
    assert np.array_equal(Or, O[toks]) and np.array_equal(Lr, L[:, toks])


# ---------------------------------------------------------------------------
# paged layout
# ---------------------------------------------------------------------------

def test_paged_equal_length_batch_matches_contiguous_exactly():
    seqlens = [96, 96, 96]
    wl = synth.small_workload(seqlens, 4, 2, 8, 32, 0.2, seed=41)
    x = synth.generate(wl)
    rng = np.random.default_rng(5)
    paged = synth.make_paged(rng, x["k"], x["v"], seqlens, 16, pool_pages=30)
    kg = oracle.gather_paged(paged["k_pool"], paged["page_table"], seqlens, 16)
    vg = oracle.gather_paged(paged["v_pool"], paged["page_table"], seqlens, 16)
    assert np.array_equal(kg, x["k"]) and np.array_equal(vg, x["v"])
    pl = oracle.plan(x["q"], kg, vg, seqlens, wl.B, wl.tau)
    O, L = oracle.attend(x["q"], kg, vg, pl)
    # each sequence alone in contiguous layout
    for s in range(3):
        sl = slice(96 * s, 96 * (s + 1))
        pls = oracle.plan(x["q"][sl], x["k"][sl], x["v"][sl], [96], wl.B, wl.tau)
        Os, Ls = oracle.attend(x["q"][sl], x["k"][sl], x["v"][sl], pls)
        assert np.array_equal(Os, O[sl]) and np.array_equal(Ls, L[:, sl])


def test_paged_pool_sentinels():
    wl = synth.small_workload([70, 10], 2, 1, 4, 8, 0.2, seed=2, page_size=64, pool_pages=5)
    x = synth.generate(wl)
    pt = x["page_table"]
    assert pt.shape == (2, 2) and pt[1, 1] == -1
    used = set(pt[pt >= 0].tolist())
    unused = [p for p in range(5) if p not in used]
    assert all(np.all(np.isnan(x["k_pool"][p])) for p in unused)
    assert np.all(x["k_pool"][pt[0, 1], 6:] == 100.0)
    assert np.all(x["v_pool"][pt[1, 0], 10:] == 100.0)


# ---------------------------------------------------------------------------
# FP8 e4m3
# ---------------------------------------------------------------------------

def _all_e4m3_values():
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue            # NaN code
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            vals += [v, -v]
    return np.array(sorted(set(vals)))


def test_e4m3_codes_are_fixed_points_and_max_is_448():
    vals = _all_e4m3_values()
    assert vals.max() == 448.0 and len(vals) == 253   # 126 magnitudes * 2 + zero
    assert np.array_equal(oracle.e4m3_round(vals), vals)
    assert oracle.e4m3_round(np.array([1e6, -500.0, 449.0]) ).tolist() == [448.0, -448.0, 448.0]


def test_e4m3_matches_torch_cast_in_range():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    y = np.concatenate([rng.standard_normal(20000) * s for s in [1e-3, 0.05, 1, 30, 140]])
    vals = _all_e4m3_values()
    mids = (vals[1:] + vals[:-1]) / 2          # exact ties
    y = np.concatenate([y, mids[np.abs(mids) < 448]]).astype(np.float32)
    y = y[np.abs(y) <= 448.0]                  # torch casts beyond the range to NaN
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.e4m3_round(y), ref)


def test_quantize_roundtrip_error_bound_and_scales():
    wl = synth.small_workload([100, 40], 2, 1, 8, 32, 0.1, seed=3)
    x = synth.generate(wl)
    codes, scales = oracle.quantize_e4m3(x["q"], wl.seqlens, wl.B)
    assert scales.shape == (4 + 2, 2)
    assert np.all(np.abs(codes) <= 448.0)
    deq = oracle.dequantize_e4m3(codes, scales, wl.seqlens, wl.B)
    # relative error of e4m3 rounding is at most 2^-4 for normal values
    big = np.abs(x["q"]) > 2.0 ** -6 * scales.max() * 4
    rel = np.abs(deq - x["q"])[big] / np.abs(x["q"])[big]
    assert rel.max() <= 2.0 ** -4 + 1e-7
    # the block absmax maps to 448 exactly
    assert np.isclose(np.abs(codes[:32, 0]).max(), 448.0)
    z = np.zeros((8, 1, 4))
    cz, sz = oracle.quantize_e4m3(z, [8], 8)
    assert np.all(cz == 0) and sz[0, 0] == 1.0


def test_e4m3_operand_rounding_alone_moves_o_by_percents():
    # The FP8 path's own definition: Q, K, V rounded to e4m3 with one absmax
    # scale per (block, head), then exact attention.  The rounding alone moves
    # O by a few percent (rel-L2) from the unquantised result -- about 4e-2 on
    # N(0, 1) inputs and 6e-2 on the low-rank generator, whose large logits
    # amplify the 2^-4 relative rounding of Q and K -- so an FP8 kernel's
    # parity is taken against the oracle on the dequantised operands, and its
    # distance to the plain oracle is a property of the format, not a defect.
    def rel(a, b):
        return float(np.linalg.norm((a - b).ravel()) / np.linalg.norm(b.ravel()))

    errs = {}
    for gen in ("normal", "lowrank"):
        wl = synth.small_workload([700, 333], 8, 2, 128, 128, 0.1, seed=711, generator=gen)
        x = synth.generate(wl)
        q, k, v = x["q"], x["k"], x["v"]
        pl = oracle.plan(q, k, v, wl.seqlens, wl.B, wl.tau)
        dq = [oracle.dequantize_e4m3(*oracle.quantize_e4m3(a, wl.seqlens, wl.B), wl.seqlens, wl.B)
              for a in (q, k, v)]
        rows = [(s, i) for s in range(2) for i in range((wl.seqlens[s] + 127) // 128)]
        _, O, _ = oracle.attend_rows(q, k, v, pl, rows)
        _, O8, _ = oracle.attend_rows(dq[0], dq[1], dq[2], pl, rows)
        _, Ov, _ = oracle.attend_rows(q, k, dq[2], pl, rows)
        errs[gen] = (rel(O8, O), rel(Ov, O))
        # V alone: a weighted mean of values each off by at most 2^-4 relative
        assert errs[gen][1] < 2.0 ** -4
    assert 2e-2 < errs["normal"][0] < 5e-2
    assert errs["lowrank"][0] > 5e-2
    assert errs["lowrank"][0] > errs["normal"][0]
