"""Pins of the chunked-prefill oracle (oracle/fp2_chunked.py) against what
the full-prefill method and the mathematics fix: the full-prefill oracle when
the chunk is the whole sequence, brute-force dense attention at tau = 0 and
whenever the correction is exact (keys constant within each block, B = 1),
the hand example of tests/golden for every chunk start, and explicit loops
for the mean of a partial first query block."""

import math
import os

import numpy as np
import pytest

import oracle
from oracle import fp2_chunked as ch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(seed, kv_lens, Hq, Hkv, d):
    rng = np.random.default_rng(seed)
    T = sum(kv_lens)
    return (rng.standard_normal((T, Hq, d)), rng.standard_normal((T, Hkv, d)) * 1.3,
            rng.standard_normal((T, Hkv, d)))


def _chunk_rows(x, q_lens, kv_lens):
    """The rows of the last q_len positions of each sequence (packed)."""
    parts, t0 = [], 0
    for Q, L in zip(q_lens, kv_lens):
        parts.append(x[t0 + L - Q:t0 + L])
        t0 += L
    return np.concatenate(parts, axis=0)


def _dense_chunk(q_full, k, v, q_lens, kv_lens):
    O, L = oracle.dense_attention(q_full, k, v, kv_lens)
    return _chunk_rows(O, q_lens, kv_lens), _chunk_rows(L.T, q_lens, kv_lens).T


@pytest.mark.parametrize("tau", [0.0, 0.3, 1.0])
def test_whole_sequence_chunk_is_the_full_prefill(tau):
    kv = [40, 23, 9]
    q, k, v = _rand(3, kv, 4, 2, 8)
    pc = ch.plan_chunk(q, k, v, kv, kv, 8, tau)
    pf = oracle.plan(q, k, v, kv, 8, tau)
    assert [list(a) for a in pc["kept"]] == [list(a) for a in pf["kept"]]
    Oc, Lc = ch.attend_chunk(q, k, v, pc)
    Of, Lf = oracle.attend(q, k, v, pf)
    assert np.allclose(Oc, Of, rtol=0, atol=1e-13) and np.allclose(Lc, Lf, rtol=0, atol=1e-13)


def test_tau0_chunk_equals_dense_attention_of_its_rows():
    # chunk starts mid-block, at the sequence start, and on a block boundary
    kv, ql = [40, 23, 17], [13, 23, 1]
    q_full, k, v = _rand(4, kv, 4, 2, 8)
    q = _chunk_rows(q_full, ql, kv)
    pl = ch.plan_chunk(q, k, v, ql, kv, 8, 0.0)
    O, L = ch.attend_chunk(q, k, v, pl)
    Od, Ld = _dense_chunk(q_full, k, v, ql, kv)
    assert np.allclose(O, Od, rtol=0, atol=1e-12) and np.allclose(L, Ld, rtol=0, atol=1e-12)


@pytest.mark.parametrize("tau", [1.0, 0.3, 0.1])
def test_constant_keys_per_block_make_the_chunk_correction_exact(tau):
    kv, ql, B = [48, 29], [21, 5], 8
    rng = np.random.default_rng(31)
    q_full = rng.standard_normal((sum(kv), 4, 8))
    v = rng.standard_normal((sum(kv), 2, 8))
    k = np.empty((sum(kv), 2, 8))
    t0 = 0
    for L in kv:
        for i in range(0, L, B):
            k[t0 + i:t0 + min(i + B, L)] = rng.standard_normal((1, 2, 8)) * 1.5
        t0 += L
    q = _chunk_rows(q_full, ql, kv)
    pl = ch.plan_chunk(q, k, v, ql, kv, B, tau)
    lay = pl["layout"]
    row_i = [i for g in range(2) for s in range(2) for i in range(int(lay["i0"][s]), int(lay["nb"][s]))]
    n_skipped = sum(i + 1 - len(c) for c, i in zip(pl["kept"], row_i))
    assert n_skipped > 0                      # the correction is exercised
    O, L = ch.attend_chunk(q, k, v, pl)
    Od, Ld = _dense_chunk(q_full, k, v, ql, kv)
    assert np.allclose(O, Od, rtol=0, atol=1e-12) and np.allclose(L, Ld, rtol=0, atol=1e-12)
    O0, _ = ch.attend_chunk(q, k, v, pl, correction=False)
    assert not np.allclose(O0, Od, atol=1e-6)   # dropping the surrogate loses mass


def _golden():
    rows = {}
    with open(os.path.join(GOLDEN, "identical_keys_hand_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            t, o, lse = line.split()
            rows[int(t)] = (float(o), float(lse))
    return rows


@pytest.mark.parametrize("Q", [1, 2, 3, 4, 6])
@pytest.mark.parametrize("tau", [1.0, 0.5])
def test_hand_example_for_every_chunk_start(Q, tau):
    # the hand example of tests/golden: the row of query block 2 has
    # Qbar = -1 whatever part of the block the chunk holds
    q_full = np.array([0, 0, 0, 0, -1, -1], dtype=np.float64).reshape(6, 1, 1)
    k = np.array([0, 0, 1, 1, 0, 0], dtype=np.float64).reshape(6, 1, 1)
    v = np.array([0, 0, 2, 4, 0, 0], dtype=np.float64).reshape(6, 1, 1)
    q = q_full[6 - Q:]
    pl = ch.plan_chunk(q, k, v, [Q], [6], 2, tau)
    assert pl["kept"][-1].tolist() == [0, 2] and pl["scores"][-1].tolist() == [0.0, -1.0, 0.0]
    O, L = ch.attend_chunk(q, k, v, pl)
    for t, (o, lse) in _golden().items():
        if t >= 6 - Q:
            assert O[t - (6 - Q), 0, 0] == pytest.approx(o, abs=1e-11)
            assert L[0, t - (6 - Q)] == pytest.approx(lse, abs=1e-11)
    Od, Ld = _dense_chunk(q_full, k, v, [Q], [6])
    assert np.allclose(O, Od, atol=1e-14) and np.allclose(L, Ld, atol=1e-14)


@pytest.mark.parametrize("off,first_equal_row", [(16, 2), (19, 3)])
def test_chunk_rows_after_its_first_block_match_the_full_prefill(off, first_equal_row):
    # a chunk that starts on a block boundary reproduces every full-prefill
    # row from its start; one that starts inside a block differs only in that
    # block (whose query mean covers fewer tokens)
    L, B, tau = 40, 8, 0.4
    q_full, k, v = _rand(5, [L], 4, 1, 8)
    q = q_full[off:]
    pc = ch.plan_chunk(q, k, v, [L - off], [L], B, tau)
    pf = oracle.plan(q_full, k, v, [L], B, tau)
    i0 = off // B
    for i in range(first_equal_row, (L + B - 1) // B):
        assert list(pc["kept"][i - i0]) == list(pf["kept"][i])
        assert np.array_equal(pc["scores"][i - i0], pf["scores"][i])
    Oc, Lc = ch.attend_chunk(q, k, v, pc)
    Of, Lf = oracle.attend(q_full, k, v, pf)
    t = first_equal_row * B
    assert np.allclose(Oc[t - off:], Of[t:], rtol=0, atol=1e-13)
    assert np.allclose(Lc[:, t - off:], Lf[:, t:], rtol=0, atol=1e-13)


def test_partial_first_query_block_mean_by_loops():
    kv, ql, B = [37, 20], [30, 3], 8
    q_full, k, v = _rand(6, kv, 2, 1, 4)
    q = _chunk_rows(q_full, ql, kv)
    pl = ch.plan_chunk(q, k, v, ql, kv, B, 0.2)
    lay = pl["layout"]
    t0q = 0
    for s, (Q, L) in enumerate(zip(ql, kv)):
        off = L - Q
        for n, i in enumerate(range(off // B, (L + B - 1) // B)):
            for h in range(2):
                for e in range(4):
                    tot, cnt = 0.0, 0
                    for p in range(i * B, min((i + 1) * B, L)):
                        if p >= off:
                            tot += float(q[t0q + p - off, h, e])
                            cnt += 1
                    assert pl["qbar"][int(lay["cu_qblocks"][s]) + n, h, e] == pytest.approx(tot / cnt, abs=1e-15)
        t0q += Q


@pytest.mark.parametrize("tau", [1.0, 0.2])
def test_block_size_one_equals_dense_for_any_tau(tau):
    kv, ql = [19, 11], [7, 11]
    q_full, k, v = _rand(7, kv, 2, 1, 4)
    q = _chunk_rows(q_full, ql, kv)
    pl = ch.plan_chunk(q, k, v, ql, kv, 1, tau)
    O, L = ch.attend_chunk(q, k, v, pl)
    Od, Ld = _dense_chunk(q_full, k, v, ql, kv)
    assert np.allclose(O, Od, rtol=0, atol=1e-12) and np.allclose(L, Ld, rtol=0, atol=1e-12)
    assert math.isfinite(float(np.sum(O)))
