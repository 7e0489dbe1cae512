"""Host check of the error bound the planner's tensor-core scorer relies on.

The scorer multiplies the tf32-rounded block means on the tensor cores
(exact products, fp32 sums) and the threshold decides outright only the
blocks whose score is farther than the bound e_j from the threshold; every
other block is re-scored in float64.  The bound (stated where the library
defines it, next to ``kres_bound``) is, for query means q_h (the G heads of a
row), key mean k_j, t(x) = tf32(fp32(x)) and c_d = d 2^-23 + 2^-22,

    |max_h fl(t(q_h) . t(k_j)) / sqrt d - max_h q_h . k_j / sqrt d|
        <= A |k_j| + B (|k_j - t(k_j)| + c_d (|k_j| + |k_j - t(k_j)|))
    A = max_h |q_h - t(q_h)| / sqrt d,  B = (max_h |q_h| + max_h |q_h - t(q_h)|) / sqrt d.

These tests restate that arithmetic in NumPy (tf32 rounding, fp32 sums in
several orders) and check the inequality on adversarial and on generated
means, so that a term dropped from the derivation shows up here.  They do not
call the library.
"""

import math

import numpy as np
import pytest


def tf32(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (nearest) -> tf32 (nearest even on the 13 dropped bits)."""
    f = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (f >> 13) & 1
    f = (f + 0xFFF + lsb) & 0xFFFFE000
    return f.astype(np.uint32).view(np.float32).astype(np.float64)


def fp32_dot(a: np.ndarray, b: np.ndarray, order: str) -> float:
    """Sum of the exact products a_i b_i, every partial sum rounded to fp32."""
    p = a * b   # exact: both factors have 11 significant bits
    if order == "reverse":
        p = p[::-1]
    if order == "steps8":
        # eight-term groups summed first (one tensor-core K-step each), then the groups
        parts = [fp32_dot(p[i:i + 8], np.ones(min(8, len(p) - i)), "forward") for i in range(0, len(p), 8)]
        return fp32_dot(np.array(parts), np.ones(len(parts)), "forward")
    s = np.float32(0.0)
    for v in p:
        s = np.float32(s + np.float32(v))
    return float(s)


def score_bound(q: np.ndarray, k: np.ndarray) -> float:
    d = q.shape[-1]
    c_d = d * 2.0 ** -23 + 2.0 ** -22
    qr = np.linalg.norm(q - tf32(q), axis=-1).max()
    qn = np.linalg.norm(q, axis=-1).max()
    kn = np.linalg.norm(k)
    kr = np.linalg.norm(k - tf32(k))
    A = qr / math.sqrt(d)
    B = (qn + qr) / math.sqrt(d)
    return A * kn + B * (kr + c_d * (kn + kr))


def tc_score(q: np.ndarray, k: np.ndarray, order: str) -> float:
    d = q.shape[-1]
    inv = float(np.float32(1.0 / math.sqrt(d)))
    return max(float(np.float32(fp32_dot(tf32(qh), tf32(k), order) * inv)) for qh in q)


def exact_score(q: np.ndarray, k: np.ndarray) -> float:
    return float((q @ k).max() / math.sqrt(q.shape[-1]))


@pytest.mark.parametrize("order", ["forward", "reverse", "steps8"])
@pytest.mark.parametrize("d", [64, 128])
def test_bound_holds_on_random_means(order, d):
    rng = np.random.default_rng(1234 + d)
    worst = 0.0
    for trial in range(60):
        G = int(rng.choice([1, 2, 4, 8]))
        scale = 10.0 ** rng.uniform(-3, 3)
        q = rng.standard_normal((G, d)) * scale * rng.uniform(0.1, 3.0, size=(G, 1))
        k = rng.standard_normal(d) * 10.0 ** rng.uniform(-3, 3)
        if trial % 3 == 0:   # a few dominant components, as in needle blocks
            k[rng.integers(0, d, 3)] *= 50.0
        err = abs(tc_score(q, k, order) - exact_score(q, k))
        e = score_bound(q, k)
        assert err <= e, (trial, err, e)
        worst = max(worst, err / e)
    assert worst > 0.0


@pytest.mark.parametrize("order", ["forward", "steps8"])
def test_bound_holds_when_every_rounding_points_the_same_way(order):
    # components just above a tf32 midpoint all round down (and the key's all
    # round the same way), so the residual terms add up instead of cancelling
    d = 128
    ulp = 2.0 ** -10                       # tf32 spacing on [1, 2)
    q = np.full((1, d), 1.0 + 0.49 * ulp)  # rounds down by 0.49 ulp
    k = np.full(d, 1.0 + 0.49 * ulp)
    err = abs(tc_score(q, k, order) - exact_score(q, k))
    assert err <= score_bound(q, k)
    # the residual terms carry this case: without them the bound would fail
    qn, kn = np.linalg.norm(q), np.linalg.norm(k)
    c_d = d * 2.0 ** -23 + 2.0 ** -22
    assert err > c_d * qn * kn / math.sqrt(d)


def test_bound_is_tight_relative_to_the_worst_case():
    # on typical means the residual norms sit well below 2^-11 |x|, which is
    # what keeps the band of blocks the threshold must re-score narrow
    rng = np.random.default_rng(7)
    d = 128
    ratios = []
    for _ in range(200):
        q = rng.standard_normal((4, d))
        k = rng.standard_normal(d)
        worst = (2 * 2.0 ** -11 + d * 2.0 ** -23) * np.linalg.norm(q, axis=-1).max() * np.linalg.norm(k) / math.sqrt(d)
        ratios.append(score_bound(q, k) / worst)
    assert 0.1 < float(np.median(ratios)) < 0.5
