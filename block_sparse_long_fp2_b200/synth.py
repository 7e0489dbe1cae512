"""Seeded synthetic inputs shaped like the long-context prefill workloads.

This module only draws random numbers and lays them out: it holds none of
the attention method's arithmetic, so both the CUDA path (tests, bench) and
the float64 oracle read the same canonical tensors from it.

All tensors are float32 arrays whose values are exactly representable in
bfloat16 (rounded to nearest-even from the float32 draw); ``bf16_bits``
turns them into the uint16 bit patterns the device receives.

Recipes (the pages measure on needle-in-a-haystack RULER prompts of real
models, which are not available; these stand in for them):

* ``needles``  -- Q, K, V ~ N(0, 1) plus planted needles: a random unit
  direction u, a query block b and a key position p in an earlier,
  non-sink block; K[p] is set to 4u and 4u is added to every query row of
  block b in the heads of that kv-head group.
Every head draws from its own generator spawned from the workload seed.

* ``normal``   -- Q, K, V ~ N(0, 1).
* ``lowrank``  -- Q, K = N(0, 1) + z W_g with W_g in R^{4 x d} ~ N(0, 1)
  per kv-head, shared by the keys of kv-head g and the queries of its
  group, and z ~ N(0, I_4) drawn per token and head (per-entry std of the
  shared part about 2).  The keys of the first 4 tokens of every sequence
  are scaled by 8 (attention sinks).  V ~ N(0, 1).
* ``lowrank+needles`` -- ``lowrank`` plus needles at uniform positions.
* ``topics``   -- block-level structure that the block means carry (the
  retrieval structure that makes the pages' real prompts 5-9 % dense): per
  kv-head, ``n_topics`` orthonormal directions w_t; every key block j draws
  a topic t_j and every query block i a topic t'_i (uniform, per kv-head);
  K = N(0, 1) + 3 w_{t_j} on the tokens of block j, Q = N(0, 1) + 3 w_{t'_i}
  on the tokens of block i (all G query heads of the kv-head), V ~ N(0, 1).
  A block's score is about 9 / sqrt(d) when the topics match and near zero
  otherwise, so a threshold between them keeps about 1 / n_topics of the
  blocks (plus the forced sink and diagonal blocks).

A paged layout places every sequence's 64-token pages at a seeded random
permutation of a larger pool.  Whole pages that no sequence uses are filled
with NaN (a stray page read shows up as NaN), and the slots after the end
of a sequence in its last page hold the finite sentinel 100.0.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------
# bfloat16 canonicalisation
# ----------------------------------------------------------------------------

def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), in place
    when possible; returns float32 holding bf16-exact values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1).view(np.uint32)
    chunk = 1 << 20
    for lo in range(0, flat.size, chunk):
        u = flat[lo:lo + chunk]
        lsb = (u >> np.uint32(16)) & np.uint32(1)
        lsb += np.uint32(0x7FFF)
        u += lsb
        u &= np.uint32(0xFFFF0000)
    return x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of a float32 array of bf16-exact values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    """float32 values of uint16 bf16 bit patterns."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# Problem description
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    seqlens: List[int]
    Hq: int
    Hkv: int
    d: int
    B: int
    tau: float
    generator: str = "lowrank"
    n_needles: int = 0
    page_size: int = 0          # 0 = contiguous K/V, else paged
    pool_pages: int = 0         # pages in the pool when paged
    dtype: str = "bf16"
    seed: int = 0
    n_topics: int = 0           # "topics" generator: topics per kv-head

    @property
    def T(self) -> int:
        return int(sum(self.seqlens))


def workloads() -> Dict[str, Workload]:
    """The named workloads: a small reference case, two single-layer shapes
    (32K and 128K), a paged continuous-batching mix and a length sweep."""
    w = {
        "pr1_ref_1k": Workload("pr1_ref_1k", [1024], 4, 1, 64, 64, 0.3, "needles", 8, seed=1000),
        "llama_32k": Workload("llama_32k", [32768], 32, 8, 128, 128, 0.1, "lowrank", 0, seed=1001),
        "qwen_128k": Workload("qwen_128k", [131072], 32, 8, 128, 128, 0.05, "lowrank+needles", 64,
                              seed=1002),
        "paged_mix": Workload("paged_mix", [4096, 9000, 16384, 30000, 65536, 1500], 32, 8, 128, 128,
                              0.1, "lowrank", 0, page_size=64, pool_pages=2048, seed=1003),
    }
    # low-density layers: the 128K shape with block-level topics, about 5, 10
    # and 20 % of the blocks kept (Table 3's 64K-128K densities are 4.6-9.4 %)
    for pct, nt in ((5, 20), (10, 10), (20, 5)):
        name = f"topics_128k_{pct}pct"
        w[name] = Workload(name, [131072], 32, 8, 128, 128, 0.5, "topics", 0, seed=1100 + pct,
                           n_topics=nt)
    for li, L in enumerate([4096, 8192, 16384, 32768, 65536, 131072]):
        for ti, tau in enumerate([0.0, 0.05, 0.2]):
            name = f"sweep_{L // 1024}k_tau{tau:g}"
            w[name] = Workload(name, [L], 32, 8, 128, 128, tau, "lowrank", 0,
                               seed=1004 + 10 * li + ti)
    return w


# ----------------------------------------------------------------------------
# Generators
# ----------------------------------------------------------------------------

def _normal(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def _fill_head(seed_seq, out: np.ndarray, h: int, W: Optional[np.ndarray]) -> None:
    """out[:, h, :] = N(0, 1) (+ z W when W is given), from the head's own
    generator so the result does not depend on thread scheduling."""
    rng = np.random.Generator(np.random.PCG64(seed_seq))
    T, _, d = out.shape
    if W is None:
        out[:, h, :] = _normal(rng, (T, d))
        return
    z = _normal(rng, (T, W.shape[0]))
    out[:, h, :] = _normal(rng, (T, d))
    out[:, h, :] += z @ W


def _fill_head_topic(seed_seq, out: np.ndarray, h: int, dirs: np.ndarray, tok_topic: np.ndarray,
                     amp: float) -> None:
    """out[:, h, :] = N(0, 1) + amp * dirs[tok_topic[t]] (the topic direction of
    the block each token t belongs to), from the head's own generator."""
    rng = np.random.Generator(np.random.PCG64(seed_seq))
    T, _, d = out.shape
    out[:, h, :] = _normal(rng, (T, d))
    chunk = 1 << 16
    for lo in range(0, T, chunk):
        hi = min(T, lo + chunk)
        out[lo:hi, h, :] += amp * dirs[tok_topic[lo:hi]]


def _fill_heads(children, out: np.ndarray, Ws) -> None:
    import concurrent.futures
    import os
    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        list(ex.map(lambda h: _fill_head(children[h], out, h, Ws[h]), range(out.shape[1])))


def _plant_needles(rng, q, k, seqlens, Hkv, B, n_needles, first_qblock=2) -> List[tuple]:
    """Plant needles; returns (seq, kv_head, q_block, key_pos) tuples."""
    Hq, d = q.shape[1], q.shape[2]
    G = Hq // Hkv
    cu = np.concatenate([[0], np.cumsum(seqlens)])
    planted = []
    for _ in range(n_needles):
        s = int(rng.integers(0, len(seqlens)))
        nb = (int(seqlens[s]) + B - 1) // B
        if nb <= first_qblock:
            continue
        b = int(rng.integers(first_qblock, nb))
        p = int(rng.integers(B, b * B))
        g = int(rng.integers(0, Hkv))
        u = _normal(rng, (d,)).astype(np.float64)
        u /= np.linalg.norm(u)
        u4 = (4.0 * u).astype(np.float32)
        k[cu[s] + p, g, :] = u4
        lo, hi = cu[s] + b * B, cu[s] + min((b + 1) * B, int(seqlens[s]))
        q[lo:hi, g * G:(g + 1) * G, :] += u4[None, None, :]
        planted.append((s, g, b, p))
    return planted


def generate(wl: Workload) -> Dict[str, object]:
    """Canonical inputs for a workload.

    Returns q [T, Hq, d], k, v [T, Hkv, d] (float32, bf16-exact), the
    contiguous cu_seqlens, and for paged workloads k_pool / v_pool
    [P, page, Hkv, d] and page_table [n, max_pages] (int32, unused = -1).
    """
    ss = np.random.SeedSequence(wl.seed)
    kids = ss.spawn(wl.Hq + 2 * wl.Hkv + 1)
    rng = np.random.Generator(np.random.PCG64(kids[-1]))      # W, needles, pages
    T, Hq, Hkv, d = wl.T, wl.Hq, wl.Hkv, wl.d
    G = Hq // Hkv
    q = np.empty((T, Hq, d), dtype=np.float32)
    k = np.empty((T, Hkv, d), dtype=np.float32)
    v = np.empty((T, Hkv, d), dtype=np.float32)
    if wl.generator.startswith("lowrank"):
        W = _normal(rng, (Hkv, 4, d))
        _fill_heads(kids[:Hq], q, [W[h // G] for h in range(Hq)])
        _fill_heads(kids[Hq:Hq + Hkv], k, [W[g] for g in range(Hkv)])
        t0 = 0
        for L in wl.seqlens:
            k[t0:t0 + min(4, L)] *= 8.0
            t0 += L
    elif wl.generator == "topics":
        nt = wl.n_topics
        assert 1 <= nt <= d
        # per kv-head orthonormal topic directions; per (kv-head, block) topics
        dirs = [np.linalg.qr(rng.standard_normal((d, nt)))[0].T.astype(np.float32)
                for _ in range(Hkv)]
        nbs = [(L + wl.B - 1) // wl.B for L in wl.seqlens]
        NB = int(sum(nbs))
        ktop = rng.integers(0, nt, size=(Hkv, NB))
        qtop = rng.integers(0, nt, size=(Hkv, NB))
        tok_block = np.concatenate([b0 + np.arange(L) // wl.B for b0, L in
                                    zip(np.concatenate([[0], np.cumsum(nbs)[:-1]]), wl.seqlens)])
        import concurrent.futures
        import os
        with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
            jobs = [ex.submit(_fill_head_topic, kids[h], q, h, dirs[h // G], qtop[h // G][tok_block], 3.0)
                    for h in range(Hq)]
            jobs += [ex.submit(_fill_head_topic, kids[Hq + g], k, g, dirs[g], ktop[g][tok_block], 3.0)
                     for g in range(Hkv)]
            for j in jobs:
                j.result()
    elif wl.generator == "needles" or wl.generator == "normal":
        _fill_heads(kids[:Hq], q, [None] * Hq)
        _fill_heads(kids[Hq:Hq + Hkv], k, [None] * Hkv)
    else:
        raise ValueError(wl.generator)
    _fill_heads(kids[Hq + Hkv:Hq + 2 * Hkv], v, [None] * Hkv)
    planted = []
    if wl.n_needles:
        planted = _plant_needles(rng, q, k, wl.seqlens, Hkv, wl.B, wl.n_needles)
    bf16_round(q)
    bf16_round(k)
    bf16_round(v)
    out = {"q": q, "k": k, "v": v, "needles": planted,
           "cu_seqlens": np.concatenate([[0], np.cumsum(wl.seqlens)]).astype(np.int32)}
    if wl.page_size:
        out.update(make_paged(rng, k, v, wl.seqlens, wl.page_size, wl.pool_pages))
    return out


def make_paged(rng, k: np.ndarray, v: np.ndarray, seqlens: Sequence[int], page: int,
               pool_pages: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Scatter contiguous k, v into a shuffled page pool.

    NaN fills unused pages; 100.0 fills the slots past a sequence's end in
    its last page.
    """
    n_pages = [(int(L) + page - 1) // page for L in seqlens]
    total = int(sum(n_pages))
    P = int(pool_pages) if pool_pages else total
    assert P >= total
    perm = rng.permutation(P)[:total]
    Hkv, d = k.shape[1], k.shape[2]
    k_pool = np.full((P, page, Hkv, d), np.nan, dtype=np.float32)
    v_pool = np.full((P, page, Hkv, d), np.nan, dtype=np.float32)
    table = np.full((len(seqlens), max(n_pages) if n_pages else 1), -1, dtype=np.int32)
    t0 = 0
    c = 0
    for s, L in enumerate(seqlens):
        L = int(L)
        for pg in range(n_pages[s]):
            pid = int(perm[c])
            c += 1
            table[s, pg] = pid
            lo = pg * page
            n = min(page, L - lo)
            k_pool[pid, :n] = k[t0 + lo:t0 + lo + n]
            v_pool[pid, :n] = v[t0 + lo:t0 + lo + n]
            if n < page:
                k_pool[pid, n:] = 100.0
                v_pool[pid, n:] = 100.0
        t0 += L
    return {"k_pool": k_pool, "v_pool": v_pool, "page_table": table}


def small_workload(seqlens, Hq, Hkv, d, B, tau, seed, generator="lowrank", n_needles=0,
                   page_size=0, pool_pages=0, n_topics=0) -> Workload:
    """A test-sized workload with the same generators."""
    return Workload(f"small_{seed}", list(seqlens), Hq, Hkv, d, B, tau, generator, n_needles,
                    page_size=page_size, pool_pages=pool_pages, seed=seed, n_topics=n_topics)


def sample_qblocks(nb: int, count: int, seed: int) -> List[int]:
    """Seeded sample of query blocks of one sequence, always holding the
    first and the last block."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if nb <= count:
        return list(range(nb))
    mid = rng.choice(np.arange(1, nb - 1), size=count - 2, replace=False)
    return sorted([0, nb - 1] + [int(x) for x in mid])
