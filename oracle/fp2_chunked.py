"""FlashPrefill V2 oracle for chunked prefill: a chunk of new queries over a
KV cache that already holds the sequence's earlier tokens.

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

The pages name chunked prefill only as a serving mode (Table 6: open-loop
serving with chunk sizes of 8K and 16K) and say nothing of how the selection
treats a chunk.  Reading taken here (the plainest one the rest supports):

  * Sequence s has kv_len L_s keys/values (earlier tokens + the chunk) and
    q_len Q_s <= L_s new queries, at positions off_s = L_s - Q_s .. L_s - 1.
  * Blocks sit on the absolute position grid of the sequence: key block j
    covers positions [jB, (j+1)B) ∩ [0, L_s) and its means Kbar_j, Vbar_j and
    count n_j are those of the full-prefill method.
  * Query block i covers the chunk's positions in [iB, (i+1)B); the rows are
    the query blocks i = floor(off_s / B) .. nb_s - 1.  Qbar_i is the mean of
    the chunk's queries in block i (the first one may be partial at its
    start: the earlier positions have no query in this call).
  * Scores, thresholding, forced blocks {0, i}, skipped blocks and the
    pseudo-token correction are those of the full-prefill method (Figure 3,
    Figure 4, max-based dynamic thresholding), with causality by absolute
    position.  With Q_s = L_s this is exactly the full prefill.

Rows are numbered r = g * NQ + (query blocks of earlier sequences) + (i - i0_s),
NQ the total number of query blocks.  Queries are packed [sum Q_s, Hq, d]
(cu_q); keys and values [sum L_s, Hkv, d] (cu_kv).

Pins (tests/test_oracle_chunked.py): Q_s = L_s equals the full-prefill
oracle; tau = 0 equals brute-force dense attention of the chunk's rows; keys
constant within each block make the correction exact for any tau (and the
hand example of tests/golden reproduces for every chunk start); a chunk that
starts on a block boundary reproduces the full prefill's rows; Qbar of a
partial first query block by explicit loops; B = 1 equals dense for any tau.
"""

from __future__ import annotations

import math
from typing import Dict, List, Sequence

import numpy as np

from .fp2_oracle import block_means, block_scores, select_blocks


def chunk_layout(q_lens: Sequence[int], kv_lens: Sequence[int], B: int) -> Dict[str, np.ndarray]:
    """Offsets of a chunked batch: cu_q, cu_kv, off (= L - Q), nb (key blocks),
    i0 (first query block), nq (query blocks) and cu_qblocks, cu_kvblocks."""
    q_lens = np.asarray(q_lens, dtype=np.int64)
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    assert q_lens.shape == kv_lens.shape
    assert np.all(q_lens >= 1) and np.all(q_lens <= kv_lens)
    off = kv_lens - q_lens
    nb = (kv_lens + B - 1) // B
    i0 = off // B
    nq = nb - i0
    return {
        "q_lens": q_lens, "kv_lens": kv_lens, "off": off, "nb": nb, "i0": i0, "nq": nq,
        "cu_q": np.concatenate([[0], np.cumsum(q_lens)]),
        "cu_kv": np.concatenate([[0], np.cumsum(kv_lens)]),
        "cu_qblocks": np.concatenate([[0], np.cumsum(nq)]),
        "cu_kvblocks": np.concatenate([[0], np.cumsum(nb)]),
    }


def query_positions(lay: Dict[str, np.ndarray], s: int, i: int, B: int) -> np.ndarray:
    """Absolute positions of the chunk's queries in query block i of sequence s."""
    lo = max(i * B, int(lay["off"][s]))
    hi = min((i + 1) * B, int(lay["kv_lens"][s]))
    return np.arange(lo, hi)


def query_block_means(q, lay: Dict[str, np.ndarray], B: int) -> np.ndarray:
    """Qbar [NQ, Hq, d] (float64): mean of the chunk's queries in each query block."""
    q = np.asarray(q)
    NQ = int(lay["cu_qblocks"][-1])
    out = np.zeros((NQ, q.shape[1], q.shape[2]))
    for s in range(len(lay["q_lens"])):
        tq0, off, c0 = int(lay["cu_q"][s]), int(lay["off"][s]), int(lay["cu_qblocks"][s])
        for n, i in enumerate(range(int(lay["i0"][s]), int(lay["nb"][s]))):
            pos = query_positions(lay, s, i, B)
            out[c0 + n] = np.asarray(q[tq0 + pos - off], dtype=np.float64).mean(axis=0)
    return out


def plan_chunk(q, k, v, q_lens: Sequence[int], kv_lens: Sequence[int], B: int,
               tau: float) -> Dict[str, object]:
    """Stage 1 for a chunked batch: Qbar of the chunk's query blocks, Kbar /
    Vbar of every key block, scores, thresholds and kept lists of every row."""
    Hq, Hkv = np.shape(q)[1], np.shape(k)[1]
    assert Hq % Hkv == 0
    G = Hq // Hkv
    lay = chunk_layout(q_lens, kv_lens, B)
    qbar = query_block_means(q, lay, B)
    kbar, counts = block_means(k, lay["kv_lens"], B)
    vbar, _ = block_means(v, lay["kv_lens"], B)
    NQ = int(lay["cu_qblocks"][-1])
    R = Hkv * NQ
    scores: List[np.ndarray] = [None] * R
    thresh: List[float] = [None] * R
    kept: List[np.ndarray] = [None] * R
    for g in range(Hkv):
        heads = list(range(g * G, (g + 1) * G))
        for s in range(len(lay["q_lens"])):
            b0, nbs = int(lay["cu_kvblocks"][s]), int(lay["nb"][s])
            c0 = int(lay["cu_qblocks"][s])
            for n, i in enumerate(range(int(lay["i0"][s]), nbs)):
                r = g * NQ + c0 + n
                sc = block_scores(qbar[c0 + n][heads], kbar[b0:b0 + nbs, g, :], i)
                scores[r] = sc
                thresh[r] = None if tau == 0.0 else float(tau * sc.max())
                kept[r] = select_blocks(sc, tau)
    return {"B": B, "tau": tau, "Hq": Hq, "Hkv": Hkv, "G": G, "layout": lay, "qbar": qbar,
            "kbar": kbar, "vbar": vbar, "counts": counts, "scores": scores,
            "thresh": thresh, "kept": kept}


def attend_chunk(q, k, v, pl: Dict[str, object], correction: bool = True):
    """Stage 2 for a chunked batch: O [sum Q, Hq, d] and LSE [Hq, sum Q]
    (natural log of the softmax denominator in 1/sqrt(d)-scaled logits,
    pseudo-tokens included), one query block row at a time."""
    q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
    B, G = int(pl["B"]), int(pl["G"])
    Hq, Hkv = int(pl["Hq"]), int(pl["Hkv"])
    lay = pl["layout"]
    NQ = int(lay["cu_qblocks"][-1])
    kbar, vbar, counts = pl["kbar"], pl["vbar"], pl["counts"]
    d = q.shape[2]
    inv_sqrt_d = 1.0 / math.sqrt(d)
    O = np.full((q.shape[0], Hq, d), np.nan)
    LSE = np.full((Hq, q.shape[0]), np.nan)
    for s in range(len(lay["q_lens"])):
        tq0, tk0 = int(lay["cu_q"][s]), int(lay["cu_kv"][s])
        off, L = int(lay["off"][s]), int(lay["kv_lens"][s])
        b0, c0 = int(lay["cu_kvblocks"][s]), int(lay["cu_qblocks"][s])
        for n, i in enumerate(range(int(lay["i0"][s]), int(lay["nb"][s]))):
            qpos = query_positions(lay, s, i, B)
            qidx = tq0 + qpos - off
            for g in range(Hkv):
                kept = pl["kept"][g * NQ + c0 + n]
                kept_set = set(int(j) for j in kept)
                skipped = [j for j in range(i) if j not in kept_set]
                kpos = np.concatenate([np.arange(j * B, min((j + 1) * B, L)) for j in kept])
                Kk = np.asarray(k[tk0 + kpos, g, :], dtype=np.float64)
                Vk = np.asarray(v[tk0 + kpos, g, :], dtype=np.float64)
                for h in range(g * G, (g + 1) * G):
                    Qh = np.asarray(q[qidx, h, :], dtype=np.float64)
                    s_exact = (Qh @ Kk.T) * inv_sqrt_d
                    s_exact = np.where(kpos[None, :] <= qpos[:, None], s_exact, -np.inf)
                    if correction and skipped:
                        jb = np.asarray(skipped)
                        s_pseudo = (Qh @ kbar[b0 + jb, g, :].T) * inv_sqrt_d \
                            + np.log(counts[b0 + jb].astype(np.float64))[None, :]
                        V_pseudo = vbar[b0 + jb, g, :]
                    else:
                        s_pseudo = np.zeros((len(qidx), 0))
                        V_pseudo = np.zeros((0, d))
                    M = np.maximum(s_exact.max(axis=1), s_pseudo.max(axis=1, initial=-np.inf))
                    w_exact = np.exp(s_exact - M[:, None])
                    w_pseudo = np.exp(s_pseudo - M[:, None])
                    den = w_exact.sum(axis=1) + w_pseudo.sum(axis=1)
                    O[qidx, h, :] = (w_exact @ Vk + w_pseudo @ V_pseudo) / den[:, None]
                    LSE[h, qidx] = M + np.log(den)
    return O, LSE
