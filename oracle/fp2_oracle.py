"""FlashPrefill V2 oracle: plan, attend and dense reference in float64 NumPy.

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.  Slow and plain on
purpose: one (sequence, kv-head, query-block) row at a time, no blocking,
fusion or reordering beyond what the method states.

Notation (follows the pages and the problem statement):
  Hq query heads, Hkv kv-heads, G = Hq / Hkv, head dim d, block size B.
  Sequence s has length L_s and nb_s = ceil(L_s / B) blocks; sequences are
  packed back to back along the token axis ("varlen", cu_seqlens).
  Query head h reads kv-head g = h // G (contiguous groups; the pages do not
  state the grouping -- this is the usual reading).
  A "row" is (s, g, i): all G query heads of kv-head g over query block i.
  Rows are numbered r = g * NB + (blocks before s) + i, NB = sum_s nb_s,
  which is the order of the CSR index ("CSR of selected blocks, per KV
  head", Table 7).

Method (FlashPrefill V2, Figure 3 / Figure 4 / abstract):
  1. Block means  Qbar_{i,h}, Kbar_j, Vbar_j  over each block's own tokens
     (a partial last block averages its real tokens only); n_j = |block j|.
  2. Score  sc_j = max_{h in group g} Qbar_{i,h} . Kbar_j / sqrt(d),
     j = 0..i  ("pattern discovery" under PackGQA).
  3. tau = 0 keeps every causally visible block.  Otherwise, with
     m = max_j sc_j, keep {j : sc_j >= tau * m} plus the sink block 0 and the
     diagonal block i ("max-based dynamic thresholding").
  4. Every other visible block j < i is skipped; it is always a full block.
  5. For a query token at position p (block i) and head h:
        s_u  = q . k_u / sqrt(d)            for tokens u in kept blocks, u <= p
        t_j  = q . Kbar_j / sqrt(d) + ln n_j  for skipped blocks j
     One softmax over both sets (Figure 4's surrogate |B_J| e^{s_J} (v_J, 1)):
        O   = (sum_u e^{s_u} v_u + sum_j e^{t_j} Vbar_j) / (sum_u e^{s_u} + sum_j e^{t_j})
        LSE = ln(sum_u e^{s_u} + sum_j e^{t_j})      (natural log, scaled logits)

Pins (tests/test_oracle.py):
  block_layout, block_means -- constant blocks, partial-block counts, B=1.
  block_scores              -- hand-written triple loop on tiny inputs; a
                               single hot head decides the max.
  select_blocks / plan      -- tau=0 keeps all; tau=1 keeps forced + argmax;
                               nested kept sets (density non-increasing in
                               tau); CSR consistent with the kept lists.
  attend                    -- tau=0 equals dense_attention (<= 1e-12);
                               identical-key blocks make the correction
                               exact (closed form, tests/golden hand example);
                               B=1 equals dense for any tau; constant V gives
                               O = v; LSE non-decreasing as tau falls (Jensen);
                               correction off drops exactly the surrogate.
  dense_attention           -- tiny case against scipy-free explicit softmax
                               loops and against the L=1 / uniform-logit
                               closed forms.
  gather_paged              -- shuffled pages reproduce the contiguous
                               layout exactly.
  e4m3_round                -- every finite e4m3 code is a fixed point; in
                               range it equals torch's float8_e4m3fn cast;
                               saturation at 448.
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------
# Layout helpers (sequence packing, blocks, rows)
# ----------------------------------------------------------------------------

def block_layout(seqlens: Sequence[int], B: int) -> Dict[str, np.ndarray]:
    """Token and block offsets of a varlen batch.

    Returns cu_seqlens [n+1], nb [n] (= ceil(L_s / B)) and cu_blocks [n+1].
    """
    seqlens = np.asarray(seqlens, dtype=np.int64)
    nb = (seqlens + B - 1) // B
    cu_seqlens = np.concatenate([[0], np.cumsum(seqlens)])
    cu_blocks = np.concatenate([[0], np.cumsum(nb)])
    return {"seqlens": seqlens, "cu_seqlens": cu_seqlens, "nb": nb, "cu_blocks": cu_blocks}


def _as64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------
# Step 1: block-mean pooling (Figure 3 "pools block-mean statistics")
# ----------------------------------------------------------------------------

def block_means(x, seqlens: Sequence[int], B: int):
    """Mean of x over each block's own tokens.

    x: [T, H, d] packed varlen tensor.  Returns (means [NB, H, d] float64,
    counts [NB] int64), blocks ordered sequence by sequence.
    """
    x = np.asarray(x)
    lay = block_layout(seqlens, B)
    T, H, d = x.shape
    NB = int(lay["cu_blocks"][-1])
    means = np.zeros((NB, H, d), dtype=np.float64)
    counts = np.zeros(NB, dtype=np.int64)
    for s, L in enumerate(lay["seqlens"]):
        t0 = int(lay["cu_seqlens"][s])
        b0 = int(lay["cu_blocks"][s])
        for i in range(int(lay["nb"][s])):
            lo = t0 + i * B
            hi = t0 + min((i + 1) * B, int(L))
            means[b0 + i] = _as64(x[lo:hi]).mean(axis=0)
            counts[b0 + i] = hi - lo
    return means, counts


# ----------------------------------------------------------------------------
# Steps 2-3: block scores and max-based thresholding
# ----------------------------------------------------------------------------

def block_scores(qbar_i: np.ndarray, kbar: np.ndarray, i: int) -> np.ndarray:
    """sc_j = max over the packed query heads of Qbar_{i,h} . Kbar_j / sqrt(d).

    qbar_i: [G, d] block means of query block i for the G heads of one group.
    kbar:   [nb, d] key block means of the same sequence and kv-head.
    Returns sc [i+1] for the causally visible blocks j = 0..i.
    """
    qbar_i = _as64(qbar_i)
    kbar = _as64(kbar)
    d = qbar_i.shape[-1]
    dots = qbar_i @ kbar[: i + 1].T            # [G, i+1]
    return dots.max(axis=0) / math.sqrt(d)


def select_blocks(sc: np.ndarray, tau: float) -> np.ndarray:
    """Kept block ids (ascending) for one row, given its scores sc[0..i].

    tau == 0 is the dense case: every visible block is kept.  Otherwise a
    block is kept when its score is at least tau times the row maximum
    (ties kept); the sink block 0 and the diagonal block i are always kept.
    """
    i = len(sc) - 1
    if tau == 0.0:
        return np.arange(i + 1, dtype=np.int64)
    m = sc.max()
    keep = sc >= tau * m
    keep[0] = True
    keep[i] = True
    return np.nonzero(keep)[0].astype(np.int64)


def plan(q, k, v, seqlens: Sequence[int], B: int, tau: float,
         rows: Optional[Sequence[tuple]] = None) -> Dict[str, object]:
    """Stage 1 of the pipeline: means, scores, kept lists, CSR and K/V means.

    q [T, Hq, d], k and v [T, Hkv, d] (contiguous; use gather_paged first for
    a paged pool).  Returns a dict with:
      qbar [NB, Hq, d], kbar / vbar [NB, Hkv, d], counts [NB],
      scores  list over rows r of sc[0..i] (float64),
      thresh  list over rows of tau * m (None for tau == 0),
      kept    list over rows of ascending kept block ids (local to the sequence),
      row_ptr [R+1] int64, col_idx [nnz] int64, with R = Hkv * NB.
    rows: optional list of (s, i) query blocks; only their rows (all
      kv-heads) are scored and selected, the others stay None and the CSR is
      not built.
    """
    Hq, Hkv = q.shape[1], k.shape[1]
    assert Hq % Hkv == 0
    G = Hq // Hkv
    lay = block_layout(seqlens, B)
    NB = int(lay["cu_blocks"][-1])
    qbar, counts = block_means(q, seqlens, B)
    kbar, _ = block_means(k, seqlens, B)
    vbar, _ = block_means(v, seqlens, B)

    R = Hkv * NB
    scores: List[Optional[np.ndarray]] = [None] * R
    thresh: List[Optional[float]] = [None] * R
    kept: List[Optional[np.ndarray]] = [None] * R
    if rows is None:
        rows = [(s, i) for s in range(len(lay["seqlens"])) for i in range(int(lay["nb"][s]))]
    for g in range(Hkv):
        heads = list(range(g * G, (g + 1) * G))
        for (s, i) in rows:
            b0 = int(lay["cu_blocks"][s])
            nbs = int(lay["nb"][s])
            kb = kbar[b0:b0 + nbs, g, :]
            r = g * NB + b0 + i
            sc = block_scores(qbar[b0 + i][heads], kb, i)
            scores[r] = sc
            thresh[r] = None if tau == 0.0 else float(tau * sc.max())
            kept[r] = select_blocks(sc, tau)
    row_ptr = col_idx = None
    if all(x is not None for x in kept):
        row_ptr = np.zeros(R + 1, dtype=np.int64)
        for r in range(R):
            row_ptr[r + 1] = row_ptr[r] + len(kept[r])
        col_idx = np.concatenate(kept) if R else np.zeros(0, dtype=np.int64)
    return {
        "B": B, "tau": tau, "Hq": Hq, "Hkv": Hkv, "G": G, "layout": lay,
        "qbar": qbar, "kbar": kbar, "vbar": vbar, "counts": counts,
        "scores": scores, "thresh": thresh, "kept": kept,
        "row_ptr": row_ptr, "col_idx": col_idx,
    }


# ----------------------------------------------------------------------------
# Steps 4-5: attention over kept blocks with mean correction
# ----------------------------------------------------------------------------

def attend_rows(q, k, v, pl: Dict[str, object], rows: Sequence[tuple],
                correction: bool = True, kept_override=None):
    """Stage 2 for the query blocks `rows` = [(s, i), ...] only.

    Returns (toks, O, LSE): toks the packed token indices of those blocks in
    order, O [len(toks), Hq, d] and LSE [Hq, len(toks)] (natural log of the
    softmax denominator in 1/sqrt(d)-scaled logits, pseudo-tokens included).

    pl: output of plan() (block means and kept lists of these rows).
    correction: add one pseudo-token per skipped block (Figure 4); False
      drops skipped blocks entirely.
    kept_override: optional {(s, g, i): kept ids} replacing the plan's
      selection for those rows.
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    B = int(pl["B"])
    G = int(pl["G"])
    Hq, Hkv = int(pl["Hq"]), int(pl["Hkv"])
    lay = pl["layout"]
    NB = int(lay["cu_blocks"][-1])
    kbar, vbar = pl["kbar"], pl["vbar"]
    counts = pl["counts"]
    d = q.shape[2]
    inv_sqrt_d = 1.0 / math.sqrt(d)
    toks, O_parts, L_parts = [], [], []
    for (s, i) in rows:
        t0 = int(lay["cu_seqlens"][s])
        L = int(lay["seqlens"][s])
        b0 = int(lay["cu_blocks"][s])
        qlo, qhi = t0 + i * B, t0 + min((i + 1) * B, L)
        qpos = np.arange(qlo, qhi) - t0                      # positions in the sequence
        O_blk = np.zeros((qhi - qlo, Hq, d))
        L_blk = np.zeros((Hq, qhi - qlo))
        for g in range(Hkv):
            r = g * NB + b0 + i
            kept = pl["kept"][r] if kept_override is None or (s, g, i) not in kept_override \
                else np.asarray(kept_override[(s, g, i)], dtype=np.int64)
            kept_set = set(int(j) for j in kept)
            skipped = [j for j in range(i) if j not in kept_set]
            # exact keys of the kept blocks
            kidx = np.concatenate([np.arange(t0 + j * B, t0 + min((j + 1) * B, L)) for j in kept])
            kpos = kidx - t0
            Kk, Vk = _as64(k[kidx, g, :]), _as64(v[kidx, g, :])
            for h in range(g * G, (g + 1) * G):
                Qh = _as64(q[qlo:qhi, h, :])                   # [n_i, d]
                s_exact = (Qh @ Kk.T) * inv_sqrt_d               # [n_i, nk]
                s_exact = np.where(kpos[None, :] <= qpos[:, None], s_exact, -np.inf)
                if correction and skipped:
                    jb = np.asarray(skipped)
                    s_pseudo = (Qh @ kbar[b0 + jb, g, :].T) * inv_sqrt_d \
                        + np.log(counts[b0 + jb].astype(np.float64))[None, :]
                    V_pseudo = vbar[b0 + jb, g, :]
                else:
                    s_pseudo = np.zeros((qhi - qlo, 0))
                    V_pseudo = np.zeros((0, d))
                M = np.maximum(s_exact.max(axis=1), s_pseudo.max(axis=1, initial=-np.inf))
                w_exact = np.exp(s_exact - M[:, None])
                w_pseudo = np.exp(s_pseudo - M[:, None])
                den = w_exact.sum(axis=1) + w_pseudo.sum(axis=1)
                num = w_exact @ Vk + w_pseudo @ V_pseudo
                O_blk[:, h, :] = num / den[:, None]
                L_blk[h, :] = M + np.log(den)
        toks.append(np.arange(qlo, qhi))
        O_parts.append(O_blk)
        L_parts.append(L_blk)
    if not toks:
        return np.zeros(0, dtype=np.int64), np.zeros((0, Hq, d)), np.zeros((Hq, 0))
    return np.concatenate(toks), np.concatenate(O_parts, axis=0), np.concatenate(L_parts, axis=1)


def attend(q, k, v, pl: Dict[str, object], correction: bool = True,
           rows: Optional[Sequence[tuple]] = None, kept_override=None):
    """Stage 2 for the whole batch (or the query blocks `rows`): O [T, Hq, d]
    and LSE [Hq, T], entries outside `rows` left NaN.  See attend_rows."""
    lay = pl["layout"]
    T, Hq, d = np.shape(q)
    if rows is None:
        rows = [(s, i) for s in range(len(lay["seqlens"])) for i in range(int(lay["nb"][s]))]
    toks, O_r, L_r = attend_rows(q, k, v, pl, rows, correction, kept_override)
    O = np.full((T, Hq, d), np.nan)
    LSE = np.full((Hq, T), np.nan)
    O[toks] = O_r
    LSE[:, toks] = L_r
    return O, LSE


def dense_attention(q, k, v, seqlens: Sequence[int]):
    """Brute-force causal GQA softmax attention (no blocks): the tau = 0
    reference.  The kv-head of query head h is found by repeating each
    kv-head G times along the head axis.
    """
    q = _as64(q)
    k = _as64(k)
    v = _as64(v)
    T, Hq, d = q.shape
    G = Hq // k.shape[1]
    k_rep = np.repeat(k, G, axis=1)
    v_rep = np.repeat(v, G, axis=1)
    O = np.zeros_like(q)
    LSE = np.zeros((Hq, T))
    t0 = 0
    for L in seqlens:
        L = int(L)
        causal = np.tril(np.ones((L, L), dtype=bool))
        for h in range(Hq):
            logits = q[t0:t0 + L, h, :] @ k_rep[t0:t0 + L, h, :].T / math.sqrt(d)
            logits = np.where(causal, logits, -np.inf)
            mx = logits.max(axis=1, keepdims=True)
            w = np.exp(logits - mx)
            den = w.sum(axis=1)
            O[t0:t0 + L, h, :] = (w @ v_rep[t0:t0 + L, h, :]) / den[:, None]
            LSE[h, t0:t0 + L] = mx[:, 0] + np.log(den)
        t0 += L
    return O, LSE


# ----------------------------------------------------------------------------
# Paged KV (page table of fixed-size pages; "paged KV cache", Figure 1)
# ----------------------------------------------------------------------------

def gather_paged(pool, page_table, seqlens: Sequence[int], page_size: int) -> np.ndarray:
    """Read a paged pool [P, page_size, H, d] into the packed layout [T, H, d].

    Token t of sequence s lives in page page_table[s][t // page_size] at slot
    t % page_size.
    """
    pool = np.asarray(pool)
    out = []
    for s, L in enumerate(seqlens):
        for t in range(int(L)):
            out.append(pool[int(page_table[s][t // page_size]), t % page_size])
    return np.stack(out, axis=0)


# ----------------------------------------------------------------------------
# FP8-e4m3 ("direct online FP8 quantization", Table 1 footnote)
# ----------------------------------------------------------------------------

E4M3_MAX = 448.0          # largest finite e4m3 (OCP FP8, "fn" variant: no infinities)
E4M3_MIN_NORMAL_EXP = -6  # exponent bias 7
E4M3_MANT_BITS = 3


def e4m3_round(y) -> np.ndarray:
    """Round to the nearest e4m3 value, ties to even, saturating to +-448.

    From the format's definition: 1 sign, 4 exponent (bias 7), 3 mantissa
    bits; normal numbers step by 2^(e-3) in [2^e, 2^(e+1)), subnormals by
    2^-9 below 2^-6.
    """
    y = _as64(y)
    a = np.abs(y)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, E4M3_MIN_NORMAL_EXP)
    quantum = np.exp2(e - E4M3_MANT_BITS)
    r = np.round(a / quantum) * quantum          # numpy rounds half to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, y)


def quantize_e4m3(x, seqlens: Sequence[int], B: int):
    """Per (block, head) absmax scaling then e4m3 rounding.

    x [T, H, d] (bf16 values).  scale = absmax / 448 (1 when the block is
    all zero); codes = e4m3_round(x / scale), the scale and the quotient
    rounded to float32 as the kernel computes them.  Returns (codes [T, H, d] float64 holding
    e4m3 values, scales [NB, H] float64).
    """
    x = _as64(x)
    lay = block_layout(seqlens, B)
    NB = int(lay["cu_blocks"][-1])
    T, H, d = x.shape
    codes = np.zeros_like(x)
    scales = np.ones((NB, H))
    for s, L in enumerate(lay["seqlens"]):
        t0 = int(lay["cu_seqlens"][s])
        b0 = int(lay["cu_blocks"][s])
        for i in range(int(lay["nb"][s])):
            lo, hi = t0 + i * B, t0 + min((i + 1) * B, int(L))
            for h in range(H):
                # The quotient decides an integer code, so it is taken in
                # float32, the precision the kernel divides in.
                blk = x[lo:hi, h, :].astype(np.float32)
                amax = np.float32(np.abs(blk).max())
                sc = amax / np.float32(E4M3_MAX) if amax > 0 else np.float32(1.0)
                scales[b0 + i, h] = sc
                codes[lo:hi, h, :] = e4m3_round(blk / sc)
    return codes, scales


def dequantize_e4m3(codes, scales, seqlens: Sequence[int], B: int) -> np.ndarray:
    """codes * scale of the (block, head) each element belongs to."""
    codes = _as64(codes)
    lay = block_layout(seqlens, B)
    out = np.zeros_like(codes)
    for s, L in enumerate(lay["seqlens"]):
        t0 = int(lay["cu_seqlens"][s])
        b0 = int(lay["cu_blocks"][s])
        for i in range(int(lay["nb"][s])):
            lo, hi = t0 + i * B, t0 + min((i + 1) * B, int(L))
            out[lo:hi] = codes[lo:hi] * scales[b0 + i][None, :, None]
    return out
