"""GPU parity of chunked prefill: a chunk of new queries per sequence over K/V
that hold the sequence's earlier tokens too, through the C ABI
(q_seqlens / cu_q_seqlens), against the float64 chunked-prefill oracle.

Block lists must match bit-exactly outside the 1e-5 threshold band on every
row of the chunk (rows of query blocks below a chunk keep nothing); O within
rel-L2 1e-2 and LSE within 1e-3 on every query of the chunk.
"""

import numpy as np
import pytest

import oracle
from oracle import fp2_chunked as ch
from block_sparse_long_fp2_b200 import binding as fb
from block_sparse_long_fp2_b200 import synth

from fp2_harness import LSE_ABS, REL_L2_BF16, compare_plan, oracle_inputs, rel_l2, to_bf16_device

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
    # name: (kv lengths, chunk lengths, Hq, Hkv, d, B, tau, generator, page_size, pool_pages)
    "mid_block": ([1000], [300], 8, 2, 128, 128, 0.1, "lowrank", 0, 0),
    "varlen_B64": ([1500, 700, 2000], [1500, 129, 1], 8, 2, 128, 64, 0.2, "normal", 0, 0),
    "paged": ([1500, 640], [200, 640], 8, 2, 128, 128, 0.1, "lowrank", 64, 40),
    "dense_d64": ([900, 300], [450, 100], 4, 1, 64, 64, 0.0, "normal", 0, 0),
    "split_rows": ([4096], [2048], 2, 1, 64, 64, 0.2, "lowrank", 0, 0),
}


def _chunk(x, q_lens, kv_lens):
    parts, t0 = [], 0
    for Q, L in zip(q_lens, kv_lens):
        parts.append(x[t0 + L - Q:t0 + L])
        t0 += L
    return np.concatenate(parts, axis=0)


class ChunkRun:
    def __init__(self, name, seed=700):
        import torch
        kv, ql, Hq, Hkv, d, B, tau, gen, page, pool = CASES[name]
        self.kv, self.ql, self.B, self.tau = kv, ql, B, tau
        self.wl = synth.small_workload(kv, Hq, Hkv, d, B, tau, seed=seed + sorted(CASES).index(name),
                                       generator=gen, page_size=page, pool_pages=pool)
        x = synth.generate(self.wl)
        self.x = x
        self.q_full, self.k64, self.v64 = oracle_inputs(x, self.wl)
        self.q64 = _chunk(self.q_full, ql, kv)
        self.Tq = sum(ql)
        self.q = to_bf16_device(_chunk(np.asarray(x["q"]), ql, kv))
        self.cu = torch.from_numpy(np.asarray(x["cu_seqlens"], dtype=np.int32)).cuda()
        self.cu_q = torch.from_numpy(np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)).cuda()
        extra = {}
        if page:
            self.k = to_bf16_device(x["k_pool"])
            self.v = to_bf16_device(x["v_pool"])
            self.pt = torch.from_numpy(np.ascontiguousarray(x["page_table"])).cuda()
            extra = dict(page_size=64, page_table=self.pt, num_pages=int(x["k_pool"].shape[0]))
        else:
            self.k = to_bf16_device(x["k"])
            self.v = to_bf16_device(x["v"])
        self.prob = fb.Problem(kv, self.cu, Hq, Hkv, d, B, tau, q_seqlens=ql,
                               cu_q_seqlens=self.cu_q, **extra)
        self.lay, self.plan_buf, self.ws = fb.allocate(self.prob)
        self.view = fb.PlanView(self.plan_buf, self.lay, Hkv, d)
        self.Hq, self.Hkv, self.d = Hq, Hkv, d

    def run(self, flags=0):
        import torch
        fb.fp2_plan(self.prob, self.q, self.k, self.v, self.plan_buf, self.ws)
        self.o = torch.full((self.Tq, self.Hq, self.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.full((self.Hq, self.Tq), float("nan"), dtype=torch.float32, device="cuda")
        fb.fp2_prefill(self.prob, self.plan_buf, self.q, self.k, self.v, self.o, self.lse, flags=flags)
        rc, st = fb.fp2_status_check(self.plan_buf)
        assert rc == fb.FP2_OK and st == 0, (rc, st)
        return self

    def kept_lists(self):
        rp = self.view.row_ptr.cpu().numpy()
        ci = self.view.col_idx.cpu().numpy()
        return {r: ci[rp[r]:rp[r + 1]].tolist() for r in range(len(rp) - 1)}


def _rows(run, pl):
    """(GPU row, oracle row) of every chunk row; the GPU rows of query blocks
    below a chunk."""
    lay = pl["layout"]
    NB = int(lay["cu_kvblocks"][-1])
    NQ = int(lay["cu_qblocks"][-1])
    active, inactive = [], []
    for g in range(run.Hkv):
        for s in range(len(run.kv)):
            b0, c0 = int(lay["cu_kvblocks"][s]), int(lay["cu_qblocks"][s])
            i0 = int(lay["i0"][s])
            for i in range(int(lay["nb"][s])):
                if i < i0:
                    inactive.append(g * NB + b0 + i)
                else:
                    active.append((g * NB + b0 + i, g * NQ + c0 + i - i0))
    return active, inactive


@pytest.mark.parametrize("name", sorted(CASES))
def test_chunked_prefill_matches_oracle(name):
    run = ChunkRun(name).run()
    pl = ch.plan_chunk(run.q64, run.k64, run.v64, run.ql, run.kv, run.B, run.tau)
    active, inactive = _rows(run, pl)
    gk = run.kept_lists()
    assert all(gk[r] == [] for r in inactive)
    # the oracle's rows renumbered as the GPU's (band-aware list comparison)
    R = len(gk)
    remap = {"kept": [None] * R, "scores": [None] * R, "thresh": [None] * R}
    for rg, ro in active:
        for key in remap:
            remap[key][rg] = pl[key][ro]
    res = compare_plan(remap, gk, rows=[rg for rg, _ in active])
    assert res["outside_band"] == 0, res
    # attention over the GPU's lists (they equal the oracle's outside the band)
    override = {}
    for rg, ro in active:
        if gk[rg] != list(pl["kept"][ro]):
            override[ro] = np.asarray(gk[rg], dtype=np.int64)
    for ro, kept in override.items():
        pl["kept"][ro] = kept
    O_ref, L_ref = ch.attend_chunk(run.q64, run.k64, run.v64, pl)
    O = run.o.float().cpu().numpy()
    L = run.lse.cpu().numpy()
    assert np.isfinite(O).all() and np.isfinite(L).all()
    assert rel_l2(O, O_ref) <= REL_L2_BF16
    assert float(np.max(np.abs(L - L_ref))) <= LSE_ABS
    if name == "split_rows":
        assert run.lay.num_split_slots > 0
    if name == "dense_d64":
        Od, Ld = oracle.dense_attention(run.q_full, run.k64, run.v64, run.kv)
        assert rel_l2(O, _chunk(Od, run.ql, run.kv)) <= REL_L2_BF16
        assert float(np.max(np.abs(L - _chunk(Ld.T, run.ql, run.kv).T))) <= LSE_ABS


def test_whole_sequence_chunk_equals_the_full_prefill_bitwise():
    # q_seqlens = seqlens runs the chunk kernels with every offset zero
    import torch
    run = ChunkRun("varlen_B64")
    kv = run.kv
    full_q = to_bf16_device(np.asarray(run.x["q"]))
    cu_q = run.cu.clone()
    prob_c = fb.Problem(kv, run.cu, run.Hq, run.Hkv, run.d, run.B, run.tau, q_seqlens=kv,
                        cu_q_seqlens=cu_q)
    prob_f = fb.Problem(kv, run.cu, run.Hq, run.Hkv, run.d, run.B, run.tau)
    outs = []
    for prob in (prob_c, prob_f):
        lay, plan, ws = fb.allocate(prob)
        fb.fp2_plan(prob, full_q, run.k, run.v, plan, ws)
        o = torch.zeros((sum(kv), run.Hq, run.d), dtype=torch.bfloat16, device="cuda")
        lse = torch.zeros((run.Hq, sum(kv)), dtype=torch.float32, device="cuda")
        fb.fp2_prefill(prob, plan, full_q, run.k, run.v, o, lse)
        rc, st = fb.fp2_status_check(plan)
        assert rc == fb.FP2_OK and st == 0
        view = fb.PlanView(plan, lay, run.Hkv, run.d)
        outs.append((view.row_ptr.cpu().numpy(), view.col_idx.cpu().numpy()[:int(view.row_ptr[-1])],
                     o.cpu(), lse.cpu()))
    (rp1, ci1, o1, l1), (rp2, ci2, o2, l2) = outs
    assert np.array_equal(rp1, rp2) and np.array_equal(ci1, ci2)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _dq_chunk_q(run):
    """The chunk's queries after direct online quantisation per (query block,
    head) over the chunk positions in the block (the first block may be
    partial), by the oracle's quantiser: codes, scales per global block and
    the dequantised values."""
    B = run.B
    nbs = [(L + B - 1) // B for L in run.kv]
    cu_b = np.concatenate([[0], np.cumsum(nbs)])
    q = np.asarray(run.q64)
    codes = np.zeros_like(q)
    deq = np.zeros_like(q)
    scales = np.ones((int(cu_b[-1]), q.shape[1]))
    t0 = 0
    for s, (L, Q) in enumerate(zip(run.kv, run.ql)):
        off = L - Q
        for i in range(off // B, nbs[s]):
            lo, hi = max(i * B, off) - off + t0, min((i + 1) * B, L) - off + t0
            c, sc = oracle.quantize_e4m3(q[lo:hi], [hi - lo], hi - lo)
            codes[lo:hi] = c
            scales[cu_b[s] + i] = sc[0]
            deq[lo:hi] = oracle.dequantize_e4m3(c, sc, [hi - lo], hi - lo)
        t0 += Q
    return codes, scales, deq


def _dq_full(a, lens, B):
    """K or V after direct online quantisation per (block, head)."""
    c, sc = oracle.quantize_e4m3(a, lens, B)
    return oracle.dequantize_e4m3(c, sc, lens, B)


@pytest.mark.parametrize("name", ["mid_block", "varlen_B64", "paged"])
def test_chunked_fp8_matches_oracle(name):
    # the e4m3 path on a chunk: Q quantised per query block over its chunk
    # positions (codes and scales bit-exact with the oracle's quantiser), K / V
    # per block; O / LSE against the chunked oracle on the quantised inputs
    # (float64 block means of the plan)
    import torch
    from fp2_harness import REL_L2_FP8
    run = ChunkRun(name).run()
    NB = int(run.lay.num_blocks)
    out = {}
    for which, src, H in ((0, run.q, run.Hq), (1, run.k, run.Hkv), (2, run.v, run.Hkv)):
        codes = torch.zeros(src.shape, dtype=torch.uint8, device="cuda")
        scales = torch.ones((NB, H), dtype=torch.float32, device="cuda")
        fb.fp2_quantize_fp8(run.prob, run.plan_buf, src, which, codes, scales)
        out[which] = (codes, scales)
    qc, qs, q_dq = _dq_chunk_q(run)
    got_c = out[0][0].view(torch.float8_e4m3fn).float().cpu().numpy()
    assert np.array_equal(got_c.astype(np.float64), qc)
    assert np.array_equal(out[0][1].cpu().numpy(), qs.astype(np.float32))
    o = torch.full((run.Tq, run.Hq, run.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((run.Hq, run.Tq), float("nan"), dtype=torch.float32, device="cuda")
    fb.fp2_prefill(run.prob, run.plan_buf, out[0][0], out[1][0], out[2][0], o, lse,
                   q_scale=out[0][1], k_scale=out[1][1], v_scale=out[2][1],
                   dtype=fb.FP2_DTYPE_E4M3)
    assert fb.fp2_status_check(run.plan_buf) == (fb.FP2_OK, 0)
    pl = ch.plan_chunk(run.q64, run.k64, run.v64, run.ql, run.kv, run.B, run.tau)
    active, _ = _rows(run, pl)
    gk = run.kept_lists()
    for rg, ro in active:
        if gk[rg] != list(pl["kept"][ro]):
            pl["kept"][ro] = np.asarray(gk[rg], dtype=np.int64)
    O_dq, L_dq = ch.attend_chunk(q_dq, _dq_full(run.k64, run.kv, run.B),
                                 _dq_full(run.v64, run.kv, run.B), pl)
    O = o.float().cpu().numpy()
    L = lse.cpu().numpy()
    assert np.isfinite(O).all() and np.isfinite(L).all()
    e = rel_l2(O, O_dq)
    l_err = float(np.max(np.abs(L - L_dq)))
    print(f"fp8 chunk {name}: rel-L2 {e:.3e}, LSE {l_err:.3e}")
    assert e <= REL_L2_FP8 and l_err <= LSE_ABS


@pytest.mark.parametrize("name", ["mid_block", "varlen_B64", "paged"])
def test_chunk_with_held_block_means(name):
    # a serving caller keeps the K / V block means of earlier blocks: passing
    # them (prev_kbar / prev_vbar) for the blocks wholly before each chunk must
    # give the same plan and outputs as pooling those blocks again; entries of
    # the other blocks are poisoned with NaN and must not be read
    import torch
    run = ChunkRun(name).run()
    full = fb.Problem(run.kv, run.cu, run.Hq, run.Hkv, run.d, run.B, run.tau,
                      **({} if not run.wl.page_size else
                         dict(page_size=64, page_table=run.pt, num_pages=int(run.x["k_pool"].shape[0]))))
    lay_f, plan_f, ws_f = fb.allocate(full)
    full_q = to_bf16_device(np.asarray(run.x["q"]))
    fb.fp2_plan(full, full_q, run.k, run.v, plan_f, ws_f)
    assert fb.fp2_status_check(plan_f) == (fb.FP2_OK, 0)
    vf = fb.PlanView(plan_f, lay_f, run.Hkv, run.d)
    kb, vb = vf.kbar.clone(), vf.vbar.clone()
    # poison every block that is not wholly before its sequence's chunk
    b0 = 0
    for L, Q in zip(run.kv, run.ql):
        nb = (L + run.B - 1) // run.B
        keep = (L - Q) // run.B
        kb[b0 + keep:b0 + nb] = float("nan")
        vb[b0 + keep:b0 + nb] = float("nan")
        b0 += nb
    extra = {} if not run.wl.page_size else dict(page_size=64, page_table=run.pt,
                                                 num_pages=int(run.x["k_pool"].shape[0]))
    prob = fb.Problem(run.kv, run.cu, run.Hq, run.Hkv, run.d, run.B, run.tau, q_seqlens=run.ql,
                      cu_q_seqlens=run.cu_q, prev_kbar=kb, prev_vbar=vb, **extra)
    lay, plan, ws = fb.allocate(prob)
    fb.fp2_plan(prob, run.q, run.k, run.v, plan, ws)
    o = torch.zeros_like(run.o)
    lse = torch.zeros_like(run.lse)
    fb.fp2_prefill(prob, plan, run.q, run.k, run.v, o, lse)
    assert fb.fp2_status_check(plan) == (fb.FP2_OK, 0)
    view = fb.PlanView(plan, lay, run.Hkv, run.d)
    assert torch.equal(view.kbar, run.view.kbar) and torch.equal(view.vbar, run.view.vbar)
    n = int(run.view.row_ptr[-1])
    assert torch.equal(view.row_ptr, run.view.row_ptr)
    assert torch.equal(view.col_idx[:n], run.view.col_idx[:n])
    assert torch.equal(o, run.o) and torch.equal(lse, run.lse)
