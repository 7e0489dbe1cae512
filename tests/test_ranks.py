"""Multi-rank host logic of bench.py on CPU: gloo ranks, no GPU.

On N GPUs the layer is split by kv-head: rank r runs its contiguous share of
the kv-heads (with their query heads) in place in the full-layer tensors, and
the ranks exchange nothing on the data path; torch.distributed only takes the
maximum of the device times over ranks, and the reported value is the whole
layer's work over that time.  These tests run that logic with world size 2 on
the gloo backend: the ranks' slices cover every kv-head exactly once, every
rank sees the same maximum, and the reference arm runs on rank 0 only.
"""

import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from block_sparse_long_fp2_b200 import synth
        wl = synth.workloads()["qwen_128k"]
        h0, hn = bench.rank_slice(wl, world, rank)
        # gather every rank's slice: together they must cover the layer once
        slices = [None] * world
        dist.all_gather_object(slices, (h0, hn))
        # the slice's problem: G * hn query heads, in place in the full tensors
        from block_sparse_long_fp2_b200 import binding as fb
        p = fb.Problem(wl.seqlens, 0x1000, (wl.Hq // wl.Hkv) * hn, hn, wl.d, wl.B, wl.tau,
                       kv_head_begin=h0, num_kv_heads_total=wl.Hkv)
        rows = int(fb.fp2_plan_sizes(p).num_rows)
        # per-rank "device times": the slower rank decides
        times = bench.max_over_ranks([10.0 + rank, 5.0 - rank], world, "cpu")
        value = bench.whole_job_value(bench.dense_equiv_flop(wl), times[0])
        # the reference arm runs on rank 0 only
        args = type("A", (), {"workload": "pr1_ref_1k", "steps": 1, "warmup": 0})()
        ref = bench.run_reference(args, rank, world)
        queue.put((rank, slices, rows, times, value,
                   None if ref is None else (ref["impl"], ref["n_gpus"], ref["cpu_baseline"]["kind"])))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_one_layer_by_kv_head():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(queue.get(timeout=240) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    (r0, sl0, rows0, times0, val0, ref0), (r1, sl1, rows1, times1, val1, ref1) = res
    import bench  # noqa: E402  (repo root is on sys.path via conftest)
    from block_sparse_long_fp2_b200 import synth
    wl = synth.workloads()["qwen_128k"]
    # both ranks saw the same slices; together they cover kv-heads 0..Hkv-1 once
    assert sl0 == sl1
    covered = sorted(h for (b, n) in sl0 for h in range(b, b + n))
    assert covered == list(range(wl.Hkv))
    # each rank plans its own rows only: the two halves' rows add up to the layer's
    nb = sum((L + wl.B - 1) // wl.B for L in wl.seqlens)
    assert rows0 + rows1 == wl.Hkv * nb
    # every rank sees the maximum over ranks of each time
    assert times0 == times1 == [11.0, 5.0]
    # whole-job value: the layer's work over the slowest rank's time
    flop = bench.dense_equiv_flop(wl)
    assert val0 == val1 == pytest.approx(flop / 11e-3 / 1e12)
    # reference arm: rank 0 reports, rank 1 does no work
    assert ref0 == ("reference", 2, "oracle") and ref1 is None


def test_kv_head_slices_cover_every_head_once():
    from block_sparse_long_fp2_b200.binding import kv_head_slice
    for H in (1, 2, 3, 8, 13):
        for world in range(1, H + 1):
            parts = [kv_head_slice(H, world, r) for r in range(world)]
            assert [h for b, n in parts for h in range(b, b + n)] == list(range(H))
            assert max(n for _, n in parts) - min(n for _, n in parts) <= 1
    with pytest.raises(ValueError):
        kv_head_slice(8, 9, 0)


def test_chunk_flop_counts():
    # a chunk that is the whole sequence counts the full causal layer; the
    # last C queries count the causal pairs of positions L - C .. L - 1
    import bench  # noqa: E402
    from block_sparse_long_fp2_b200 import synth
    wl = synth.workloads()["qwen_128k"]
    L = wl.seqlens[0]
    assert bench.chunk_dense_equiv_flop(wl, [L]) == bench.dense_equiv_flop(wl)
    C = 8192
    pairs = sum(p + 1 for p in range(L - C, L))
    assert bench.chunk_dense_equiv_flop(wl, [C]) == 4.0 * wl.d * wl.Hq * pairs
