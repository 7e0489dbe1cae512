"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

The path partitions into independent layers, so a run on N GPUs gives each
rank its own layer (its own seed) and exchanges nothing on the data path;
torch.distributed only takes the maximum of the device times over ranks, and
the reported value is the work of all ranks over that time.  These tests run
that logic with world size 2 on the gloo backend (no GPU).
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
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from block_sparse_long_fp2_b200 import synth
        wl = bench.rank_workload("pr1_ref_1k", rank)
        x = synth.generate(wl)
        # per-rank "device times": the slower rank decides
        times = bench.max_over_ranks([10.0 + rank, 5.0 - rank], world, "cpu")
        value = bench.whole_job_value(bench.dense_equiv_flop(wl), world, times[0])
        # the reference arm runs on rank 0 only
        args = type("A", (), {"workload": "pr1_ref_1k", "steps": 1, "warmup": 0})()
        ref = bench.run_reference(args, rank, world)
        queue.put((rank, wl.seed, float(np.asarray(x["q"]).sum()), times, value,
                   None if ref is None else (ref["impl"], ref["n_gpus"], ref["cpu_baseline"]["kind"])))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_independent_layers_and_max_time():
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
    (r0, seed0, sum0, times0, val0, ref0), (r1, seed1, sum1, times1, val1, ref1) = res
    # independent layers: different seeds, different inputs
    assert seed0 != seed1 and sum0 != sum1
    # every rank sees the maximum over ranks of each time
    assert times0 == times1 == [11.0, 5.0]
    # whole-job value: both ranks' work over the slowest rank's time
    import bench  # noqa: E402  (repo root is on sys.path via conftest)
    from block_sparse_long_fp2_b200 import synth
    flop = bench.dense_equiv_flop(synth.workloads()["pr1_ref_1k"])
    assert val0 == val1 == pytest.approx(2 * flop / 11e-3 / 1e12)
    # reference arm: rank 0 reports, rank 1 does no work
    assert ref0 == ("reference", 2, "oracle") and ref1 is None


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
