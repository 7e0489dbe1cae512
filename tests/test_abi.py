"""The C-ABI library loads, exports what include/fp2.h declares, and its
host-only entry points validate arguments (no GPU needed)."""

import ctypes
import os
import re

import numpy as np
import pytest

from block_sparse_long_fp2_b200 import binding as fb
from block_sparse_long_fp2_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fbuild.build()
    return fb.lib()


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            names |= set(re.findall(r"^\s*(?:int|const char\*)\s+(fp2_\w+)\s*\(", text, re.M))
    return names


def test_header_declares_the_entry_points():
    assert {"fp2_version", "fp2_strerror", "fp2_plan_sizes", "fp2_plan", "fp2_quantize_fp8",
            "fp2_prefill", "fp2_status_check"} <= _declared()


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version_and_strerror(lib):
    assert fb.fp2_version() == 3
    assert fb.strerror(0) == "ok"
    for code in [-1, -2, -3, -4, -5, -6]:
        assert fb.strerror(code) not in ("", "unknown error")
    assert fb.strerror(-99) == "unknown error"


def _problem(seqlens=(1000, 37), Hq=32, Hkv=8, d=128, B=128, tau=0.1, page_size=0,
             page_table=None, num_pages=0):
    # device pointers are never dereferenced by fp2_plan_sizes: fake non-null values
    p = fb.Problem(seqlens, 0x1000, Hq, Hkv, d, B, tau)
    p.c.page_size = page_size
    p.c.num_pages = num_pages
    if page_table is not None:
        p.c.page_table = 0x2000
        p.c.page_table_stride = page_table
    return p


def _schedule_sizes(seqlens, Hq, Hkv, B):
    # The documented split rule of fp2_prefill's work schedule, restated: the
    # tile bound of row i is i + 1 + ceil(i / B); rows split only when the
    # longest bound exceeds both 32 and the layer's mean tiles per CTA over 148
    # CTAs, with split size max(8, ceil(mean / 2), ceil(longest / 32)).
    G = Hq // Hkv
    pairs = (G * B // 128 + 1) // 2
    rows = [i for L in seqlens for i in range((L + B - 1) // B)]
    bound = [i + 1 + (i + B - 1) // B for i in rows]
    share = -(-sum(bound) * Hkv * pairs // 148)
    longest = max(bound)
    c = max(8, (share + 1) // 2, -(-longest // 32))
    if longest <= share or longest < 32:
        c = 0
    splits = [-(-u // c) if c else 1 for u in bound]
    return sum(splits) * Hkv * pairs, sum(x for x in splits if x > 1) * Hkv


@pytest.mark.parametrize("shape", [((1024,), 4, 1, 64), ((4096,), 32, 8, 128), ((4096,), 2, 1, 64),
                                   ((3000, 700), 2, 1, 64), ((131072,), 32, 8, 128),
                                   ((4096, 9000, 16384, 30000, 65536, 1500), 32, 8, 128),
                                   ((1, 2, 129, 3, 130), 8, 2, 128), ((9000,), 2, 1, 64)])
def test_schedule_sizes_follow_the_split_rule(lib, shape):
    seqlens, Hq, Hkv, B = shape
    lay = fb.fp2_plan_sizes(_problem(seqlens, Hq, Hkv, 128 if B == 128 else 64, B))
    items, slots = _schedule_sizes(seqlens, Hq, Hkv, B)
    assert (lay.num_work_items, lay.num_split_slots) == (items, slots)
    # every row has at least one item per query-tile pair
    G = Hq // Hkv
    assert lay.num_work_items >= lay.num_rows * ((G * B // 128 + 1) // 2)


def test_plan_sizes_counts(lib):
    lay = fb.fp2_plan_sizes(_problem())
    nb = [8, 1]
    assert lay.num_tokens == 1037 and lay.num_blocks == 9 and lay.num_rows == 72
    assert lay.nnz_cap == 8 * (8 * 9 // 2 + 1)
    assert lay.mask_words == 1 and lay.max_blocks_per_seq == 8
    offs = [lay.off_status, lay.off_row_ptr, lay.off_col_idx, lay.off_kept_mask, lay.off_kbar,
            lay.off_vbar, lay.off_kbar_bf16, lay.off_vbar_bf16, lay.off_kbar_e4m3,
            lay.off_vbar_e4m3, lay.off_kbar_scale, lay.off_vbar_scale, lay.off_kbar_e4m3_lo]
    assert lay.off_status == 0
    assert all(o % 256 == 0 for o in offs)
    assert len(set(offs)) == len(offs) and max(offs) < lay.plan_bytes
    assert lay.off_col_idx - lay.off_row_ptr >= 4 * 73
    assert lay.workspace_bytes >= 8 * 9 * 32 * 128 + 4 * lay.nnz_cap
    assert sum(n * (n + 1) // 2 for n in nb) * 8 == lay.nnz_cap


def test_plan_sizes_128k_index_memory(lib):
    # the CSR of a 128K prefill with 8 kv-heads is at most the dense count
    lay = fb.fp2_plan_sizes(_problem(seqlens=(131072,), tau=0.05))
    assert lay.nnz_cap == 8 * 1024 * 1025 // 2
    assert lay.mask_words == 32


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=30, Hkv=8), fb.FP2_ERR_INVALID_ARG),          # Hq % Hkv
    (dict(d=96), fb.FP2_ERR_UNSUPPORTED),
    (dict(B=32), fb.FP2_ERR_UNSUPPORTED),
    (dict(Hq=8, Hkv=8, B=64), fb.FP2_ERR_UNSUPPORTED),     # G * B not a multiple of 128
    (dict(tau=-0.1), fb.FP2_ERR_INVALID_ARG),
    (dict(tau=float("nan")), fb.FP2_ERR_INVALID_ARG),
    (dict(seqlens=(10, 0)), fb.FP2_ERR_INVALID_ARG),
    (dict(page_size=32), fb.FP2_ERR_UNSUPPORTED),
    (dict(page_size=64, page_table=None, num_pages=4), fb.FP2_ERR_INVALID_ARG),
    (dict(page_size=64, page_table=15, num_pages=40), fb.FP2_ERR_INVALID_ARG),  # stride < 16 pages
])
def test_plan_sizes_rejects(lib, kw, code):
    with pytest.raises(fb.Fp2Error) as e:
        fb.fp2_plan_sizes(_problem(**kw))
    assert e.value.code == code


def _chunk_problem(seqlens, q_seqlens, Hq=32, Hkv=8, B=128):
    p = _problem(seqlens, Hq, Hkv, 128, B)
    p.q_seqlens_np = np.ascontiguousarray(np.asarray(q_seqlens, dtype=np.int32))
    p.c.q_seqlens = p.q_seqlens_np.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    p.c.cu_q_seqlens = 0x3000
    return p


@pytest.mark.parametrize("q_seqlens", [(0, 37), (1001, 37), (1000, 38)])
def test_chunk_lengths_checked(lib, q_seqlens):
    with pytest.raises(fb.Fp2Error) as e:
        fb.fp2_plan_sizes(_chunk_problem((1000, 37), q_seqlens))
    assert e.value.code == fb.FP2_ERR_INVALID_ARG


def test_chunk_needs_both_lengths_and_offsets(lib):
    p = _chunk_problem((1000, 37), (10, 37))
    p.c.cu_q_seqlens = None
    with pytest.raises(fb.Fp2Error) as e:
        fb.fp2_plan_sizes(p)
    assert e.value.code == fb.FP2_ERR_INVALID_ARG


def test_chunked_planning_from_an_fp8_cache_is_rejected(lib):
    # rejected on the host before anything is enqueued
    p = _chunk_problem((1000, 37), (10, 37))
    lay = fb.fp2_plan_sizes(p)
    rc = lib.fp2_plan_kv8(p.ref, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x100000,
                          lay.plan_bytes, 0x200000, lay.workspace_bytes, None)
    assert rc == fb.FP2_ERR_UNSUPPORTED


def test_chunk_schedule_counts_only_the_chunk_rows(lib):
    # 131072 keys, the last 8192 queries: query blocks 960..1023 of 1024
    full = fb.fp2_plan_sizes(_problem((131072,), 32, 8, 128, 128))
    lay = fb.fp2_plan_sizes(_chunk_problem((131072,), (8192,)))
    assert lay.num_rows == full.num_rows
    assert lay.num_work_items == 8 * 2 * 64
    # a chunk starting inside block 10 (position 1300) has rows 10..15
    lay = fb.fp2_plan_sizes(_chunk_problem((2000,), (700,)))
    assert lay.num_work_items == 8 * 2 * 6


def test_paged_problem_accepted(lib):
    lay = fb.fp2_plan_sizes(_problem(page_size=64, page_table=16, num_pages=40))
    assert lay.num_blocks == 9


def test_null_problem_and_buffers_rejected(lib):
    L = fb.lib()
    assert L.fp2_plan_sizes(None, None) == fb.FP2_ERR_INVALID_ARG
    p = _problem()
    assert L.fp2_plan(p.ref, None, None, None, None, 0, None, 0, None) == fb.FP2_ERR_INVALID_ARG
    lay = fb.fp2_plan_sizes(p)
    # capacity is checked before anything is enqueued
    rc = L.fp2_plan(p.ref, 0x10000, 0x10000, 0x10000, 0x100000, lay.plan_bytes - 256, 0x200000,
                    lay.workspace_bytes, None)
    assert rc == fb.FP2_ERR_CAPACITY
    rc = L.fp2_prefill(p.ref, 0x100000, lay.plan_bytes, 0x10000, 0x10000, 0x10000, None, None,
                       None, 7, 0x10000, 0x10000, 0, None)
    assert rc == fb.FP2_ERR_INVALID_ARG   # unknown dtype
    rc = L.fp2_prefill(p.ref, 0x100000, lay.plan_bytes, 0x10008, 0x10000, 0x10000, None, None,
                       None, 0, 0x10000, 0x10000, 0, None)
    assert rc == fb.FP2_ERR_INVALID_ARG   # q not 16-byte aligned
    rc = L.fp2_prefill(p.ref, 0x100000, lay.plan_bytes, 0x10000, 0x10000, 0x10000, None, None,
                       None, 0, 0x10000, 0x10000, 0x8000, None)
    assert rc == fb.FP2_ERR_INVALID_ARG   # unknown flag
    rc = L.fp2_quantize_fp8(p.ref, 0x100000, lay.plan_bytes, 0x10000, 3, 0x10000, 0x10000, None)
    assert rc == fb.FP2_ERR_INVALID_ARG   # which out of range
    rc = L.fp2_plan_kv8(p.ref, 0x10000, 0x10000, 0x10000, None, 0x10000, 0x100000, lay.plan_bytes,
                        0x200000, lay.workspace_bytes, None)
    assert rc == fb.FP2_ERR_INVALID_ARG   # missing K scales
    rc = L.fp2_plan_kv8(p.ref, 0x10000, 0x10008, 0x10000, 0x10000, 0x10000, 0x100000,
                        lay.plan_bytes, 0x200000, lay.workspace_bytes, None)
    assert rc == fb.FP2_ERR_INVALID_ARG   # K codes not 16-byte aligned
    rc = L.fp2_plan_kv8(p.ref, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x100000,
                        lay.plan_bytes, 0x200000, lay.workspace_bytes - 256, None)
    assert rc == fb.FP2_ERR_CAPACITY


def test_no_cpu_fallback_in_product_path():
    # the package never imports the oracle
    pkg = os.path.join(ROOT, "block_sparse_long_fp2_b200")
    for f in os.listdir(pkg):
        if f.endswith(".py"):
            src = open(os.path.join(pkg, f)).read()
            assert "import oracle" not in src and "from oracle" not in src, f


def test_head_slice_arguments_and_sizes():
    # a slice of the layer's kv-heads: its plan is sized for its own heads, and
    # a slice that does not fit in the tensors' heads is rejected on the host
    lib = fb.lib()
    full = fb.Problem([1000, 300], 0x1000, 32, 8, 128, 128, 0.1)
    half = fb.Problem([1000, 300], 0x1000, 16, 4, 128, 128, 0.1, kv_head_begin=4,
                      num_kv_heads_total=8)
    compact = fb.Problem([1000, 300], 0x1000, 16, 4, 128, 128, 0.1)
    lf, lh, lc = fb.fp2_plan_sizes(full), fb.fp2_plan_sizes(half), fb.fp2_plan_sizes(compact)
    assert lh.num_rows * 2 == lf.num_rows and lh.nnz_cap * 2 == lf.nnz_cap
    assert (lh.plan_bytes, lh.workspace_bytes) == (lc.plan_bytes, lc.workspace_bytes)
    lay = fb.fp2_plan_layout()
    for begin, total in ((5, 8), (-1, 8), (0, 3), (0, -2)):
        bad = fb.Problem([1000, 300], 0x1000, 16, 4, 128, 128, 0.1, kv_head_begin=begin,
                         num_kv_heads_total=total)
        assert lib.fp2_plan_sizes(bad.ref, ctypes.byref(lay)) == fb.FP2_ERR_INVALID_ARG, (begin, total)
