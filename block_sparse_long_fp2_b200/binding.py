"""Thin ctypes binding of libfp2 (``include/fp2.h``).

Argument marshalling only: torch tensors become device pointers, Python
sequences become host arrays, and every call goes straight to the C entry
point of the same name.  All computation happens in the library's CUDA
kernels.  A missing library is an error (there is no fallback).
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp2.so")
DEBUG_LIB_PATH = os.path.join(_PKG, "libfp2_debug.so")

FP2_OK = 0
FP2_ERR_INVALID_ARG = -1
FP2_ERR_UNSUPPORTED = -2
FP2_ERR_CAPACITY = -3
FP2_ERR_CUDA = -4
FP2_ERR_TIMEOUT = -5
FP2_ERR_DEVICE_CHECK = -6

FP2_STATUS_BAD_SEQLENS = 0x1
FP2_STATUS_BAD_PAGE = 0x2
FP2_STATUS_TIMEOUT = 0x4
FP2_STATUS_BOUNDS = 0x8

FP2_DTYPE_BF16 = 0
FP2_DTYPE_E4M3 = 1

FP2_NO_CORRECTION = 0x1
FP2_DEBUG_DROP_Q_LOAD = 0x100

EXPORTED = ["fp2_version", "fp2_strerror", "fp2_plan_sizes", "fp2_plan", "fp2_quantize_fp8",
            "fp2_quantize_fp8_qkv", "fp2_prefill", "fp2_status_check", "fp2_plan_static",
            "fp2_plan_kv8"]

# Size of the library-held scratch of fp2_plan_static (FP2_STATIC_WORKSPACE_BYTES).
FP2_STATIC_WORKSPACE_BYTES = 32 << 20


class Fp2Error(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


class fp2_problem(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32),
        ("seqlens", ctypes.POINTER(ctypes.c_int32)),
        ("cu_seqlens", ctypes.c_void_p),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("tau", ctypes.c_double),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("page_table", ctypes.c_void_p),
        ("page_table_stride", ctypes.c_int32),
        ("q_seqlens", ctypes.POINTER(ctypes.c_int32)),
        ("cu_q_seqlens", ctypes.c_void_p),
        ("kv_head_begin", ctypes.c_int32),
        ("num_kv_heads_total", ctypes.c_int32),
        ("prev_kbar", ctypes.c_void_p),
        ("prev_vbar", ctypes.c_void_p),
    ]


class fp2_plan_layout(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int64),
        ("num_blocks", ctypes.c_int64),
        ("num_rows", ctypes.c_int64),
        ("nnz_cap", ctypes.c_int64),
        ("mask_words", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("off_row_ptr", ctypes.c_size_t),
        ("off_col_idx", ctypes.c_size_t),
        ("off_kept_mask", ctypes.c_size_t),
        ("off_kbar", ctypes.c_size_t),
        ("off_vbar", ctypes.c_size_t),
        ("off_kbar_bf16", ctypes.c_size_t),
        ("off_vbar_bf16", ctypes.c_size_t),
        ("off_kbar_e4m3", ctypes.c_size_t),
        ("off_vbar_e4m3", ctypes.c_size_t),
        ("off_kbar_scale", ctypes.c_size_t),
        ("off_vbar_scale", ctypes.c_size_t),
        ("off_status", ctypes.c_size_t),
        ("off_meta", ctypes.c_size_t),
        ("plan_bytes", ctypes.c_size_t),
        ("workspace_bytes", ctypes.c_size_t),
        ("num_work_items", ctypes.c_int64),
        ("num_split_slots", ctypes.c_int64),
        ("off_kbar_e4m3_lo", ctypes.c_size_t),
    ]


_lib = None
_loaded = {}


def use_debug_library(on: bool) -> None:
    """Route every call through libfp2_debug.so (the FP2_DEBUG build, whose
    index checks record FP2_STATUS_BOUNDS) instead of libfp2.so, or back."""
    global LIB_PATH, _lib
    LIB_PATH = DEBUG_LIB_PATH if on else os.path.join(_PKG, "libfp2.so")
    _lib = None


def lib():
    """The loaded libfp2 (raises if it has not been built)."""
    global _lib
    if _lib is None and LIB_PATH in _loaded:
        _lib = _loaded[LIB_PATH]
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libfp2 is not built ({LIB_PATH} missing); run "
                               "`python -m block_sparse_long_fp2_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.fp2_version.restype = ctypes.c_int
        L.fp2_strerror.restype = ctypes.c_char_p
        L.fp2_strerror.argtypes = [ctypes.c_int]
        L.fp2_plan_sizes.argtypes = [ctypes.POINTER(fp2_problem), ctypes.POINTER(fp2_plan_layout)]
        L.fp2_plan.argtypes = [ctypes.POINTER(fp2_problem), ctypes.c_void_p, ctypes.c_void_p,
                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                               ctypes.c_size_t, ctypes.c_void_p]
        L.fp2_plan_static.argtypes = [ctypes.POINTER(fp2_problem), ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_size_t, ctypes.c_void_p]
        L.fp2_plan_kv8.argtypes = [ctypes.POINTER(fp2_problem), ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                   ctypes.c_size_t, ctypes.c_void_p]
        L.fp2_quantize_fp8.argtypes = [ctypes.POINTER(fp2_problem), ctypes.c_void_p,
                                       ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.fp2_quantize_fp8_qkv.argtypes = [ctypes.POINTER(fp2_problem), ctypes.c_void_p,
                                           ctypes.c_size_t] + [ctypes.c_void_p] * 10
        L.fp2_prefill.argtypes = [ctypes.POINTER(fp2_problem), ctypes.c_void_p, ctypes.c_size_t,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_uint32, ctypes.c_void_p]
        L.fp2_status_check.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                       ctypes.POINTER(ctypes.c_int32)]
        for name in EXPORTED:
            getattr(L, name).restype = ctypes.c_int if name != "fp2_strerror" else ctypes.c_char_p
        _lib = L
        _loaded[LIB_PATH] = L
    return _lib


def strerror(code: int) -> str:
    return lib().fp2_strerror(int(code)).decode()


def _check(rc: int, what: str) -> None:
    if rc != FP2_OK:
        raise Fp2Error(rc, what)


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    return int(t.data_ptr())


def _stream_ptr(stream) -> int:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


class Problem:
    """Owns the host seqlens array and the fp2_problem struct pointing at it.

    cu_seqlens and page_table are device tensors (int32) kept alive here.
    """

    def __init__(self, seqlens: Sequence[int], cu_seqlens, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, tau: float, page_size: int = 0,
                 page_table=None, num_pages: int = 0, q_seqlens: Optional[Sequence[int]] = None,
                 cu_q_seqlens=None, kv_head_begin: int = 0, num_kv_heads_total: int = 0,
                 prev_kbar=None, prev_vbar=None):
        self.seqlens_np = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
        self.cu_seqlens = cu_seqlens
        self.page_table = page_table
        self.c = fp2_problem()
        self.c.num_seqs = len(self.seqlens_np)
        self.c.seqlens = self.seqlens_np.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        self.c.cu_seqlens = _ptr(cu_seqlens)
        self.c.num_q_heads = num_q_heads
        self.c.num_kv_heads = num_kv_heads
        self.c.head_dim = head_dim
        self.c.block_size = block_size
        self.c.tau = float(tau)
        self.c.page_size = page_size
        self.c.num_pages = num_pages
        self.c.page_table = _ptr(page_table)
        self.c.page_table_stride = int(page_table.shape[1]) if page_table is not None else 0
        # chunked prefill: new queries per sequence (host) and their prefix sums (device)
        self.q_seqlens_np = None
        self.cu_q_seqlens = cu_q_seqlens
        if q_seqlens is not None:
            self.q_seqlens_np = np.ascontiguousarray(np.asarray(q_seqlens, dtype=np.int32))
            self.c.q_seqlens = self.q_seqlens_np.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
            self.c.cu_q_seqlens = _ptr(cu_q_seqlens)
        # a slice of the layer's kv-heads, run in place in full-layer tensors
        self.c.kv_head_begin = int(kv_head_begin)
        self.c.num_kv_heads_total = int(num_kv_heads_total)
        # chunked prefill: block means already held for blocks before the chunk
        self.prev = (prev_kbar, prev_vbar)
        self.c.prev_kbar = _ptr(prev_kbar)
        self.c.prev_vbar = _ptr(prev_vbar)

    @property
    def ref(self):
        return ctypes.byref(self.c)


def fp2_version() -> int:
    return lib().fp2_version()


def fp2_plan_sizes(problem: Problem) -> fp2_plan_layout:
    out = fp2_plan_layout()
    _check(lib().fp2_plan_sizes(problem.ref, ctypes.byref(out)), "fp2_plan_sizes")
    return out


def fp2_plan(problem: Problem, q, k, v, plan, workspace, stream=None) -> None:
    _check(lib().fp2_plan(problem.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(plan), plan.numel(),
                          _ptr(workspace), workspace.numel(), _stream_ptr(stream)), "fp2_plan")


def fp2_plan_static(problem: Problem, q, k, v, plan, stream=None) -> None:
    """fp2_plan with the library's own fixed scratch instead of a caller
    workspace (for callers that cannot allocate device memory)."""
    _check(lib().fp2_plan_static(problem.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(plan),
                                 plan.numel(), _stream_ptr(stream)), "fp2_plan_static")


def fp2_plan_kv8(problem: Problem, q, k_e4m3, v_e4m3, k_scale, v_scale, plan, workspace,
                 stream=None) -> None:
    """fp2_plan from an FP8 KV cache: e4m3 K/V codes with per-(block, kv-head)
    scales, bf16 Q."""
    _check(lib().fp2_plan_kv8(problem.ref, _ptr(q), _ptr(k_e4m3), _ptr(v_e4m3), _ptr(k_scale),
                              _ptr(v_scale), _ptr(plan), plan.numel(), _ptr(workspace),
                              workspace.numel(), _stream_ptr(stream)), "fp2_plan_kv8")


def fp2_quantize_fp8(problem: Problem, plan, x, which: int, x_e4m3, scales, stream=None) -> None:
    _check(lib().fp2_quantize_fp8(problem.ref, _ptr(plan), plan.numel(), _ptr(x), int(which),
                                  _ptr(x_e4m3), _ptr(scales), _stream_ptr(stream)),
           "fp2_quantize_fp8")


def fp2_quantize_fp8_qkv(problem: Problem, plan, q, k, v, q8, k8, v8, qs, ks, vs,
                         stream=None) -> None:
    """fp2_quantize_fp8 of q, k and v in one launch."""
    _check(lib().fp2_quantize_fp8_qkv(problem.ref, _ptr(plan), plan.numel(), _ptr(q), _ptr(k),
                                      _ptr(v), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(qs), _ptr(ks),
                                      _ptr(vs), _stream_ptr(stream)), "fp2_quantize_fp8_qkv")


def fp2_prefill(problem: Problem, plan, q, k, v, o, lse, q_scale=None, k_scale=None,
                v_scale=None, dtype: int = FP2_DTYPE_BF16, flags: int = 0, stream=None) -> None:
    _check(lib().fp2_prefill(problem.ref, _ptr(plan), plan.numel(), _ptr(q), _ptr(k), _ptr(v),
                             _ptr(q_scale), _ptr(k_scale), _ptr(v_scale), int(dtype), _ptr(o),
                             _ptr(lse), int(flags), _stream_ptr(stream)), "fp2_prefill")


def fp2_status_check(plan, stream=None) -> tuple:
    """(return code, raw status bits); synchronises the stream."""
    st = ctypes.c_int32(0)
    rc = lib().fp2_status_check(_ptr(plan), plan.numel(), _stream_ptr(stream), ctypes.byref(st))
    return rc, st.value


# ---------------------------------------------------------------------------
# views of the plan buffer (reading results; no computation)
# ---------------------------------------------------------------------------

class PlanView:
    """Typed torch views into a plan buffer given its layout."""

    def __init__(self, plan, layout: fp2_plan_layout, num_kv_heads: int, head_dim: int):
        import torch
        self.plan = plan
        L = layout
        R, NB = int(L.num_rows), int(L.num_blocks)

        def view(off, n, dtype, shape):
            nbytes = n * torch.empty((), dtype=dtype).element_size()
            return plan[off:off + nbytes].view(dtype).view(*shape)

        mean_shape = (NB, num_kv_heads, head_dim)
        n_mean = NB * num_kv_heads * head_dim
        self.row_ptr = view(L.off_row_ptr, R + 1, torch.int32, (R + 1,))
        self.col_idx = view(L.off_col_idx, int(L.nnz_cap), torch.int32, (int(L.nnz_cap),))
        self.kept_mask = view(L.off_kept_mask, R * L.mask_words, torch.int32, (R, L.mask_words))
        self.kbar = view(L.off_kbar, n_mean, torch.float32, mean_shape)
        self.vbar = view(L.off_vbar, n_mean, torch.float32, mean_shape)
        self.kbar_bf16 = view(L.off_kbar_bf16, n_mean, torch.bfloat16, mean_shape)
        self.vbar_bf16 = view(L.off_vbar_bf16, n_mean, torch.bfloat16, mean_shape)
        self.status = view(L.off_status, 1, torch.int32, (1,))


def kv_head_slice(num_kv_heads: int, world: int, rank: int) -> tuple:
    """(first kv-head, kv-heads) of rank's share of a layer split over world
    ranks by kv-head: contiguous, as equal as the counts allow, earlier ranks
    taking the remainder."""
    if not 1 <= world <= num_kv_heads or not 0 <= rank < world:
        raise ValueError(f"cannot split {num_kv_heads} kv-heads over {world} ranks")
    base, extra = divmod(num_kv_heads, world)
    begin = rank * base + min(rank, extra)
    return begin, base + (1 if rank < extra else 0)


def allocate(problem: Problem, device="cuda"):
    """Plan buffer and workspace sized by fp2_plan_sizes (uint8 tensors)."""
    import torch
    lay = fp2_plan_sizes(problem)
    plan = torch.empty(int(lay.plan_bytes), dtype=torch.uint8, device=device)
    ws = torch.empty(int(lay.workspace_bytes), dtype=torch.uint8, device=device)
    return lay, plan, ws
