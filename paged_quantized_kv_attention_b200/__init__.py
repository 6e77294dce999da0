"""Python binding of libpagedattn.so (paged quantised-KV GQA attention, sm_100a).

Argument marshalling only: every function here converts torch tensors / numpy
arrays into raw pointers and sizes and calls the C entry point of the same name
(see include/paged_attn.h for layouts, ownership and errors).  All compute runs
in the library's CUDA kernels; there is no CPU fallback.  If the shared library
is missing, importing the functions raises immediately.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE = 0, -1, -2, -3
PA_ERR_BAD_BLOCK_TABLE, PA_ERR_CUDA, PA_ERR_DEVICE = -4, -5, -6
PA_KV_INT8, PA_KV_INT4, PA_KV_FP8_E4M3 = 0, 1, 2
PA_F16, PA_BF16, PA_F32 = 0, 1, 2
PA_DEVERR_BAD_BLOCK, PA_DEVERR_TIMEOUT, PA_DEVERR_BAD_SCALE, PA_DEVERR_BAD_LENGTH = 1, 2, 4, 8
PA_NOALLOC_MAX_WORKSPACE_BYTES = 16 << 20

EXPORTED = ["paged_attn_plan", "paged_attn_forward", "paged_attn_forward_noalloc",
            "paged_attn_workspace_init",
            "paged_attn_read_device_error", "paged_kv_pack_int4", "paged_kv_unpack_int4",
            "paged_kv_gather_decode", "paged_kv_append", "paged_attn_merge", "paged_attn_stream_read",
            "paged_attn_last_error", "paged_attn_version"]


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("status %d: %s" % (status, message))
        self.status = status


class paged_attn_params(ctypes.Structure):  # noqa: N801 (mirrors the C struct name)
    _fields_ = [("batch", ctypes.c_int), ("num_heads", ctypes.c_int),
                ("kv_num_heads", ctypes.c_int), ("head_size", ctypes.c_int),
                ("block_size", ctypes.c_int), ("num_blocks", ctypes.c_int),
                ("max_blocks_per_seq", ctypes.c_int), ("kv_dtype", ctypes.c_int),
                ("q_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("causal", ctypes.c_int),
                ("num_sms", ctypes.c_int), ("split_blocks", ctypes.c_int),
                ("total_q", ctypes.c_int), ("max_query_len", ctypes.c_int),
                ("max_seqlen_k", ctypes.c_int), ("rows_per_cta", ctypes.c_int),
                ("num_row_groups", ctypes.c_int), ("num_splits", ctypes.c_int),
                ("blocks_per_split", ctypes.c_int), ("num_work_items", ctypes.c_int),
                ("workspace_bytes", ctypes.c_size_t),
                ("workspace", ctypes.c_void_p), ("profile_events", ctypes.c_void_p),
                ("stall_consumers", ctypes.c_int), ("lse_out", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libpagedattn.so (built in-tree by __graft_entry__.build())."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libpagedattn.so is not built (%s); run "
                              "`python -c 'import __graft_entry__ as g; g.build()'`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        PP = ctypes.POINTER(paged_attn_params)
        L.paged_attn_plan.argtypes = [P, P, PP, ctypes.POINTER(ctypes.c_size_t)]
        L.paged_attn_forward.argtypes = [P] * 9 + [PP, P]
        L.paged_attn_forward_noalloc.argtypes = [P] * 9 + [PP, P]
        L.paged_attn_workspace_init.argtypes = [P, S, P]
        L.paged_attn_read_device_error.argtypes = [P, I, ctypes.POINTER(ctypes.c_uint32), P]
        L.paged_kv_pack_int4.argtypes = [P, P, ctypes.c_int64, I, P]
        L.paged_kv_unpack_int4.argtypes = [P, P, ctypes.c_int64, I, P]
        L.paged_kv_gather_decode.argtypes = [P, P, PP, I, I, I, I, P, P]
        L.paged_kv_append.argtypes = [P] * 9 + [PP, P]
        L.paged_attn_merge.argtypes = [P, I, P, I, ctypes.c_int64, I, P, I, P, P]
        L.paged_attn_stream_read.argtypes = [P, S, P, P]
        L.paged_attn_last_error.restype = ctypes.c_char_p
        L.paged_attn_version.restype = ctypes.c_char_p
        for name in EXPORTED[:-2]:
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int):
    if status != PA_OK:
        raise PagedAttnError(status, lib().paged_attn_last_error().decode())


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if isinstance(t, np.ndarray):
        return ctypes.c_void_p(t.ctypes.data)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(getattr(stream, "cuda_stream", stream))


def make_params(*, batch, num_heads, kv_num_heads, head_size, block_size, num_blocks,
                max_blocks_per_seq, kv_dtype, q_dtype, out_dtype, softmax_scale=0.0, causal=1,
                num_sms=0, split_blocks=0) -> paged_attn_params:
    p = paged_attn_params()
    p.batch, p.num_heads, p.kv_num_heads = batch, num_heads, kv_num_heads
    p.head_size, p.block_size, p.num_blocks = head_size, block_size, num_blocks
    p.max_blocks_per_seq, p.kv_dtype = max_blocks_per_seq, kv_dtype
    p.q_dtype, p.out_dtype = q_dtype, out_dtype
    p.softmax_scale, p.causal, p.num_sms, p.split_blocks = softmax_scale, causal, num_sms, split_blocks
    return p


def paged_attn_plan(cu_seqlens_q_host, seqlens_k_host, params: paged_attn_params) -> int:
    """Fill the planned fields of ``params``; returns the workspace bytes needed."""
    cu = np.ascontiguousarray(np.asarray(cu_seqlens_q_host), dtype=np.int32)
    sk = np.ascontiguousarray(np.asarray(seqlens_k_host), dtype=np.int32)
    need = ctypes.c_size_t(0)
    _check(lib().paged_attn_plan(_ptr(cu), _ptr(sk), ctypes.byref(params), ctypes.byref(need)))
    return need.value


def paged_attn_forward(q, k_cache, v_cache, k_scale, v_scale, block_table, seqlens_k,
                       cu_seqlens_q, out, params: paged_attn_params, stream=None):
    _check(lib().paged_attn_forward(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                                    _ptr(v_scale), _ptr(block_table), _ptr(seqlens_k),
                                    _ptr(cu_seqlens_q), _ptr(out), ctypes.byref(params),
                                    _stream(stream)))


def paged_attn_forward_noalloc(q, k_cache, v_cache, k_scale, v_scale, block_table, seqlens_k,
                               cu_seqlens_q, out, params: paged_attn_params, stream=None):
    """paged_attn_forward without a caller workspace: the library's own static
    device scratch (PA_NOALLOC_MAX_WORKSPACE_BYTES) is used instead, for callers
    that cannot allocate device memory.  params.workspace is ignored."""
    _check(lib().paged_attn_forward_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                                            _ptr(v_scale), _ptr(block_table), _ptr(seqlens_k),
                                            _ptr(cu_seqlens_q), _ptr(out), ctypes.byref(params),
                                            _stream(stream)))


def paged_attn_workspace_init(workspace, nbytes: int, stream=None):
    _check(lib().paged_attn_workspace_init(_ptr(workspace), nbytes, _stream(stream)))


def paged_attn_read_device_error(workspace, clear: bool = True, stream=None):
    """(status, bits) of the sticky device error word; never raises for set bits.
    ``workspace`` None reads the word of paged_attn_forward_noalloc's scratch."""
    bits = ctypes.c_uint32(0)
    st = lib().paged_attn_read_device_error(_ptr(workspace), int(clear), ctypes.byref(bits),
                                            _stream(stream))
    if st not in (PA_OK, PA_ERR_BAD_BLOCK_TABLE, PA_ERR_DEVICE):
        _check(st)
    return st, bits.value


def paged_kv_pack_int4(src, dst, rows: int, head_size: int, stream=None):
    _check(lib().paged_kv_pack_int4(_ptr(src), _ptr(dst), rows, head_size, _stream(stream)))


def paged_kv_unpack_int4(src, dst, rows: int, head_size: int, stream=None):
    _check(lib().paged_kv_unpack_int4(_ptr(src), _ptr(dst), rows, head_size, _stream(stream)))


def paged_kv_gather_decode(cache, block_table, params: paged_attn_params, b: int, kv: int,
                           len_b: int, dst_dtype: int, dst, stream=None):
    _check(lib().paged_kv_gather_decode(_ptr(cache), _ptr(block_table), ctypes.byref(params), b,
                                        kv, len_b, dst_dtype, _ptr(dst), _stream(stream)))


def paged_kv_append(k_new, v_new, k_cache, v_cache, k_scale, v_scale, block_table, seqlens_k,
                    cu_seqlens_q, params: paged_attn_params, stream=None):
    """Quantise the new tokens' K/V rows ([total_q, Hk, D], params.q_dtype) into
    the caches at their slots (see paged_kv_append in paged_attn.h)."""
    _check(lib().paged_kv_append(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                 _ptr(k_scale), _ptr(v_scale), _ptr(block_table), _ptr(seqlens_k),
                                 _ptr(cu_seqlens_q), ctypes.byref(params), _stream(stream)))


def paged_attn_merge(parts, parts_dtype: int, lse_parts, n_parts: int, rows: int, head_size: int,
                     out, out_dtype: int, lse_out=None, stream=None):
    """Log-sum-exp merge of results over disjoint key sets (see paged_attn.h)."""
    _check(lib().paged_attn_merge(_ptr(parts), parts_dtype, _ptr(lse_parts), n_parts, rows,
                                  head_size, _ptr(out), out_dtype, _ptr(lse_out), _stream(stream)))


def paged_attn_stream_read(src, nbytes: int, sink, stream=None):
    _check(lib().paged_attn_stream_read(_ptr(src), nbytes, _ptr(sink), _stream(stream)))


def paged_attn_last_error() -> str:
    return lib().paged_attn_last_error().decode()


def paged_attn_version() -> str:
    return lib().paged_attn_version().decode()


class PagedAttention:
    """Convenience wrapper: plans one batch shape and owns the workspace.

    Tensor arguments are torch CUDA tensors in the layouts of paged_attn.h; the
    workspace is allocated with torch once per plan and zeroed by the library.
    """

    def __init__(self, cu_seqlens_q_host, seqlens_k_host, **problem):
        import torch
        self.params = make_params(**problem)
        self.workspace_bytes = paged_attn_plan(cu_seqlens_q_host, seqlens_k_host, self.params)
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device="cuda")
        self.params.workspace = self.workspace.data_ptr()
        paged_attn_workspace_init(self.workspace, self.workspace_bytes)

    def __call__(self, q, k_cache, v_cache, k_scale, v_scale, block_table, seqlens_k,
                 cu_seqlens_q, out, stream=None):
        paged_attn_forward(q, k_cache, v_cache, k_scale, v_scale, block_table, seqlens_k,
                           cu_seqlens_q, out, self.params, stream)
        return out

    def device_error(self, clear: bool = True):
        return paged_attn_read_device_error(self.workspace, clear)
