"""FP64 CPU oracle for paged quantised-KV GQA attention (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the CPU-baseline
leg of the benchmark are the only callers.  The product package never imports
this module, and this module never imports the product package.  The C source
(``oracle.c``) is compiled with gcc into ``liboracle.so`` beside it.

Every function takes and returns numpy arrays; floating point inputs are passed
as float64 holding the exact values of the original fp16/bf16/fp32 data.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

KV_INT8, KV_INT4, KV_FP8_E4M3 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain gcc, no fast-math)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "oracle.h")))
    if force or stale:
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("num_heads", ctypes.c_int),
                ("kv_num_heads", ctypes.c_int), ("head_size", ctypes.c_int),
                ("block_size", ctypes.c_int), ("num_blocks", ctypes.c_int),
                ("max_blocks_per_seq", ctypes.c_int), ("kv_dtype", ctypes.c_int),
                ("softmax_scale", ctypes.c_double), ("causal", ctypes.c_int)]


def _load():
    global _lib
    if _lib is None:
        # ORACLE_LIB lets the mutation tests load a deliberately broken copy.
        _lib = ctypes.CDLL(os.environ.get("ORACLE_LIB") or build())
        P = ctypes.c_void_p
        _lib.oracle_cache_head_size.argtypes = [ctypes.c_int, ctypes.c_int]
        _lib.oracle_decode.argtypes = [ctypes.c_int, P, ctypes.c_int]
        _lib.oracle_decode.restype = ctypes.c_double
        _lib.oracle_pack_int4.argtypes = [P, ctypes.c_int64, ctypes.c_int, P]
        _lib.oracle_unpack_int4.argtypes = [P, ctypes.c_int64, ctypes.c_int, P]
        _lib.oracle_quantise.argtypes = [ctypes.c_int, ctypes.c_float, ctypes.c_float]
        _lib.oracle_append.argtypes = [ctypes.POINTER(_Problem)] + [P] * 9
        for fn in (_lib.oracle_paged_attn, _lib.oracle_paged_attn_folded):
            fn.argtypes = [ctypes.POINTER(_Problem)] + [P] * 9
        _lib.oracle_paged_attn_partial.argtypes = [ctypes.POINTER(_Problem)] + [P] * 12
        _lib.oracle_lse_combine.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, P, P, P]
        _lib.oracle_gather_decode.argtypes = [ctypes.POINTER(_Problem), P, P, P, ctypes.c_int,
                                              ctypes.c_int, P]
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def cache_head_size(kv_dtype: int, head_size: int) -> int:
    return _load().oracle_cache_head_size(kv_dtype, head_size)


def decode_row(kv_dtype: int, row: np.ndarray, head_size: int) -> np.ndarray:
    """Exact decoded values of one cache row (bytes) as float64 [head_size]."""
    lib = _load()
    row = _c(row, np.uint8)
    return np.array([lib.oracle_decode(kv_dtype, _ptr(row), d) for d in range(head_size)])


def pack_int4(vals: np.ndarray) -> np.ndarray:
    vals = _c(vals, np.int8)
    rows, hs = vals.reshape(-1, vals.shape[-1]).shape
    out = np.zeros((rows, (hs + 1) // 2), dtype=np.uint8)
    if _load().oracle_pack_int4(_ptr(vals), rows, hs, _ptr(out)) != 0:
        raise ValueError("INT4 value out of [-8, 7]")
    return out.reshape(vals.shape[:-1] + ((hs + 1) // 2,))


def unpack_int4(packed: np.ndarray, head_size: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    rows = packed.reshape(-1, packed.shape[-1]).shape[0]
    out = np.zeros((rows, head_size), dtype=np.int8)
    _load().oracle_unpack_int4(_ptr(packed), rows, head_size, _ptr(out))
    return out.reshape(packed.shape[:-1] + (head_size,))


def _problem(w) -> _Problem:
    return _Problem(w["batch"], w["num_heads"], w["kv_num_heads"], w["head_size"],
                    w["block_size"], w["num_blocks"], w["max_blocks_per_seq"], w["kv_dtype"],
                    float(w.get("softmax_scale", 0.0)), int(w.get("causal", 1)))


def _arrays(w):
    return dict(q=_c(w["q"], np.float64), k=_c(w["k_cache"], np.uint8),
                v=_c(w["v_cache"], np.uint8), ks=_c(w["k_scale"], np.float64),
                vs=_c(w["v_scale"], np.float64), bt=_c(w["block_table"], np.int32),
                sk=_c(w["seqlens_k"], np.int32), cq=_c(w["cu_seqlens_q"], np.int32))


def paged_attn(w: dict, folded: bool = False) -> np.ndarray:
    """Attention output [T_q, H, D] (float64) for the problem dict ``w``.

    ``w`` holds the sizes (batch, num_heads, kv_num_heads, head_size,
    block_size, num_blocks, max_blocks_per_seq, kv_dtype, softmax_scale,
    causal) and the arrays (q as float64 [T_q, H, D], k_cache/v_cache uint8,
    k_scale/v_scale float64 [Hk, D], block_table, seqlens_k, cu_seqlens_q).
    """
    lib = _load()
    a = _arrays(w)
    T = int(a["cq"][-1])
    out = np.zeros((T, w["num_heads"], w["head_size"]), dtype=np.float64)
    fn = lib.oracle_paged_attn_folded if folded else lib.oracle_paged_attn
    rc = fn(ctypes.byref(_problem(w)), _ptr(a["q"]), _ptr(a["k"]), _ptr(a["v"]), _ptr(a["ks"]),
            _ptr(a["vs"]), _ptr(a["bt"]), _ptr(a["sk"]), _ptr(a["cq"]), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the problem (contract violation)")
    return out


def paged_attn_partial(w: dict, key_begin, key_end):
    """(o [T_q, H, D], lse [T_q, H]) over keys [key_begin[b], key_end[b])."""
    lib = _load()
    a = _arrays(w)
    T = int(a["cq"][-1])
    o = np.zeros((T, w["num_heads"], w["head_size"]), dtype=np.float64)
    lse = np.zeros((T, w["num_heads"]), dtype=np.float64)
    kb, ke = _c(key_begin, np.int32), _c(key_end, np.int32)
    rc = lib.oracle_paged_attn_partial(ctypes.byref(_problem(w)), _ptr(a["q"]), _ptr(a["k"]),
                                       _ptr(a["v"]), _ptr(a["ks"]), _ptr(a["vs"]), _ptr(a["bt"]),
                                       _ptr(a["sk"]), _ptr(a["cq"]), _ptr(kb), _ptr(ke), _ptr(o),
                                       _ptr(lse))
    if rc != 0:
        raise ValueError("oracle rejected the problem (contract violation)")
    return o, lse


def lse_combine(o_parts: np.ndarray, lse_parts: np.ndarray) -> np.ndarray:
    """Merge partials o_parts [S, rows, D], lse_parts [S, rows] -> [rows, D]."""
    o_parts = _c(o_parts, np.float64)
    lse_parts = _c(lse_parts, np.float64)
    S, rows, D = o_parts.shape
    out = np.zeros((rows, D), dtype=np.float64)
    if _load().oracle_lse_combine(S, rows, D, _ptr(o_parts), _ptr(lse_parts), _ptr(out)) != 0:
        raise ValueError("bad combine arguments")
    return out


def gather_decode(w: dict, cache: np.ndarray, b: int, kv: int) -> np.ndarray:
    """Decoded (unscaled) keys of sequence b, head kv, contiguous [L_b, D]."""
    bt = _c(w["block_table"], np.int32)
    sk = _c(w["seqlens_k"], np.int32)
    cache = _c(cache, np.uint8)
    L = int(sk[b])
    out = np.zeros((L, w["head_size"]), dtype=np.float64)
    rc = _load().oracle_gather_decode(ctypes.byref(_problem(w)), _ptr(cache), _ptr(bt),
                                      _ptr(sk), b, kv, _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the gather")
    return out


def quantise(kv_dtype: int, x: float, s: float) -> int:
    """Cache code of value x under scale s (signed code for INT8/INT4, byte for FP8)."""
    return int(_load().oracle_quantise(kv_dtype, float(x), float(s)))


def append(w: dict, k_new: np.ndarray, v_new: np.ndarray):
    """Quantise-and-append: copies of w's k_cache / v_cache with the new rows
    k_new / v_new ([T_q, Hk, D], exact values) written at their slots."""
    lib = _load()
    kc = np.array(w["k_cache"], dtype=np.uint8, copy=True, order="C")
    vc = np.array(w["v_cache"], dtype=np.uint8, copy=True, order="C")
    kn, vn = _c(k_new, np.float64), _c(v_new, np.float64)
    ks, vs = _c(w["k_scale"], np.float32), _c(w["v_scale"], np.float32)
    bt, sk, cq = _c(w["block_table"], np.int32), _c(w["seqlens_k"], np.int32), _c(
        w["cu_seqlens_q"], np.int32)
    rc = lib.oracle_append(ctypes.byref(_problem(w)), _ptr(kn), _ptr(vn), _ptr(ks), _ptr(vs),
                           _ptr(bt), _ptr(sk), _ptr(cq), _ptr(kc), _ptr(vc))
    if rc != 0:
        raise ValueError("oracle rejected the problem (contract violation)")
    return kc, vc
