"""Seeded synthetic inputs for paged quantised-KV attention.

This module only draws random numbers and lays them out (cache pools, block
tables, ragged lengths); it holds none of the attention arithmetic, no
dequantisation and no packing routine.  It is the one piece shared by the tests,
the benchmark and the smoke check; the CUDA library and the FP64 oracle both
consume what it produces and neither depends on the other.

Packed INT4 caches are drawn as uniform random bytes: every nibble of a uniform
byte is uniform over its 16 codes, i.e. uniform over [-8, 7] in 4-bit two's
complement, which is the stated value distribution, without running an encoder.
FP8-e4m3 caches are drawn as float32 normals and cast with torch's
float8_e4m3fn conversion (round to nearest even).

The five named workloads follow the shapes and distributions of the pages'
cases (INT8 decode, INT4 decode with a per-channel K scale folded into Q,
long-context split decode, ragged prefill with zero-new-token sequences, large
FP8 batch).  Seeds are 1000 + workload index, numpy PCG64.
"""
from __future__ import annotations

import math

import numpy as np
import torch

KV_INT8, KV_INT4, KV_FP8_E4M3 = 0, 1, 2
F16, BF16 = 0, 1
KV_NAMES = {KV_INT8: "int8", KV_INT4: "int4", KV_FP8_E4M3: "fp8_e4m3"}
TORCH_DTYPE = {F16: torch.float16, BF16: torch.bfloat16}

_CHUNK = 1 << 24  # elements per RNG call for large caches (fixed: keeps streams stable)


def cache_bytes_per_row(kv_dtype: int, head_size: int) -> int:
    """Bytes per token per KV head as laid out in the cache arrays."""
    return (head_size + 1) // 2 if kv_dtype == KV_INT4 else head_size


def _fill(rng: np.random.Generator, n: int, kind: str, dist: str) -> np.ndarray:
    """Draw n cache bytes of the given kind/distribution, in fixed-size chunks."""
    out = np.empty(n, dtype=np.uint8)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        if kind == "int4":
            out[s:s + m] = rng.integers(0, 256, m, dtype=np.uint8)
        elif kind == "int8" and dist == "uniform127":
            out[s:s + m] = rng.integers(-127, 128, m, dtype=np.int8).view(np.uint8)
        elif kind == "int8" and dist == "normal40":
            x = np.rint(rng.standard_normal(m, dtype=np.float32) * np.float32(40.0))
            out[s:s + m] = np.clip(x, -127, 127).astype(np.int8).view(np.uint8)
        elif kind == "fp8":
            x = rng.standard_normal(m, dtype=np.float32) * np.float32(4.0)
            out[s:s + m] = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        else:
            raise ValueError((kind, dist))
    return out


def _scales(rng, Hk, D, lo, hi, boost_frac=0.0, boost=100.0):
    s = rng.uniform(lo, hi, size=(Hk, D)).astype(np.float32)
    n = int(round(boost_frac * Hk * D))
    if n:
        idx = rng.choice(Hk * D, size=n, replace=False)
        s.reshape(-1)[idx] *= np.float32(boost)
    return s


def make_problem(*, seed: int, batch: int, num_heads: int, kv_num_heads: int, head_size: int,
                 block_size: int, kv_dtype: int, q_dtype: int, out_dtype: int,
                 seqlens_k, q_lens, pool_blocks=None, pool_factor: float = 1.0,
                 kv_dist: str = "uniform127", k_scale_range=(0.005, 0.02),
                 v_scale_range=(0.005, 0.02), k_boost_frac: float = 0.0, causal: int = 1,
                 softmax_scale: float = 0.0, rng=None, name: str = "custom") -> dict:
    """Build one problem with explicit per-sequence key lengths and new-token counts.

    seqlens_k[b] counts all keys of sequence b (new ones included) and
    q_lens[b] <= seqlens_k[b] is its number of new tokens.  The physical pool
    holds ``pool_blocks`` blocks (default: pool_factor x the blocks needed);
    the block table is a seeded random permutation of the pool and unused slots
    hold -1.
    """
    rng = rng if rng is not None else np.random.default_rng(seed)
    seqlens_k = np.asarray(seqlens_k, dtype=np.int32).reshape(batch)
    q_lens = np.asarray(q_lens, dtype=np.int32).reshape(batch)
    assert np.all(q_lens >= 0) and np.all(q_lens <= seqlens_k)
    nblk = (seqlens_k + block_size - 1) // block_size
    needed = int(nblk.sum())
    if pool_blocks is None:
        pool_blocks = max(1, int(math.ceil(pool_factor * needed)))
    assert pool_blocks >= needed
    maxb = max(1, int(nblk.max()) if batch else 1)
    perm = rng.permutation(pool_blocks).astype(np.int32)
    block_table = np.full((batch, maxb), -1, dtype=np.int32)
    pos = 0
    for b in range(batch):
        block_table[b, :nblk[b]] = perm[pos:pos + nblk[b]]
        pos += int(nblk[b])
    cu = np.zeros(batch + 1, dtype=np.int32)
    cu[1:] = np.cumsum(q_lens)
    chs = cache_bytes_per_row(kv_dtype, head_size)
    k_scale = _scales(rng, kv_num_heads, head_size, *k_scale_range, boost_frac=k_boost_frac)
    v_scale = _scales(rng, kv_num_heads, head_size, *v_scale_range)
    T = int(cu[-1])
    qf = rng.standard_normal((T, num_heads, head_size), dtype=np.float32)
    q = torch.from_numpy(qf).to(TORCH_DTYPE[q_dtype])
    kind = {KV_INT8: "int8", KV_INT4: "int4", KV_FP8_E4M3: "fp8"}[kv_dtype]
    shape = (pool_blocks, block_size, kv_num_heads, chs)
    n = int(np.prod(shape))
    k_cache = _fill(rng, n, kind, kv_dist).reshape(shape)
    v_cache = _fill(rng, n, kind, kv_dist).reshape(shape)
    return dict(name=name, seed=seed, batch=batch, num_heads=num_heads,
                kv_num_heads=kv_num_heads, head_size=head_size, block_size=block_size,
                num_blocks=pool_blocks, max_blocks_per_seq=maxb, kv_dtype=kv_dtype,
                q_dtype=q_dtype, out_dtype=out_dtype, causal=causal,
                softmax_scale=softmax_scale, q=q, k_cache=k_cache, v_cache=v_cache,
                k_scale=k_scale, v_scale=v_scale, block_table=block_table,
                seqlens_k=seqlens_k, cu_seqlens_q=cu)


NAMES = ["c1_tiny_int8", "c2_int4_decode", "c3_int8_long_split", "c4_ragged_prefill_int8",
         "c5_fp8_large_batch"]

DESCRIPTIONS = {
    "c1_tiny_int8": "INT8 decode B=2 L={37,64} H=4 Hk=1 D=64 bs=16, fp16 Q/out",
    "c2_int4_decode": "INT4 decode B=16 L~U[512,4096] H=32 Hk=8 D=128 bs=16, fp16 Q/out",
    "c3_int8_long_split": "INT8 split-KV decode B=4 L=32768 H=64 Hk=8 D=128 bs=32, bf16 Q/out",
    "c4_ragged_prefill_int8": "INT8 ragged causal prefill B=64 p~U[0,2048] q~U{0..16} H=32 "
                              "Hk=8 D=128 bs=16, fp16 Q/out",
    "c5_fp8_large_batch": "FP8-e4m3 decode B=128 L=8192 H=64 Hk=8 D=128 bs=16, bf16 Q/out",
}


def make(name: str) -> dict:
    """One of the five named workloads, at full size."""
    idx = NAMES.index(name) + 1
    seed = 1000 + idx
    rng = np.random.default_rng(seed)
    if name == "c1_tiny_int8":
        return make_problem(seed=seed, rng=rng, name=name, batch=2, num_heads=4, kv_num_heads=1,
                            head_size=64, block_size=16, kv_dtype=KV_INT8, q_dtype=F16,
                            out_dtype=F16, seqlens_k=[37, 64], q_lens=[1, 1], pool_blocks=16,
                            kv_dist="uniform127", k_scale_range=(0.005, 0.02),
                            v_scale_range=(0.005, 0.02))
    if name == "c2_int4_decode":
        B = 16
        L = rng.integers(512, 4097, size=B)
        return make_problem(seed=seed, rng=rng, name=name, batch=B, num_heads=32,
                            kv_num_heads=8, head_size=128, block_size=16, kv_dtype=KV_INT4,
                            q_dtype=F16, out_dtype=F16, seqlens_k=L, q_lens=np.ones(B),
                            pool_factor=2.0, k_scale_range=(0.01, 0.1),
                            v_scale_range=(0.01, 0.1), k_boost_frac=0.01)
    if name == "c3_int8_long_split":
        B = 4
        return make_problem(seed=seed, rng=rng, name=name, batch=B, num_heads=64,
                            kv_num_heads=8, head_size=128, block_size=32, kv_dtype=KV_INT8,
                            q_dtype=BF16, out_dtype=BF16, seqlens_k=np.full(B, 32768),
                            q_lens=np.ones(B), pool_factor=1.0, kv_dist="normal40",
                            k_scale_range=(0.005, 0.02), v_scale_range=(0.005, 0.02))
    if name == "c4_ragged_prefill_int8":
        B = 64
        past = rng.integers(0, 2049, size=B)
        ql = rng.integers(0, 17, size=B)
        ql[rng.choice(B, size=8, replace=False)] = 0
        return make_problem(seed=seed, rng=rng, name=name, batch=B, num_heads=32,
                            kv_num_heads=8, head_size=128, block_size=16, kv_dtype=KV_INT8,
                            q_dtype=F16, out_dtype=F16, seqlens_k=past + ql, q_lens=ql,
                            pool_factor=2.0, kv_dist="uniform127", k_scale_range=(0.01, 0.1),
                            v_scale_range=(0.01, 0.1), k_boost_frac=0.01, causal=1)
    if name == "c5_fp8_large_batch":
        B = 128
        return make_problem(seed=seed, rng=rng, name=name, batch=B, num_heads=64,
                            kv_num_heads=8, head_size=128, block_size=16,
                            kv_dtype=KV_FP8_E4M3, q_dtype=BF16, out_dtype=BF16,
                            seqlens_k=np.full(B, 8192), q_lens=np.ones(B), pool_factor=1.0,
                            kv_dist="fp8", k_scale_range=(0.05, 0.5),
                            v_scale_range=(0.05, 0.5))
    raise KeyError(name)


def shrink(name: str, seed: int, max_len: int, batch: int | None = None) -> dict:
    """A small problem with the named workload's head layout, dtypes and
    distributions but short sequences, for oracle-sized parity runs."""
    full = {"c1_tiny_int8": dict(H=4, Hk=1, D=64, bs=16, kv=KV_INT8, qd=F16, od=F16,
                                 dist="uniform127", ks=(0.005, 0.02), vs=(0.005, 0.02), kb=0.0),
            "c2_int4_decode": dict(H=32, Hk=8, D=128, bs=16, kv=KV_INT4, qd=F16, od=F16,
                                   dist="uniform127", ks=(0.01, 0.1), vs=(0.01, 0.1), kb=0.01),
            "c3_int8_long_split": dict(H=64, Hk=8, D=128, bs=32, kv=KV_INT8, qd=BF16, od=BF16,
                                       dist="normal40", ks=(0.005, 0.02), vs=(0.005, 0.02),
                                       kb=0.0),
            "c4_ragged_prefill_int8": dict(H=32, Hk=8, D=128, bs=16, kv=KV_INT8, qd=F16, od=F16,
                                           dist="uniform127", ks=(0.01, 0.1), vs=(0.01, 0.1),
                                           kb=0.01),
            "c5_fp8_large_batch": dict(H=64, Hk=8, D=128, bs=16, kv=KV_FP8_E4M3, qd=BF16,
                                       od=BF16, dist="fp8", ks=(0.05, 0.5), vs=(0.05, 0.5),
                                       kb=0.0)}[name]
    rng = np.random.default_rng(seed)
    B = batch if batch is not None else 3
    if name == "c4_ragged_prefill_int8":
        past = rng.integers(0, max_len + 1, size=B)
        ql = rng.integers(0, 17, size=B)
        ql[0] = 0
        L = past + ql
    else:
        L = rng.integers(1, max_len + 1, size=B)
        ql = np.ones(B, dtype=np.int64)
    return make_problem(seed=seed, rng=rng, name=name + "_small", batch=B, num_heads=full["H"],
                        kv_num_heads=full["Hk"], head_size=full["D"], block_size=full["bs"],
                        kv_dtype=full["kv"], q_dtype=full["qd"], out_dtype=full["od"],
                        seqlens_k=L, q_lens=ql, pool_factor=2.0, kv_dist=full["dist"],
                        k_scale_range=full["ks"], v_scale_range=full["vs"],
                        k_boost_frac=full["kb"], causal=1)


def oracle_view(w: dict) -> dict:
    """The problem with float64 copies of q and the scales (exact values)."""
    d = dict(w)
    d["q"] = w["q"].double().numpy()
    d["k_scale"] = w["k_scale"].astype(np.float64)
    d["v_scale"] = w["v_scale"].astype(np.float64)
    return d
