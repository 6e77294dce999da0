"""Test-side helpers: build paged problems from dense per-sequence values.

Written independently of both the oracle and the CUDA library: the INT4 packing
here is the plain bit layout (channel 2j -> low nibble of byte j, channel 2j+1 ->
high nibble, 4-bit two's complement) typed out with Python integer operations,
and FP8 values are decoded with torch's float8_e4m3fn.
"""
from __future__ import annotations

import numpy as np
import torch

from workloads import KV_FP8_E4M3, KV_INT4, KV_INT8


def pack_nibbles(vals: np.ndarray) -> np.ndarray:
    """int values in [-8, 7], last axis = channels (even) -> packed bytes."""
    v = vals.astype(np.int64) & 0xF
    return (v[..., 0::2] | (v[..., 1::2] << 4)).astype(np.uint8)


def random_codes(rng, kv_dtype, shape):
    """(cache bytes with the channel axis last, exact decoded values)."""
    if kv_dtype == KV_INT8:
        vals = rng.integers(-127, 128, size=shape).astype(np.int8)
        return vals.view(np.uint8), vals.astype(np.float64)
    if kv_dtype == KV_INT4:
        vals = rng.integers(-8, 8, size=shape)
        return pack_nibbles(vals), vals.astype(np.float64)
    codes = rng.integers(0, 256, size=shape).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C  # no NaN codes in attention inputs
    vals = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    return codes, vals


def paged_problem(rng, *, kv_dtype, lens, q_lens, H, Hk, D, bs, pool_factor=2.0, causal=1,
                  k_scale=None, v_scale=None, q=None, softmax_scale=0.0):
    """Dense per-sequence K/V values scattered into a paged cache.

    Returns (problem dict for the oracle, dense dict with the exact values).
    """
    B = len(lens)
    lens = np.asarray(lens, dtype=np.int32)
    q_lens = np.asarray(q_lens, dtype=np.int32)
    nblk = (lens + bs - 1) // bs
    need = int(nblk.sum())
    pool = max(1, int(np.ceil(pool_factor * need)))
    perm = rng.permutation(pool).astype(np.int32)
    maxb = max(1, int(nblk.max()) if B else 1)
    bt = np.full((B, maxb), -1, dtype=np.int32)
    chs = (D + 1) // 2 if kv_dtype == KV_INT4 else D
    kc = rng.integers(0, 256, size=(pool, bs, Hk, chs)).astype(np.uint8)  # junk everywhere
    vc = rng.integers(0, 256, size=(pool, bs, Hk, chs)).astype(np.uint8)
    if kv_dtype == KV_FP8_E4M3:
        kc[(kc & 0x7F) == 0x7F] = 0
        vc[(vc & 0x7F) == 0x7F] = 0
    Kd, Vd = [], []
    pos = 0
    for b in range(B):
        bt[b, :nblk[b]] = perm[pos:pos + nblk[b]]
        pos += int(nblk[b])
        kb, kvals = random_codes(rng, kv_dtype, (int(lens[b]), Hk, D))
        vb, vvals = random_codes(rng, kv_dtype, (int(lens[b]), Hk, D))
        for t in range(int(lens[b])):
            phys, slot = bt[b, t // bs], t % bs
            kc[phys, slot] = kb[t]
            vc[phys, slot] = vb[t]
        Kd.append(kvals)
        Vd.append(vvals)
    cu = np.zeros(B + 1, dtype=np.int32)
    cu[1:] = np.cumsum(q_lens)
    T = int(cu[-1])
    if k_scale is None:
        k_scale = rng.uniform(0.01, 0.1, size=(Hk, D))
    if v_scale is None:
        v_scale = rng.uniform(0.01, 0.1, size=(Hk, D))
    if q is None:
        q = rng.standard_normal((T, H, D))
    prob = dict(batch=B, num_heads=H, kv_num_heads=Hk, head_size=D, block_size=bs,
                num_blocks=pool, max_blocks_per_seq=maxb, kv_dtype=kv_dtype,
                softmax_scale=softmax_scale, causal=causal, q=np.asarray(q, dtype=np.float64),
                k_cache=kc, v_cache=vc, k_scale=np.asarray(k_scale, dtype=np.float64),
                v_scale=np.asarray(v_scale, dtype=np.float64), block_table=bt,
                seqlens_k=lens, cu_seqlens_q=cu)
    return prob, dict(K=Kd, V=Vd)


def brute_force(prob, dense):
    """Contiguous, non-paged attention with numpy matrix products."""
    H, Hk, D = prob["num_heads"], prob["kv_num_heads"], prob["head_size"]
    G = H // Hk
    scale = prob["softmax_scale"] or 1.0 / np.sqrt(D)
    cu = prob["cu_seqlens_q"]
    out = np.zeros((int(cu[-1]), H, D))
    for b in range(prob["batch"]):
        L = int(prob["seqlens_k"][b])
        qb = int(cu[b + 1] - cu[b])
        for i in range(qb):
            nk = (L - qb + i + 1) if prob["causal"] else L
            for h in range(H):
                kv = h // G
                khat = dense["K"][b][:nk, kv, :] * prob["k_scale"][kv]
                vhat = dense["V"][b][:nk, kv, :] * prob["v_scale"][kv]
                s = scale * (khat @ prob["q"][cu[b] + i, h])
                w = np.exp(s - s.max())
                out[cu[b] + i, h] = (w / w.sum()) @ vhat
    return out
