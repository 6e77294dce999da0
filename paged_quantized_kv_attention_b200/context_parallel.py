"""Context parallelism: one long sequence's KV cache spread over several GPUs.

Each rank holds a contiguous run of every sequence's KV blocks and runs
``paged_attn_forward`` over its own keys with ``params.lse_out`` set and
``out_dtype = PA_F32`` (its partial rows unrounded).  The ranks then exchange
the rows so that each merges the rows it owns: one all-to-all of the fp32
(output, log-sum-exp) rows, where rank r receives every rank's part of its own
block of rows; ``paged_attn_merge`` combines them exactly as the flash-decoding
split of the GQA GEMV decode page (Code analysis 2) combines its workers'
partials; one all-gather of the merged rows (in the output type) gives every
rank the whole result.  Both collectives go over ``torch.distributed`` (NCCL
over NVLink on GPUs).  Per rank the exchange moves about T H (4 D + 4) bytes out
and T H 2 D bytes in (T rows, H heads, head size D), independent of the rank
count.

Only new tokens that see every key of their sequence can be split this way; the
helpers accept decode steps (at most one new token per sequence), whose token
sees all keys.  A causal prefill row would need the rank's key offset in its
mask, and a multi-token non-causal row would give a rank more new tokens than
keys.  The helpers here are host-side plumbing; every arithmetic step runs in
the library's kernels.
"""
from __future__ import annotations

import numpy as np


def shard_ranges(seqlens_k, block_size: int, world: int) -> np.ndarray:
    """Key ranges [lo, hi) of every sequence per rank, shape [world, batch, 2]:
    the sequence's blocks dealt out in contiguous runs, as even as whole blocks
    allow (rank r takes blocks [r n / world, (r + 1) n / world))."""
    L = np.asarray(seqlens_k, dtype=np.int64)
    nblk = (L + block_size - 1) // block_size
    out = np.zeros((world, len(L), 2), dtype=np.int64)
    for r in range(world):
        b0 = (r * nblk) // world
        b1 = ((r + 1) * nblk) // world
        out[r, :, 0] = np.minimum(b0 * block_size, L)
        out[r, :, 1] = np.minimum(b1 * block_size, L)
    return out


def local_problem(block_table, cu_seqlens_q, ranges_r, block_size: int):
    """Rank-local view of the batch for one rank's key ranges [batch, 2]:
    (local block table, local seqlens_k, local cu_seqlens_q, rows) where
    sequences without a key on this rank get no new-token rows, and ``rows``
    lists the global token index of every local row."""
    bt = np.asarray(block_table)
    cu = np.asarray(cu_seqlens_q, dtype=np.int64)
    if np.any(np.diff(cu) > 1):
        raise ValueError("context parallelism splits decode rows only: at most one new token "
                         "per sequence (a rank's key range may be shorter than more new tokens)")
    B = bt.shape[0]
    lo, hi = ranges_r[:, 0], ranges_r[:, 1]
    nloc = (hi - lo + block_size - 1) // block_size
    maxb = max(1, int(nloc.max()) if B else 1)
    lbt = np.full((B, maxb), -1, dtype=np.int32)
    lq = np.zeros(B, dtype=np.int64)
    rows = []
    for b in range(B):
        if hi[b] > lo[b]:
            first = lo[b] // block_size
            lbt[b, :nloc[b]] = bt[b, first:first + nloc[b]]
            lq[b] = cu[b + 1] - cu[b]
            rows.extend(range(int(cu[b]), int(cu[b + 1])))
    lcu = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    return lbt, (hi - lo).astype(np.int32), lcu, np.asarray(rows, dtype=np.int64)


def merge_across_ranks(out_local, lse_local, rows_local, total_q: int, out_dtype=None,
                       group=None, merge=None):
    """Merge every rank's partial rows into the full result [total_q, H, D].

    ``out_local`` [n, H, D] are this rank's rows (fp32 from a forward call with
    out_dtype PA_F32) at the global token indices ``rows_local``, ``lse_local``
    [n, H] their log-sum-exps; rows this rank does not hold count as empty parts
    (log-sum-exp -inf).  The rows are dealt in contiguous blocks of ceil(T / W)
    to the W ranks: one all-to-all brings each rank every part of its block, the
    merge combines them into ``out_dtype`` (default bf16), and one all-gather
    returns the merged blocks to every rank.  ``merge`` defaults to the library's
    ``paged_attn_merge``; it is called as merge(parts [W, rows, H, D],
    lses [W, rows, H], out [rows, H, D])."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    H, D = out_local.shape[1], out_local.shape[2]
    out_dtype = out_dtype if out_dtype is not None else torch.bfloat16
    per = -(-total_q // world)  # rows owned by each rank
    Tp = per * world
    dev = out_local.device
    full = torch.zeros((Tp, H, D), dtype=out_local.dtype, device=dev)
    lse = torch.full((Tp, H), float("-inf"), dtype=lse_local.dtype, device=dev)
    if len(rows_local):
        idx = torch.as_tensor(rows_local, device=dev)
        full.index_copy_(0, idx, out_local)
        lse.index_copy_(0, idx, lse_local)
    parts = torch.empty((world, per, H, D), dtype=full.dtype, device=dev)
    lses = torch.empty((world, per, H), dtype=lse.dtype, device=dev)
    dist.all_to_all_single(parts.view(-1), full.view(-1), group=group)
    dist.all_to_all_single(lses.view(-1), lse.view(-1), group=group)
    mine = torch.empty((per, H, D), dtype=out_dtype, device=dev)
    if merge is None:
        from . import PA_BF16, PA_F16, PA_F32, paged_attn_merge
        src = {torch.float32: PA_F32, torch.bfloat16: PA_BF16, torch.float16: PA_F16}[parts.dtype]
        paged_attn_merge(parts, src, lses, world, per * H, D, mine,
                         PA_BF16 if out_dtype == torch.bfloat16 else PA_F16)
    else:
        merge(parts, lses, mine)
    gathered = torch.empty((Tp, H, D), dtype=out_dtype, device=dev)
    dist.all_gather_into_tensor(gathered, mine, group=group)
    return gathered[:total_q]
