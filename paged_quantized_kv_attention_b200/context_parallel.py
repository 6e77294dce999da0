"""Context parallelism: one long sequence's KV cache spread over several GPUs.

Each rank holds a contiguous run of every sequence's KV blocks, runs
``paged_attn_forward`` over its own keys with ``params.lse_out`` set, and the
ranks exchange their (output, log-sum-exp) rows; ``paged_attn_merge`` then
combines them exactly as the flash-decoding split of the GQA GEMV decode page
(Code analysis 2) combines its workers' partials.  The exchange is one
all-gather per call over ``torch.distributed`` (NCCL over NVLink on GPUs).

Only new tokens that see every key of their sequence (decode, or a non-causal
call) can be split this way: a causal new token would need the rank's key
offset in its mask.  The helpers here are host-side plumbing; every arithmetic
step runs in the library's kernels.
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


def merge_across_ranks(out_local, lse_local, rows_local, total_q: int, group=None, merge=None):
    """All-gather every rank's rows (output [n, H, D], log-sum-exp [n, H] at
    global token indices ``rows_local``) and merge them into [total_q, H, D].

    Rows a rank does not hold count as empty parts (log-sum-exp -inf).  ``merge``
    defaults to the library's ``paged_attn_merge``; it is called as
    merge(parts [W, total_q, H, D], lses [W, total_q, H], out)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    H, D = out_local.shape[1], out_local.shape[2]
    full = out_local.new_zeros((total_q, H, D))
    lse = torch.full((total_q, H), float("-inf"), dtype=lse_local.dtype, device=out_local.device)
    if len(rows_local):
        idx = torch.as_tensor(rows_local, device=out_local.device)
        full.index_copy_(0, idx, out_local)
        lse.index_copy_(0, idx, lse_local)
    parts = [torch.empty_like(full) for _ in range(world)]
    lses = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(parts, full, group=group)
    dist.all_gather(lses, lse, group=group)
    parts_t, lses_t = torch.stack(parts), torch.stack(lses)
    out = torch.empty_like(full)
    if merge is None:
        from . import PA_BF16, PA_F16, paged_attn_merge
        paged_attn_merge(parts_t, lses_t, world, total_q * H, D,
                         PA_BF16 if full.dtype == torch.bfloat16 else PA_F16, out)
    else:
        merge(parts_t, lses_t, out)
    return out
