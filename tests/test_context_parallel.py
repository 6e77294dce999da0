"""Context parallelism (one sequence's KV spread over ranks): host sharding, the
all-gather over torch.distributed (gloo ranks on the CPU) and, on one GPU, the
rank-local forward calls with their log-sum-exps merged by paged_attn_merge."""
import os

import numpy as np
import pytest
import torch

import oracle
import paged_quantized_kv_attention_b200 as pa
import workloads
from paged_quantized_kv_attention_b200 import context_parallel as cp
from tests._dense import paged_problem
from workloads import KV_FP8_E4M3, KV_INT4, KV_INT8


def _problem(seed, kv=KV_INT8, lens=(300, 47, 1000, 17), bs=16):
    rng = np.random.default_rng(seed)
    prob, _ = paged_problem(rng, kv_dtype=kv, lens=list(lens), q_lens=[1] * len(lens), H=8, Hk=2,
                            D=128, bs=bs)
    return prob


def test_shard_ranges_partition_every_sequence():
    L = np.array([0, 1, 15, 16, 17, 300, 1000])
    for world in (1, 2, 3, 8):
        r = cp.shard_ranges(L, 16, world)
        assert r.shape == (world, len(L), 2)
        for b, Lb in enumerate(L):
            # contiguous, in rank order, block aligned, covering [0, L)
            assert r[0, b, 0] == 0 and r[-1, b, 1] == Lb
            for k in range(world - 1):
                assert r[k, b, 1] == r[k + 1, b, 0]
            assert all(r[k, b, 0] % 16 == 0 for k in range(world) if r[k, b, 1] > r[k, b, 0])
            sizes = [(r[k, b, 1] - r[k, b, 0] + 15) // 16 for k in range(world)]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("world", [2, 3, 5])
def test_local_problems_rebuild_the_full_attention(world):
    """Host-side rank views: each rank's block table, lengths and rows, run through
    the oracle as an ordinary problem, merge (oracle combine) into the unsplit
    attention (1e-12); a rank without keys for a sequence gets no rows for it."""
    prob = _problem(31, lens=(300, 47, 1000, 17, 5))
    T, H, D = int(prob["cu_seqlens_q"][-1]), prob["num_heads"], prob["head_size"]
    ranges = cp.shard_ranges(prob["seqlens_k"], prob["block_size"], world)
    parts = np.zeros((world, T, H, D))
    lses = np.full((world, T, H), -np.inf)
    for r in range(world):
        lbt, lL, lcu, rows = cp.local_problem(prob["block_table"], prob["cu_seqlens_q"], ranges[r],
                                              prob["block_size"])
        assert len(rows) == int(lcu[-1])
        if len(rows) == 0:
            continue
        loc = dict(prob, block_table=lbt, seqlens_k=lL, cu_seqlens_q=lcu,
                   max_blocks_per_seq=lbt.shape[1], q=prob["q"][rows])
        o, l = oracle.paged_attn_partial(loc, np.zeros_like(lL), lL)
        parts[r, rows], lses[r, rows] = o, l
    merged = oracle.lse_combine(parts.reshape(world, T * H, D), lses.reshape(world, T * H))
    ref = oracle.paged_attn(prob)
    assert np.max(np.abs(merged.reshape(T, H, D) - ref)) <= 1e-12 * np.max(np.abs(ref))


def _oracle_rank(prob, ranges_r):
    """Rank-local (output, lse) rows from the oracle's partial attention."""
    o, lse = oracle.paged_attn_partial(prob, ranges_r[:, 0], ranges_r[:, 1])
    rows = [t for b in range(prob["batch"]) if ranges_r[b, 1] > ranges_r[b, 0]
            for t in range(int(prob["cu_seqlens_q"][b]), int(prob["cu_seqlens_q"][b + 1]))]
    return o[rows], lse[rows], np.asarray(rows, dtype=np.int64)


def _gloo_rank(rank, world, port, result):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    prob = _problem(5)
    ranges = cp.shard_ranges(prob["seqlens_k"], prob["block_size"], world)
    o, lse, rows = _oracle_rank(prob, ranges[rank])

    def merge(parts, lses, out):  # the oracle's combine stands in for the kernel on the CPU
        W, T, H, D = parts.shape
        m = oracle.lse_combine(parts.reshape(W, T * H, D).numpy(), lses.reshape(W, T * H).numpy())
        out.copy_(torch.from_numpy(m.reshape(T, H, D)))

    T = int(prob["cu_seqlens_q"][-1])
    out = cp.merge_across_ranks(torch.from_numpy(o), torch.from_numpy(lse), rows, T,
                                out_dtype=torch.float64, merge=merge)
    if rank == 0:
        ref = oracle.paged_attn(prob)
        result.put(float(np.max(np.abs(out.numpy() - ref)) / np.max(np.abs(ref))))
    dist.barrier()
    dist.destroy_process_group()


def test_gloo_two_ranks_merge_to_the_unsplit_result():
    """World size 2 over gloo: shards, the all-to-all of each rank's rows to their
    owners, the merge and the all-gather give the oracle's unsplit attention
    (1e-12)."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    ps = [ctx.Process(target=_gloo_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in ps)
    assert q.get(timeout=5) < 1e-12


# ----------------------------------------------------------------- on one GPU


def _gpu_forward(w, lse=True, **over):
    from tests import _gpu
    d = _gpu.to_device(w)
    p, nb = _gpu.plan(w, **over)
    ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")
    p.workspace = ws.data_ptr()
    T, H, D = int(w["cu_seqlens_q"][-1]), w["num_heads"], w["head_size"]
    odt = {0: torch.float16, 1: torch.bfloat16, 2: torch.float32}[w["out_dtype"]]
    out = torch.empty((T, H, D), dtype=odt, device="cuda")
    lse_t = torch.empty((T, H), dtype=torch.float32, device="cuda")
    if lse:
        p.lse_out = lse_t.data_ptr()
    pa.paged_attn_forward(d["q"], d["k_cache"], d["v_cache"], d["k_scale"], d["v_scale"],
                          d["block_table"], d["seqlens_k"], d["cu_seqlens_q"], out, p)
    torch.cuda.synchronize()
    assert pa.paged_attn_read_device_error(ws)[1] == 0
    return out, lse_t, p


def _as_w(prob, q_dtype=1):
    w = dict(prob)
    w["q"] = torch.from_numpy(prob["q"]).to(torch.bfloat16 if q_dtype else torch.float16)
    w["k_scale"] = prob["k_scale"].astype(np.float32)
    w["v_scale"] = prob["v_scale"].astype(np.float32)
    w["q_dtype"] = w["out_dtype"] = q_dtype
    return w


@pytest.mark.gpu
@pytest.mark.parametrize("split", [-1, 3])
def test_forward_lse_out_matches_the_oracle(split):
    """lse_out of an unsplit call (written by the fused kernel) and of a split
    call (written by the combine) equals the oracle's log-sum-exp."""
    prob = _problem(11)
    w = _as_w(prob)
    _, lse, p = _gpu_forward(w, split_blocks=split)
    assert (p.num_splits > 1) == (split > 0)
    L = prob["seqlens_k"]
    _, ref = oracle.paged_attn_partial(workloads.oracle_view(w), np.zeros_like(L), L)
    got = lse.double().cpu().numpy()
    assert np.max(np.abs(got - ref)) <= 1e-4 * max(1.0, np.max(np.abs(ref)))


@pytest.mark.gpu
@pytest.mark.parametrize("kv", [KV_INT8, KV_INT4, KV_FP8_E4M3])
@pytest.mark.parametrize("world", [2, 3])
def test_rank_local_calls_merge_to_the_full_result(kv, world):
    """The ranks emulated one after another on one GPU (no kernel waits on
    another): each runs the forward over its own key ranges with lse_out, the
    rows are merged by paged_attn_merge, and the result meets the parity bar
    against the oracle's unsplit attention."""
    from tests import _gpu
    prob = _problem(20 + kv + world, kv=kv)
    w = _as_w(prob)
    w["out_dtype"] = pa.PA_F32  # the ranks' partial rows, unrounded
    T, H, D = int(w["cu_seqlens_q"][-1]), w["num_heads"], w["head_size"]
    ranges = cp.shard_ranges(prob["seqlens_k"], prob["block_size"], world)
    parts = torch.zeros((world, T, H, D), dtype=torch.float32, device="cuda")
    lses = torch.full((world, T, H), float("-inf"), dtype=torch.float32, device="cuda")
    for r in range(world):
        lbt, lL, lcu, rows = cp.local_problem(prob["block_table"], prob["cu_seqlens_q"], ranges[r],
                                              prob["block_size"])
        wr = dict(w, block_table=lbt, seqlens_k=lL, cu_seqlens_q=lcu,
                  max_blocks_per_seq=lbt.shape[1], q=w["q"][torch.as_tensor(rows)])
        if len(rows) == 0:
            continue
        o, l, _ = _gpu_forward(wr)
        idx = torch.as_tensor(rows, device="cuda")
        parts[r].index_copy_(0, idx, o)
        lses[r].index_copy_(0, idx, l)
    out = torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda")
    pa.paged_attn_merge(parts, pa.PA_F32, lses, world, T * H, D, out, pa.PA_BF16)
    torch.cuda.synchronize()
    ref = oracle.paged_attn(workloads.oracle_view(w))
    got = out.double().cpu().numpy()
    assert np.max(np.abs(got - ref)) <= _gpu.TOL[1] * _gpu.vmax(w)


def test_local_problem_is_for_decode_rows_only():
    """A rank's key range can be shorter than a sequence's new tokens, so only
    decode steps (at most one new token per sequence) are split across ranks."""
    prob = _problem(7)
    ranges = cp.shard_ranges(prob["seqlens_k"], prob["block_size"], 2)
    cu = np.array([0, 1, 3, 4, 5], dtype=np.int32)  # sequence 1 has two new tokens
    with pytest.raises(ValueError):
        cp.local_problem(prob["block_table"], cu, ranges[0], prob["block_size"])


@pytest.mark.gpu
def test_fp32_output_matches_the_rounded_one():
    """out_dtype PA_F32 gives the unrounded rows: rounding them to bf16 gives the
    bf16 call's output to within one bf16 rounding, and both meet the bar."""
    from tests import _gpu
    prob = _problem(31)
    w = _as_w(prob)
    o16, _, _ = _gpu_forward(w)
    w32 = dict(w, out_dtype=pa.PA_F32)
    o32, _, _ = _gpu_forward(w32)
    assert o32.dtype == torch.float32
    ref = oracle.paged_attn(workloads.oracle_view(w))
    vm = _gpu.vmax(w)
    assert np.max(np.abs(o32.double().cpu().numpy() - ref)) <= _gpu.TOL[0] * vm
    diff = (o32.to(torch.bfloat16).float() - o16.float()).abs().max().item()
    assert diff <= 2 ** -7 * vm
