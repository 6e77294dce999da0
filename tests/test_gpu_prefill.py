"""GPU parity of the tensor-core prefill path (tcgen05 MMAs, TMEM accumulators)
against the FP64 oracle, through the C ABI.

The planner sends units with more than 16 query rows per KV head (new tokens x
GQA group) over an INT8 cache with head_size 128 to this kernel (work items of
one KV head and up to 64 rows, padded to 16, 32, 48 or 64; 128-key tiles).
Cases: ragged causal prefill with zero-new-token sequences, every row padding,
lengths on and off the 128-key tile and the 16/32-token block edges, more than
one row group, forced KV splits (the combine kernel), an odd KV head count,
non-causal calls, bf16 queries and output, fp32 output, the per-row
log-sum-exp, extreme K scales, a bad block id.  Tolerance as for the
decode path: max|out - ref| <= 2e-3 * max|dequant(V)| (fp16 out), 8e-3 (bf16).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_quantized_kv_attention_b200 as pa
import workloads
from tests import _gpu
from tests._dense import paged_problem
from workloads import KV_INT8

pytestmark = pytest.mark.gpu


def _as_workload(prob, q_dtype=0, out_dtype=0):
    w = dict(prob)
    w["q"] = torch.from_numpy(prob["q"]).to(torch.bfloat16 if q_dtype else torch.float16)
    w["k_scale"] = prob["k_scale"].astype(np.float32)
    w["v_scale"] = prob["v_scale"].astype(np.float32)
    w["q_dtype"], w["out_dtype"] = q_dtype, out_dtype
    return w


def _check(w, out):
    ref = oracle.paged_attn(workloads.oracle_view(w))
    got = out.float().cpu().double().numpy()[: ref.shape[0]]
    vm = _gpu.vmax(w)
    tol = _gpu.TOL[w["out_dtype"]] * vm
    assert np.all(np.isfinite(got)), "non-finite output"
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert err <= tol, "max err %.3g > tol %.3g (Vmax %.3g)" % (err, tol, vm)


def _run_checked(w, **over):
    out, p, ws = _gpu.run(w, **over)
    assert p.rows_per_cta == 64, "the planner did not choose the tensor-core prefill kernel"
    st, bits = pa.paged_attn_read_device_error(ws)
    assert st == pa.PA_OK and bits == 0, bits
    _check(w, out)
    return out, p


@pytest.mark.parametrize("bs", [16, 32])
def test_ragged_causal_prefill(bs):
    """Lengths around the 64- and 128-key marks and the block edges, q_len 0..16."""
    rng = np.random.default_rng(500 + bs)
    lens = [5, 64, 65, 130, 0, 191, 300, 17, 1000, 48]
    ql = [5, 16, 7, 12, 0, 16, 1, 17 - 1, 13, 9]
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=lens, q_lens=ql, H=32, Hk=8, D=128, bs=bs)
    _run_checked(_as_workload(prob))


def test_more_than_one_row_group():
    """q_len 20 and 40 with G = 4: 80 and 160 rows, two and three row groups."""
    rng = np.random.default_rng(611)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[20, 300, 90], q_lens=[20, 40, 17], H=16,
                            Hk=4, D=128, bs=16)
    _, p = _run_checked(_as_workload(prob))
    assert p.num_row_groups == 3


@pytest.mark.parametrize("split_blocks", [1, 3, 8])
def test_forced_splits_merge_in_the_combine(split_blocks):
    rng = np.random.default_rng(620 + split_blocks)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[700, 90, 1200, 33], q_lens=[16, 5, 9, 8],
                            H=32, Hk=8, D=128, bs=16)
    _, p = _run_checked(_as_workload(prob), split_blocks=split_blocks)
    assert p.num_splits > 1


def test_odd_kv_head_count():
    """Hk = 3, G = 8: 24 query heads."""
    rng = np.random.default_rng(630)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[150, 70], q_lens=[10, 7], H=24, Hk=3,
                            D=128, bs=16)
    _run_checked(_as_workload(prob))


def test_non_causal_bf16():
    rng = np.random.default_rng(640)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[333, 64, 90], q_lens=[12, 6, 16], H=32,
                            Hk=8, D=128, bs=32, causal=0)
    _run_checked(_as_workload(prob, 1, 1))


@pytest.mark.parametrize("split_blocks", [-1, 5])
def test_fp32_output(split_blocks):
    """out_dtype PA_F32: unrounded rows, unsplit and through the combine."""
    rng = np.random.default_rng(645)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[410, 70, 129], q_lens=[11, 3, 16], H=32,
                            Hk=8, D=128, bs=16)
    _run_checked(_as_workload(prob, 0, 2), split_blocks=split_blocks)


def test_every_row_padding_and_tile_edge():
    """Units of 4..64 rows (R padded to 16, 32, 48, 64) with lengths at the
    128-key tile edges (127, 128, 129, 256, 257)."""
    rng = np.random.default_rng(646)
    lens = [127, 128, 129, 256, 257, 300, 64, 200]
    ql = [1, 4, 5, 8, 9, 12, 13, 16]
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=lens, q_lens=ql, H=32, Hk=8, D=128, bs=16)
    _run_checked(_as_workload(prob))


def test_c4_workload_small():
    for seed in (3, 4):
        w = workloads.shrink("c4_ragged_prefill_int8", seed, max_len=700, batch=12)
        _run_checked(w)


def test_lse_out_matches_the_oracle():
    """The per-row natural-log log-sum-exp of the scaled logits, unsplit and split."""
    rng = np.random.default_rng(650)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[400, 77], q_lens=[16, 9], H=16, Hk=4,
                            D=128, bs=16, causal=0)
    w = _as_workload(prob)
    T, H = int(prob["cu_seqlens_q"][-1]), prob["num_heads"]
    zeros = np.zeros(prob["batch"], dtype=np.int32)
    _, ref_lse = oracle.paged_attn_partial(workloads.oracle_view(w), zeros, prob["seqlens_k"])
    for sb in (-1, 4):
        lse = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
        d = _gpu.to_device(w)
        p, nb = _gpu.plan(w, split_blocks=sb)
        ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        p.workspace = ws.data_ptr()
        p.lse_out = lse.data_ptr()
        out = torch.empty((T, H, 128), dtype=torch.float16, device="cuda")
        pa.paged_attn_forward(d["q"], d["k_cache"], d["v_cache"], d["k_scale"], d["v_scale"],
                              d["block_table"], d["seqlens_k"], d["cu_seqlens_q"], out, p)
        torch.cuda.synchronize()
        assert p.rows_per_cta == 64
        got = lse.cpu().double().numpy()
        assert np.max(np.abs(got - ref_lse)) <= 1e-4 * max(1.0, np.max(np.abs(ref_lse)))


def test_run_to_run_bitwise_deterministic():
    w = workloads.shrink("c4_ragged_prefill_int8", 8, max_len=900, batch=10)
    d = _gpu.to_device(w)
    a, p, _ = _gpu.run(w, d)
    b, _, _ = _gpu.run(w, d)
    assert p.rows_per_cta == 64
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("kmag", [3.0e38, 1.0e-30])
def test_extreme_k_scales_follow_the_oracle(kmag):
    rng = np.random.default_rng(660)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[100, 45], q_lens=[16, 5], H=16, Hk=4,
                            D=128, bs=16)
    prob["k_scale"] = prob["k_scale"] / prob["k_scale"].max() * kmag
    _run_checked(_as_workload(prob))


def test_bad_block_id_is_flagged_not_faulted():
    rng = np.random.default_rng(670)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[100, 45], q_lens=[16, 5], H=16, Hk=4,
                            D=128, bs=16)
    w = _as_workload(prob)
    w["block_table"] = w["block_table"].copy()
    w["block_table"][0, 2] = w["num_blocks"] + 3
    out, p, ws = _gpu.run(w)
    assert p.rows_per_cta == 64
    st, bits = pa.paged_attn_read_device_error(ws)
    assert bits & pa.PA_DEVERR_BAD_BLOCK
    assert bool(torch.isfinite(out.float()).all())
