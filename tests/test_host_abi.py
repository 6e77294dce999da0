"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every
declared entry point, and its planner and argument checks behave as documented.
"""
import os
import re

import numpy as np
import pytest

import paged_quantized_kv_attention_b200 as pa
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "paged_attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:pa_status|const char\*)\s+(\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 10
    L = pa.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(pa.EXPORTED)
    assert "sm_100a" in pa.paged_attn_version()


def _params(**kw):
    base = dict(batch=4, num_heads=32, kv_num_heads=8, head_size=128, block_size=16,
                num_blocks=1024, max_blocks_per_seq=256, kv_dtype=pa.PA_KV_INT8,
                q_dtype=pa.PA_F16, out_dtype=pa.PA_F16, num_sms=148)
    base.update(kw)
    return pa.make_params(**base)


def test_plan_exact_max_query_len_golden():
    """The exact max_query_len page: the host max replaces token_count - batch + 1."""
    with open(os.path.join(GOLDEN, "max_query_len.txt")) as f:
        rows = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    for ln in rows:
        cu_s, exact, heur = [x.strip() for x in ln.split("|")]
        cu = np.array([int(x) for x in cu_s.split(",")], dtype=np.int32)
        B = len(cu) - 1
        assert cu[-1] - B + 1 == int(heur)  # the fixture's heuristic column is what it claims
        lens = np.diff(cu) + 5
        p = _params(batch=B, max_blocks_per_seq=8)
        pa.paged_attn_plan(cu, lens, p)
        assert p.max_query_len == int(exact)
        assert p.total_q == cu[-1]
        G = 32 // 8
        rows_needed = int(exact) * G
        assert p.num_row_groups == -(-rows_needed // p.rows_per_cta)
        assert p.num_row_groups >= 0  # never negative, unlike the heuristic


def test_plan_zero_new_tokens_everywhere_is_a_no_op():
    cu = np.zeros(5, dtype=np.int32)
    p = _params(batch=4)
    pa.paged_attn_plan(cu, np.array([3, 0, 7, 1]), p)
    assert p.max_query_len == 0 and p.num_row_groups == 0 and p.total_q == 0
    # forward returns OK without touching any pointer (no GPU needed)
    pa.paged_attn_forward(None, None, None, None, None, None, None, None, None, p, stream=0)


def _count_items(cu, L, G, Hk, bs, rows, T, max_splits):
    """Work items by the documented split rule: a sequence with n KV blocks gets
    s = min(max_splits, ceil(n / T)) splits of ceil(n / s) blocks (empty ones
    dropped), times its groups of KV heads (4 per item; 1 for the 64-row items
    of the tensor-core prefill kernel) times its row groups."""
    hp = 1 if rows == 64 else 4
    total, most = 0, 1
    for b in range(len(L)):
        qb = int(cu[b + 1] - cu[b])
        if qb == 0:
            continue
        n = -(-int(L[b]) // bs)
        s = max(1, min(max_splits, -(-n // T)))
        per = -(-n // s)
        s = -(-n // per)
        most = max(most, s)
        total += (-(-Hk // hp)) * (-(-qb * G // rows)) * s
    return total, most


@pytest.mark.parametrize("name,split", [("c1_tiny_int8", False), ("c2_int4_decode", True),
                                        ("c3_int8_long_split", True),
                                        ("c4_ragged_prefill_int8", None),
                                        ("c5_fp8_large_batch", None)])
def test_plan_split_decisions_on_the_workload_shapes(name, split):
    """Flash-decoding split (the GQA GEMV decode page's rule, sized for the
    resident CTAs): the tiny case stays whole, the cases whose (sequence, KV
    head) units underfill the device are split, and the planned item count is
    the documented split rule applied to the host lengths."""
    rng = np.random.default_rng(0)
    if name == "c1_tiny_int8":
        B, H, Hk, D, bs, L, ql = 2, 4, 1, 64, 16, np.array([37, 64]), np.ones(2, int)
    elif name == "c2_int4_decode":
        B, H, Hk, D, bs = 16, 32, 8, 128, 16
        L, ql = rng.integers(512, 4097, B), np.ones(B, int)
    elif name == "c3_int8_long_split":
        B, H, Hk, D, bs, L, ql = 4, 64, 8, 128, 32, np.full(4, 32768), np.ones(4, int)
    elif name == "c4_ragged_prefill_int8":
        B, H, Hk, D, bs = 64, 32, 8, 128, 16
        ql = rng.integers(0, 17, B)
        L = rng.integers(0, 2049, B) + ql
    else:
        B, H, Hk, D, bs, L, ql = 128, 64, 8, 128, 16, np.full(128, 8192), np.ones(128, int)
    cu = np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)
    maxb = int(-(-L.max() // bs))
    kvd = pa.PA_KV_INT4 if name == "c2_int4_decode" else pa.PA_KV_INT8
    p = _params(batch=B, num_heads=H, kv_num_heads=Hk, head_size=D, block_size=bs,
                num_blocks=maxb * B, max_blocks_per_seq=maxb, kv_dtype=kvd)
    ws = pa.paged_attn_plan(cu, L, p)
    if split is not None:
        assert (p.num_splits > 1) == split
    assert 1 <= p.num_splits <= 128 and p.blocks_per_split >= 1
    items, most = _count_items(cu, L, H // Hk, Hk, bs, p.rows_per_cta, p.blocks_per_split, 128)
    assert p.num_work_items == items
    assert p.num_splits == most
    assert ws >= 256 and ws % 256 == 0
    if p.num_splits > 1:
        # fp16 partial rows (D halves) and one fp32 log-sum-exp per split row
        assert ws >= 256 + p.num_splits * p.total_q * H * (2 * D + 4)
    if name == "c3_int8_long_split":
        # equal sequences: one round of items over 148 SMs x 3 resident CTAs
        assert p.num_work_items <= 148 * 3


def test_plan_forced_and_disabled_split():
    cu = np.array([0, 1], dtype=np.int32)
    L = np.array([1000], dtype=np.int32)
    p = _params(batch=1, split_blocks=10)
    pa.paged_attn_plan(cu, L, p)
    assert p.blocks_per_split == 10 and p.num_splits == 7  # ceil(63 / 10)
    p = _params(batch=1, split_blocks=-1)
    pa.paged_attn_plan(cu, L, p)
    assert p.num_splits == 1


@pytest.mark.parametrize("mut,status", [
    (dict(head_size=96), pa.PA_ERR_UNSUPPORTED),
    (dict(block_size=8), pa.PA_ERR_UNSUPPORTED),
    (dict(num_heads=30), pa.PA_ERR_INVALID_ARG),
    (dict(kv_dtype=7), pa.PA_ERR_INVALID_ARG),
    (dict(q_dtype=3), pa.PA_ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), pa.PA_ERR_INVALID_ARG),
    (dict(causal=2), pa.PA_ERR_INVALID_ARG),
])
def test_plan_rejects_bad_problems(mut, status):
    p = _params(**mut)
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_attn_plan(np.array([0, 1, 2, 3, 4]), np.array([5, 5, 5, 5]), p)
    assert ei.value.status == status
    assert pa.paged_attn_last_error() != ""


@pytest.mark.parametrize("cu,L", [
    ([0, 3, 4, 5, 6], [2, 5, 5, 5]),      # more new tokens than keys
    ([1, 2, 3, 4, 5], [5, 5, 5, 5]),      # cu[0] != 0
    ([0, 3, 2, 4, 5], [5, 5, 5, 5]),      # decreasing offsets
    ([0, 1, 2, 3, 4], [5, 5, 5, 5000]),   # longer than the block table allows
])
def test_plan_rejects_contract_violations(cu, L):
    p = _params()
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_attn_plan(np.array(cu), np.array(L), p)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG


def test_forward_checks_arguments_before_any_launch():
    cu = np.array([0, 1], dtype=np.int32)
    p = _params(batch=1)
    pa.paged_attn_plan(cu, np.array([40]), p)
    fake = np.zeros(64, dtype=np.uint8)  # host memory: never dereferenced by these checks
    args = [fake] * 9
    # missing workspace
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_attn_forward(*args, p, stream=0)
    assert ei.value.status == pa.PA_ERR_WORKSPACE
    # a NULL device pointer
    p.workspace = fake.ctypes.data & ~0xFF
    bad = list(args)
    bad[3] = None
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_attn_forward(*bad, p, stream=0)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG
    # params not produced by the planner
    q = pa.paged_attn_params.from_buffer_copy(p)
    q.rows_per_cta = 3
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_attn_forward(*args, q, stream=0)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG


def test_append_checks_arguments_before_any_launch():
    cu = np.array([0, 3], dtype=np.int32)
    p = _params(batch=1)
    pa.paged_attn_plan(cu, np.array([40]), p)
    buf = np.zeros(4096, dtype=np.uint8)
    al = buf[(-buf.ctypes.data) % 256:]  # 256-aligned host memory, never dereferenced here
    args = [al] * 9
    # a NULL pointer
    p.workspace, p.workspace_bytes = al.ctypes.data, 256
    bad = list(args)
    bad[4] = None
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_kv_append(*bad, p, stream=0)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG
    # misaligned new rows
    bad = list(args)
    bad[0] = al[4:]
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_kv_append(*bad, p, stream=0)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG
    # no workspace for the error word
    p.workspace, p.workspace_bytes = None, 0
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_kv_append(*args, p, stream=0)
    assert ei.value.status == pa.PA_ERR_WORKSPACE
    # no new tokens: nothing to do, nothing launched
    p0 = _params(batch=1)
    pa.paged_attn_plan(np.array([0, 0], dtype=np.int32), np.array([40]), p0)
    pa.paged_kv_append(*args, p0, stream=0)


def test_merge_checks_arguments_before_any_launch():
    buf = np.zeros(1024, dtype=np.uint8)
    al = buf[(-buf.ctypes.data) % 16:]
    for bad in (dict(n_parts=0), dict(n_parts=65), dict(head_size=96), dict(src=7),
                dict(dst=pa.PA_F32), dict(dst=7)):
        kw = dict(n_parts=2, head_size=128, src=pa.PA_F32, dst=pa.PA_F16)
        kw.update(bad)
        with pytest.raises(pa.PagedAttnError):
            pa.paged_attn_merge(al, kw["src"], al, kw["n_parts"], 4, kw["head_size"], al, kw["dst"],
                                stream=0)
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_attn_merge(None, pa.PA_F16, al, 2, 4, 128, al, pa.PA_F16, stream=0)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PagedAttnError):  # fp32 parts must be 16-byte aligned
        pa.paged_attn_merge(al[8:], pa.PA_F32, al, 2, 4, 128, al, pa.PA_F16, stream=0)
    pa.paged_attn_merge(al, pa.PA_F32, al, 2, 0, 128, al, pa.PA_F16, stream=0)  # no rows: no launch


def test_forward_accepts_fp32_output_and_rejects_it_for_queries():
    p = _params(out_dtype=pa.PA_F32)
    pa.paged_attn_plan(np.array([0, 1, 2, 3, 4], dtype=np.int32), np.array([40, 5, 9, 100]), p)
    p = _params(q_dtype=pa.PA_F32)
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_attn_plan(np.array([0, 1, 2, 3, 4], dtype=np.int32), np.array([40, 5, 9, 100]), p)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG


def test_codec_entry_points_check_arguments():
    with pytest.raises(pa.PagedAttnError):
        pa.paged_kv_pack_int4(None, None, 4, 128, stream=0)
    buf = np.zeros(1024, dtype=np.uint8)
    with pytest.raises(pa.PagedAttnError):
        pa.paged_kv_pack_int4(buf, buf, 4, 12, stream=0)  # head_size not a multiple of 8


def test_workload_generators_follow_the_stated_shapes():
    w = workloads.make("c1_tiny_int8")
    assert w["k_cache"].shape == (16, 16, 1, 64)
    assert list(w["seqlens_k"]) == [37, 64]
    bt = w["block_table"]
    used = bt[bt >= 0]
    assert len(used) == 7 and len(set(used.tolist())) == 7
    assert w["q"].dtype.__str__() == "torch.float16"
    k = w["k_cache"].view(np.int8)
    assert k.min() >= -127 and k.max() <= 127
    assert w["k_scale"].min() >= 0.005 and w["k_scale"].max() <= 0.02


def test_noalloc_rejects_plans_beyond_its_static_scratch():
    """The no-alloc forward refuses, before any device work, a plan whose
    workspace exceeds the library's static scratch."""
    B, ql, L = 8, 16, 4096
    cu = np.arange(0, B * ql + 1, ql, dtype=np.int32)
    p = _params(batch=B, num_heads=64, kv_num_heads=8, max_blocks_per_seq=L // 16,
                num_blocks=B * L // 16, split_blocks=8)
    need = pa.paged_attn_plan(cu, np.full(B, L, dtype=np.int32), p)
    assert need > pa.PA_NOALLOC_MAX_WORKSPACE_BYTES
    fake = np.zeros(64, dtype=np.uint8)  # host memory: never dereferenced
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_attn_forward_noalloc(*([fake] * 9), p, stream=0)
    assert ei.value.status == pa.PA_ERR_WORKSPACE
    assert "static scratch" in pa.paged_attn_last_error()
    unplanned = pa.make_params(batch=1, num_heads=8, kv_num_heads=8, head_size=128,
                               block_size=16, num_blocks=4, max_blocks_per_seq=4,
                               kv_dtype=pa.PA_KV_INT8, q_dtype=pa.PA_F16, out_dtype=pa.PA_F16)
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.paged_attn_forward_noalloc(*([fake] * 9), unplanned, stream=0)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG


def test_plan_sends_many_row_units_to_the_tensor_core_prefill_kernel():
    """Units with more than 16 rows (new tokens x GQA group) over an INT8 cache
    with head_size 128 are planned as 64-row items of the tcgen05 prefill kernel
    (the workspace then holds one unit of query digit planes per sequence, KV
    head and row group: 3 x 64 rows x 128 bytes and 64 multipliers); other
    formats and shapes keep the 4/8/16-row kernel."""
    cu = np.array([0, 16, 21], dtype=np.int32)
    L = np.array([300, 40], dtype=np.int32)
    for kvd, D, want in ((pa.PA_KV_INT8, 128, 64), (pa.PA_KV_INT4, 128, 16),
                         (pa.PA_KV_FP8_E4M3, 128, 16), (pa.PA_KV_INT8, 64, 16)):
        p = _params(batch=2, num_heads=32, kv_num_heads=8, head_size=D, block_size=16,
                    num_blocks=64, max_blocks_per_seq=32, kv_dtype=kvd, split_blocks=-1)
        ws = pa.paged_attn_plan(cu, L, p)
        assert p.rows_per_cta == want, (kvd, D, p.rows_per_cta)
        if want == 64:
            unit = 3 * 64 * 128 + 64 * 4
            assert p.num_row_groups == 1
            assert ws == 256 + -(-(2 * 8 * unit) // 256) * 256  # no split here
    # decode rows (4 per KV head) stay on the decode kernel
    p = _params(batch=2, num_heads=32, kv_num_heads=8, head_size=128, block_size=16,
                num_blocks=64, max_blocks_per_seq=32, kv_dtype=pa.PA_KV_INT8)
    pa.paged_attn_plan(np.array([0, 1, 2], dtype=np.int32), L, p)
    assert p.rows_per_cta == 4
