"""GPU parity: the CUDA path through the C ABI against the FP64 oracle.

Tolerance (stated by the workload description): max|out - ref| <= 2e-3 *
max|dequant(V)| for fp16 output and 8e-3 * max|dequant(V)| for bf16 output,
with fp32 accumulation; integer stages are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_quantized_kv_attention_b200 as pa
import workloads
from tests import _gpu
from tests._dense import pack_nibbles, paged_problem
from workloads import KV_FP8_E4M3, KV_INT4, KV_INT8

pytestmark = pytest.mark.gpu
ALL_KV = [KV_INT8, KV_INT4, KV_FP8_E4M3]


def _check(w, out, rows=None, seqs=None):
    ov = workloads.oracle_view(w)
    ref = oracle.paged_attn(ov)
    got = out.float().cpu().double().numpy()[: ref.shape[0]]
    vm = _gpu.vmax(w, seqs)
    err = np.max(np.abs(got - ref)) if ref.size else 0.0
    tol = _gpu.TOL[w["out_dtype"]] * vm
    assert np.all(np.isfinite(got)), "non-finite output"
    assert err <= tol, "max err %.3g > tol %.3g (Vmax %.3g)" % (err, tol, vm)
    return err / max(vm, 1e-30)


# ------------------------------------------------------------- integer stages


def test_int4_pack_unpack_bit_exact():
    vals = np.stack(np.meshgrid(np.arange(-8, 8), np.arange(-8, 8), indexing="ij"), -1)
    vals = np.tile(vals.reshape(-1), 4).reshape(-1, 128).astype(np.int8)  # 16 rows x 128
    src = torch.from_numpy(vals).cuda()
    dst = torch.empty((vals.shape[0], 64), dtype=torch.uint8, device="cuda")
    pa.paged_kv_pack_int4(src, dst, vals.shape[0], 128)
    back = torch.empty_like(src)
    pa.paged_kv_unpack_int4(dst, back, vals.shape[0], 128)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(dst.cpu().numpy(), oracle.pack_int4(vals))
    np.testing.assert_array_equal(dst.cpu().numpy(), pack_nibbles(vals))
    np.testing.assert_array_equal(back.cpu().numpy(), vals)


@pytest.mark.parametrize("kv", ALL_KV)
@pytest.mark.parametrize("dst_dtype", [0, 1])
def test_gather_decode_bit_exact(kv, dst_dtype):
    """Paged gather + code->fp16/bf16 conversion of every byte value, bit-exact."""
    rng = np.random.default_rng(5 + kv)
    prob, _ = paged_problem(rng, kv_dtype=kv, lens=[37, 64, 1], q_lens=[1, 1, 1], H=8, Hk=2,
                            D=128, bs=16)
    # make sure every byte value appears (NaN codes included for FP8)
    flat = prob["k_cache"].reshape(-1)
    flat[: 256] = np.arange(256, dtype=np.uint8)
    prob["k_cache"] = flat.reshape(prob["k_cache"].shape)
    p = pa.make_params(batch=3, num_heads=8, kv_num_heads=2, head_size=128, block_size=16,
                       num_blocks=prob["num_blocks"], max_blocks_per_seq=prob["max_blocks_per_seq"],
                       kv_dtype=kv, q_dtype=0, out_dtype=0)
    cache = torch.from_numpy(prob["k_cache"]).cuda()
    bt = torch.from_numpy(prob["block_table"]).cuda()
    for b in range(3):
        for h in range(2):
            L = int(prob["seqlens_k"][b])
            dt = torch.bfloat16 if dst_dtype else torch.float16
            dst = torch.empty((L, 128), dtype=dt, device="cuda")
            pa.paged_kv_gather_decode(cache, bt, p, b, h, L, dst_dtype, dst)
            torch.cuda.synchronize()
            got = dst.double().cpu().numpy()
            ref = oracle.gather_decode(prob, prob["k_cache"], b, h)
            np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
            ok = ~np.isnan(ref)
            np.testing.assert_array_equal(got[ok], ref[ok])
    # the block holding all 256 codes is decoded by some (b, kv): check directly
    all_codes = prob["k_cache"].reshape(-1)[:256]
    assert len(set(all_codes.tolist())) == 256


# ------------------------------------------------------------- small parity


@pytest.mark.parametrize("name", workloads.NAMES)
@pytest.mark.parametrize("seed", [11, 12])
def test_parity_small_shapes(name, seed):
    """Each workload's head layout, dtypes and distributions at oracle-friendly
    lengths that span several blocks and end in a ragged tail."""
    w = workloads.shrink(name, seed, max_len=300, batch=4)
    out, p, ws = _gpu.run(w)
    _check(w, out)
    st, bits = pa.paged_attn_read_device_error(ws)
    assert st == pa.PA_OK and bits == 0


def test_parity_c1_full():
    w = workloads.make("c1_tiny_int8")
    out, p, _ = _gpu.run(w)
    _check(w, out)


@pytest.mark.parametrize("kv", ALL_KV)
@pytest.mark.parametrize("lens", [[1], [16], [17], [31, 32, 33], [1, 2, 3, 4, 5, 6, 7, 8]])
def test_edge_lengths(kv, lens):
    rng = np.random.default_rng(sum(lens) + kv)
    for bs in (16, 32):
        for H, Hk in ((8, 1), (4, 4), (16, 2)):
            prob, _ = paged_problem(rng, kv_dtype=kv, lens=lens, q_lens=[1] * len(lens), H=H,
                                    Hk=Hk, D=64 if bs == 32 else 128, bs=bs)
            w = _as_workload(prob, q_dtype=0, out_dtype=0)
            out, _, _ = _gpu.run(w)
            _check(w, out)


@pytest.mark.parametrize("kv", ALL_KV)
@pytest.mark.parametrize("B,qmax,D", [(300, 1, 64), (170, 4, 128)])
def test_many_sequences_use_the_sparse_item_numbering(kv, B, qmax, D):
    """More sequences than the producer's shared-memory item table holds (256, or
    160 for the two-n-tile kernels with 128-byte rows): every sequence gets the
    largest item count and empty items are skipped.  Zero-new-token sequences mixed
    in; decode (300 sequences) and up to 16 rows per KV head (170 sequences)."""
    rng = np.random.default_rng(B + kv)
    ql = rng.integers(0, qmax + 1, size=B)
    lens = rng.integers(1, 60, size=B) + ql
    prob, _ = paged_problem(rng, kv_dtype=kv, lens=lens.tolist(), q_lens=ql.tolist(), H=8, Hk=2,
                            D=D, bs=16)
    w = _as_workload(prob, q_dtype=0, out_dtype=0)
    out, p, ws = _gpu.run(w)
    assert pa.paged_attn_read_device_error(ws)[1] == 0
    _check(w, out)


def _as_workload(prob, q_dtype, out_dtype):
    w = dict(prob)
    w["q"] = torch.from_numpy(prob["q"]).to(torch.bfloat16 if q_dtype else torch.float16)
    w["k_scale"] = prob["k_scale"].astype(np.float32)
    w["v_scale"] = prob["v_scale"].astype(np.float32)
    w["q_dtype"], w["out_dtype"] = q_dtype, out_dtype
    return w


@pytest.mark.parametrize("kv", ALL_KV)
def test_prefill_causal_with_zero_new_token_rows(kv):
    """Ragged prefill: q_len 0..16 with zero rows, bottom-right causal mask; the
    output rows past total_q keep their sentinel."""
    rng = np.random.default_rng(77 + kv)
    lens = [0, 5, 40, 16, 100, 3, 64]
    ql = [0, 5, 16, 0, 9, 1, 13]
    prob, _ = paged_problem(rng, kv_dtype=kv, lens=lens, q_lens=ql, H=32, Hk=8, D=128, bs=16)
    w = _as_workload(prob, 0, 0)
    out, p, _ = _gpu.run(w, extra_rows=3, sentinel=0x7BCD)
    assert p.max_query_len == 16
    _check(w, out)
    tail = out[-3:].view(torch.int16).cpu()
    assert bool((tail == 0x7BCD).all())
    body = out[:-3].view(torch.int16).cpu()
    assert not bool((body == 0x7BCD).all(dim=-1).any())


@pytest.mark.parametrize("kv", ALL_KV)
def test_split_and_unsplit_agree(kv):
    """Flash-decoding split + LSE combine against the single-pass kernel and the
    oracle (the GQA GEMV decode page's flash-vs-naive parity)."""
    rng = np.random.default_rng(88 + kv)
    prob, _ = paged_problem(rng, kv_dtype=kv, lens=[700, 33, 1500, 257], q_lens=[1, 1, 1, 1],
                            H=64, Hk=8, D=128, bs=32)
    w = _as_workload(prob, 1, 1)
    o1, p1, _ = _gpu.run(w, split_blocks=-1)
    o2, p2, _ = _gpu.run(w, split_blocks=8)
    assert p1.num_splits == 1 and p2.num_splits > 1
    _check(w, o1)
    _check(w, o2)
    vm = _gpu.vmax(w)
    assert float((o1.float() - o2.float()).abs().max()) <= _gpu.TOL[1] * vm


def test_run_to_run_bitwise_deterministic():
    w = workloads.shrink("c3_int8_long_split", 5, max_len=2000, batch=3)
    d = _gpu.to_device(w)
    a, _, _ = _gpu.run(w, d)
    b, _, _ = _gpu.run(w, d)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_bf16_queries_of_large_magnitude_stay_finite():
    """The per-row power-of-two normaliser keeps folded queries inside fp16 range."""
    rng = np.random.default_rng(99)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[50, 20], q_lens=[1, 1], H=8, Hk=2,
                            D=128, bs=16)
    prob["q"] = prob["q"] * 1.0e6
    w = _as_workload(prob, 1, 1)
    w["q"] = torch.from_numpy(prob["q"]).to(torch.bfloat16)
    ov = workloads.oracle_view(w)
    out, _, _ = _gpu.run(w)
    ref = oracle.paged_attn(ov)
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - ref)) <= _gpu.TOL[1] * _gpu.vmax(w)


def test_bad_block_id_is_flagged_not_faulted():
    rng = np.random.default_rng(3)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[40, 40], q_lens=[1, 1], H=8, Hk=2,
                            D=128, bs=16)
    w = _as_workload(prob, 0, 0)
    w["block_table"] = w["block_table"].copy()
    w["block_table"][1, 1] = w["num_blocks"] + 5  # outside the pool
    out, p, ws = _gpu.run(w)
    st, bits = pa.paged_attn_read_device_error(ws)
    assert st == pa.PA_ERR_BAD_BLOCK_TABLE and bits & pa.PA_DEVERR_BAD_BLOCK
    st, bits = pa.paged_attn_read_device_error(ws)  # cleared by the previous read
    assert st == pa.PA_OK and bits == 0
    # sequence 0 is unaffected
    ov = workloads.oracle_view(w)
    ov["block_table"] = prob["block_table"]
    ref = oracle.paged_attn(ov)
    got = out.double().cpu().numpy()
    vm = _gpu.vmax(dict(w, block_table=prob["block_table"]), [0])
    assert np.max(np.abs(got[0] - ref[0])) <= _gpu.TOL[0] * vm


def test_non_finite_k_scale_is_flagged():
    rng = np.random.default_rng(4)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[40], q_lens=[1], H=8, Hk=2, D=128,
                            bs=16)
    w = _as_workload(prob, 0, 0)
    w["k_scale"] = w["k_scale"].copy()
    w["k_scale"][1, 3] = np.inf
    out, p, ws = _gpu.run(w)
    st, bits = pa.paged_attn_read_device_error(ws)
    assert bits & pa.PA_DEVERR_BAD_SCALE


@pytest.mark.parametrize("which,val", [("k", np.nan), ("v", np.nan), ("v", -np.inf)])
def test_nan_or_infinite_scale_is_flagged(which, val):
    """A NaN K scale (which a max over the channels would skip), or a non-finite
    V scale, sets the defined error bit; nothing faults."""
    rng = np.random.default_rng(5)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT4, lens=[40, 70], q_lens=[1, 1], H=8, Hk=2,
                            D=128, bs=16)
    w = _as_workload(prob, 0, 0)
    key = which + "_scale"
    w[key] = w[key].copy()
    w[key][1, 77] = val
    out, p, ws = _gpu.run(w)
    st, bits = pa.paged_attn_read_device_error(ws)
    assert bits & pa.PA_DEVERR_BAD_SCALE


@pytest.mark.parametrize("kv", ALL_KV)
@pytest.mark.parametrize("kmag", [3.0e38, 1.0e30, 1.0e-30])
def test_extreme_k_scales_follow_the_oracle(kv, kmag):
    """K scales up to FLT_MAX (and down to 1e-30): finite outputs equal to the
    oracle's (which, for huge scales, is the V row of the largest logit)."""
    rng = np.random.default_rng(int(np.log10(kmag) + 100) + kv)
    Hk, D = 2, 128
    k_scale = (kmag * rng.uniform(0.25, 1.0, size=(Hk, D))).astype(np.float32)
    prob, _ = paged_problem(rng, kv_dtype=kv, lens=[60, 33, 90], q_lens=[1, 4, 1], H=8, Hk=Hk,
                            D=D, bs=16, k_scale=k_scale)
    w = _as_workload(prob, 1, 1)
    assert np.all(np.isfinite(w["k_scale"]))
    for split in (-1, 2):
        out, p, ws = _gpu.run(w, split_blocks=split)
        st, bits = pa.paged_attn_read_device_error(ws)
        assert bits == 0
        got = out.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        _check(w, out)


def test_queries_near_bf16_max_stay_finite():
    """bf16 queries of magnitude 1e38 (the multiplier would overflow without its
    cap): finite outputs equal to the oracle's."""
    rng = np.random.default_rng(98)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[50, 20], q_lens=[1, 2], H=8, Hk=2,
                            D=128, bs=16)
    w = _as_workload(prob, 1, 1)
    w["q"] = (w["q"].float().clamp(-3.0, 3.0) * 1.0e38).to(torch.bfloat16)  # |q| <= 3e38
    assert bool(torch.isfinite(w["q"]).all())
    out, _, ws = _gpu.run(w)
    assert pa.paged_attn_read_device_error(ws)[1] == 0
    _check(w, out)


# ------------------------------------------------------------- full sizes, sampled


@pytest.mark.parametrize("name", ["c2_int4_decode", "c3_int8_long_split",
                                  "c4_ragged_prefill_int8", "c5_fp8_large_batch"])
def test_parity_full_size_sampled(name):
    """Full workload in the launch configuration the benchmark times; the oracle
    recomputes 16 whole sequences (all their heads and tokens; all of them when
    the workload has fewer)."""
    w = workloads.make(name)
    out, p, ws = _gpu.run(w)
    got = out.float().cpu().double().numpy()
    rng = np.random.default_rng(2024)
    qlens = np.diff(w["cu_seqlens_q"])
    cand = np.nonzero(qlens > 0)[0]
    # 16 whole sequences (every one when there are fewer), always the first and
    # the last so that both ends of the item numbering are in the sample; each
    # sequence is checked over all of its query heads, so every KV head and
    # head group is covered
    pick = {int(cand[0]), int(cand[-1])}
    rest = [int(b) for b in cand if int(b) not in pick]
    pick.update(int(b) for b in rng.choice(rest, size=min(14, len(rest)), replace=False))
    seqs = sorted(pick)
    cu = w["cu_seqlens_q"]
    for b in seqs:
        s = _gpu.sub_problem(w, int(b))
        ref = oracle.paged_attn(workloads.oracle_view(s))
        g = got[cu[b]:cu[b + 1]]
        vm = _gpu.vmax(w, [int(b)])
        assert np.max(np.abs(g - ref)) <= _gpu.TOL[w["out_dtype"]] * vm, (name, b)
    assert np.all(np.isfinite(got))
    st, bits = pa.paged_attn_read_device_error(ws)
    assert st == pa.PA_OK and bits == 0


def test_repeated_calls_share_one_workspace():
    """Work and split counters rewind at the end of every call: back-to-back calls
    on one workspace (persistent CTAs, many split items, shallow stage rings)
    give bit-identical, oracle-checked results."""
    w = workloads.shrink("c3_int8_long_split", 21, max_len=6000, batch=3)
    d = _gpu.to_device(w)
    p, ws_bytes = _gpu.plan(w, split_blocks=4)
    assert p.num_splits > 8
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    pa.paged_attn_workspace_init(ws, ws_bytes)
    p.workspace = ws.data_ptr()
    outs = []
    for _ in range(4):
        out = torch.empty((int(w["cu_seqlens_q"][-1]), w["num_heads"], w["head_size"]),
                          dtype=torch.bfloat16, device="cuda")
        pa.paged_attn_forward(d["q"], d["k_cache"], d["v_cache"], d["k_scale"], d["v_scale"],
                              d["block_table"], d["seqlens_k"], d["cu_seqlens_q"], out, p)
        outs.append(out)
    torch.cuda.synchronize()
    st, bits = pa.paged_attn_read_device_error(ws)
    assert st == pa.PA_OK and bits == 0
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    _check(w, outs[-1])


@pytest.mark.parametrize("kv", ALL_KV)
def test_full_length_beyond_the_dense_item_table(kv):
    """300 decode sequences of up to 2048 keys: more sequences than the kernel's
    shared-memory item table holds, so the sparse item numbering runs at full
    lengths (with splits); 16 sampled sequences are recomputed by the oracle."""
    B = 300
    rng = np.random.default_rng(4242 + kv)
    L = rng.integers(1, 2049, size=B)
    w = workloads.make_problem(seed=4242 + kv, rng=rng, batch=B, num_heads=32, kv_num_heads=8,
                               head_size=128, block_size=16, kv_dtype=kv, q_dtype=workloads.F16,
                               out_dtype=workloads.F16, seqlens_k=L, q_lens=np.ones(B),
                               pool_factor=1.0, kv_dist="fp8" if kv == KV_FP8_E4M3 else "uniform127",
                               k_scale_range=(0.01, 0.1), v_scale_range=(0.01, 0.1),
                               k_boost_frac=0.01)
    out, p, ws = _gpu.run(w)
    got = out.float().cpu().double().numpy()
    seqs = sorted({0, B - 1} | {int(b) for b in rng.choice(np.arange(1, B - 1), 14, replace=False)})
    for b in seqs:
        ref = oracle.paged_attn(workloads.oracle_view(_gpu.sub_problem(w, b)))
        vm = _gpu.vmax(w, [b])
        assert np.max(np.abs(got[b:b + 1] - ref)) <= _gpu.TOL[0] * vm, b
    st, bits = pa.paged_attn_read_device_error(ws)
    assert st == pa.PA_OK and bits == 0


def test_stream_read_checksum():
    """The read-ceiling kernel reads every 16-byte word once: the XOR of its
    per-block checksums equals the XOR of all words of the buffer."""
    n = (64 << 20) + 48  # a ragged tail past the unrolled loop
    buf = torch.randint(0, 256, (n,), dtype=torch.uint8, device="cuda")
    sink = torch.zeros(16 * 148 * 8, dtype=torch.uint8, device="cuda")
    pa.paged_attn_stream_read(buf, n, sink)
    torch.cuda.synchronize()
    words = buf.cpu().numpy().view(np.uint32).reshape(-1, 4)
    want = np.bitwise_xor.reduce(words, axis=0)
    got = np.bitwise_xor.reduce(sink.cpu().numpy().view(np.uint32).reshape(-1, 4), axis=0)
    np.testing.assert_array_equal(got, want)


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    """The consumer warps wait on a barrier that nothing signals (the
    stall_consumers diagnostic): the wait's bound runs out, the kernel records
    PA_DEVERR_TIMEOUT and returns (its producer drains every copy it issued), and
    the next call on the re-initialised workspace is correct."""
    w = workloads.shrink("c2_int4_decode", 41, max_len=300, batch=3)
    d = _gpu.to_device(w)
    p, nb = _gpu.plan(w, split_blocks=-1)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    pa.paged_attn_workspace_init(ws, ws.numel())
    p.workspace = ws.data_ptr()
    p.stall_consumers = 1
    out = torch.empty((int(w["cu_seqlens_q"][-1]), w["num_heads"], w["head_size"]),
                      dtype=torch.float16, device="cuda")
    pa.paged_attn_forward(d["q"], d["k_cache"], d["v_cache"], d["k_scale"], d["v_scale"],
                          d["block_table"], d["seqlens_k"], d["cu_seqlens_q"], out, p)
    torch.cuda.synchronize()
    st, bits = pa.paged_attn_read_device_error(ws)
    assert bits & pa.PA_DEVERR_TIMEOUT and st == pa.PA_ERR_DEVICE
    p.stall_consumers = 0
    pa.paged_attn_workspace_init(ws, ws.numel())
    pa.paged_attn_forward(d["q"], d["k_cache"], d["v_cache"], d["k_scale"], d["v_scale"],
                          d["block_table"], d["seqlens_k"], d["cu_seqlens_q"], out, p)
    torch.cuda.synchronize()
    assert pa.paged_attn_read_device_error(ws) == (pa.PA_OK, 0)
    _check(w, out)
