"""GPU parity of the quantise-and-append cache writer against the oracle.

Every cache byte is an integer decision, so the comparison is bit for bit over
the whole K and V caches (the written rows and every untouched byte).  The
codes are decided in IEEE single precision on both sides.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_quantized_kv_attention_b200 as pa
import workloads
from tests import _gpu
from tests._dense import paged_problem
from workloads import KV_FP8_E4M3, KV_INT4, KV_INT8

pytestmark = pytest.mark.gpu
ALL_KV = [KV_INT8, KV_INT4, KV_FP8_E4M3]


def _problem(kv, seed, lens, q_lens, *, Hk=4, D=128, bs=16, bf16=False):
    rng = np.random.default_rng(seed)
    prob, _ = paged_problem(rng, kv_dtype=kv, lens=lens, q_lens=q_lens, H=2 * Hk, Hk=Hk, D=D,
                            bs=bs)
    T = int(prob["cu_seqlens_q"][-1])
    tdt = torch.bfloat16 if bf16 else torch.float16
    # quotients x / s (s ~ U[0.01, 0.1]) spanning each format's range, some past it;
    # one value in eight is small (FP8 subnormals, zero codes)
    mag = 0.15 if kv == KV_INT4 else 3.0

    def draw():
        x = rng.standard_normal((T, Hk, D)) * mag
        x[rng.random((T, Hk, D)) < 0.125] *= 1e-3
        return torch.from_numpy(x).to(tdt)

    k_new, v_new = draw(), draw()
    prob["k_scale"] = rng.uniform(0.01, 0.1, size=(Hk, D)).astype(np.float32)
    prob["v_scale"] = rng.uniform(0.01, 0.1, size=(Hk, D)).astype(np.float32)
    prob["q"] = torch.zeros((T, 2 * Hk, D), dtype=tdt)
    prob["q_dtype"] = prob["out_dtype"] = 1 if bf16 else 0
    return prob, k_new, v_new


def _run(prob, k_new, v_new):
    """Append on the GPU; returns (k_cache, v_cache, error bits)."""
    d = _gpu.to_device(prob)
    p, nb = _gpu.plan(prob)
    ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")
    p.workspace = ws.data_ptr()
    p.workspace_bytes = ws.numel()
    pa.paged_kv_append(k_new.cuda(), v_new.cuda(), d["k_cache"], d["v_cache"], d["k_scale"],
                       d["v_scale"], d["block_table"], d["seqlens_k"], d["cu_seqlens_q"], p)
    torch.cuda.synchronize()
    _, bits = pa.paged_attn_read_device_error(ws)
    return d["k_cache"].cpu().numpy(), d["v_cache"].cpu().numpy(), bits


def _oracle(prob, k_new, v_new):
    return oracle.append(prob, k_new.double().numpy(), v_new.double().numpy())


@pytest.mark.parametrize("kv", ALL_KV)
@pytest.mark.parametrize("D,bs,bf16", [(128, 16, False), (64, 32, True), (128, 32, True)])
def test_append_bit_exact(kv, D, bs, bf16):
    """Ragged new-token counts (one sequence with none), tokens crossing block
    boundaries, values past the code range (saturation): every byte of both
    caches equals the oracle's."""
    prob, kn, vn = _problem(kv, 100 + kv * 7 + D + bs, [5, 40, 17, 3, 64, 33], [2, 17, 0, 3, 16, 33],
                            D=D, bs=bs, bf16=bf16)
    kc, vc, bits = _run(prob, kn, vn)
    ko, vo = _oracle(prob, kn, vn)
    assert bits == 0
    np.testing.assert_array_equal(kc, ko)
    np.testing.assert_array_equal(vc, vo)


@pytest.mark.parametrize("kv", ALL_KV)
def test_append_ties_and_specials(kv):
    """Power-of-two scales with values on exact half steps (ties to even), zeros
    of both signs, infinities and NaN: the same codes as the oracle."""
    prob, kn, vn = _problem(kv, 300 + kv, [16], [16], Hk=2, D=64)
    prob["k_scale"][:] = 0.25
    prob["v_scale"][:] = 2.0 ** -3
    rng = np.random.default_rng(9)
    steps = rng.integers(-300, 300, size=kn.shape) + 0.5
    kn = torch.from_numpy(steps * 0.25).to(torch.float16)
    flat = vn.view(-1)
    flat[:6] = torch.tensor([0.0, -0.0, float("inf"), float("-inf"), float("nan"), 1e4],
                            dtype=vn.dtype)
    kc, vc, bits = _run(prob, kn, vn)
    ko, vo = _oracle(prob, kn, vn)
    np.testing.assert_array_equal(kc, ko)
    np.testing.assert_array_equal(vc, vo)


@pytest.mark.parametrize("kv", ALL_KV)
def test_append_codes_next_to_a_rounding_boundary(kv):
    """Inputs whose exact quotient x / s sits just past a boundary between two
    codes, where x times a rounded 1 / s would store the neighbouring code: the
    kernel stores the code of the correctly rounded quotient (decided here from
    the exact rational, independently of the oracle) and agrees with the oracle
    on every byte."""
    from tests._quotient_points import boundary_points
    D, Hk = 64, 2
    pts = boundary_points(kv, 64, seed=800 + kv)
    pts = [pts[(i * 37) % len(pts)] for i in range(2 * Hk * D)]  # each point on several channels
    prob, kn, vn = _problem(kv, 900 + kv, [3], [3], Hk=Hk, D=D)
    xs = np.array([x for x, _, _ in pts], dtype=np.float64).reshape(2, Hk, D)
    ss = np.array([s for _, s, _ in pts], dtype=np.float32).reshape(2, Hk, D)
    want = np.array([c for _, _, c in pts]).reshape(2, Hk, D)
    prob["k_scale"], prob["v_scale"] = ss[0].copy(), ss[1].copy()
    kn[1] = torch.from_numpy(xs[0]).to(torch.float16)  # token 1: the boundary values
    vn[1] = torch.from_numpy(xs[1]).to(torch.float16)
    kc, vc, bits = _run(prob, kn, vn)
    ko, vo = _oracle(prob, kn, vn)
    assert bits == 0
    np.testing.assert_array_equal(kc, ko)
    np.testing.assert_array_equal(vc, vo)
    bt, bs = prob["block_table"], prob["block_size"]
    phys, slot = bt[0, 1 // bs], 1 % bs
    for cache, w in ((kc, want[0]), (vc, want[1])):
        row = cache[phys, slot]  # [Hk, chs]
        if kv == KV_INT4:
            nib = np.stack([row & 0xF, row >> 4], axis=-1).reshape(Hk, D).astype(np.int16)
            got = np.where(nib >= 8, nib - 16, nib)
        elif kv == KV_INT8:
            got = row.view(np.int8).astype(np.int16)
        else:
            got = row.astype(np.int16)
        np.testing.assert_array_equal(got, w)


def test_append_bad_block_id_is_flagged_and_skipped():
    """A new token whose page id is outside the pool is not written and sets
    the BAD_BLOCK bit; the other sequences' rows are written as usual."""
    prob, kn, vn = _problem(KV_INT8, 400, [20, 30], [4, 5])
    bad = prob["block_table"].copy()
    bad[1, 1] = prob["num_blocks"] + 7  # page of sequence 1's new tokens (positions 25..29)
    ok_prob = dict(prob)
    ok_prob["block_table"] = bad
    kc, vc, bits = _run(ok_prob, kn, vn)
    assert bits & pa.PA_DEVERR_BAD_BLOCK
    # sequence 0 alone, through the oracle
    only0 = dict(prob)
    only0["cu_seqlens_q"] = np.array([0, 4, 4], dtype=np.int32)
    only0["seqlens_k"] = np.array([20, 25], dtype=np.int32)  # sequence 1 appends nothing
    ko, vo = oracle.append(only0, kn[:4].double().numpy(), vn[:4].double().numpy())
    np.testing.assert_array_equal(kc, ko)
    np.testing.assert_array_equal(vc, vo)


@pytest.mark.parametrize("kv", ALL_KV)
def test_append_then_attend_matches_oracle(kv):
    """The writer feeding the forward call: the attention over the GPU-appended
    cache equals the oracle's attention over the oracle-appended cache."""
    prob, kn, vn = _problem(kv, 500 + kv, [48, 70, 9], [16, 1, 9], Hk=2, D=128)
    rng = np.random.default_rng(77)
    prob["q"] = torch.from_numpy(rng.standard_normal(tuple(prob["q"].shape))).to(torch.float16)
    prob["q_dtype"] = prob["out_dtype"] = 0
    kc, vc, bits = _run(prob, kn, vn)
    assert bits == 0
    after = dict(prob)
    after["k_cache"], after["v_cache"] = kc, vc
    out, _, _ = _gpu.run(after)
    ref = oracle.paged_attn(workloads.oracle_view(after))
    got = out.double().cpu().numpy()[: ref.shape[0]]
    assert np.max(np.abs(got - ref)) <= _gpu.TOL[0] * _gpu.vmax(after)


def test_append_full_size_sampled():
    """The long-prompt append at full size (32768 new tokens, 8 KV heads, D=128,
    INT8, bf16): a sample of 64 rows equals the oracle's codes."""
    T, Hk, D, bs = 32768, 8, 128, 16
    rng = np.random.default_rng(600)
    nblk = T // bs
    pool = 2 * nblk
    kc = torch.zeros((pool, bs, Hk, D), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    bt = rng.permutation(pool)[:nblk].astype(np.int32).reshape(1, nblk)
    ks = rng.uniform(0.01, 0.1, size=(Hk, D)).astype(np.float32)
    vs = rng.uniform(0.01, 0.1, size=(Hk, D)).astype(np.float32)
    kn = (torch.randn((T, Hk, D), generator=torch.Generator().manual_seed(1)) * 3).to(torch.bfloat16)
    vn = (torch.randn((T, Hk, D), generator=torch.Generator().manual_seed(2)) * 3).to(torch.bfloat16)
    cu = np.array([0, T], dtype=np.int32)
    sk = np.array([T], dtype=np.int32)
    p = pa.make_params(batch=1, num_heads=Hk, kv_num_heads=Hk, head_size=D, block_size=bs,
                       num_blocks=pool, max_blocks_per_seq=nblk, kv_dtype=KV_INT8, q_dtype=1,
                       out_dtype=1)
    nb = pa.paged_attn_plan(cu, sk, p)
    ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device="cuda")
    p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    dev = lambda a: torch.from_numpy(a).cuda()
    pa.paged_kv_append(kn.cuda(), vn.cuda(), kc, vc, dev(ks), dev(vs), dev(bt), dev(sk), dev(cu), p)
    torch.cuda.synchronize()
    assert pa.paged_attn_read_device_error(ws)[1] == 0
    for t in rng.choice(T, 64, replace=False):
        phys, slot = int(bt[0, t // bs]), int(t % bs)
        for kvh in (0, Hk - 1):
            for new, cache, sc in ((kn, kc, ks), (vn, vc, vs)):
                want = [oracle.quantise(KV_INT8, float(new[t, kvh, d]), float(sc[kvh, d])) & 0xFF
                        for d in range(D)]
                got = cache[phys, slot, kvh].cpu().numpy().tolist()
                assert got == want
