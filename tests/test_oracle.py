"""Pins of the FP64 oracle against facts fixed by the pages and by mathematics.

Nothing here calls the CUDA library.  Each test states what it pins:
codec facts (INT4 nibble layout, e4m3 code points), closed forms (Q = 0 mean,
one key, two keys), invariants (block permutation, linearity, identical GQA
heads, causal prefix), a contiguous brute force, split/combine equivalence
and the scale fold of the INT4 paged-KV page (onnxruntime PR 32515, Code
analysis 3).
"""
import os

import numpy as np
import pytest
import torch

import oracle
from tests._dense import brute_force, pack_nibbles, paged_problem
from workloads import KV_FP8_E4M3, KV_INT4, KV_INT8

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
KV_BY_NAME = {"int8": KV_INT8, "int4": KV_INT4, "fp8_e4m3": KV_FP8_E4M3}
ALL_KV = [KV_INT8, KV_INT4, KV_FP8_E4M3]


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(1e-300, np.max(np.abs(b)))


# ---------------------------------------------------------------- codecs


def test_cache_head_size_golden():
    for kv, hs, chs in _rows("cache_head_size.txt"):
        assert oracle.cache_head_size(KV_BY_NAME[kv], int(hs)) == int(chs)
    # INT4 is exactly half of INT8 for an even head size
    for hs in (64, 128, 256):
        assert 2 * oracle.cache_head_size(KV_INT4, hs) == oracle.cache_head_size(KV_INT8, hs)


def test_int4_roundtrip_exhaustive():
    lo, hi = np.meshgrid(np.arange(-8, 8), np.arange(-8, 8), indexing="ij")
    vals = np.stack([lo.ravel(), hi.ravel()], axis=1).astype(np.int8)  # 256 rows x 2 channels
    packed = oracle.pack_int4(vals)
    assert packed.shape == (256, 1)
    assert len(set(packed.ravel().tolist())) == 256  # bijective on bytes
    np.testing.assert_array_equal(oracle.unpack_int4(packed, 2), vals)
    # the byte layout matches the stated nibble order (channel 2j low nibble)
    np.testing.assert_array_equal(packed, pack_nibbles(vals))
    with pytest.raises(ValueError):
        oracle.pack_int4(np.array([[8, 0]], dtype=np.int8))


def test_int4_odd_head_size_padding():
    vals = np.array([[1, -2, 3]], dtype=np.int8)
    packed = oracle.pack_int4(vals)
    assert packed.shape == (1, 2) and packed[0, 1] == 3  # high nibble of the pad byte is 0
    np.testing.assert_array_equal(oracle.unpack_int4(packed, 3), vals)


def test_int8_decode_all_bytes():
    for byte in range(256):
        got = oracle.decode_row(KV_INT8, np.array([byte], dtype=np.uint8), 1)[0]
        assert got == np.array([byte], dtype=np.uint8).view(np.int8)[0]


def test_e4m3_golden_points():
    for code, val in _rows("e4m3_points.txt"):
        got = oracle.decode_row(KV_FP8_E4M3, np.array([int(code, 16)], dtype=np.uint8), 1)[0]
        if val == "nan":
            assert np.isnan(got)
        else:
            assert got == float(val) and np.signbit(got) == val.startswith("-")


def test_e4m3_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.decode_row(KV_FP8_E4M3, codes[i:i + 1], 1)[0] for i in range(256)])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    # sign symmetry
    np.testing.assert_array_equal(got[1:127], -got[129:255])


# ---------------------------------------------------------------- closed forms


@pytest.mark.parametrize("kv", ALL_KV)
def test_q_zero_gives_mean_of_v(kv):
    rng = np.random.default_rng(1)
    lens, ql = [5, 23, 16], [1, 3, 2]
    prob, dense = paged_problem(rng, kv_dtype=kv, lens=lens, q_lens=ql, H=4, Hk=2, D=8, bs=4)
    prob["q"][:] = 0.0
    out = oracle.paged_attn(prob)
    cu = prob["cu_seqlens_q"]
    for b, (L, qb) in enumerate(zip(lens, ql)):
        for i in range(qb):
            nk = L - qb + i + 1
            for h in range(4):
                kv_h = h // 2
                mean = (dense["V"][b][:nk, kv_h, :] * prob["v_scale"][kv_h]).mean(axis=0)
                assert _rel(out[cu[b] + i, h], mean) < 1e-13


@pytest.mark.parametrize("kv", ALL_KV)
def test_single_key_returns_its_v_row(kv):
    rng = np.random.default_rng(2)
    prob, dense = paged_problem(rng, kv_dtype=kv, lens=[1, 1], q_lens=[1, 1], H=6, Hk=3, D=16,
                                bs=16)
    out = oracle.paged_attn(prob)
    for b in range(2):
        for h in range(6):
            kv_h = h // 2
            np.testing.assert_array_equal(out[b, h], dense["V"][b][0, kv_h] * prob["v_scale"][kv_h])


def test_two_keys_closed_form():
    rng = np.random.default_rng(3)
    prob, dense = paged_problem(rng, kv_dtype=KV_INT8, lens=[2], q_lens=[1], H=2, Hk=1, D=32,
                                bs=16, softmax_scale=0.37)
    out = oracle.paged_attn(prob)
    for h in range(2):
        k = dense["K"][0][:, 0, :] * prob["k_scale"][0]
        v = dense["V"][0][:, 0, :] * prob["v_scale"][0]
        s1, s2 = 0.37 * (k[0] @ prob["q"][0, h]), 0.37 * (k[1] @ prob["q"][0, h])
        sig = lambda x: 1.0 / (1.0 + np.exp(-x))  # noqa: E731
        ref = sig(s1 - s2) * v[0] + sig(s2 - s1) * v[1]
        assert _rel(out[0, h], ref) < 1e-13


def test_one_hot_logit_selects_its_row():
    rng = np.random.default_rng(4)
    D = 16
    prob, dense = paged_problem(rng, kv_dtype=KV_INT8, lens=[40], q_lens=[1], H=1, Hk=1, D=D,
                                bs=8, k_scale=np.ones((1, D)), v_scale=np.ones((1, D)))
    # make key 17 the only one aligned with q, by a wide margin
    j = 17
    kbytes = np.zeros(D, dtype=np.int8)
    kbytes[0] = 127
    for t in range(40):
        phys, slot = prob["block_table"][0, t // 8], t % 8
        row = np.zeros(D, dtype=np.int8)
        row[0] = 127 if t == j else 0
        prob["k_cache"][phys, slot, 0] = row.view(np.uint8)
    prob["q"][:] = 0.0
    prob["q"][0, 0, 0] = 10.0  # logit gap 10 * 127 / 4 = 317
    out = oracle.paged_attn(prob)
    np.testing.assert_allclose(out[0, 0], dense["V"][0][j, 0], rtol=0, atol=1e-100)


# ---------------------------------------------------------------- invariants


@pytest.mark.parametrize("kv", ALL_KV)
def test_matches_contiguous_brute_force(kv):
    rng = np.random.default_rng(10 + kv)
    lens, ql = [1, 17, 33, 64, 9], [1, 4, 0, 7, 9]
    prob, dense = paged_problem(rng, kv_dtype=kv, lens=lens, q_lens=ql, H=8, Hk=2, D=32, bs=16)
    out = oracle.paged_attn(prob)
    assert _rel(out, brute_force(prob, dense)) < 1e-12


def test_non_causal_matches_brute_force():
    rng = np.random.default_rng(20)
    prob, dense = paged_problem(rng, kv_dtype=KV_INT8, lens=[12, 30], q_lens=[3, 5], H=4, Hk=4,
                                D=16, bs=4, causal=0)
    assert _rel(oracle.paged_attn(prob), brute_force(prob, dense)) < 1e-12


@pytest.mark.parametrize("kv", ALL_KV)
def test_block_permutation_invariance(kv):
    rng = np.random.default_rng(30 + kv)
    prob, _ = paged_problem(rng, kv_dtype=kv, lens=[45, 3, 64], q_lens=[2, 1, 5], H=4, Hk=2, D=16,
                            bs=8)
    out = oracle.paged_attn(prob)
    perm = rng.permutation(prob["num_blocks"])  # new position of each old block
    p2 = dict(prob)
    p2["k_cache"] = np.empty_like(prob["k_cache"])
    p2["v_cache"] = np.empty_like(prob["v_cache"])
    p2["k_cache"][perm] = prob["k_cache"]
    p2["v_cache"][perm] = prob["v_cache"]
    bt = prob["block_table"].copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    p2["block_table"] = bt
    np.testing.assert_array_equal(oracle.paged_attn(p2), out)


def test_linearity_in_scales():
    rng = np.random.default_rng(40)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT4, lens=[20, 7], q_lens=[1, 2], H=4, Hk=2, D=16,
                            bs=4)
    out = oracle.paged_attn(prob)
    p2 = dict(prob, v_scale=prob["v_scale"] * 2.0)
    np.testing.assert_array_equal(oracle.paged_attn(p2), 2.0 * out)
    p3 = dict(prob, k_scale=prob["k_scale"] * 3.0, softmax_scale=(1.0 / 4.0) / 3.0)
    assert _rel(oracle.paged_attn(p3), out) < 1e-13


def test_identical_heads_in_group_give_identical_rows():
    rng = np.random.default_rng(50)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[30], q_lens=[3], H=8, Hk=2, D=16, bs=8)
    prob["q"][:, 1:4] = prob["q"][:, 0:1]  # heads 0..3 share kv head 0
    out = oracle.paged_attn(prob)
    for h in (1, 2, 3):
        np.testing.assert_array_equal(out[:, h], out[:, 0])
    assert not np.array_equal(out[:, 4], out[:, 0])


def test_causal_row_equals_truncated_decode():
    """New token i of a prefill sees exactly the first L - q + i + 1 keys."""
    rng = np.random.default_rng(60)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[29], q_lens=[6], H=2, Hk=1, D=16, bs=4)
    out = oracle.paged_attn(prob)
    for i in range(6):
        p2 = dict(prob, seqlens_k=np.array([29 - 6 + i + 1], dtype=np.int32),
                  cu_seqlens_q=np.array([0, 1], dtype=np.int32), q=prob["q"][i:i + 1])
        np.testing.assert_array_equal(oracle.paged_attn(p2)[0], out[i])


def test_zero_new_token_sequence_writes_nothing():
    rng = np.random.default_rng(70)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[10, 50, 12], q_lens=[2, 0, 3], H=2,
                            Hk=1, D=16, bs=8)
    out = oracle.paged_attn(prob)
    assert out.shape[0] == 5
    keep = [0, 2]
    p2 = dict(prob, batch=2, seqlens_k=prob["seqlens_k"][keep],
              block_table=prob["block_table"][keep],
              cu_seqlens_q=np.array([0, 2, 5], dtype=np.int32))
    np.testing.assert_array_equal(oracle.paged_attn(p2), out)


def test_contract_violations_rejected():
    rng = np.random.default_rng(80)
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=[4], q_lens=[2], H=2, Hk=1, D=8, bs=4)
    bad = dict(prob, cu_seqlens_q=np.array([0, 5], dtype=np.int32),
               q=np.zeros((5, 2, 8)))  # more new tokens than keys
    with pytest.raises(ValueError):
        oracle.paged_attn(bad)
    bt = prob["block_table"].copy()
    bt[0, 0] = prob["num_blocks"]  # physical block out of range
    with pytest.raises(ValueError):
        oracle.paged_attn(dict(prob, block_table=bt))


@pytest.mark.parametrize("kv", ALL_KV)
def test_fold_equals_explicit_dequant(kv):
    rng = np.random.default_rng(90 + kv)
    ks = rng.uniform(0.01, 0.1, size=(2, 32))
    ks.reshape(-1)[rng.choice(64, 3, replace=False)] *= 100.0
    prob, _ = paged_problem(rng, kv_dtype=kv, lens=[50, 17], q_lens=[1, 4], H=4, Hk=2, D=32,
                            bs=16, k_scale=ks)
    assert _rel(oracle.paged_attn(prob, folded=True), oracle.paged_attn(prob)) < 1e-13


def test_split_combine_equals_unsplit():
    """Flash-decoding partition + log-sum-exp merge reproduces the unsplit rows
    (the GQA GEMV decode page's flash-vs-naive parity, held here to 1e-12)."""
    rng = np.random.default_rng(100)
    lens, ql = [100, 37, 64], [1, 1, 3]
    prob, _ = paged_problem(rng, kv_dtype=KV_INT8, lens=lens, q_lens=ql, H=4, Hk=2, D=16, bs=16)
    ref = oracle.paged_attn(prob)
    cuts = [np.array([0, 10, 10, 55, 100]), np.array([0, 37, 37, 37, 37]),
            np.array([0, 1, 2, 40, 64])]  # includes empty splits
    os_, ls_ = [], []
    for s in range(4):
        kb = np.array([c[s] for c in cuts], dtype=np.int32)
        ke = np.array([c[s + 1] for c in cuts], dtype=np.int32)
        o, lse = oracle.paged_attn_partial(prob, kb, ke)
        os_.append(o.reshape(-1, 16))
        ls_.append(lse.reshape(-1))
    out = oracle.lse_combine(np.stack(os_), np.stack(ls_)).reshape(ref.shape)
    assert _rel(out, ref) < 1e-12


def test_gather_decode_matches_dense():
    rng = np.random.default_rng(110)
    prob, dense = paged_problem(rng, kv_dtype=KV_INT4, lens=[37, 64], q_lens=[1, 1], H=4, Hk=2,
                                D=16, bs=16)
    for b in range(2):
        for kv in range(2):
            np.testing.assert_array_equal(oracle.gather_decode(prob, prob["k_cache"], b, kv),
                                          dense["K"][b][:, kv, :])


def test_stored_tiny_int8_output_reproduces():
    """Regression guard: the stored FP64 output of the tiny INT8 workload
    (written by tests/golden/make_golden.py from the oracle) still matches."""
    import workloads
    w = workloads.make("c1_tiny_int8")
    out = oracle.paged_attn(workloads.oracle_view(w))
    ref = np.loadtxt(os.path.join(GOLDEN, "c1_tiny_int8_oracle.txt")).reshape(out.shape)
    np.testing.assert_allclose(out, ref, rtol=1e-15, atol=0)


# ---------------------------------------------------------------- cache writer


def test_quantise_exact_codes_at_power_of_two_scales():
    """x = code * s with s a power of two is exact in fp32: the code comes back,
    and decoding it times s gives x again (symmetric per-channel format)."""
    for kv, lo, hi in ((KV_INT8, -127, 127), (KV_INT4, -8, 7)):
        for s in (2.0 ** -7, 0.5, 1.0, 8.0):
            for c in range(lo, hi + 1):
                assert oracle.quantise(kv, c * s, s) == c


def test_quantise_ties_round_to_even_and_saturate():
    s = 0.25
    for kv in (KV_INT8, KV_INT4):
        # 0.5, 1.5, 2.5, -0.5, -1.5, -2.5 steps: halves go to the even neighbour
        assert [oracle.quantise(kv, (c + 0.5) * s, s) for c in (0, 1, 2, -1, -2, -3)] == \
            [0, 2, 2, 0, -2, -2]
        assert oracle.quantise(kv, 0.49 * s, s) == 0
        assert oracle.quantise(kv, 0.51 * s, s) == 1
    assert oracle.quantise(KV_INT8, 1e6, s) == 127 and oracle.quantise(KV_INT8, -1e6, s) == -127
    assert oracle.quantise(KV_INT4, 1e6, s) == 7 and oracle.quantise(KV_INT4, -1e6, s) == -8
    assert oracle.quantise(KV_INT8, float("inf"), s) == 127
    assert oracle.quantise(KV_INT8, float("nan"), s) == 0


@pytest.mark.parametrize("kv", [KV_INT8, KV_INT4, KV_FP8_E4M3])
def test_quantise_decides_from_the_correctly_rounded_quotient(kv):
    """Next to a rounding boundary the code is the one nearest to the exact
    quotient x / s (decided with rationals; every correctly rounded fp32
    quotient lies on the same side of the boundary), at inputs where x times a
    rounded 1 / s would give the neighbouring code."""
    from tests._quotient_points import boundary_points
    pts = boundary_points(kv, 48, seed=700 + kv)
    got = [oracle.quantise(kv, x, s) for x, s, _ in pts]
    want = [c for _, _, c in pts]
    assert got == want


def test_quantise_e4m3_round_trips_every_code():
    """encode(decode(c)) == c for every non-NaN code (the decode table is pinned
    by the printed code points and torch); 0x80 is the signed zero."""
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        v = oracle.decode_row(KV_FP8_E4M3, np.array([c], dtype=np.uint8), 1)[0]
        assert oracle.quantise(KV_FP8_E4M3, float(v), 1.0) == c, hex(c)
    assert oracle.quantise(KV_FP8_E4M3, float("nan"), 1.0) == 0x7F
    assert oracle.quantise(KV_FP8_E4M3, 1e9, 1.0) == 0x7E      # saturates at 448
    assert oracle.quantise(KV_FP8_E4M3, -1e9, 1.0) == 0xFE
    assert oracle.quantise(KV_FP8_E4M3, float("inf"), 1.0) == 0x7E
    assert oracle.quantise(KV_FP8_E4M3, float("-inf"), 1.0) == 0xFE
    assert oracle.quantise(KV_FP8_E4M3, 1.0625, 1.0) == 0x38    # tie 1 | 1.125 -> even
    assert oracle.quantise(KV_FP8_E4M3, 1.1875, 1.0) == 0x3A    # tie 1.125 | 1.25 -> even


def test_quantise_e4m3_matches_torch_cast_in_range():
    """Inside the finite range the writer's FP8 code is torch's round-to-nearest-
    even float32 -> float8_e4m3fn cast of the fp32 quotient."""
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(4000) * 40, rng.standard_normal(2000) * 0.01,
                        rng.uniform(-440, 440, 2000)]).astype(np.float32)
    s = np.float32(1.0)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.quantise(KV_FP8_E4M3, float(v), float(s)) for v in x], dtype=np.uint8)
    np.testing.assert_array_equal(got, want)


def _append_case(kv, rng, lens, q_lens, bs=16, Hk=2, D=16):
    prob, _ = paged_problem(rng, kv_dtype=kv, lens=lens, q_lens=q_lens, H=2 * Hk, Hk=Hk, D=D,
                            bs=bs)
    T = int(prob["cu_seqlens_q"][-1])
    k_new = rng.standard_normal((T, Hk, D)) * 3.0
    v_new = rng.standard_normal((T, Hk, D)) * 3.0
    if kv == KV_FP8_E4M3:
        k_new, v_new = k_new * 40.0, v_new * 40.0
    # the new rows arrive as fp16: their exact values
    k_new = k_new.astype(np.float16).astype(np.float64)
    v_new = v_new.astype(np.float16).astype(np.float64)
    prob["k_scale"] = rng.uniform(0.01, 0.1, size=(Hk, D)).astype(np.float32)
    prob["v_scale"] = rng.uniform(0.01, 0.1, size=(Hk, D)).astype(np.float32)
    return prob, k_new, v_new


@pytest.mark.parametrize("kv", ALL_KV)
def test_append_places_rows_at_their_slots_only(kv):
    """Placement: exactly the bytes of the new tokens' rows change; decoding them
    gives the codes of the new values; every other byte keeps its old value."""
    rng = np.random.default_rng(61 + kv)
    lens, ql = [5, 40, 17, 3], [2, 17, 0, 3]  # crosses block boundaries; one empty sequence
    prob, k_new, v_new = _append_case(kv, rng, lens, ql)
    kc, vc = oracle.append(prob, k_new, v_new)
    bs, Hk, D = prob["block_size"], prob["kv_num_heads"], prob["head_size"]
    changed_k = np.zeros(kc.shape[:3], dtype=bool)
    cu = prob["cu_seqlens_q"]
    for b in range(len(lens)):
        qb = int(cu[b + 1] - cu[b])
        for i in range(qb):
            t = lens[b] - qb + i
            phys, slot = prob["block_table"][b, t // bs], t % bs
            changed_k[phys, slot, :] = True
            for kvh in range(Hk):
                for new, cache, sc in ((k_new, kc, prob["k_scale"]), (v_new, vc, prob["v_scale"])):
                    got = oracle.decode_row(kv, cache[phys, slot, kvh], D)
                    for d in range(D):
                        code = oracle.quantise(kv, new[cu[b] + i, kvh, d], sc[kvh, d])
                        want = oracle.decode_row(kv, np.array([code & 0xFF], np.uint8), 1)[0] \
                            if kv == KV_FP8_E4M3 else code
                        if np.isnan(want):
                            assert np.isnan(got[d])
                        else:
                            assert got[d] == want
    np.testing.assert_array_equal(kc[~changed_k], prob["k_cache"][~changed_k])
    np.testing.assert_array_equal(vc[~changed_k], prob["v_cache"][~changed_k])


def test_append_dequant_error_is_half_a_step():
    """In range, |s * code - x| <= s / 2 for the integer caches (nearest code)."""
    rng = np.random.default_rng(67)
    for kv in (KV_INT8, KV_INT4):
        prob, k_new, v_new = _append_case(kv, rng, [30], [30])
        k_new = np.clip(k_new, -0.05, 0.05)  # inside the code range at these scales
        kc, _ = oracle.append(prob, k_new, v_new)
        bs, D = prob["block_size"], prob["head_size"]
        for t in range(30):
            phys, slot = prob["block_table"][0, t // bs], t % bs
            for kvh in range(prob["kv_num_heads"]):
                deq = oracle.decode_row(kv, kc[phys, slot, kvh], D) * prob["k_scale"][kvh]
                assert np.all(np.abs(deq - k_new[t, kvh]) <= prob["k_scale"][kvh] / 2 * (1 + 1e-6))


def test_append_rejects_bad_block_ids():
    rng = np.random.default_rng(71)
    prob, k_new, v_new = _append_case(KV_INT8, rng, [20], [4])
    prob["block_table"] = prob["block_table"].copy()
    prob["block_table"][0, 1] = prob["num_blocks"]  # the page of the new tokens
    with pytest.raises(ValueError):
        oracle.append(prob, k_new, v_new)
