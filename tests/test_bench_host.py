"""Host-side checks of the bench's measurement arithmetic (no GPU): the
algorithmic bytes and flops behind every roofline fraction, the L2 rule of the
timing (inputs read from HBM each step), the roofline's choice of bound, the
kernel-source gate on the committed ncu traffic, and the warm-up contract.
"""
import numpy as np
import pytest

import bench
import workloads
from workloads import KV_FP8_E4M3, KV_INT4, KV_INT8


def _shape(kv, B, H, Hk, D, bs, L, ql, causal=1):
    """The fields the measurement formulas read (no cache arrays)."""
    L = np.asarray(L, dtype=np.int64)
    ql = np.asarray(ql, dtype=np.int64)
    return dict(kv_dtype=kv, batch=B, num_heads=H, kv_num_heads=Hk, head_size=D, block_size=bs,
                seqlens_k=L, cu_seqlens_q=np.concatenate([[0], np.cumsum(ql)]).astype(np.int32),
                causal=causal)


def test_fp8_large_batch_moves_its_whole_cache_once():
    """128 sequences of 8192 keys, 8 KV heads, 128 one-byte channels, K and V:
    2 x 128 x 8192 x 8 x 128 bytes of cache (the 2.15 GB the workload is named
    for) plus queries, outputs, scales, block table and lengths."""
    B, H, Hk, D, bs = 128, 64, 8, 128, 16
    w = _shape(KV_FP8_E4M3, B, H, Hk, D, bs, [8192] * B, [1] * B)
    ab = bench.algorithmic_bytes(w)
    kv = 2 * B * 8192 * Hk * D
    assert ab["kv"] == kv == 2147483648
    extra = B * H * D * 2 * 2 + 2 * Hk * D * 4 + B * (8192 // bs) * 4 + 4 * B + 4 * (B + 1)
    assert ab["total"] == kv + extra


def test_int4_rows_are_half_the_bytes_and_silent_sequences_move_nothing():
    """INT4 packs two codes per byte; a sequence with no new token reads no key."""
    w8 = _shape(KV_INT8, 3, 8, 2, 128, 16, [100, 60, 33], [1, 0, 2])
    w4 = _shape(KV_INT4, 3, 8, 2, 128, 16, [100, 60, 33], [1, 0, 2])
    assert bench.algorithmic_bytes(w8)["kv"] == (100 + 33) * 2 * 2 * 128
    assert bench.algorithmic_bytes(w4)["kv"] == (100 + 33) * 2 * 2 * 64


@pytest.mark.parametrize("causal", [1, 0])
def test_flops_count_every_visible_key_of_every_row(causal):
    """4 D flops (QK and PV) per visible (row, key) pair, counted here by brute
    force over the mask: a causal new token i of a sequence with `past` earlier
    keys sees past + i + 1 keys; a non-causal one sees them all."""
    rng = np.random.default_rng(7)
    B, H, Hk, D = 6, 16, 4, 128
    ql = rng.integers(0, 6, size=B)
    L = ql + rng.integers(0, 40, size=B)
    w = _shape(KV_INT8, B, H, Hk, D, 16, L, ql, causal=causal)
    pairs = 0
    for b in range(B):
        past = int(L[b] - ql[b])
        for i in range(int(ql[b])):
            for k in range(int(L[b])):
                if not causal or k <= past + i:
                    pairs += H
    assert bench.algorithmic_flops(w) == 4 * D * pairs


@pytest.mark.parametrize("name", workloads.NAMES)
def test_timed_steps_read_their_inputs_from_hbm(name):
    """Between two uses of one input copy more than 3 x L2 bytes are read, or the
    L2 is flushed before every step."""
    w = workloads.shrink(name, 1, max_len=64, batch=2)
    # the L2 rule is applied to the full workload's footprint
    full = {"c1_tiny_int8": (KV_INT8, 2, 4, 1, 64, 16, [37, 64], [1, 1]),
            "c2_int4_decode": (KV_INT4, 16, 32, 8, 128, 16, [2300] * 16, [1] * 16),
            "c3_int8_long_split": (KV_INT8, 4, 64, 8, 128, 32, [32768] * 4, [1] * 4),
            "c4_ragged_prefill_int8": (KV_INT8, 64, 32, 8, 128, 16, [1030] * 64, [8] * 64),
            "c5_fp8_large_batch": (KV_FP8_E4M3, 128, 64, 8, 128, 16, [8192] * 128, [1] * 128)}[name]
    assert w["kv_dtype"] == full[0]
    shape = _shape(*full)
    replicas, flush = bench.l2_plan(shape)
    foot = bench.algorithmic_bytes(shape)["total"]
    assert flush or replicas * foot > 3 * bench.L2_BYTES
    assert flush or replicas <= bench.MAX_REPLICAS


def test_roofline_takes_the_slower_of_hbm_and_tensor_time():
    """A decode shape is HBM-bound: frac = (bytes / copy peak) / measured time.
    The same rows against a tiny cache with many new tokens turn tensor-bound."""
    peak, _ = bench.measured_peaks()
    tpk, _ = bench.measured_tensor_peak()
    w = _shape(KV_INT8, 4, 64, 8, 128, 32, [32768] * 4, [1] * 4, causal=1)
    ab = bench.algorithmic_bytes(w)
    blk = bench.roofline_block(w, ab, 0.1, "c3_int8_long_split")
    assert blk["bound"] == "hbm" and blk["unit"] == "GB/s"
    assert blk["frac"] == pytest.approx(ab["total"] / (peak * 1e9) / 1e-4, rel=1e-3)
    assert blk["achieved"] == pytest.approx(ab["total"] / 1e-4 / 1e9, rel=1e-3)
    dense = _shape(KV_INT8, 1, 256, 1, 128, 16, [65536], [4096], causal=0)
    abd = bench.algorithmic_bytes(dense)
    blk = bench.roofline_block(dense, abd, 1.0, "c4_ragged_prefill_int8")
    assert blk["bound"] == "tensor" and blk["unit"] == "TFLOP/s"
    assert blk["frac"] == pytest.approx(bench.algorithmic_flops(dense) / (tpk * 1e12) / 1e-3, rel=1e-3)


def test_committed_traffic_is_used_only_for_the_kernel_source_it_was_taken_on(tmp_path, monkeypatch):
    """profiles/ncu_traffic.txt lines carry the kernel source hash; a line whose
    hash differs from the current source gives no traffic figure."""
    (tmp_path / "profiles").mkdir()
    sha = bench.kernel_source_sha("decode")
    (tmp_path / "profiles" / "ncu_traffic.txt").write_text(
        "# header\nc2_int4_decode %s 123\nc3_int8_long_split 0000000000000000 456\n" % sha)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # kernel_source_sha reads the sources under ROOT: point it back at the repo
    monkeypatch.setattr(bench, "kernel_source_sha", lambda kind="decode": sha if kind == "decode" else "x")
    assert bench.ncu_traffic("c2_int4_decode") == 123
    assert bench.ncu_traffic("c3_int8_long_split") is None
    assert bench.ncu_traffic("c4_ragged_prefill_int8") is None


def test_fewer_than_three_warmup_steps_are_refused(monkeypatch):
    monkeypatch.setattr("sys.argv", ["bench.py", "--warmup", "2"])
    with pytest.raises(SystemExit) as ei:
        bench.main()
    assert ei.value.code == 2
