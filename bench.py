#!/usr/bin/env python
"""Benchmark of paged quantised-KV attention on B200 (one JSON line on rank 0).

A step is one call of the whole hot path (the query-fragment pre-pass, the fused
attention kernel and, when the planner splits the KV, the log-sum-exp combine,
chained by programmatic dependent launch) over one batch of seeded synthetic input
whose cache is already resident in HBM.  Consecutive steps read different
copies ("replicas") of the whole input set, rotating through enough of them that
the bytes read between two uses of one copy exceed three times the 126 MB L2, so
every step reads its KV cache from HBM; a workload too small for that (the tiny
case) instead flushes L2 by writing a 256 MB buffer before each step, outside the
timed span.  Each step is timed with CUDA events on the launching stream.

Headline workload (N=1): the largest configuration, FP8 e4m3 large-batch decode,
B=128, q_len=1, 64 query / 8 KV heads, head_size 128, block_size 16, seqlens_k =
8192 (2.15 GB of KV per call).  The other workloads (INT4 decode, INT8 long-context
split decode, INT8 ragged causal prefill, the tiny INT8 case, the cache writer)
are reported under "workloads" with the same method, each with its own roofline
block.  A read-only 16-byte-vector stream over a 2 GiB buffer
(paged_attn_stream_read) is timed beside them as the measured read ceiling.

Metric: effective HBM bandwidth = algorithmic bytes per call / time per call
(KV bytes of the sequences with new tokens + Q in + out + scales + block-table
entries read + lengths), plus us/call and tokens/s.

--impl reference times the FP64 CPU oracle (single thread) on a bounded sample
of the same workload, which is the comparison arm of this build.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

HEADLINE = "c5_fp8_large_batch"
EXTRA = ["c2_int4_decode", "c3_int8_long_split", "c4_ragged_prefill_int8", "c1_tiny_int8"]
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20
MAX_REPLICAS = 16
SPIN_CYCLES = 1000000  # ~0.5 ms of GPU work queued ahead of every timed span


def algorithmic_bytes(w: dict) -> dict:
    """Bytes the method must move per call (the measurement section's formula)."""
    D, H, Hk, bs = w["head_size"], w["num_heads"], w["kv_num_heads"], w["block_size"]
    chs = workloads.cache_bytes_per_row(w["kv_dtype"], D)
    ql = np.diff(w["cu_seqlens_q"]).astype(np.int64)
    L = w["seqlens_k"].astype(np.int64)
    act = ql > 0
    kv = int((L[act] * Hk * 2 * chs).sum())
    T = int(w["cu_seqlens_q"][-1])
    qo = T * H * D * (2 + 2)
    scales = 2 * Hk * D * 4
    bt = int(((L[act] + bs - 1) // bs).sum()) * 4
    meta = 4 * w["batch"] + 4 * (w["batch"] + 1)
    total = kv + qo + scales + bt + meta
    return dict(total=total, kv=kv, qo=qo, tokens=T, fwd=total)


# Source files of the dominant kernel of each workload (the decode kernel, or
# the tensor-core prefill kernel for the ragged prefill workload).
KERNEL_SOURCES = {"decode": ("pa_attention.cu", "pa_device.cuh"),
                  "prefill": ("pa_prefill.cu", "pa_tc.cuh", "pa_device.cuh")}


def kernel_of(name: str) -> str:
    return "prefill" if name == "c4_ragged_prefill_int8" else "decode"


def kernel_source_sha(kind: str = "decode") -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "paged_quantized_kv_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(name: str):
    """DRAM bytes (read + write) per launch of the workload's dominant kernel from
    the committed ncu summary profiles/ncu_traffic.txt, if it was taken on the
    current kernel source (else None).  Line format: workload kernel_source_sha
    bytes_per_launch."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    try:
        with open(path) as f:
            for ln in f:
                parts = ln.split()
                if len(parts) >= 3 and not ln.startswith("#") and parts[0] == name:
                    if parts[1] == kernel_source_sha(kernel_of(name)):
                        return int(parts[2])
    except (OSError, ValueError):
        return None
    return None


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor peak (TFLOP/s, burst) of MEASURED_PEAKS.json, else the
    fallback figure."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, ValueError, KeyError):
        return 1590.0, "fallback"


def algorithmic_flops(w: dict) -> int:
    """Useful tensor work per call: 2 D flops for QK and 2 D for PV per visible
    key of every row (rows = new tokens x query heads; causal rows see their
    past plus the new tokens up to themselves)."""
    D, H = w["head_size"], w["num_heads"]
    cu = w["cu_seqlens_q"].astype(np.int64)
    L = w["seqlens_k"].astype(np.int64)
    keys = 0
    for b in range(w["batch"]):
        qb = int(cu[b + 1] - cu[b])
        if qb == 0:
            continue
        past = int(L[b]) - qb
        if w["causal"]:
            keys += qb * past + qb * (qb + 1) // 2
        else:
            keys += qb * int(L[b])
    return 4 * D * H * keys


def roofline_block(w: dict, ab: dict, kern_ms: float, name: str) -> dict:
    """Roofline of the call's kernels for one workload: bound = the larger of the
    HBM time (algorithmic bytes / measured copy peak) and the tensor time
    (algorithmic flops / measured bf16 peak); achieved in that bound's unit."""
    peak, kind = measured_peaks()
    tpk, tkind = measured_tensor_peak()
    flops = algorithmic_flops(w)
    t_hbm = ab["total"] / (peak * 1e9)
    t_mma = flops / (tpk * 1e12)
    sec = kern_ms * 1e-3
    kname = "pa_prefill_kernel" if kernel_of(name) == "prefill" else "pa_fwd_kernel"
    if t_mma > t_hbm:
        return {"bound": "tensor", "kernel": kname, "achieved": round(flops / sec / 1e12, 2), "peak": tpk,
                "unit": "TFLOP/s", "frac": round(t_mma / sec, 4), "peak_kind": tkind,
                "algorithmic_flops_per_launch": flops, "traffic": ncu_traffic(name)}
    return {"bound": "hbm", "kernel": kname, "achieved": round(ab["total"] / sec / 1e9, 1), "peak": peak,
            "unit": "GB/s", "frac": round(t_hbm / sec, 4), "peak_kind": kind,
            "algorithmic_bytes_per_launch": ab["total"], "algorithmic_flops_per_launch": flops,
            "frac_of_tensor_peak": round(t_mma / sec, 4), "traffic": ncu_traffic(name)}


READ_CEILING_BYTES = 2 << 30


def read_ceiling(dev: str, steps: int = 10) -> dict:
    """Measured read-only ceiling: paged_attn_stream_read (16-byte loads on every
    SM) over a 2 GiB buffer, CUDA events on the launching stream, best and mean
    of `steps` launches after 3 warm-up launches."""
    import paged_quantized_kv_attention_b200 as pa
    buf = torch.empty(READ_CEILING_BYTES, dtype=torch.uint8, device=dev)
    buf.fill_(1)
    sink = torch.empty(16 * 148 * 64, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(3):
        pa.paged_attn_stream_read(buf, READ_CEILING_BYTES, sink, stream)
    ms = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pa.paged_attn_stream_read(buf, READ_CEILING_BYTES, sink, stream)
        e1.record(stream)
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    del buf
    torch.cuda.empty_cache()
    peak, kind = measured_peaks()
    best = READ_CEILING_BYTES / (min(ms) * 1e-3) / 1e9
    mean = READ_CEILING_BYTES / (statistics.mean(ms) * 1e-3) / 1e9
    return {"kernel": "pa_stream_read_kernel (paged_attn_stream_read)", "bytes": READ_CEILING_BYTES,
            "gbs_best": round(best, 1), "gbs_mean": round(mean, 1),
            "vs_%s_copy_peak" % kind: round(mean / peak, 4)}


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.ok = [], 0, False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report nulls
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.reasons |= int(r) & ~0x1
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def setup(w: dict, dev: str, replicas: int = 1):
    """Device copies of the workload: a list of `replicas` independent input sets
    (each with its own output), one plan and one workspace shared by all."""
    import paged_quantized_kv_attention_b200 as pa
    from_np = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    odt = torch.bfloat16 if w["out_dtype"] == 1 else torch.float16
    T = int(w["cu_seqlens_q"][-1])
    reps = []
    for _ in range(replicas):
        d = dict(q=w["q"].to(dev), k_cache=from_np(w["k_cache"]), v_cache=from_np(w["v_cache"]),
                 k_scale=from_np(w["k_scale"].astype(np.float32)),
                 v_scale=from_np(w["v_scale"].astype(np.float32)),
                 block_table=from_np(w["block_table"]), seqlens_k=from_np(w["seqlens_k"]),
                 cu_seqlens_q=from_np(w["cu_seqlens_q"]))
        d["out"] = torch.empty((T, w["num_heads"], w["head_size"]), dtype=odt, device=dev)
        reps.append(d)
    p = pa.make_params(batch=w["batch"], num_heads=w["num_heads"], kv_num_heads=w["kv_num_heads"],
                       head_size=w["head_size"], block_size=w["block_size"],
                       num_blocks=w["num_blocks"], max_blocks_per_seq=w["max_blocks_per_seq"],
                       kv_dtype=w["kv_dtype"], q_dtype=w["q_dtype"], out_dtype=w["out_dtype"],
                       causal=w["causal"])
    ws_bytes = pa.paged_attn_plan(w["cu_seqlens_q"], w["seqlens_k"], p)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    pa.paged_attn_workspace_init(ws, ws_bytes)
    p.workspace = ws.data_ptr()
    for d in reps:
        d["ws"] = ws
    return reps, p


def l2_plan(w: dict):
    """(replicas, flush): rotate replicas so that > 3 x L2 bytes are read between
    two uses of one copy; fall back to flushing when that needs too many copies."""
    foot = algorithmic_bytes(w)["total"]
    need = -(-3 * L2_BYTES // max(foot, 1))
    if need <= MAX_REPLICAS:
        return max(1, int(need)), False
    return 1, True


def l2_desc(replicas: int, flush: bool, w: dict) -> str:
    if flush:
        return "flushed before every step (256 MB write, outside the timed span)"
    foot = algorithmic_bytes(w)["total"] / 1e6
    return ("inputs larger than L2: %d rotating replica(s) of the whole input set, %.0f MB read "
            "per step, %.0f MB between two uses of one copy" % (replicas, foot, foot * replicas))


def _event_handles(evs):
    import ctypes
    arr = (ctypes.c_void_p * 2)(evs[0].cuda_event, evs[1].cuda_event)
    return arr


def _args(d):
    return (d["q"], d["k_cache"], d["v_cache"], d["k_scale"], d["v_scale"], d["block_table"],
            d["seqlens_k"], d["cu_seqlens_q"], d["out"])


def time_device(w, reps, p, steps, warmup, flush):
    """Per-step device time of the whole call and of the fused kernel (ms lists).
    `flush` is the L2 flush buffer, or None when replicas rotate."""
    import ctypes

    import paged_quantized_kv_attention_b200 as pa
    stream = torch.cuda.current_stream()
    R = len(reps)
    for i in range(max(warmup, R)):
        if flush is not None:
            flush.zero_()
        pa.paged_attn_forward(*_args(reps[i % R]), p, stream)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for e in ev:  # create the events before handing their handles to the library
        for x in e:
            x.record(stream)
    torch.cuda.synchronize()
    holders = []
    for i in range(steps):
        if flush is not None:
            flush.zero_()  # L2 flush, between the timed spans
        torch.cuda._sleep(SPIN_CYCLES)  # keep the GPU busy while the host enqueues the span
        h = _event_handles(ev[i][:2])
        holders.append(h)
        p.profile_events = ctypes.cast(h, ctypes.c_void_p)
        pa.paged_attn_forward(*_args(reps[i % R]), p, stream)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    p.profile_events = None
    call_ms = [ev[i][0].elapsed_time(ev[i][2]) for i in range(steps)]
    kern_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(steps)]
    return call_ms, kern_ms


def time_e2e(w, reps, p, steps, warmup, flush):
    """Through the public API with host buffers: H2D of the step's inputs from pinned
    memory, host planning, forward, D2H of the output; device-timed per step.  The
    step's inputs (Q, block table, lengths) travel in one copy: they are packed into
    one pinned host buffer and land in one device buffer whose views the call uses."""
    import paged_quantized_kv_attention_b200 as pa
    stream = torch.cuda.current_stream()
    d0 = reps[0]
    names = ("q", "block_table", "seqlens_k", "cu_seqlens_q")
    offs, off = {}, 0
    for k in names:  # 256-byte aligned sections
        offs[k] = off
        off += (d0[k].numel() * d0[k].element_size() + 255) // 256 * 256
    packed_h = torch.empty(off, dtype=torch.uint8).pin_memory()
    for k in names:
        src = d0[k].cpu().contiguous().view(torch.uint8).reshape(-1)
        packed_h[offs[k]:offs[k] + src.numel()].copy_(src)
    views = []
    for d in reps:  # one packed device buffer per replica, read by the call through views
        buf = torch.empty(off, dtype=torch.uint8, device=d0["q"].device)
        v = dict(d)
        v["_packed"] = buf
        for k in names:
            n = d0[k].numel() * d0[k].element_size()
            v[k] = buf[offs[k]:offs[k] + n].view(d0[k].dtype).view(d0[k].shape)
        views.append(v)
    cu_h, sk_h = w["cu_seqlens_q"].copy(), w["seqlens_k"].copy()
    out_h = torch.empty(d0["out"].shape, dtype=d0["out"].dtype).pin_memory()
    h2d = sum(d0[k].numel() * d0[k].element_size() for k in names)
    d2h = out_h.numel() * out_h.element_size()
    R = len(reps)

    def one(d):
        d["_packed"].copy_(packed_h, non_blocking=True)
        pa.paged_attn_plan(cu_h, sk_h, p)
        pa.paged_attn_forward(*_args(d), p, stream)
        out_h.copy_(d["out"], non_blocking=True)

    for i in range(max(warmup, R)):
        if flush is not None:
            flush.zero_()
        one(views[i % R])
    torch.cuda.synchronize()
    ms = []
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        torch.cuda._sleep(SPIN_CYCLES)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        one(views[i % R])
        e1.record(stream)
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    return ms, h2d, d2h


def cpu_oracle_sample(w: dict, budget_s: float):
    """The FP64 oracle as it stands, single-threaded, over whole sequences of the
    workload until about budget_s seconds of CPU work; returns (GB/s, detail)."""
    import oracle
    ov = workloads.oracle_view(w)
    cu = w["cu_seqlens_q"]
    done_bytes, t_used, seqs, keys = 0, 0.0, 0, 0
    for b in range(w["batch"]):
        if cu[b + 1] == cu[b]:
            continue
        s = sub_problem(ov, b)
        t0 = time.perf_counter()
        oracle.paged_attn(s)
        t_used += time.perf_counter() - t0
        done_bytes += algorithmic_bytes(s)["total"]
        seqs += 1
        keys += int(s["seqlens_k"][0])
        if t_used >= budget_s:
            break
    gbs = done_bytes / t_used / 1e9 if t_used > 0 else None
    return gbs, dict(seconds=round(t_used, 3), sequences=seqs, keys=keys, bytes=done_bytes)


def sub_problem(w: dict, b: int) -> dict:
    cu = w["cu_seqlens_q"]
    s = dict(w)
    s["batch"] = 1
    s["block_table"] = np.ascontiguousarray(w["block_table"][b:b + 1])
    s["seqlens_k"] = np.ascontiguousarray(w["seqlens_k"][b:b + 1])
    s["cu_seqlens_q"] = np.array([0, cu[b + 1] - cu[b]], dtype=np.int32)
    s["q"] = w["q"][int(cu[b]):int(cu[b + 1])]
    return s


def first_sequences(w: dict, B: int) -> dict:
    """The workload cut to its first B sequences (same cache pools, heads and
    dtypes): a smaller instance of the same shape, for profiler captures."""
    if B is None or B >= w["batch"]:
        return w
    s = dict(w)
    cu = w["cu_seqlens_q"]
    s["batch"] = B
    s["block_table"] = np.ascontiguousarray(w["block_table"][:B])
    s["seqlens_k"] = np.ascontiguousarray(w["seqlens_k"][:B])
    s["cu_seqlens_q"] = np.ascontiguousarray(cu[:B + 1])
    s["q"] = w["q"][:int(cu[B])]
    return s


def measure(name: str, steps: int, warmup: int, dev: str, flush_buf, with_e2e: bool,
            batch=None):
    w = first_sequences(workloads.make(name), batch)
    ab = algorithmic_bytes(w)
    replicas, use_flush = l2_plan(w)
    flush = flush_buf if use_flush else None
    reps, p = setup(w, dev, replicas)
    call_ms, kern_ms = time_device(w, reps, p, steps, warmup, flush)
    call = statistics.mean(call_ms)
    kern = statistics.mean(kern_ms)
    peak, peak_kind = measured_peaks()
    res = dict(w=w, ab=ab, p=p, call_ms=call, kern_ms=kern,
               value=ab["total"] / (call * 1e-3) / 1e9,
               kernel_gbs=ab["fwd"] / (kern * 1e-3) / 1e9, peak=peak, peak_kind=peak_kind,
               launches_per_step=2 + (1 if p.num_splits > 1 else 0), l2=l2_desc(replicas, use_flush, w))
    if with_e2e:
        e2e_ms, h2d, d2h = time_e2e(w, reps, p, max(5, steps // 2), 2, flush)
        res["e2e"] = dict(value=ab["total"] / (statistics.mean(e2e_ms) * 1e-3) / 1e9,
                          unit="GB/s", h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h,
                          ms_per_step=statistics.mean(e2e_ms))
    del reps
    torch.cuda.empty_cache()
    return res


# Quantise-and-append (the cache writer that precedes the attention call):
# (name, description, new tokens, sequences, Hk, D, block_size, kv dtype, bf16 input)
APPEND = [("append_prefill_32k_int8", "append of a 32768-token prompt: Hk=8 D=128 bs=16 INT8, "
           "bf16 K/V in", 32768, 1, 8, 128, 16, workloads.KV_INT8, True),
          ("append_decode_int4", "decode-step append: 16 sequences x 1 token, Hk=8 D=128 bs=16 "
           "INT4, fp16 K/V in", 16, 16, 8, 128, 16, workloads.KV_INT4, False)]


def measure_append(spec, steps: int, warmup: int, dev: str, flush_buf):
    """Device time of paged_kv_append (CUDA events on the launching stream)."""
    import paged_quantized_kv_attention_b200 as pa
    name, desc, T, B, Hk, D, bs, kv, bf16 = spec
    rng = np.random.default_rng(2024)
    per = T // B
    cu = np.arange(0, T + 1, per, dtype=np.int32)
    sk = np.full(B, 4096 if B > 1 else T, dtype=np.int32)  # decode: 4095 past keys each
    nblk = int(-(-sk.max() // bs))
    pool = B * nblk * 2
    bt = rng.permutation(pool)[:B * nblk].astype(np.int32).reshape(B, nblk)
    chs = D // 2 if kv == workloads.KV_INT4 else D
    dt = torch.bfloat16 if bf16 else torch.float16
    kc = torch.zeros((pool, bs, Hk, chs), dtype=torch.uint8, device=dev)
    vc = torch.zeros_like(kc)
    kn = (torch.randn((T, Hk, D), device=dev) * 3).to(dt)
    vn = (torch.randn((T, Hk, D), device=dev) * 3).to(dt)
    ks = torch.from_numpy(rng.uniform(0.01, 0.1, (Hk, D)).astype(np.float32)).to(dev)
    vs = torch.from_numpy(rng.uniform(0.01, 0.1, (Hk, D)).astype(np.float32)).to(dev)
    p = pa.make_params(batch=B, num_heads=Hk, kv_num_heads=Hk, head_size=D, block_size=bs,
                       num_blocks=pool, max_blocks_per_seq=nblk, kv_dtype=kv,
                       q_dtype=1 if bf16 else 0, out_dtype=1 if bf16 else 0)
    nb = pa.paged_attn_plan(cu, sk, p)
    ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device=dev)
    p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    args = (kn, vn, kc, vc, ks, vs, torch.from_numpy(bt).to(dev), torch.from_numpy(sk).to(dev),
            torch.from_numpy(cu).to(dev))
    big = 2 * T * Hk * D * 2 > L2_BYTES  # the new rows alone stream through L2 every step
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        pa.paged_kv_append(*args, p, stream)
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        if not big:
            flush_buf.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pa.paged_kv_append(*args, p, stream)
        e1.record(stream)
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    st, bits = pa.paged_attn_read_device_error(ws)
    k_ms = statistics.median(ms)
    nbytes = (2 * T * Hk * D * 2 + 2 * T * Hk * chs + 2 * Hk * D * 4 + T * 4 + 2 * (B + 1) * 4)
    peak, kind = measured_peaks()
    gbs = nbytes / (k_ms * 1e-3) / 1e9
    return {"desc": desc, "us_per_call": round(k_ms * 1e3, 3), "gbs": round(gbs, 1),
            "frac_of_measured_peak" if kind == "measured" else "frac_of_fallback_peak":
                round(gbs / peak, 4),
            "algorithmic_bytes": nbytes, "device_error_bits": bits,
            "l2": "inputs larger than L2" if big else "flushed before every call (256 MB write)",
            "kernel": "pa_append_kernel"}


def summary_of(name, r):
    return {"workload": name, "desc": workloads.DESCRIPTIONS[name],
            "gbs": round(r["value"], 1), "us_per_call": round(r["call_ms"] * 1e3, 2),
            "tokens_per_s": round(r["ab"]["tokens"] / (r["call_ms"] * 1e-3), 1),
            "kernel_us": round(r["kern_ms"] * 1e3, 2),
            "kernel_gbs": round(r["kernel_gbs"], 1),
            "kernel_frac_of_%s_peak" % r["peak_kind"]: round(r["kernel_gbs"] / r["peak"], 3),
            "num_splits": r["p"].num_splits, "algorithmic_bytes": r["ab"]["total"], "l2": r["l2"],
            "launches_per_call": r["launches_per_step"],
            "roofline": roofline_block(r["w"], r["ab"], r["kern_ms"], name)}


def run_ours(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = "cuda:%d" % torch.cuda.current_device()
    import paged_quantized_kv_attention_b200 as pa
    pa.lib()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    # headline workload: identical per-rank replica (weak scaling, no collective on the path)
    w_name = args.workload
    sampler = ClockSampler(torch.cuda.current_device())
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        r = measure(w_name, args.steps, args.warmup, dev, flush, with_e2e=True, batch=args.batch)
    torch.cuda.synchronize()
    if dist is not None:
        t = torch.tensor([r["call_ms"], r["e2e"]["ms_per_step"]], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.barrier()
        r["call_ms"], r["e2e"]["ms_per_step"] = float(t[0]), float(t[1])
    extra = {}
    ceiling = None
    if not args.no_extra:
        ceiling = read_ceiling(dev)
        for name in EXTRA:
            if name == w_name:
                continue
            rr = measure(name, max(3, min(args.steps, 20)), args.warmup, dev, flush,
                         with_e2e=False)
            extra[name] = summary_of(name, rr)
        for spec in APPEND:
            extra[spec[0]] = measure_append(spec, max(5, min(args.steps, 20)), 3, dev, flush)
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return
    ab = r["ab"]
    value = world * ab["total"] / (r["call_ms"] * 1e-3) / 1e9
    e2e_value = world * ab["total"] / (r["e2e"]["ms_per_step"] * 1e-3) / 1e9
    cpu = None
    if world == 1 and not args.no_cpu:
        gbs, det = cpu_oracle_sample(r["w"], args.cpu_seconds)
        cpu = {"value": gbs, "unit": "GB/s", "cores": 1, "host_cores": os.cpu_count(),
               "kind": "oracle",
               "sample": "FP64 oracle, one thread (of %d host cores), whole sequences of the "
                         "same workload in order until ~%.0f s: %d sequences, %d keys, %.1f s" %
                         (os.cpu_count(), args.cpu_seconds, det["sequences"], det["keys"],
                          det["seconds"])}
    line = {
        "metric": "paged quantized-KV attention: effective HBM GB/s (% of ~8 TB/s), us/call",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(r["call_ms"], 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded numpy PCG64; cache resident in HBM)",
        "config": {"workload": w_name if args.batch is None else
                   "%s (first %d sequences)" % (w_name, r["w"]["batch"]),
                   "desc": workloads.DESCRIPTIONS[w_name],
                   "kv_dtype": workloads.KV_NAMES[r["w"]["kv_dtype"]],
                   "global_batch": r["w"]["batch"] * world, "seq_len": int(r["w"]["seqlens_k"].max()),
                   "parallelism": "replicas x%d" % world,
                   "l2": r["l2"], "timing": "per-step CUDA events on the launching stream",
                   "num_splits": r["p"].num_splits, "blocks_per_split": r["p"].blocks_per_split},
        "us_per_call": round(r["call_ms"] * 1e3, 3),
        "tokens_per_s": round(world * ab["tokens"] / (r["call_ms"] * 1e-3), 1),
        "pct_of_8tbs": round(100 * value / world / 8000.0, 2),
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": r["e2e"]["h2d_bytes_per_step"],
                "d2h_bytes_per_step": r["e2e"]["d2h_bytes_per_step"],
                "us_per_step": round(r["e2e"]["ms_per_step"] * 1e3, 2)},
        "gpu_launches": args.steps * r["launches_per_step"],
        "roofline": dict(roofline_block(r["w"], ab, r["kern_ms"], w_name),
                         timed="the dominant kernel with the other kernels of the call, "
                               "which overlap it: the whole call on the device",
                         kernel_us=round(r["kern_ms"] * 1e3, 3),
                         read_ceiling_gbs=ceiling["gbs_mean"] if ceiling else None),
        "read_ceiling": ceiling,
        "clocks": sampler.summary(),
        "cpu_baseline": cpu,
        "workloads": extra,
    }
    print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()


def run_reference(args):
    """The comparison arm: the FP64 oracle on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = workloads.make(args.workload)
    ov = workloads.oracle_view(w)
    cu = w["cu_seqlens_q"]
    seqs = [b for b in range(w["batch"]) if cu[b + 1] > cu[b]]
    for i in range(args.warmup):
        oracle.paged_attn(sub_problem(ov, seqs[i % len(seqs)]))
    t_total, bytes_total, keys = 0.0, 0, 0
    for i in range(args.steps):
        s = sub_problem(ov, seqs[i % len(seqs)])
        t0 = time.perf_counter()
        oracle.paged_attn(s)
        t_total += time.perf_counter() - t0
        bytes_total += algorithmic_bytes(s)["total"]
        keys += int(s["seqlens_k"][0])
    value = bytes_total / t_total / 1e9
    world = int(os.environ.get("WORLD_SIZE", "1"))
    sample = ("FP64 oracle, one thread, one whole sequence of %s per step (%d steps, %d keys)"
              % (args.workload, args.steps, keys))
    line = {"impl": "reference",
            "metric": "paged quantized-KV attention: effective HBM GB/s (% of ~8 TB/s), us/call",
            "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * t_total / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy PCG64)",
            "config": {"workload": args.workload, "desc": workloads.DESCRIPTIONS[args.workload]},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=workloads.NAMES)
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--batch", type=int, default=None,
                    help="cut the workload to its first BATCH sequences (a smaller instance "
                         "of the same shape, for profiler captures; not a bench line)")
    ap.add_argument("--writer", action="store_true",
                    help="time only the quantise-and-append writer workloads (one JSON line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.writer:
        torch.cuda.set_device(0)
        flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda:0")
        print(json.dumps({"writer": {spec[0]: measure_append(spec, args.steps, args.warmup,
                                                             "cuda:0", flush)
                                     for spec in APPEND}}))
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
