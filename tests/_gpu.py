"""GPU-side helpers for the parity tests: upload a workload, run the C-ABI path."""
from __future__ import annotations

import numpy as np
import torch

import paged_quantized_kv_attention_b200 as pa
import oracle

TOL = {0: 2e-3, 1: 8e-3, 2: 2e-3}  # fp16 / bf16 / fp32 output: max|out - ref| <= TOL * max|dequant(V)|


def to_device(w: dict) -> dict:
    dev = "cuda"
    return dict(q=w["q"].to(dev), k_cache=torch.from_numpy(w["k_cache"]).to(dev),
                v_cache=torch.from_numpy(w["v_cache"]).to(dev),
                k_scale=torch.from_numpy(np.ascontiguousarray(w["k_scale"], np.float32)).to(dev),
                v_scale=torch.from_numpy(np.ascontiguousarray(w["v_scale"], np.float32)).to(dev),
                block_table=torch.from_numpy(w["block_table"]).to(dev),
                seqlens_k=torch.from_numpy(w["seqlens_k"]).to(dev),
                cu_seqlens_q=torch.from_numpy(w["cu_seqlens_q"]).to(dev))


def plan(w: dict, **over):
    p = pa.make_params(batch=w["batch"], num_heads=w["num_heads"], kv_num_heads=w["kv_num_heads"],
                       head_size=w["head_size"], block_size=w["block_size"],
                       num_blocks=w["num_blocks"], max_blocks_per_seq=w["max_blocks_per_seq"],
                       kv_dtype=w["kv_dtype"], q_dtype=w["q_dtype"], out_dtype=w["out_dtype"],
                       softmax_scale=w.get("softmax_scale", 0.0), causal=w.get("causal", 1),
                       **over)
    ws = pa.paged_attn_plan(w["cu_seqlens_q"], w["seqlens_k"], p)
    return p, ws


def run(w: dict, d: dict | None = None, extra_rows: int = 0, sentinel=None, **over):
    """Run the forward path; returns (out [T_q(+extra), H, D] on device, params, workspace)."""
    d = d if d is not None else to_device(w)
    p, ws_bytes = plan(w, **over)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    pa.paged_attn_workspace_init(ws, ws.numel())
    p.workspace = ws.data_ptr()
    T = int(w["cu_seqlens_q"][-1])
    odt = {0: torch.float16, 1: torch.bfloat16, 2: torch.float32}[w["out_dtype"]]
    out = torch.empty((T + extra_rows, w["num_heads"], w["head_size"]), dtype=odt, device="cuda")
    if sentinel is not None:
        out.view(torch.int16).fill_(sentinel)
    pa.paged_attn_forward(d["q"], d["k_cache"], d["v_cache"], d["k_scale"], d["v_scale"],
                          d["block_table"], d["seqlens_k"], d["cu_seqlens_q"], out, p)
    torch.cuda.synchronize()
    return out, p, ws


def vmax(w: dict, seqs=None) -> float:
    """max |v_scale * decode(V)| over the valid tokens of the chosen sequences."""
    ov = dict(w)
    best = 0.0
    for b in (range(w["batch"]) if seqs is None else seqs):
        if w["seqlens_k"][b] == 0:
            continue
        for kv in range(w["kv_num_heads"]):
            vals = oracle.gather_decode(ov, w["v_cache"], b, kv)
            vs = w["v_scale"][kv].astype(np.float64)
            best = max(best, float(np.nanmax(np.abs(vals * vs))))
    return best


def sub_problem(w: dict, b: int) -> dict:
    """Sequence b alone (same cache pools), for oracle runs on sampled rows."""
    cu = w["cu_seqlens_q"]
    s = dict(w)
    s["batch"] = 1
    s["block_table"] = np.ascontiguousarray(w["block_table"][b:b + 1])
    s["seqlens_k"] = np.ascontiguousarray(w["seqlens_k"][b:b + 1])
    s["cu_seqlens_q"] = np.array([0, cu[b + 1] - cu[b]], dtype=np.int32)
    s["q"] = w["q"][int(cu[b]):int(cu[b + 1])]
    return s
