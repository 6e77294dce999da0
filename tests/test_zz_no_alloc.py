"""paged_attn_forward_noalloc: the forward call for callers that cannot allocate.

Some callers (an operator inside a framework that owns every device buffer, a
memory plan frozen at start-up and replayed, a real-time loop) may not call
cudaMalloc where they run attention, so they cannot pass a workspace.  The
library then uses its own static device scratch.  These tests call that entry
point through the C ABI twice in a row and check each result against the
ordinary entry point (own workspace) within the parity tolerance
(2e-3 * max|dequant(V)| for fp16 output, 8e-3 for bf16).

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import paged_quantized_kv_attention_b200 as pa
import workloads
from tests import _gpu

pytestmark = pytest.mark.gpu


def _new_out(w):
    odt = torch.bfloat16 if w["out_dtype"] == 1 else torch.float16
    return torch.empty((int(w["cu_seqlens_q"][-1]), w["num_heads"], w["head_size"]), dtype=odt,
                       device="cuda")


@pytest.mark.parametrize("name,over", [
    ("c3_int8_long_split", dict(split_blocks=4)),  # many splits: partials in the scratch
    ("c2_int4_decode", {}),
    ("c4_ragged_prefill_int8", {}),
])
def test_noalloc_matches_forward_on_two_calls(name, over):
    w = workloads.shrink(name, 31, max_len=3000 if name.startswith("c3") else 600, batch=4)
    d = _gpu.to_device(w)
    ref, p, _ = _gpu.run(w, d, **over)
    if over:
        assert p.num_splits > 1
    assert p.workspace_bytes <= pa.PA_NOALLOC_MAX_WORKSPACE_BYTES
    tol = _gpu.TOL[w["out_dtype"]] * _gpu.vmax(w)
    q = pa.paged_attn_params.from_buffer_copy(p)
    q.workspace = None  # ignored by the no-alloc entry point
    for _ in range(2):
        out = _new_out(w)
        out.fill_(float("nan"))
        pa.paged_attn_forward_noalloc(d["q"], d["k_cache"], d["v_cache"], d["k_scale"],
                                      d["v_scale"], d["block_table"], d["seqlens_k"],
                                      d["cu_seqlens_q"], out, q)
        torch.cuda.synchronize()
        got = out.double()
        assert bool(torch.isfinite(got).all())
        err = float((got - ref.double()).abs().max())
        assert err <= tol, "no-alloc vs forward: max err %.3g > tol %.3g" % (err, tol)


def test_noalloc_device_error_reads_back():
    """A block-table entry outside the pool is a condition only the device sees:
    the no-alloc call records it in its scratch's error word, which
    paged_attn_read_device_error(NULL) returns; the next call starts clean."""
    w = workloads.shrink("c2_int4_decode", 37, max_len=400, batch=3)
    d = _gpu.to_device(w)
    p, _ = _gpu.plan(w)
    bad = d["block_table"].clone()
    bad[1, 0] = w["num_blocks"] + 5
    out = _new_out(w)
    pa.paged_attn_forward_noalloc(d["q"], d["k_cache"], d["v_cache"], d["k_scale"], d["v_scale"],
                                  bad, d["seqlens_k"], d["cu_seqlens_q"], out, p)
    st, bits = pa.paged_attn_read_device_error(None, clear=False)
    assert bits & pa.PA_DEVERR_BAD_BLOCK and st == pa.PA_ERR_BAD_BLOCK_TABLE
    pa.paged_attn_forward_noalloc(d["q"], d["k_cache"], d["v_cache"], d["k_scale"], d["v_scale"],
                                  d["block_table"], d["seqlens_k"], d["cu_seqlens_q"], out, p)
    st, bits = pa.paged_attn_read_device_error(None)
    assert (st, bits) == (pa.PA_OK, 0)
