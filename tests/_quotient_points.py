"""Values next to a code's rounding boundary, with their codes decided exactly.

A symmetric per-channel cache stores the code nearest to x / s (value = scale x
code; the INT4 paged-KV page, onnxruntime PR 32515, Code analysis 2-3).  The
writer takes that quotient in IEEE single precision.  Near a boundary between
two codes (k + 1/2 for the integer caches, the midpoint of two neighbouring
e4m3 values for FP8) a correctly rounded x / s and the product of x with a
rounded 1 / s can fall on different sides.  This module builds such inputs and
decides their codes from the exact rational quotient, which needs neither the
oracle nor the kernel:

  * x is an fp16 value (the writer's input type), s a positive fp32 scale;
  * the exact quotient x / s lies more than one fp32 ulp (of the boundary B)
    away from B, so every correctly rounded fp32 quotient stays on the same side
    of B as the exact one, and the code is the one nearest to the exact value;
  * x * fl(1 / s), computed in fp32, lands on the other side (or on B itself,
    where ties to even pick the other code).

The search is targeted: pick a boundary B and an fp16 x, put s within a few
fp32 ulps of x / B, and keep the pairs that meet both conditions.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import torch

KV_INT8, KV_INT4, KV_FP8_E4M3 = 0, 1, 2


def _e4m3_values() -> np.ndarray:
    """Values of the 127 non-negative finite e4m3fn codes 0x00..0x7E, from
    torch's float8_e4m3fn type (a library outside this repository)."""
    codes = torch.arange(0x7F, dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _nearest_int_code(q: Fraction, lo: int, hi: int) -> int:
    """Nearest integer to q (never a tie here), clamped to [lo, hi]."""
    k = int(q.__floor__())
    c = k + 1 if q - k > Fraction(1, 2) else k
    return max(lo, min(hi, c))


def _nearest_e4m3_code(q: Fraction, table: np.ndarray) -> int:
    """Byte of the e4m3fn value nearest to q (never a tie here; |q| < 448)."""
    a = abs(q)
    best, best_d = 0, None
    for c, v in enumerate(table):
        d = abs(Fraction(float(v)) - a)
        if best_d is None or d < best_d:
            best, best_d = c, d
    return (0x80 if q < 0 else 0) | best


def _product_code(kv: int, x: np.float32, s: np.float32) -> int:
    """The code a writer that multiplies by the rounded inverse scale stores."""
    inv = np.float32(1.0) / s
    qm = np.float32(x * inv)
    if kv == KV_FP8_E4M3:
        return int(torch.tensor([float(qm)], dtype=torch.float32)
                   .to(torch.float8_e4m3fn).view(torch.uint8).item())
    lo, hi = (-8, 7) if kv == KV_INT4 else (-127, 127)
    return int(max(lo, min(hi, np.rint(qm))))


def boundary_points(kv: int, n: int, seed: int):
    """n triples (x, s, code): x exactly representable in fp16, s > 0 in fp32,
    code the exact-quotient code (signed integer, or the e4m3 byte), at inputs
    where the inverse-multiply form stores a different code."""
    rng = np.random.default_rng(seed)
    table = _e4m3_values()
    if kv == KV_FP8_E4M3:
        mids = (table[1:] + table[:-1]) / 2  # midpoints of neighbouring magnitudes
        mids = mids[(mids > 2.0 ** -8) & (mids < 440.0)]
    out, tries = [], 0
    while len(out) < n:
        tries += 1
        assert tries < 200000, "boundary search did not converge"
        if kv == KV_FP8_E4M3:
            B = float(rng.choice(mids))
        else:
            top = 7 if kv == KV_INT4 else 127
            B = float(rng.integers(0, top)) + 0.5  # boundary between k and k + 1
        if rng.random() < 0.5:
            B = -B
        x = np.float16(rng.uniform(0.5, 60.0) * (1 if B > 0 else -1))
        x32 = np.float32(x)
        if x32 == 0:
            continue
        s = np.float32(float(x32) / B)
        for _ in range(int(rng.integers(0, 4))):  # a few ulps either way
            s = np.nextafter(s, np.float32(np.inf) if rng.random() < 0.5 else np.float32(0))
        if not (s > 0) or not np.isfinite(s):
            continue
        q = Fraction(float(x32)) / Fraction(float(s))
        Bf = Fraction(B)
        u = Fraction(float(np.spacing(np.float32(abs(B)))))
        if abs(q - Bf) <= u:  # too close: the fp32 quotient might sit on B
            continue
        if kv == KV_FP8_E4M3:
            want = _nearest_e4m3_code(q, table)
        else:
            lo, hi = (-8, 7) if kv == KV_INT4 else (-127, 127)
            want = _nearest_int_code(q, lo, hi)
        if _product_code(kv, x32, s) == want:
            continue  # both forms agree here: not a separating point
        out.append((float(x32), float(s), want))
    return out
