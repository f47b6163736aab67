"""The GPU quantiser's code rule, emulated in numpy, against the float64
definition (oracle/quant.py takes codes as rint of the float64 quotient).

The kernel (lossless_draft_verify_vc_b200/csrc/vc_compress.cu, codes2_fast
and code_near) takes q = fp32(fp32(x - z) * fp32(1 / s)), clamps it to
[0, levels], rounds by adding 1.5 * 2^23, and calls a quotient "near" when
it lies within 2^-17 of a tie.  A near quotient is decided exactly: when
d = fp32(x - z) is exact (two-sum error 0), the sign of d - T s for the tie
T = k + 1/2 (one FMA, so the sign is exact) puts it above, below or on T
(on T the even code wins); otherwise the float64 division decides.  Here
every fp32 operation is numpy float32 arithmetic (IEEE round to nearest),
and the FMA's sign is the sign of the exact float64 value d - T s (both
products of fp32 numbers with few bits, so float64 holds them exactly).
Inputs: random bf16 x with fp16 z and s drawn as the quantiser forms them
from a group's range, plus constructed exact ties, near ties and
differences too wide for fp32."""

import numpy as np
import pytest

F32 = np.float32
MAGIC = F32(12582912.0)       # 1.5 * 2^23
NEAR = F32(0.5) - F32(2.0 ** -17)


def bf16(x):
    """Round float64 values to bfloat16 (nearest, ties to even), as float64."""
    b = np.asarray(x, np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def rule_f64(x, z, s, levels):
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s != 0, np.rint((x - z) / np.where(s != 0, s, 1.0)), 0.0)
    return np.clip(q, 0, levels).astype(np.int64)


def rule_kernel(x, z, s, levels):
    x32, nz32, s32 = x.astype(F32), (-z).astype(F32), s.astype(F32)
    with np.errstate(divide="ignore"):
        inv = np.where(s32 != 0, F32(1) / np.where(s32 != 0, s32, F32(1)), F32(0)).astype(F32)
    d = (x32 + nz32).astype(F32)
    q = (d * inv).astype(F32)
    qc = np.clip(q, F32(0), F32(levels)).astype(F32)
    m = (qc + MAGIC).astype(F32)
    r = (m - MAGIC).astype(F32)
    code = r.astype(np.int64)
    e = (qc - r).astype(F32)
    near = (np.abs(e) > NEAR) & (s32 != 0)
    # exact decision for the near ones
    bv = (d - x32).astype(F32)
    av = (d - bv).astype(F32)
    err = ((x32 - av).astype(F32) + (nz32 - bv).astype(F32)).astype(F32)
    T = np.where(qc > r, r + F32(0.5), r - F32(0.5)).astype(np.float64)
    t = d.astype(np.float64) - T * s32.astype(np.float64)   # exact; its sign is the FMA's
    lo = T - 0.5
    exact = np.where(t > 0, T + 0.5, np.where(t < 0, lo, np.where(lo % 2 == 0, lo, T + 0.5)))
    exact = np.clip(exact, 0, levels).astype(np.int64)
    f64 = rule_f64(x32.astype(np.float64), -nz32.astype(np.float64), s32.astype(np.float64), levels)
    near_code = np.where(err != 0, f64, exact)
    return np.where(near, near_code, code), near, err != 0


def group_params(lo, hi, levels):
    s = (np.asarray(hi - lo, np.float64) / levels).astype(np.float16).astype(np.float64)
    z = np.asarray(lo, np.float64).astype(np.float16).astype(np.float64)
    return z, s


@pytest.mark.parametrize("bits", [2, 4])
def test_random_groups_match_the_float64_rule(bits):
    levels = (1 << bits) - 1
    rng = np.random.default_rng(bits)
    n = 400000
    scale = np.exp(rng.uniform(-6, 6, n))
    a = bf16(rng.standard_normal(n) * scale)
    b = bf16(rng.standard_normal(n) * scale)
    lo, hi = np.minimum(a, b), np.maximum(a, b)
    x = bf16(lo + rng.uniform(0, 1, n) * (hi - lo))
    x = np.where(rng.uniform(size=n) < 0.05, lo, np.where(rng.uniform(size=n) < 0.05, hi, x))
    z, s = group_params(lo, hi, levels)
    got, near, _ = rule_kernel(x, z, s, levels)
    assert np.array_equal(got, rule_f64(x, z, s, levels))
    assert near.any()  # bf16 data against fp16 parameters meets exact ties


@pytest.mark.parametrize("bits", [2, 4])
def test_constructed_ties_and_wide_differences(bits):
    levels = (1 << bits) - 1
    rng = np.random.default_rng(10 + bits)
    n = 200000
    # exact ties: s with few significant bits, x = z + (k + 1/2) s
    e = rng.integers(-12, 6, n).astype(np.float64)
    s = (rng.integers(1, 16, n) * 2.0 ** e).astype(np.float16).astype(np.float64)
    z = bf16(rng.standard_normal(n) * 2.0 ** rng.integers(-4, 6, n)).astype(np.float16).astype(np.float64)
    k = rng.integers(0, levels, n)
    x = bf16(z + (k + 0.5) * s)
    # nudge some by one bf16 step either way (near, not on, the tie)
    step = np.abs(x) * 2.0 ** -7
    x = np.where(rng.uniform(size=n) < 0.3, bf16(x + step), x)
    x = np.where(rng.uniform(size=n) < 0.3, bf16(x - step), x)
    # differences too wide for fp32: tiny x against a large zero
    wide = rng.uniform(size=n) < 0.2
    z = np.where(wide, -1000.0, z)
    s = np.where(wide, 400.0, s)
    x = np.where(wide, bf16(2.0 ** rng.integers(-40, -20, n) * np.sign(rng.standard_normal(n))), x)
    got, near, inexact = rule_kernel(x, z, s, levels)
    want = rule_f64(x, z, s, levels)
    assert np.array_equal(got, want)
    assert near.sum() > n // 10 and (near & inexact).any()
    # without the exact decision the rule would differ on some of them
    fast_only = np.clip(np.rint(((x.astype(F32) - z.astype(F32)).astype(F32) *
                                 (F32(1) / s.astype(F32))).astype(F32)), 0, levels).astype(np.int64)
    assert not np.array_equal(fast_only, want)
