"""Pins of the decoder-layer oracle (oracle/layer.py), CPU only.

bf16 rounding is checked against hand-worked ties and against torch's
float32 -> bfloat16 conversion on float32 inputs (no double rounding
there); the rotary embedding against its closed form at D = 2, identity at
position 0, norm preservation and the relative-position property; RMSNorm
against constants; the whole layer against zero projections (the output is
the input) and against a loop-by-loop restatement of every step on a tiny
shape, which fixes the weight layouts, the cache rows written and the
rounding points."""

import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import layer as L


def test_bf16_round_hand_worked_ties_and_torch():
    one = 1.0
    assert L.bf16_round(one + 2 ** -8) == 1.0                  # tie -> even (1.0)
    assert L.bf16_round(one + 3 * 2 ** -8) == one + 2 ** -6    # tie -> even (1 + 2^-6)
    assert L.bf16_round(one + 2 ** -8 + 2 ** -20) == one + 2 ** -7
    assert L.bf16_round(-3.0) == -3.0 and L.bf16_round(0.0) == 0.0
    assert np.isinf(L.bf16_round(1e39)) and np.isnan(L.bf16_round(np.nan))
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(L.bf16_round(x.astype(np.float64)), want)


def test_rope_closed_form_identity_norm_and_relative_position():
    # D = 2: one pair, inverse frequency 1, a rotation by the position
    x = np.array([[[[0.6, -0.8]]]])  # [B=1, n=1, H=1, D=2]
    for p in (0.0, 1.0, 7.5):
        got = L.rope(x, np.array([[p]]))[0, 0, 0]
        want = [0.6 * math.cos(p) + 0.8 * math.sin(p), 0.6 * math.sin(p) - 0.8 * math.cos(p)]
        assert np.allclose(got, want, rtol=0, atol=1e-15)
    rng = np.random.default_rng(1)
    q = rng.standard_normal((1, 1, 1, 64))
    k = rng.standard_normal((1, 1, 1, 64))
    assert np.array_equal(L.rope(q, np.array([[0.0]])), q)
    r = L.rope(q, np.array([[123.0]]))
    assert np.allclose(np.linalg.norm(r), np.linalg.norm(q), rtol=1e-14)
    d1 = (L.rope(q, np.array([[40.0]])) * L.rope(k, np.array([[10.0]]))).sum()
    d2 = (L.rope(q, np.array([[1030.0]])) * L.rope(k, np.array([[1000.0]]))).sum()
    assert d1 == pytest.approx(d2, rel=1e-9)


def test_rms_norm_of_constants_and_scale():
    w = np.array([1.0, 2.0, -0.5, 3.0])
    c = np.full(4, -2.0)
    assert np.allclose(L.rms_norm(c, w, eps=0.0), -w)
    x = np.array([3.0, 4.0, 0.0, 0.0])
    assert np.allclose(L.rms_norm(x, np.ones(4), eps=0.0), x / math.sqrt(25 / 4))


def _weights(rng, dm, Hq, Hkv, D, F, scale=0.2):
    b = L.bf16_round
    return dict(w1=b(1 + 0.1 * rng.standard_normal(dm)), w2=b(1 + 0.1 * rng.standard_normal(dm)),
                wqkv=b(scale * rng.standard_normal(((Hq + 2 * Hkv) * D, dm))),
                wo=b(scale * rng.standard_normal((dm, Hq * D))),
                wgu=b(scale * rng.standard_normal((2 * F, dm))), wd=b(scale * rng.standard_normal((dm, F))))


def test_zero_output_projections_return_the_input():
    rng = np.random.default_rng(2)
    B, nq, dm, Hq, Hkv, D, F, T = 2, 3, 16, 4, 2, 8, 12, 9
    W = _weights(rng, dm, Hq, Hkv, D, F)
    W["wo"] = np.zeros_like(W["wo"])
    W["wd"] = np.zeros_like(W["wd"])
    x = L.bf16_round(rng.standard_normal((B, nq, dm)))
    kc = L.bf16_round(rng.standard_normal((B, Hkv, T, D)))
    vc = L.bf16_round(rng.standard_normal((B, Hkv, T, D)))
    out, kc2, vc2 = L.verify_layer(x, W, kc, vc, Hq, Hkv)
    assert np.array_equal(out, x)
    assert np.array_equal(kc2[:, :, :T - nq], kc[:, :, :T - nq])  # older rows untouched


def _loop_layer(x, W, kc, vc, Hq, Hkv, theta=500000.0, eps=1e-5):
    """Every step with explicit loops over tokens, heads and channels."""
    b16 = L.bf16_round
    B, nq, dm = x.shape
    T, D = kc.shape[2], kc.shape[3]
    g = Hq // Hkv
    half = D // 2
    F = W["wgu"].shape[0] // 2
    kc = kc.copy()
    vc = vc.copy()
    out = np.zeros_like(x)
    qs = np.zeros((B, nq, Hq, D))
    for b in range(B):
        for i in range(nq):
            pos = T - nq + i
            ms = sum(float(t) * float(t) for t in x[b, i]) / dm
            h = [b16(x[b, i, c] / math.sqrt(ms + eps) * W["w1"][c]) for c in range(dm)]
            row = [b16(sum(W["wqkv"][r, c] * h[c] for c in range(dm))) for r in range((Hq + 2 * Hkv) * D)]

            def rot(vec):
                res = [0.0] * D
                for j in range(half):
                    ang = pos * theta ** (-2.0 * j / D)
                    res[j] = b16(vec[j] * math.cos(ang) - vec[j + half] * math.sin(ang))
                    res[j + half] = b16(vec[j] * math.sin(ang) + vec[j + half] * math.cos(ang))
                return res

            for hq in range(Hq):
                qs[b, i, hq] = rot(row[hq * D:(hq + 1) * D])
            for hk in range(Hkv):
                kc[b, hk, pos] = rot(row[(Hq + hk) * D:(Hq + hk + 1) * D])
                vc[b, hk, pos] = row[(Hq + Hkv + hk) * D:(Hq + Hkv + hk + 1) * D]
    for b in range(B):
        for i in range(nq):
            attn = []
            for hq in range(Hq):
                hk = hq // g
                n = T - nq + i + 1
                s = [sum(qs[b, i, hq, c] * kc[b, hk, t, c] for c in range(D)) / math.sqrt(D) for t in range(n)]
                m = max(s)
                p = [math.exp(z - m) for z in s]
                den = sum(p)
                attn += [b16(sum(p[t] * vc[b, hk, t, c] for t in range(n)) / den) for c in range(D)]
            x2 = [b16(x[b, i, c] + sum(W["wo"][c, r] * attn[r] for r in range(Hq * D))) for c in range(dm)]
            ms = sum(t * t for t in x2) / dm
            h2 = [b16(x2[c] / math.sqrt(ms + eps) * W["w2"][c]) for c in range(dm)]
            gu = [b16(sum(W["wgu"][r, c] * h2[c] for c in range(dm))) for r in range(2 * F)]
            a = [b16(gu[f] / (1 + math.exp(-gu[f])) * gu[F + f]) for f in range(F)]
            out[b, i] = [b16(x2[c] + sum(W["wd"][c, f] * a[f] for f in range(F))) for c in range(dm)]
    return out, kc, vc


def test_layer_equals_the_loop_restatement_on_a_tiny_shape():
    rng = np.random.default_rng(3)
    B, nq, dm, Hq, Hkv, D, F, T = 1, 2, 8, 4, 2, 4, 6, 5
    W = _weights(rng, dm, Hq, Hkv, D, F, scale=0.5)
    x = L.bf16_round(rng.standard_normal((B, nq, dm)))
    kc = L.bf16_round(rng.standard_normal((B, Hkv, T, D)))
    vc = L.bf16_round(rng.standard_normal((B, Hkv, T, D)))
    got, gk, gv = L.verify_layer(x, W, kc, vc, Hq, Hkv)
    want, wk, wv = _loop_layer(x, W, kc, vc, Hq, Hkv)
    # the loop sums in another order: each bf16 rounding may land one ulp apart
    # only when the exact value sits on a tie, which random data never hits
    assert np.array_equal(gk, wk) and np.array_equal(gv, wv)
    assert np.array_equal(got, want)
