"""One decoder layer of the verifier on random weights (oracle; test
infrastructure only).

What the pages fix
------------------
[P1] "The Core Idea": verification is one pass of the same model over the
block of drafted tokens with the full cache, giving one prediction per
drafted position plus one.  [P2] "Methodology": drafter and verifier use
the same model weights and differ only in KV fidelity; the models are
Llama, Mistral and Qwen decoders.  The pages give no layer arithmetic.

Readings taken where the pages are silent
-----------------------------------------
* A Llama-style pre-norm decoder layer: h = RMSNorm(x) w1 (eps 1e-5);
  [q | k | v] = h Wqkv^T; rotary position embedding on q and k; the block's
  own k and v are written into the full cache at rows T - nq .. T - 1 (row i
  of the block at position T - nq + i); causal verification attention
  (attention.verify_attention); x2 = x + attn Wo^T; h2 = RMSNorm(x2) w2;
  [g | u] = h2 Wgu^T; a = silu(g) * u; out = x2 + a Wd^T.
* Rotary embedding, the "rotate half" form: channel j < D/2 pairs with
  j + D/2; angle = position * theta^(-2j / D) with theta 500000 (the
  Llama-3.1 base; no frequency scaling: the weights are random).
* Activations are bf16 between the layer's operations, as in a bf16 serving
  model: the result of every step above (norm outputs, each projection, the
  rotated q and k, the attention output, each residual sum, the SwiGLU
  product) is rounded to bf16, round to nearest even, and the next step
  starts from the rounded value.  Each step itself is computed exactly in
  float64 from its bf16 inputs, so this function is the plain definition
  with the rounding points written out.
* Weights are bf16, row-major [out][in]: Wqkv [(Hq + 2 Hkv) D][d_model],
  Wo [d_model][Hq D], Wgu [2 d_ff][d_model] (gate rows first), Wd
  [d_model][d_ff]; w1, w2 [d_model].
"""

from __future__ import annotations

import numpy as np

from . import attention


def bf16_round(x) -> np.ndarray:
    """x (float64) rounded once to the nearest bf16 value (ties to even),
    returned as float64; inf and nan pass through, overflow gives inf."""
    x = np.asarray(x, np.float64)
    out = np.array(x, copy=True)
    fin = np.isfinite(x) & (x != 0)
    m, e = np.frexp(x[fin])  # x = m 2^e, 0.5 <= |m| < 1
    r = np.rint(m * 256.0) / 256.0  # 8 significant bits, half to even
    v = np.ldexp(r, e)
    v[np.abs(v) > 3.3895313892515355e38] = np.inf * np.sign(v[np.abs(v) > 3.3895313892515355e38])
    out[fin] = v
    return out


def rms_norm(x: np.ndarray, w: np.ndarray, eps: float = 1e-5) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * w over the last axis (float64)."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w, np.float64)


def rope(x: np.ndarray, pos: np.ndarray, theta: float = 500000.0) -> np.ndarray:
    """Rotary embedding, rotate-half form, of x [..., n, H, D] at positions
    pos [..., n] (float64)."""
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    half = D // 2
    inv = theta ** (-2.0 * np.arange(half, dtype=np.float64) / D)
    ang = np.asarray(pos, np.float64)[..., None, None] * inv  # [..., n, 1, half]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def silu(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, np.float64)
    return x / (1.0 + np.exp(-x))


def verify_layer(x: np.ndarray, weights: dict, k_cache: np.ndarray, v_cache: np.ndarray, Hq: int, Hkv: int,
                 theta: float = 500000.0, eps: float = 1e-5):
    """One decoder layer over the verification block.

    x: [B, nq, d_model] bf16 values; k_cache, v_cache: [B, Hkv, T, D] bf16
    values (rows T - nq .. T - 1 are overwritten by the block's own k, v).
    weights: w1, wqkv, wo, w2, wgu, wd as described in the header.
    Returns (out [B, nq, d_model], k_cache, v_cache) as float64 arrays of
    bf16 values; the caches are new arrays."""
    x = np.asarray(x, np.float64)
    B, nq, dm = x.shape
    T, D = k_cache.shape[2], k_cache.shape[3]
    W = {k: np.asarray(v, np.float64) for k, v in weights.items()}
    h = bf16_round(rms_norm(x, W["w1"], eps))
    qkv = bf16_round(h @ W["wqkv"].T)  # [B, nq, (Hq + 2 Hkv) D]
    q = qkv[..., :Hq * D].reshape(B, nq, Hq, D)
    k = qkv[..., Hq * D:(Hq + Hkv) * D].reshape(B, nq, Hkv, D)
    v = qkv[..., (Hq + Hkv) * D:].reshape(B, nq, Hkv, D)
    pos = np.broadcast_to(np.arange(T - nq, T, dtype=np.float64), (B, nq))
    q = bf16_round(rope(q, pos, theta))
    k = bf16_round(rope(k, pos, theta))
    kc = np.array(k_cache, np.float64, copy=True)
    vc = np.array(v_cache, np.float64, copy=True)
    kc[:, :, T - nq:, :] = k.transpose(0, 2, 1, 3)
    vc[:, :, T - nq:, :] = v.transpose(0, 2, 1, 3)
    o, _ = attention.verify_attention(q, kc, vc)  # [B, nq, Hq, D]
    attn = bf16_round(o).reshape(B, nq, Hq * D)
    x2 = bf16_round(x + attn @ W["wo"].T)
    h2 = bf16_round(rms_norm(x2, W["w2"], eps))
    gu = bf16_round(h2 @ W["wgu"].T)
    F = gu.shape[-1] // 2
    a = bf16_round(silu(gu[..., :F]) * gu[..., F:])
    out = bf16_round(x2 + a @ W["wd"].T)
    return out, kc, vc
