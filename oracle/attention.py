"""fp64 softmax attention for the three attention steps (oracle; test
infrastructure only).

What the pages fix
------------------
[P1] "The Core Idea": the same model drafts one token at a time from the
compressed cache, then one verification pass with the full cache produces a
prediction for every drafted position plus one more.  [P2] "Key
Contributions": drafting reads the compressed KV in HBM; verification checks
multiple tokens in parallel against the full KV.

Readings taken where the pages are silent
-----------------------------------------
* Attention is standard scaled dot-product softmax attention,
  o = softmax(q . K^T * sm_scale) . V, sm_scale = 1/sqrt(D) unless given.
* Grouped-query attention: query head hq reads KV head hq // g with
  g = Hq / Hkv.
* Verification: the block holds nq query rows whose own keys are the last nq
  rows of the T-row cache; row i (0 <= i < nq) sees keys 0 .. T - nq + i
  (causal).  With nq = K + 1 the rows are the last accepted token followed
  by the K drafted tokens, giving K + 1 predictions.
* Everything is computed in float64 from the exact bf16 / dequantised fp32
  inputs.  No blocking, no split over the context, no rescaling tricks beyond
  subtracting the row maximum before exponentiation (which changes nothing
  mathematically).
"""

from __future__ import annotations

import math

import numpy as np

from . import quant


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, sm_scale: float):
    """o = softmax(q k^T * sm_scale) v for one KV head.

    q: [M, D] query rows, k, v: [N, D] with N >= 1.  Returns (o [M, D],
    lse [M]) in float64; lse is the natural log of the softmax denominator
    sum_j exp(s_j) with s_j the scaled scores."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    if k.shape[0] == 0:
        raise ValueError("attention over an empty key set is undefined")
    s = (q @ k.T) * float(sm_scale)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ v) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


def _check_gqa(Hq: int, Hkv: int) -> int:
    if Hkv <= 0 or Hq % Hkv:
        raise ValueError("Hq must be a positive multiple of Hkv")
    return Hq // Hkv


def draft_attention_dense(q: np.ndarray, k: np.ndarray, v: np.ndarray, sm_scale: float | None = None):
    """Single-token decode attention over a dense cache.

    q: [B, Hq, D]; k, v: [B, Hkv, N, D].  Returns o [B, Hq, D] float64.
    This is the textbook operation the two draft steps reduce to."""
    q = np.asarray(q, np.float64)
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    g = _check_gqa(Hq, Hkv)
    scale = default_scale(D) if sm_scale is None else sm_scale
    out = np.empty((B, Hq, D), np.float64)
    for b in range(B):
        for h in range(Hkv):
            o, _ = softmax_attention(q[b, h * g:(h + 1) * g], k[b, h], v[b, h], scale)
            out[b, h * g:(h + 1) * g] = o
    return out


def draft_attention_quant(q: np.ndarray, cache: dict, sm_scale: float | None = None):
    """Draft attention over a quantised cache ([P2] "Key Contributions":
    draft one token at a time from the compressed KV; [P1] "Verifying
    Without Giving Back the Speedup": drafting reads the compressed cache).

    The compressed cache is first dequantised by the reference rule
    (oracle.quant), the bf16 residual rows are appended, then plain softmax
    attention runs over all L_q + R rows."""
    k_hat, v_hat = quant.dequantize_cache(cache)
    return draft_attention_dense(q, k_hat, v_hat, sm_scale)


def gather_rows(store: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """rows[b, h, j] = store[b, h, idx[b, h, j]] ([P2] "Key Contributions": a
    token-dropping compressor is described by its kept / dropped positions;
    "Limitations": the same count for every layer-head)."""
    store = np.asarray(store)
    idx = np.asarray(idx, np.int64)
    B, H, n = idx.shape
    if np.any(idx < 0) or np.any(idx >= store.shape[2]):
        raise ValueError("kept position outside the store")
    out = np.empty((B, H, n, store.shape[3]), store.dtype)
    for b in range(B):
        for h in range(H):
            out[b, h] = store[b, h, idx[b, h]]
    return out


def draft_attention_sparse(q: np.ndarray, k_store: np.ndarray, v_store: np.ndarray,
                           idx: np.ndarray, sm_scale: float | None = None):
    """Draft attention over a token-dropped cache: attention over the kept
    rows only."""
    return draft_attention_dense(q, gather_rows(k_store, idx), gather_rows(v_store, idx), sm_scale)


def verify_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, sm_scale: float | None = None):
    """Causal block verification attention ([P1] "The Core Idea": one
    forward pass over the full cache yields a prediction for every drafted
    position plus one; [P2] "Key Contributions": verify multiple tokens in
    parallel against the full KV).

    q: [B, nq, Hq, D]; k, v: [B, Hkv, T, D] with T >= nq.  Row i sees keys
    0 .. T - nq + i.  Returns (o [B, nq, Hq, D], lse [B, nq, Hq]) float64."""
    q = np.asarray(q, np.float64)
    B, nq, Hq, D = q.shape
    Hkv, T = k.shape[1], k.shape[2]
    if T < nq:
        raise ValueError("the cache must hold the verified block")
    g = _check_gqa(Hq, Hkv)
    scale = default_scale(D) if sm_scale is None else sm_scale
    o = np.empty((B, nq, Hq, D), np.float64)
    lse = np.empty((B, nq, Hq), np.float64)
    for b in range(B):
        for hq in range(Hq):
            h = hq // g
            for i in range(nq):
                n_vis = T - nq + i + 1
                oi, li = softmax_attention(q[b, i, hq][None, :], k[b, h, :n_vis], v[b, h, :n_vis], scale)
                o[b, i, hq] = oi[0]
                lse[b, i, hq] = li[0]
    return o, lse
