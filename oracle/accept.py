"""Greedy acceptance (oracle; test infrastructure only).

What the pages fix ([P1] "The Core Idea", the worked example and the
vericache_step sketch; [P2] "Key Contributions"):
  * the verifier yields K + 1 predictions: one per drafted position plus one
    after the last drafted token;
  * drafted tokens are compared with the verifier's predictions left to right;
  * at the first mismatch the verified prefix is kept, the verifier's token is
    emitted as the correction and the rest of the draft is discarded;
  * if every drafted token matches, the whole draft is kept and the extra
    (bonus) prediction is emitted.

Readings taken where the pages are silent:
  * greedy prediction = argmax over the vocabulary of the verifier's logit
    row, compared in fp32 (bf16 logits convert exactly);
  * ties go to the LOWEST index; -0.0 and +0.0 tie; a NaN counts as the
    maximum and the first NaN wins (the numpy / torch argmax convention);
  * accept_len a in [0, K] counts accepted drafted tokens; the emitted run is
    draft[:a] + [target[a]], a + 1 tokens, and correction = target[a] (the
    bonus token when a = K).
"""

from __future__ import annotations

import numpy as np


def greedy_predictions(logits: np.ndarray) -> np.ndarray:
    """target[..., i] = argmax_v logits[..., i, v] (first index of the max,
    first NaN if any)."""
    x = np.asarray(logits, np.float32)
    if x.shape[-1] == 0:
        raise ValueError("empty vocabulary")
    return np.argmax(x, axis=-1).astype(np.int32)


def accept_one(draft, verified):
    """One request, in the pages' order: walk the draft left to right, stop at
    the first token that differs from the verifier's prediction.

    draft: K ints, verified: K + 1 ints.  Returns (accept_len, correction,
    emitted list)."""
    draft = [int(t) for t in draft]
    verified = [int(t) for t in verified]
    if len(verified) != len(draft) + 1:
        raise ValueError("the verifier gives one prediction per drafted token plus one")
    for i, token in enumerate(draft):
        if token != verified[i]:
            return i, verified[i], draft[:i] + [verified[i]]
    return len(draft), verified[-1], draft + [verified[-1]]


def accept(logits: np.ndarray, draft: np.ndarray):
    """Batched acceptance.

    logits: [B, K + 1, V] (fp32 or bf16 values); draft: [B, K] int.
    Returns (target [B, K + 1] int32, accept_len [B] int32,
    correction [B] int32)."""
    logits = np.asarray(logits, np.float32)
    draft = np.asarray(draft, np.int64)
    B, K1, _ = logits.shape
    if draft.shape != (B, K1 - 1):
        raise ValueError("draft must be [B, K] with K + 1 logit rows")
    target = greedy_predictions(logits)
    acc = np.empty(B, np.int32)
    cor = np.empty(B, np.int32)
    for b in range(B):
        a, c, _ = accept_one(draft[b], target[b])
        acc[b] = a
        cor[b] = c
    return target, acc, cor
