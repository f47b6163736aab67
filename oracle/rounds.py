"""The VeriCache round over a toy greedy "model" (oracle; test infrastructure
only).

[P1] "The Core Idea" states the round: draft ``draft_len`` tokens with the
compressed cache, verify every drafted position with the full cache in one
pass (draft_len + 1 predictions), accept up to the first mismatch, emit the
correction or the bonus token.  [P1] and [P2] "Results" claim the emitted
stream equals greedy decoding with the full cache.  There are no model weights
here, so that claim is pinned on a toy model: a deterministic next-token rule
over a token prefix, and a "lossy" copy of it that agrees except where a
seeded hash says otherwise.  The toy stands in for "same weights, different
cache fidelity" and nothing else.

The verifier's predictions go through greedy logits rows and oracle.accept,
so the test that uses this module exercises the acceptance rule end to end.
"""

from __future__ import annotations

import numpy as np

from . import accept as _accept


def _mix(x: int) -> int:
    """splitmix64 finaliser (public-domain integer hash), used only to make a
    deterministic toy next-token rule."""
    x = (x + 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
    return x ^ (x >> 31)


def _prefix_hash(prefix) -> int:
    h = 0x1234567
    for t in prefix:
        h = _mix(h ^ (int(t) + 1))
    return h


class ToyModel:
    """Deterministic greedy next-token rule over a vocabulary of ``vocab``."""

    def __init__(self, vocab: int, seed: int = 0):
        self.vocab = vocab
        self.seed = seed

    def logits(self, prefix) -> np.ndarray:
        """A logit row whose unique argmax is the next token."""
        h = _prefix_hash(prefix) ^ self.seed
        row = np.array([(_mix(h ^ v) >> 40) / float(1 << 24) for v in range(self.vocab)], np.float32)
        row[_mix(h) % self.vocab] = 2.0
        return row

    def next_token(self, prefix) -> int:
        return int(np.argmax(self.logits(prefix)))


class LossyToyModel:
    """The same rule, except that at a seeded fraction of prefixes it
    predicts a different token (the "compressed cache" drafter)."""

    def __init__(self, full: ToyModel, flip_rate: float, seed: int = 1):
        self.full = full
        self.flip_rate = flip_rate
        self.seed = seed

    def next_token(self, prefix) -> int:
        t = self.full.next_token(prefix)
        u = (_mix(_prefix_hash(prefix) ^ (self.seed * 0x51ED27)) >> 11) / float(1 << 53)
        if u < self.flip_rate:
            return (t + 1 + (_mix(t ^ self.seed) % (self.full.vocab - 1))) % self.full.vocab
        return t


def vericache_step(prefix, drafter: LossyToyModel, verifier: ToyModel, draft_len: int):
    """One round: draft autoregressively with the drafter, compute the
    verifier's draft_len + 1 logit rows (position i sees prefix + draft[:i]),
    then accept by the greedy rule.  Returns the emitted tokens."""
    draft = []
    for _ in range(draft_len):
        draft.append(drafter.next_token(list(prefix) + draft))
    rows = np.stack([verifier.logits(list(prefix) + draft[:i]) for i in range(draft_len + 1)])
    _, acc, cor = _accept.accept(rows[None], np.array([draft], np.int64))
    a = int(acc[0])
    return draft[:a] + [int(cor[0])]


def generate(prefix, drafter, verifier, draft_len: int, n_tokens: int):
    """Run rounds until at least n_tokens are emitted; returns the first
    n_tokens emitted tokens."""
    out = []
    cur = list(prefix)
    while len(out) < n_tokens:
        emitted = vericache_step(cur, drafter, verifier, draft_len)
        out += emitted
        cur += emitted
    return out[:n_tokens]


def greedy_generate(prefix, model: ToyModel, n_tokens: int):
    """Plain greedy decoding with the full model (the output VeriCache must
    reproduce)."""
    out = []
    cur = list(prefix)
    for _ in range(n_tokens):
        t = model.next_token(cur)
        out.append(t)
        cur.append(t)
    return out
