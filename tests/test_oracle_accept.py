"""Pins for the oracle's greedy acceptance (CPU only): the pages' worked
example, brute force over tiny vocabularies against independent definitions,
and the end-to-end claim that the emitted stream equals full-cache greedy
decoding (on a toy model)."""

import itertools
import json
import os

import numpy as np
import pytest

from oracle import accept as ACC
from oracle import rounds


def test_worked_example(golden_dir):
    with open(os.path.join(golden_dir, "worked_example_accept.json")) as f:
        ex = json.load(f)
    draft = ex["draft"]
    K = len(draft)
    verified = ex["verified_prefix"] + [9] * (K + 1 - len(ex["verified_prefix"]))
    a, c, emitted = ACC.accept_one(draft, verified)
    assert (a, c, emitted) == (ex["expected_accept_len"], ex["expected_correction"], ex["expected_emitted"])
    # the same through logits rows
    V = 32
    logits = np.zeros((1, K + 1, V), np.float32)
    for i, t in enumerate(verified):
        logits[0, i, t] = 1.0
    tgt, acc, cor = ACC.accept(logits, np.array([draft]))
    assert tgt[0].tolist() == verified and acc[0] == 5 and cor[0] == 23


def _argmax_by_definition(row):
    """Smallest v with row[v] >= row[u] for every u (NaN: smallest NaN index)."""
    nan = [i for i, x in enumerate(row) if x != x]
    if nan:
        return nan[0]
    for v in range(len(row)):
        if all(row[v] >= row[u] for u in range(len(row))):
            return v
    raise AssertionError


def test_argmax_brute_force_all_rows_with_ties():
    vals = [-1.0, 0.0, 2.0]
    for row in itertools.product(vals, repeat=4):
        got = int(ACC.greedy_predictions(np.array([row], np.float32))[0])
        assert got == _argmax_by_definition(row), row


def test_argmax_signed_zero_and_nan():
    assert ACC.greedy_predictions(np.array([[-0.0, 0.0, -1.0]], np.float32))[0] == 0
    assert ACC.greedy_predictions(np.array([[0.0, -0.0]], np.float32))[0] == 0
    assert ACC.greedy_predictions(np.array([[1.0, np.nan, 5.0, np.nan]], np.float32))[0] == 1
    assert ACC.greedy_predictions(np.array([[-np.inf, -np.inf]], np.float32))[0] == 0


@pytest.mark.parametrize("K", [0, 1, 2, 3])
def test_accept_brute_force(K):
    """All drafts and verifier predictions over a vocabulary of 3: the accepted
    length is the longest k with draft[:k] == target[:k]; the emitted run is
    that prefix plus target[k]."""
    V = 3
    for draft in itertools.product(range(V), repeat=K):
        for target in itertools.product(range(V), repeat=K + 1):
            a_def = max(k for k in range(K + 1) if list(draft[:k]) == list(target[:k]))
            a, c, emitted = ACC.accept_one(draft, target)
            assert a == a_def and c == target[a_def]
            assert emitted == list(draft[:a_def]) + [target[a_def]]
            assert len(emitted) == a + 1


def test_accept_batched_shapes_and_bonus():
    rng = np.random.default_rng(0)
    B, K, V = 3, 4, 7
    logits = rng.standard_normal((B, K + 1, V)).astype(np.float32)
    tgt = logits.argmax(-1)
    draft = tgt[:, :K].copy()
    draft[1, 2] = (draft[1, 2] + 1) % V
    draft[2, 0] = (draft[2, 0] + 1) % V
    t, a, c = ACC.accept(logits, draft)
    assert a.tolist() == [K, 2, 0]
    assert c.tolist() == [tgt[0, K], tgt[1, 2], tgt[2, 0]]


@pytest.mark.parametrize("flip,draft_len", [(0.0, 5), (0.05, 8), (0.3, 4), (1.0, 3)])
def test_rounds_reproduce_greedy_decoding(flip, draft_len):
    """The pages' central claim on a toy model: whatever the drafter does,
    the emitted stream equals greedy decoding with the full model."""
    full = rounds.ToyModel(vocab=11, seed=5)
    lossy = rounds.LossyToyModel(full, flip_rate=flip, seed=3)
    prefix = [1, 2, 3]
    want = rounds.greedy_generate(prefix, full, 60)
    got = rounds.generate(prefix, lossy, full, draft_len, 60)
    assert got == want


def test_rounds_emit_draft_plus_bonus_when_drafter_is_exact():
    full = rounds.ToyModel(vocab=13, seed=2)
    out = rounds.vericache_step([4, 4], rounds.LossyToyModel(full, 0.0), full, 6)
    assert len(out) == 7
