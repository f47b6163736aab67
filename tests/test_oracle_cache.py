"""Pins of the cache-maintenance oracle (oracle/cache.py), CPU only.

The maintained quantised cache must equal, record for record and row for
row, the cache built at once from the committed rows (each record is the
quantisation of one fixed group of consecutive committed rows); discarded
draft rows must never enter it; its residual never exceeds R_cap; and the
pages' worked example (draft A..H, verifier A B C D E X) keeps the block's
first six rows (x and A..E) and drops F, G, H."""

import numpy as np
import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from oracle import attention as A
from oracle import cache as CM
from oracle import quant as Q


def _rows(Hkv, n, D, seed):
    k, v = synth.kv_full(1, Hkv, n, D, seed=seed)
    return k[0].float().numpy(), v[0].float().numpy()


@pytest.mark.parametrize("bits,G,D,R_cap,nq", [(2, 32, 64, 128, 31), (4, 64, 64, 96, 31), (2, 32, 128, 40, 9),
                                               (4, 32, 64, 32, 32)])
def test_maintained_cache_equals_the_cache_built_from_the_committed_rows(bits, G, D, R_cap, nq):
    Hkv = 2
    rng = np.random.default_rng(bits * 1000 + G + R_cap)
    # an initial cache built from a prompt, then rounds
    k0, v0 = _rows(Hkv, 3 * G + 17, D, seed=1)
    R0 = 17
    base = Q.build_quant_cache(k0[None], v0[None], bits, G, R0)
    state = dict(bits=bits, group=G, D=D, L_q=base["L_q"], R=R0, records=base["records"][0],
                 k_res=base["k_res"][0], v_res=base["v_res"][0])
    committed_k, committed_v = [k0], [v0]
    for r in range(12):
        kb, vb = _rows(Hkv, nq, D, seed=100 + r)
        a = int(rng.integers(0, nq))
        state = CM.commit(state, kb, vb, a, R_cap)
        committed_k.append(kb[:, :a + 1])
        committed_v.append(vb[:, :a + 1])
        ck = np.concatenate(committed_k, axis=1)
        cv = np.concatenate(committed_v, axis=1)
        assert state["L_q"] + state["R"] == ck.shape[1]
        assert state["R"] <= R_cap and state["L_q"] % G == 0
        want = Q.build_quant_cache(ck[None], cv[None], bits, G, state["R"])
        assert np.array_equal(state["records"], want["records"][0])
        assert np.array_equal(state["k_res"], want["k_res"][0]) and np.array_equal(state["v_res"], want["v_res"][0])


def test_discarded_rows_never_enter_the_cache():
    Hkv, D, G, bits, R_cap, nq = 1, 64, 32, 2, 64, 8
    state = CM.empty_state(Hkv, D, bits, G)
    for r in range(30):
        kb, vb = _rows(Hkv, nq, D, seed=200 + r)
        a = r % nq
        kb[:, a + 1:] = 1e4  # rejected drafts: a marker no committed row has
        vb[:, a + 1:] = 1e4
        state = CM.commit(state, kb, vb, a, R_cap)
        kh, vh = Q.dequantize_cache(CM.as_cache(state))
        assert np.abs(kh).max() < 1e3 and np.abs(vh).max() < 1e3


def test_worked_example_keeps_x_and_the_accepted_prefix_only():
    # block rows: x, A, B, C, D, E, F, G, H; verifier agrees up to E (a = 5)
    Hkv, D, G, bits = 1, 64, 32, 2
    labels = np.arange(9, dtype=np.float32)  # row i carries value i in every channel
    kb = np.repeat(labels[None, :, None], D, axis=2)
    vb = -kb
    state = CM.commit(CM.empty_state(Hkv, D, bits, G), kb, vb, 5, 128)
    assert state["R"] == 6 and state["L_q"] == 0
    assert list(state["k_res"][0, :, 0]) == [0, 1, 2, 3, 4, 5]


def test_one_record_per_commit_and_refusals():
    Hkv, D, G, bits, R_cap = 1, 64, 32, 2, 32
    state = CM.empty_state(Hkv, D, bits, G)
    kb, vb = _rows(Hkv, 32, D, seed=5)
    state = CM.commit(state, kb, vb, 31, R_cap)  # 32 rows: fills the residual exactly
    assert (state["L_q"], state["R"]) == (0, 32)
    state = CM.commit(state, kb, vb, 0, R_cap)  # one more: the oldest 32 become a record
    assert (state["L_q"], state["R"]) == (32, 1)
    with pytest.raises(ValueError):
        CM.commit(state, kb, vb, 32, R_cap)  # accepted length outside the block


def test_draft_attention_on_the_maintained_cache_equals_the_cache_built_at_once():
    Hkv, D, G, bits, R_cap, nq, g = 2, 64, 32, 2, 48, 16, 4
    state = CM.empty_state(Hkv, D, bits, G)
    ks, vs = [], []
    rng = np.random.default_rng(3)
    for r in range(20):
        kb, vb = _rows(Hkv, nq, D, seed=300 + r)
        a = int(rng.integers(0, nq))
        state = CM.commit(state, kb, vb, a, R_cap)
        ks.append(kb[:, :a + 1])
        vs.append(vb[:, :a + 1])
    q = synth.normal((1, Hkv * g, D), seed=9).float().numpy()
    got = A.draft_attention_quant(q, CM.as_cache(state))
    want = A.draft_attention_quant(q, Q.build_quant_cache(np.concatenate(ks, 1)[None], np.concatenate(vs, 1)[None],
                                                          bits, G, state["R"]))
    assert np.array_equal(got, want)
