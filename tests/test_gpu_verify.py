"""Parity of the tcgen05 block-verification attention kernel with the oracle."""

import numpy as np
import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import attention as A
from tests.vcutil import ATTN_TOL, np32, row_rel_err

pytestmark = pytest.mark.gpu
dev = "cuda"
LSE_TOL = 2e-3  # absolute, natural-log units


def run_verify(q, k, v, nq, sm_scale=0.0, with_lse=True):
    B, Hkv, T, D = k.shape
    Hq = q.shape[2]
    sh = vc.shape(B, Hq, Hkv, D, sm_scale)
    ws = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq))
    out = torch.full((B, nq, Hq, D), float("nan"), device=dev)
    lse = torch.full((B, nq, Hq), float("nan"), device=dev) if with_lse else None
    vc.vc_verify_attn(sh, q, k, v, T, nq, out, lse, ws)
    torch.cuda.synchronize()
    return out, lse, ws


def case(B, nq, Hq, Hkv, D, T, seed, sm_scale=0.0):
    k, v = synth.kv_full(B, Hkv, T, D, seed=seed)
    q = synth.normal((B, nq, Hq, D), seed=seed + 1)
    out, lse, _ = run_verify(q.to(dev), k.to(dev), v.to(dev), nq, sm_scale)
    wo, wl = A.verify_attention(np32(q), np32(k), np32(v), sm_scale or None)
    return np32(out), np32(lse), wo, wl


def test_tiny_single_layer_eight_rows():
    """B=1, Hq=4, Hkv=2, D=64, T=512, 8 verification rows."""
    o, l, wo, wl = case(1, 8, 4, 2, 64, 512, seed=1)
    assert row_rel_err(o, wo) <= ATTN_TOL
    assert np.abs(l - wl).max() <= LSE_TOL


@pytest.mark.parametrize("B,nq,Hq,Hkv,D,T", [
    (2, 31, 32, 8, 128, 2000),   # Llama-style GQA, K = 30 drafts + 1
    (1, 31, 40, 8, 128, 3001),   # g = 5: two row tiles in one block (8 units)
    (1, 31, 64, 8, 128, 1500),   # g = 8: two row tiles in one block
    (3, 31, 64, 8, 128, 700),    # g = 8, 24 units: one block per row tile
    (2, 31, 16, 2, 64, 900),     # g = 8, D = 64, two row tiles in one block
    (1, 1, 4, 4, 128, 100),      # one row, g = 1
    (1, 32, 4, 1, 64, 32),       # T == nq: the block is the whole cache
    (1, 31, 4, 1, 128, 96),      # one full tile plus a ragged tail
    (3, 8, 6, 3, 64, 777),
    (1, 31, 32, 8, 128, 32768),  # many chunks per head
])
def test_shapes_row_tiles_and_tails(B, nq, Hq, Hkv, D, T):
    o, l, wo, wl = case(B, nq, Hq, Hkv, D, T, seed=T + Hq)
    assert row_rel_err(o, wo) <= ATTN_TOL
    assert np.abs(l - wl).max() <= LSE_TOL


def test_explicit_scale_and_no_lse():
    B, nq, Hq, Hkv, D, T = 1, 16, 8, 2, 128, 1000
    k, v = synth.kv_full(B, Hkv, T, D, seed=3)
    q = synth.normal((B, nq, Hq, D), seed=4)
    out, _, _ = run_verify(q.to(dev), k.to(dev), v.to(dev), nq, 0.25, with_lse=False)
    wo, _ = A.verify_attention(np32(q), np32(k), np32(v), 0.25)
    assert row_rel_err(np32(out), wo) <= ATTN_TOL


def test_last_row_equals_decode_attention():
    B, nq, Hq, Hkv, D, T = 1, 5, 8, 2, 128, 3000
    k, v = synth.kv_full(B, Hkv, T, D, seed=5)
    q = synth.normal((B, nq, Hq, D), seed=6)
    out, _, _ = run_verify(q.to(dev), k.to(dev), v.to(dev), nq)
    dec = A.draft_attention_dense(np32(q)[:, -1], np32(k), np32(v))
    assert row_rel_err(np32(out)[:, -1], dec) <= ATTN_TOL


def test_equal_keys_give_mean_of_visible_values():
    B, nq, Hq, Hkv, D, T = 1, 4, 2, 1, 64, 300
    k = torch.full((B, Hkv, T, D), 0.25, dtype=torch.bfloat16)
    v = synth.normal((B, Hkv, T, D), seed=7)
    q = synth.normal((B, nq, Hq, D), seed=8)
    out, _, _ = run_verify(q.to(dev), k.to(dev), v.to(dev), nq)
    vv = np32(v)[0, 0].astype(np.float64)
    want = np.stack([np.broadcast_to(vv[:T - nq + i + 1].mean(0), (Hq, D)) for i in range(nq)])
    assert row_rel_err(np32(out)[0], want) <= ATTN_TOL


def test_repeat_calls_reuse_workspace():
    B, nq, Hq, Hkv, D, T = 2, 31, 32, 8, 128, 5000
    k, v = synth.kv_full(B, Hkv, T, D, seed=9)
    q = synth.normal((B, nq, Hq, D), seed=10).to(dev)
    kd, vd = k.to(dev), v.to(dev)
    o1, l1, ws = run_verify(q, kd, vd, nq)
    sh = vc.shape(B, Hq, Hkv, D)
    o2 = torch.empty_like(o1)
    l2 = torch.empty_like(l1)
    vc.vc_verify_attn(sh, q, kd, vd, T, nq, o2, l2, ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert vc.vc_workspace_flags(ws) == 0
