"""Parity of the token-dropped draft attention kernel with the oracle."""

import math

import numpy as np
import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import attention as A
from tests.vcutil import ATTN_TOL, np32, row_rel_err

pytestmark = pytest.mark.gpu
dev = "cuda"


def run_sparse(q, k, v, idx, Hq, sm_scale=0.0):
    B, Hkv, T, D = k.shape
    sh = vc.shape(B, Hq, Hkv, D, sm_scale)
    sc = vc.sparse_cache(k, v, idx)
    ws = vc.workspace(vc.vc_draft_attn_sparse_workspace_size(sh, sc))
    out = torch.full((B, Hq, D), float("nan"), device=dev)
    vc.vc_draft_attn_sparse(sh, sc, q, out, ws)
    torch.cuda.synchronize()
    return out, ws


def case(B, Hq, Hkv, D, T, n_keep, seed, sm_scale=0.0):
    k, v = synth.kv_full(B, Hkv, T, D, seed=seed)
    q = synth.normal((B, Hq, D), seed=seed + 1)
    idx = synth.kept_positions(B, Hkv, T, n_keep, seed=seed + 2)
    out, ws = run_sparse(q.to(dev), k.to(dev), v.to(dev), idx.to(dev), Hq, sm_scale)
    want = A.draft_attention_sparse(np32(q), np32(k), np32(v), idx.numpy(), sm_scale or None)
    return np32(out), want, ws


def test_tiny_single_layer_keep_128_of_512():
    got, want, _ = case(1, 4, 2, 64, 512, 128, seed=10)
    assert row_rel_err(got, want) <= ATTN_TOL


@pytest.mark.parametrize("B,Hq,Hkv,D,T,n_keep", [
    (1, 4, 2, 64, 100, 1),        # a single kept row
    (2, 8, 2, 128, 300, 15),      # one ragged tile
    (2, 8, 2, 128, 300, 17),      # a full tile plus one row
    (3, 5, 1, 128, 5000, 1234),   # g = 5 (Qwen-style GQA)
    (1, 8, 1, 64, 2000, 999),     # g = 8
    (1, 3, 3, 128, 700, 700),     # g = 1, every position kept
    (1, 40, 8, 128, 20000, 5000), # many chunks per head
])
def test_shapes_tiles_and_ragged_tails(B, Hq, Hkv, D, T, n_keep):
    got, want, _ = case(B, Hq, Hkv, D, T, n_keep, seed=B * 1000 + n_keep)
    assert row_rel_err(got, want) <= ATTN_TOL


def test_explicit_scale():
    got, want, _ = case(1, 4, 2, 128, 900, 300, seed=5, sm_scale=0.3)
    assert row_rel_err(got, want) <= ATTN_TOL


def test_all_positions_equals_dense_decode():
    B, Hq, Hkv, D, T = 1, 8, 2, 128, 777
    k, v = synth.kv_full(B, Hkv, T, D, seed=21)
    q = synth.normal((B, Hq, D), seed=22)
    idx = torch.arange(T, dtype=torch.int32).expand(B, Hkv, T).contiguous()
    out, _ = run_sparse(q.to(dev), k.to(dev), v.to(dev), idx.to(dev), Hq)
    want = A.draft_attention_dense(np32(q), np32(k), np32(v))
    assert row_rel_err(np32(out), want) <= ATTN_TOL


def test_equal_keys_give_mean_of_kept_values():
    B, Hq, Hkv, D, T = 1, 4, 1, 64, 400
    k = torch.ones(B, Hkv, T, D, dtype=torch.bfloat16) * 0.5
    v = synth.normal((B, Hkv, T, D), seed=3)
    q = synth.normal((B, Hq, D), seed=4)
    idx = synth.kept_positions(B, Hkv, T, 123, seed=5)
    out, _ = run_sparse(q.to(dev), k.to(dev), v.to(dev), idx.to(dev), Hq)
    mean = np32(v)[0, 0, idx[0, 0].numpy().astype(np.int64)].astype(np.float64).mean(0)
    assert row_rel_err(np32(out)[0], np.broadcast_to(mean, (Hq, D))) <= ATTN_TOL


def test_gather_is_bit_exact():
    B, Hkv, T, D, n = 2, 3, 500, 128, 77
    k, v = synth.kv_full(B, Hkv, T, D, seed=31)
    idx = synth.kept_positions(B, Hkv, T, n, seed=32)
    sh = vc.shape(B, 3 * Hkv, Hkv, D)
    kd, vd, idd = k.to(dev), v.to(dev), idx.to(dev)
    ko = torch.empty(B, Hkv, n, D, dtype=torch.bfloat16, device=dev)
    vo = torch.empty_like(ko)
    vc.vc_debug_gather(sh, vc.sparse_cache(kd, vd, idd), ko, vo)
    torch.cuda.synchronize()
    assert torch.equal(ko.cpu(), torch.from_numpy(A.gather_rows(k.float().numpy(), idx.numpy())).bfloat16())
    assert torch.equal(vo.cpu(), torch.from_numpy(A.gather_rows(v.float().numpy(), idx.numpy())).bfloat16())


def test_out_of_range_position_is_flagged_and_skipped():
    B, Hq, Hkv, D, T = 1, 4, 1, 64, 300
    k, v = synth.kv_full(B, Hkv, T, D, seed=41)
    q = synth.normal((B, Hq, D), seed=42)
    idx = synth.kept_positions(B, Hkv, T, 50, seed=43)
    bad = idx.clone()
    bad[0, 0, 7] = T + 5
    out, ws = run_sparse(q.to(dev), k.to(dev), v.to(dev), bad.to(dev), Hq)
    assert vc.vc_workspace_flags(ws) & vc.VC_FLAG_BAD_INDEX
    keep = np.delete(idx.numpy(), 7, axis=-1)
    want = A.draft_attention_sparse(np32(q), np32(k), np32(v), keep)
    assert row_rel_err(np32(out), want) <= ATTN_TOL
    assert vc.vc_workspace_flags(ws) == 0   # reading clears the flag


def test_repeat_calls_reuse_workspace():
    B, Hq, Hkv, D, T, n = 1, 8, 2, 128, 30000, 9000
    k, v = synth.kv_full(B, Hkv, T, D, seed=51)
    q = synth.normal((B, Hq, D), seed=52).to(dev)
    idx = synth.kept_positions(B, Hkv, T, n, seed=53).to(dev)
    kd, vd = k.to(dev), v.to(dev)
    o1, ws = run_sparse(q, kd, vd, idx, Hq)
    sh = vc.shape(B, Hq, Hkv, D)
    o2 = torch.empty_like(o1)
    vc.vc_draft_attn_sparse(sh, vc.sparse_cache(kd, vd, idx), q, o2, ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
