"""Parity of the quantised draft attention kernel and its dequantiser with the
oracle."""

import numpy as np
import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import attention as A
from oracle import quant as Q
from tests.vcutil import ATTN_TOL, np32, quant_cache_to_torch, row_rel_err

pytestmark = pytest.mark.gpu
dev = "cuda"


def make(B, Hkv, T, D, bits, G, R, seed):
    k, v = synth.kv_full(B, Hkv, T, D, seed=seed)
    cache = Q.build_quant_cache(np32(k), np32(v), bits, G, R)
    return k, v, cache


def run_quant(q, tc, Hq, Hkv, D, sm_scale=0.0):
    B = q.shape[0]
    sh = vc.shape(B, Hq, Hkv, D, sm_scale)
    qc = vc.quant_cache(tc)
    ws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qc))
    out = torch.full((B, Hq, D), float("nan"), device=dev)
    vc.vc_draft_attn_quant(sh, qc, q, out, ws)
    torch.cuda.synchronize()
    return np32(out), ws


@pytest.mark.parametrize("bits,G,D", [(2, 32, 64), (2, 32, 128), (2, 64, 128), (4, 64, 128), (4, 32, 64),
                                      (4, 64, 64), (2, 64, 64), (4, 32, 128)])
def test_dequant_bit_exact(bits, G, D):
    B, Hkv, T = 2, 3, 4 * G
    k, v, cache = make(B, Hkv, T, D, bits, G, 0, seed=bits * 7 + G + D)
    tc = quant_cache_to_torch(cache, dev)
    ko = torch.empty(B, Hkv, T, D, device=dev)
    vo = torch.empty_like(ko)
    vc.vc_debug_dequant(vc.shape(B, 2 * Hkv, Hkv, D), vc.quant_cache(tc), ko, vo)
    torch.cuda.synchronize()
    kc, sk, zk, vcd, sv, zv = Q.cache_parts(cache)
    kw = Q.dequantize_keys(kc, sk, zk, G)
    vw = Q.dequantize_values(vcd, sv, zv, G)
    assert np.array_equal(ko.cpu().numpy().view(np.uint32), kw.view(np.uint32))
    assert np.array_equal(vo.cpu().numpy().view(np.uint32), vw.view(np.uint32))


def test_tiny_kivi2_single_layer():
    """B=1, Hq=4, Hkv=2, D=64, T=512, 2-bit, group 32, last 32 tokens bf16."""
    B, Hq, Hkv, D, T = 1, 4, 2, 64, 512
    k, v, cache = make(B, Hkv, T, D, 2, 32, 32, seed=1)
    q = synth.normal((B, Hq, D), seed=2)
    got, _ = run_quant(q.to(dev), quant_cache_to_torch(cache, dev), Hq, Hkv, D)
    want = A.draft_attention_quant(np32(q), cache)
    assert row_rel_err(got, want) <= ATTN_TOL


@pytest.mark.parametrize("B,Hq,Hkv,D,T,bits,G,R,R_cap", [
    (2, 8, 2, 128, 32 * 20 + 128, 2, 32, 128, 128),    # Llama-style group, full residual window
    (1, 8, 1, 128, 64 * 9 + 100, 4, 64, 100, 128),     # g = 8, 4-bit, partial residual
    (1, 5, 1, 128, 32 * 37 + 3, 2, 32, 3, 16),         # g = 5
    (3, 3, 3, 64, 32 * 5, 2, 32, 0, 1),                # no residual
    (1, 4, 2, 64, 40, 2, 32, 40, 64),                  # everything in the residual
    (2, 2, 1, 128, 64 * 3 + 1, 4, 64, 1, 8),           # one residual row
    (1, 32, 8, 128, 32 * 300 + 128, 2, 32, 128, 128),  # Llama-3.1-8B heads, many chunks
    (1, 16, 2, 64, 64 * 40, 4, 64, 0, 1),
])
def test_shapes_groups_and_tails(B, Hq, Hkv, D, T, bits, G, R, R_cap):
    k, v, cache = make(B, Hkv, T, D, bits, G, R, seed=T + Hq)
    q = synth.normal((B, Hq, D), seed=T)
    got, _ = run_quant(q.to(dev), quant_cache_to_torch(cache, dev, R_cap=R_cap), Hq, Hkv, D)
    want = A.draft_attention_quant(np32(q), cache)
    assert row_rel_err(got, want) <= ATTN_TOL


def test_on_grid_data_equal_unquantised_attention():
    """Keys and values on their quantisation grid: attention over the codes
    equals plain attention over the bf16 data (oracle, dense)."""
    B, Hq, Hkv, D, G, R = 1, 8, 2, 128, 32, 32
    Lq = 32 * 12
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 4, size=(B, Hkv, Lq, D))
    codes[..., 0::G, :] = 0
    codes[..., 1::G, :] = 3
    vcodes = rng.integers(0, 4, size=(B, Hkv, Lq, D))
    vcodes[..., :, 0::G] = 0
    vcodes[..., :, 1::G] = 3
    k = np.concatenate([-1.0 + 0.5 * codes, rng.standard_normal((B, Hkv, R, D))], 2).astype(np.float32)
    v = np.concatenate([-0.75 + 0.25 * vcodes, rng.standard_normal((B, Hkv, R, D))], 2).astype(np.float32)
    k = torch.from_numpy(k).bfloat16().float().numpy()
    v = torch.from_numpy(v).bfloat16().float().numpy()
    cache = Q.build_quant_cache(k, v, 2, G, R)
    q = synth.normal((B, Hq, D), seed=3)
    got, _ = run_quant(q.to(dev), quant_cache_to_torch(cache, dev), Hq, Hkv, D)
    assert row_rel_err(got, A.draft_attention_dense(np32(q), k, v)) <= ATTN_TOL


def test_explicit_scale_and_repeat():
    B, Hq, Hkv, D, T = 2, 8, 2, 128, 32 * 50 + 128
    k, v, cache = make(B, Hkv, T, D, 2, 32, 128, seed=77)
    q = synth.normal((B, Hq, D), seed=78).to(dev)
    tc = quant_cache_to_torch(cache, dev)
    got, ws = run_quant(q, tc, Hq, Hkv, D, sm_scale=0.2)
    assert row_rel_err(got, A.draft_attention_quant(np32(q), cache, 0.2)) <= ATTN_TOL
    sh = vc.shape(B, Hq, Hkv, D, 0.2)
    out2 = torch.empty(B, Hq, D, device=dev)
    vc.vc_draft_attn_quant(sh, vc.quant_cache(tc), q, out2, ws)
    torch.cuda.synchronize()
    assert np.array_equal(np32(out2), got)


def test_static_cache_flag_changes_nothing_but_the_start():
    """VC_CACHE_STATIC lets the kernel copy its first records before the
    previous kernel of the stream ends; the results must be bit-identical to
    the same calls without it, in a chain of back-to-back calls over
    alternating caches (each call overlapping the previous one's tail)."""
    B, Hq, Hkv, D, G, R = 3, 12, 3, 128, 32, 128
    caches = []
    for s_ in range(2):
        k, v, cache = make(B, Hkv, 32 * 40 + R, D, 2, G, R, seed=300 + s_)
        caches.append(quant_cache_to_torch(cache, dev))
    qs = [synth.normal((B, Hq, D), seed=400 + i).to(dev) for i in range(6)]
    sh = vc.shape(B, Hq, Hkv, D)
    outs = {}
    for flags in (0, vc.VC_CACHE_STATIC):
        qcs = [vc.quant_cache(dict(c, flags=flags)) for c in caches]
        ws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qcs[0]))
        res = []
        for i, q in enumerate(qs):
            out = torch.empty(B, Hq, D, device=dev)
            vc.vc_draft_attn_quant(sh, qcs[i % 2], q, out, ws)
            res.append(out)
        torch.cuda.synchronize()
        assert vc.vc_workspace_flags(ws) == 0
        outs[flags] = [np32(o) for o in res]
    for a_, b_ in zip(outs[0], outs[vc.VC_CACHE_STATIC]):
        assert np.array_equal(a_, b_)
