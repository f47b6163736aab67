"""Parity at the benchmark's full sizes, in the launch configurations the
benchmark times (the work split depends only on the shapes, which are the
benchmark's): every kernel runs on the whole problem on the GPU, and the
oracle recomputes sampled (request, KV head) units one by one on the host.

Workloads: Llama-3.1-8B shapes (8 requests x 32K, KIVI-2 group 32, 128-row
residual), the 500K context, the Llama-70B shape (g = 8, 4-bit group 64),
each both on random records and with sampled units holding oracle-quantised
draws with lognormal key outliers,
the Qwen-32B shape (g = 5, 25000 kept rows of 100000), and acceptance over
the Llama vocabulary (128256 bf16 logits, 31 rows, 8 requests)."""

import numpy as np
import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import accept as ACC
from oracle import attention as A
from oracle import quant as Q
from tests.vcutil import ATTN_TOL, np32, row_rel_err

pytestmark = pytest.mark.gpu
dev = "cuda"


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _unit_cache(c, b, h, D):
    """The oracle's cache dict for one (request, KV head) of a device cache."""
    R = int(c["R"])
    return dict(bits=c["bits"], group=c["group"], L_q=c["L_q"], R=R, D=D,
                records=c["records"][b:b + 1, h:h + 1].cpu().numpy(),
                k_res=np32(c["k_res"][b:b + 1, h:h + 1, :R]), v_res=np32(c["v_res"][b:b + 1, h:h + 1, :R]))


@pytest.mark.parametrize("B,Hq,Hkv,D,T,bits,G,R,units", [
    (8, 32, 8, 128, 32768, 2, 32, 128, [0, 13, 37, 63]),    # Llama-3.1-8B, 8 x 32K
    (1, 32, 8, 128, 500000, 2, 32, 128, [0, 5]),             # 500K context
    (1, 64, 8, 128, 131072, 4, 64, 128, [2, 7]),             # Llama-70B shape, 4-bit group 64
])
def test_quant_draft_full_size_sampled(B, Hq, Hkv, D, T, bits, G, R, units):
    c = synth.random_quant_cache(B, Hkv, T - R, R, D, bits, G, seed=T + bits, device=dev)
    q = synth.normal((B, Hq, D), seed=5, device=dev)
    sh = vc.shape(B, Hq, Hkv, D)
    qc = vc.quant_cache(c)
    ws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qc))
    out = torch.full((B, Hq, D), float("nan"), device=dev)
    vc.vc_draft_attn_quant(sh, qc, q, out, ws)
    torch.cuda.synchronize()
    g = Hq // Hkv
    got = np32(out)
    assert np.isfinite(got).all()
    for u in units:
        b, h = divmod(u, Hkv)
        want = A.draft_attention_quant(np32(q[b:b + 1, h * g:(h + 1) * g]), _unit_cache(c, b, h, D))
        assert row_rel_err(got[b:b + 1, h * g:(h + 1) * g], want) <= ATTN_TOL, (b, h)
    del c, ws, out
    _free()


@pytest.mark.parametrize("B,Hq,Hkv,D,T,bits,G,R,units", [
    (8, 32, 8, 128, 32768, 2, 32, 128, [0, 13, 37, 63]),    # Llama-3.1-8B, 8 x 32K
    (1, 32, 8, 128, 500000, 2, 32, 128, [3]),                # 500K context
    (1, 64, 8, 128, 131072, 4, 64, 128, [2, 7]),             # Llama-70B shape, 4-bit group 64, g = 8
])
def test_quant_draft_full_size_realistic_units(B, Hq, Hkv, D, T, bits, G, R, units):
    """The numerically hardest regime at full context: the sampled units hold
    real draws (keys with lognormal per-channel outliers, values N(0, 1))
    quantised by the oracle, so scores span the outlier channels' range and
    the long softmax sums stress the folded-operand precision; the other
    units are random records.  Each sampled unit is compared with the oracle
    on its own quantised cache."""
    c = synth.random_quant_cache(B, Hkv, T - R, R, D, bits, G, seed=T + 7 * bits, device=dev)
    oracle_units = {}
    for u in units:
        b, h = divmod(u, Hkv)
        k, v = synth.kv_full(1, 1, T, D, seed=1000 + u)
        oc = Q.build_quant_cache(np32(k), np32(v), bits, G, R)
        c["records"][b, h].copy_(torch.from_numpy(np.ascontiguousarray(oc["records"][0, 0])).to(dev))
        c["k_res"][b, h, :R].copy_(k[0, 0, T - R:].to(dev))
        c["v_res"][b, h, :R].copy_(v[0, 0, T - R:].to(dev))
        oracle_units[u] = oc
        del k, v
    q = synth.normal((B, Hq, D), seed=6, device=dev)
    sh = vc.shape(B, Hq, Hkv, D)
    qc = vc.quant_cache(c)
    ws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qc))
    out = torch.full((B, Hq, D), float("nan"), device=dev)
    vc.vc_draft_attn_quant(sh, qc, q, out, ws)
    torch.cuda.synchronize()
    assert vc.vc_workspace_flags(ws) == 0
    g = Hq // Hkv
    got = np32(out)
    assert np.isfinite(got).all()
    for u in units:
        b, h = divmod(u, Hkv)
        want = A.draft_attention_quant(np32(q[b:b + 1, h * g:(h + 1) * g]), oracle_units[u])
        assert row_rel_err(got[b:b + 1, h * g:(h + 1) * g], want) <= ATTN_TOL, (b, h)
    del c, ws, out
    _free()


def test_sparse_draft_full_size_sampled():
    """Qwen-32B shape: 25000 kept rows of a 100000-row store per head."""
    B, Hq, Hkv, D, T, nk = 1, 40, 8, 128, 100000, 25000
    k, v = synth.kv_full(B, Hkv, T, D, seed=31, device=dev)
    idx = synth.kept_positions(B, Hkv, T, nk, seed=32, device=dev)
    q = synth.normal((B, Hq, D), seed=33, device=dev)
    sh = vc.shape(B, Hq, Hkv, D)
    sc = vc.sparse_cache(k, v, idx)
    ws = vc.workspace(vc.vc_draft_attn_sparse_workspace_size(sh, sc))
    out = torch.full((B, Hq, D), float("nan"), device=dev)
    vc.vc_draft_attn_sparse(sh, sc, q, out, ws)
    torch.cuda.synchronize()
    g = Hq // Hkv
    got = np32(out)
    for h in (0, 3, 7):
        want = A.draft_attention_sparse(np32(q[:, h * g:(h + 1) * g]), np32(k[:, h:h + 1]), np32(v[:, h:h + 1]),
                                        idx[:, h:h + 1].cpu().numpy())
        assert row_rel_err(got[:, h * g:(h + 1) * g], want) <= ATTN_TOL, h
    del k, v, ws, out
    _free()


@pytest.mark.parametrize("B,Hq,Hkv,D,T,units", [
    (8, 32, 8, 128, 32768, [0, 29, 63]),   # Llama-3.1-8B, 8 x 32K, nq = 31
    (1, 32, 8, 128, 500000, [6]),          # 500K context
    (1, 40, 8, 128, 100000, [1]),          # Qwen-32B shape (g = 5: two row tiles)
])
def test_verify_full_size_sampled(B, Hq, Hkv, D, T, units):
    nq = 31
    k, v = synth.kv_full(B, Hkv, T, D, seed=T + 3, device=dev)
    q = synth.normal((B, nq, Hq, D), seed=T + 4, device=dev)
    sh = vc.shape(B, Hq, Hkv, D)
    ws = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq))
    out = torch.full((B, nq, Hq, D), float("nan"), device=dev)
    lse = torch.full((B, nq, Hq), float("nan"), device=dev)
    vc.vc_verify_attn(sh, q, k, v, T, nq, out, lse, ws)
    torch.cuda.synchronize()
    g = Hq // Hkv
    got, got_lse = np32(out), np32(lse)
    for u in units:
        b, h = divmod(u, Hkv)
        # float64 once per unit, so the oracle's per-row calls do not convert again
        k64 = np32(k[b:b + 1, h:h + 1]).astype(np.float64)
        v64 = np32(v[b:b + 1, h:h + 1]).astype(np.float64)
        want, want_lse = A.verify_attention(np32(q[b:b + 1, :, h * g:(h + 1) * g]), k64, v64)
        del k64, v64
        assert row_rel_err(got[b:b + 1, :, h * g:(h + 1) * g], want) <= ATTN_TOL, (b, h)
        assert np.abs(got_lse[b:b + 1, :, h * g:(h + 1) * g] - want_lse).max() <= ATTN_TOL, (b, h)
    del k, v, ws, out
    _free()


def test_accept_full_size_every_row():
    """Llama vocabulary, bf16 logits, 8 requests x 31 rows: every target,
    accepted length and correction bit-exact against the oracle."""
    B, K, V = 8, 30, 128256
    draft = synth.tokens((B, K), V, seed=41)
    lens = synth.geometric_accept_lengths(B, K, 0.2, seed=41)
    logits = synth.planted_logits(B, K, V, draft, lens, seed=42, dtype=torch.bfloat16)
    ws = vc.workspace(vc.vc_accept_workspace_size(B, K, V))
    tgt = torch.empty(B, K + 1, dtype=torch.int32, device=dev)
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    cor = torch.empty(B, dtype=torch.int32, device=dev)
    vc.vc_accept(logits.to(dev), B, K, V, draft.to(dev), tgt, acc, cor, ws)
    torch.cuda.synchronize()
    t, a, c = ACC.accept(logits.float().numpy(), draft.numpy())
    assert np.array_equal(tgt.cpu().numpy(), t)
    assert np.array_equal(acc.cpu().numpy(), a)
    assert np.array_equal(cor.cpu().numpy(), c)
    assert acc.cpu().tolist() == lens


def test_streamed_verify_full_layer_bit_identical():
    """One Qwen-32B-shaped layer (409.6 MB of K and V) streamed from pinned
    host memory gives bit-identical results to the resident call, and one
    streamed (request, KV head) unit of the second layer matches the oracle."""
    B, Hq, Hkv, D, T, nq, NL = 1, 40, 8, 128, 100000, 31, 2
    kv = [synth.kv_full(B, Hkv, T, D, seed=60 + l) for l in range(NL)]
    hk = [k.pin_memory() for k, _ in kv]
    hv = [v.pin_memory() for _, v in kv]
    q = synth.normal((NL, B, nq, Hq, D), seed=62, device=dev)
    sh = vc.shape(B, Hq, Hkv, D)
    ws = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq))
    resident = []
    for l in range(NL):
        o = torch.empty(B, nq, Hq, D, device=dev)
        vc.vc_verify_attn(sh, q[l], kv[l][0].to(dev), kv[l][1].to(dev), T, nq, o, None, ws)
        resident.append(o)
    torch.cuda.synchronize()
    stage_k = [torch.empty_like(hk[0], device=dev) for _ in range(2)]
    stage_v = [torch.empty_like(hv[0], device=dev) for _ in range(2)]
    copy, comp = torch.cuda.Stream(), torch.cuda.current_stream()
    ks = vc.KvStream(hk, hv, stage_k, stage_v, copy)
    ks.prefetch(0)
    ks.prefetch(1)
    outs = []
    for l in range(NL):
        kp, vp = ks.acquire(l, comp)
        o = torch.empty(B, nq, Hq, D, device=dev)
        vc.vc_verify_attn(sh, q[l], kp, vp, T, nq, o, None, ws, comp)
        ks.release(l, comp)
        outs.append(o)
    torch.cuda.synchronize()
    ks.close()
    for l in range(NL):
        assert torch.equal(outs[l], resident[l]), l
    g, h = Hq // Hkv, 5
    want, _ = A.verify_attention(np32(q[1][:, :, h * g:(h + 1) * g]), np32(kv[1][0][:, h:h + 1]).astype(np.float64),
                                 np32(kv[1][1][:, h:h + 1]).astype(np.float64))
    assert row_rel_err(np32(outs[1])[:, :, h * g:(h + 1) * g], want) <= ATTN_TOL
    del stage_k, stage_v, ws
    _free()
