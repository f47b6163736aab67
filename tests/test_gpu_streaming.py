"""Host-streamed verification (vc_kvstream) and the staggering scheduler
(vc_sched) on the GPU: streamed results are bit-identical to the resident
ones, and rounds run by either policy reproduce direct calls."""

import numpy as np
import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import quant as Q
from tests.vcutil import np32, quant_cache_to_torch

pytestmark = pytest.mark.gpu
dev = "cuda"


def _verify(sh, q, k, v, T, nq, ws):
    out = torch.empty(q.shape, device=dev)
    vc.vc_verify_attn(sh, q, k, v, T, nq, out, None, ws)
    return out


def test_streamed_verification_is_bit_identical_to_resident():
    NL, B, Hq, Hkv, D, T, nq = 5, 2, 8, 2, 128, 700, 31
    kv = [synth.kv_full(B, Hkv, T, D, seed=10 + l) for l in range(NL)]
    hk = [k.pin_memory() for k, _ in kv]
    hv = [v.pin_memory() for _, v in kv]
    qs = synth.normal((NL, B, nq, Hq, D), seed=3).to(dev)
    sh = vc.shape(B, Hq, Hkv, D)
    ws = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq))
    resident = [_verify(sh, qs[l], kv[l][0].to(dev), kv[l][1].to(dev), T, nq, ws) for l in range(NL)]
    torch.cuda.synchronize()
    stage_k = [torch.empty_like(hk[0], device=dev) for _ in range(2)]
    stage_v = [torch.empty_like(hv[0], device=dev) for _ in range(2)]
    copy = torch.cuda.Stream()
    comp = torch.cuda.current_stream()
    ks = vc.KvStream(hk, hv, stage_k, stage_v, copy)
    outs = []
    ks.prefetch(0)
    ks.prefetch(1)
    for l in range(NL):
        kp, vp = ks.acquire(l, comp)
        o = torch.empty(B, nq, Hq, D, device=dev)
        vc.vc_verify_attn(sh, qs[l], kp, vp, T, nq, o, None, ws, comp)
        ks.release(l, comp)
        if l + 2 < NL:
            ks.prefetch(l + 2)
        outs.append(o)
    torch.cuda.synchronize()
    for l in range(NL):
        assert torch.equal(outs[l], resident[l]), l
    # protocol errors are refused on the host
    with pytest.raises(vc.VcError):
        ks.acquire(0, comp)           # layer 0's slot now holds layer 4
    ks2 = vc.KvStream(hk, hv, stage_k, stage_v, copy)
    ks2.prefetch(0)
    with pytest.raises(vc.VcError) as e:
        ks2.prefetch(2)               # slot 0 still holds layer 0 (not released)
    assert e.value.status == vc.VC_ERR_INVALID_ARG
    ks2.close()
    ks.close()


def _request(i, NL, K, B, Hq, Hkv, D, T, R, V, kind, stream):
    nq = K + 1
    sh = vc.shape(B, Hq, Hkv, D)
    kv = [synth.kv_full(B, Hkv, T, D, seed=100 * i + l) for l in range(NL)]
    if kind == vc.VC_DRAFT_QUANT:
        tcs = [quant_cache_to_torch(Q.build_quant_cache(np32(k), np32(v), 2, 32, R), dev) for k, v in kv]
        caches = [vc.quant_cache(t) for t in tcs]
        dws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, caches[0]))
    else:
        idx = synth.kept_positions(B, Hkv, T, T // 4, seed=7 + i).to(dev)
        dkv = [(k.to(dev), v.to(dev)) for k, v in kv]
        caches = [vc.sparse_cache(k, v, idx) for k, v in dkv]
        dws = vc.workspace(vc.vc_draft_attn_sparse_workspace_size(sh, caches[0]))
    q_draft = synth.normal((K, NL, B, Hq, D), seed=20 + i).to(dev)
    q_ver = synth.normal((NL, B, nq, Hq, D), seed=30 + i).to(dev)
    toks = synth.tokens((B, K), V, seed=40 + i)
    lens = synth.geometric_accept_lengths(B, K, 0.3, seed=40 + i)
    logits = synth.planted_logits(B, K, V, toks, lens, seed=50 + i).to(dev)
    hk = [k.pin_memory() for k, _ in kv]
    hv = [v.pin_memory() for _, v in kv]
    st_k = [torch.empty_like(hk[0], device=dev) for _ in range(2)]
    st_v = [torch.empty_like(hv[0], device=dev) for _ in range(2)]
    out = dict(d=torch.empty(B, Hq, D, device=dev), v=torch.empty(B, nq, Hq, D, device=dev),
               t=torch.empty(B, K + 1, dtype=torch.int32, device=dev), a=torch.empty(B, dtype=torch.int32, device=dev),
               c=torch.empty(B, dtype=torch.int32, device=dev))
    vws = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq))
    aws = vc.workspace(vc.vc_accept_workspace_size(B, K, V))
    req = vc.make_sched_request(sh, kind, caches, q_draft, out["d"], dws, hk, hv, st_k, st_v, q_ver, out["v"], vws,
                                T, nq, logits, V, toks.to(dev), out["t"], out["a"], out["c"], aws, stream)
    ref = dict(sh=sh, kind=kind, caches=caches, q_draft=q_draft, q_ver=q_ver, kv=kv, lens=lens, logits=logits,
               toks=toks.to(dev), T=T, nq=nq)
    return req, out, ref


@pytest.mark.parametrize("policy", [0, 1])
def test_scheduler_rounds_reproduce_direct_calls(policy):
    NL, K, B, Hq, Hkv, D, T, R, V = 3, 4, 2, 8, 2, 128, 32 * 20 + 64, 64, 5000
    streams = [torch.cuda.Stream() for _ in range(3)]
    kinds = [vc.VC_DRAFT_QUANT, vc.VC_DRAFT_QUANT, vc.VC_DRAFT_SPARSE]
    built = [_request(i, NL, K, B, Hq, Hkv, D, T, R, V, kinds[i], streams[i]) for i in range(3)]
    copy = torch.cuda.Stream()
    s = vc.Sched([b[0] for b in built], NL, K, policy, copy, timeout_ms=120000)
    stats = s.run_rounds(2)
    torch.cuda.synchronize()
    s.close()
    assert stats["rounds"] == 2 and stats["requests"] == 3
    assert stats["elapsed_ms"] > 0 and stats["link_busy_ms"] > 0
    for req, out, ref in built:
        sh = ref["sh"]
        assert out["a"].cpu().tolist() == ref["lens"]
        # the last draft call and the last verification, recomputed directly
        d = torch.empty_like(out["d"])
        if ref["kind"] == vc.VC_DRAFT_QUANT:
            ws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, ref["caches"][-1]))
            vc.vc_draft_attn_quant(sh, ref["caches"][-1], ref["q_draft"][K - 1, NL - 1], d, ws)
        else:
            ws = vc.workspace(vc.vc_draft_attn_sparse_workspace_size(sh, ref["caches"][-1]))
            vc.vc_draft_attn_sparse(sh, ref["caches"][-1], ref["q_draft"][K - 1, NL - 1], d, ws)
        vws = vc.workspace(vc.vc_verify_attn_workspace_size(sh, ref["T"], ref["nq"]))
        k, v = ref["kv"][-1]
        vo = _verify(sh, ref["q_ver"][NL - 1], k.to(dev), v.to(dev), ref["T"], ref["nq"], vws)
        torch.cuda.synchronize()
        assert torch.equal(d, out["d"])
        assert torch.equal(vo, out["v"])
