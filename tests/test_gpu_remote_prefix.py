"""Remote prefix caching on the GPU: bandwidth-limited links (vc_link) and the
scheduler's fetch phase (vc_sched_set_links / vc_sched_set_fetch).

A paced link must deliver the bytes intact and no faster than its rate.  A
scheduled run whose requests' compressed caches start as zeros on the device
and arrive over the remote link must reproduce the direct calls on the real
caches (so every draft ran after its fetch), with the planted acceptance,
under both policies; its fetch and streaming times must respect the two
link rates."""

import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import quant as Q
from tests.vcutil import np32, quant_cache_to_torch

pytestmark = pytest.mark.gpu
dev = "cuda"


@pytest.mark.parametrize("gbps,nbytes,chunk", [(2.0, 48 << 20, 4 << 20), (1.2, 12 << 20, 1 << 20),
                                               (40.0, 256 << 20, 0)])
def test_paced_link_delivers_intact_at_its_rate(gbps, nbytes, chunk):
    src = torch.randint(0, 255, (nbytes,), dtype=torch.uint8).pin_memory()
    dst = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream()
    link = vc.Link(stream, gbps, chunk)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    link.copy(dst, src)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    want = nbytes / (gbps * 1e9) * 1e3
    assert ms >= 0.95 * want, (ms, want)
    assert ms <= 1.3 * want + 2.0, (ms, want)
    assert torch.equal(dst.cpu(), src)
    assert link.flags() == 0
    link.close()


def test_unpaced_link_is_a_plain_copy():
    src = torch.arange(1 << 20, dtype=torch.int32).pin_memory()
    dst = torch.zeros(1 << 20, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream()
    link = vc.Link(stream, 0.0)
    link.copy(dst, src)
    torch.cuda.synchronize()
    assert torch.equal(dst.cpu(), src)
    link.close()


def _request(i, NL, K, B, Hq, Hkv, D, T, R, V, stream):
    """A quantised-draft request whose draft caches live in pinned host memory
    and start as zeros on the device (they arrive by the fetch)."""
    nq = K + 1
    sh = vc.shape(B, Hq, Hkv, D)
    kv = [synth.kv_full(B, Hkv, T, D, seed=300 * i + l) for l in range(NL)]
    host_caches = [quant_cache_to_torch(Q.build_quant_cache(np32(k), np32(v), 2, 32, R), "cpu") for k, v in kv]
    fetch_src, fetch_dst, dev_caches = [], [], []
    for hc in host_caches:
        dc = dict(hc)
        for key in ("records", "k_res", "v_res"):
            h = hc[key].contiguous().pin_memory()
            d = torch.zeros_like(h, device=dev)
            fetch_src.append(h)
            fetch_dst.append(d)
            dc[key] = d
        dev_caches.append(dc)
    caches = [vc.quant_cache(t) for t in dev_caches]
    dws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, caches[0]))
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
    req = vc.make_sched_request(sh, vc.VC_DRAFT_QUANT, caches, q_draft, out["d"], dws, hk, hv, st_k, st_v, q_ver,
                                out["v"], vws, T, nq, logits, V, toks.to(dev), out["t"], out["a"], out["c"], aws,
                                stream)
    ref = dict(sh=sh, caches=caches, dev_caches=dev_caches, host_caches=host_caches, q_draft=q_draft, lens=lens,
               fetch_src=fetch_src, fetch_dst=fetch_dst, kv_bytes=2 * NL * hk[0].numel() * 2)
    return req, out, ref


@pytest.mark.parametrize("policy", [vc.VC_SCHED_LOCKSTEP, vc.VC_SCHED_STAGGER])
def test_fetched_caches_reproduce_direct_calls(policy):
    NL, K, B, Hq, Hkv, D, T, R, V = 3, 4, 2, 8, 2, 128, 32 * 60 + 64, 64, 5000
    remote_gbps, local_gbps = 2.0, 20.0
    streams = [torch.cuda.Stream() for _ in range(3)]
    built = [_request(i, NL, K, B, Hq, Hkv, D, T, R, V, streams[i]) for i in range(3)]
    copy, remote = torch.cuda.Stream(), torch.cuda.Stream()
    s = vc.Sched([b[0] for b in built], NL, K, policy, copy, timeout_ms=120000)
    s.set_links(remote, remote_gbps, local_gbps, chunk_bytes=1 << 20)
    for i, (_, _, ref) in enumerate(built):
        s.set_fetch(i, ref["fetch_src"], ref["fetch_dst"])
    stats = s.run_rounds(2)
    torch.cuda.synchronize()
    s.close()
    fetch_bytes = sum(t.numel() * t.element_size() for _, _, ref in built for t in ref["fetch_src"])
    stream_bytes = 2 * sum(ref["kv_bytes"] for _, _, ref in built)  # two rounds
    assert stats["fetch_ms"] >= 0.95 * fetch_bytes / (remote_gbps * 1e9) * 1e3
    assert stats["elapsed_ms"] >= 0.95 * fetch_bytes / (remote_gbps * 1e9) * 1e3
    assert stats["link_busy_ms"] >= 0.95 * stream_bytes / (local_gbps * 1e9) * 1e3
    # the last request's first draft starts only after every fetch (device time)
    assert stats["first_draft_ms"] >= 0.95 * fetch_bytes / (remote_gbps * 1e9) * 1e3
    for req, out, ref in built:
        assert out["a"].cpu().tolist() == ref["lens"]
        for hc, dc in zip(ref["host_caches"], ref["dev_caches"]):
            for key in ("records", "k_res", "v_res"):
                assert torch.equal(dc[key].cpu(), hc[key])
        sh = ref["sh"]
        d = torch.empty_like(out["d"])
        ws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, ref["caches"][-1]))
        vc.vc_draft_attn_quant(sh, ref["caches"][-1], ref["q_draft"][K - 1, NL - 1], d, ws)
        torch.cuda.synchronize()
        assert torch.equal(d, out["d"])
