"""The allocation-free quantised draft attention entry point.

Some callers cannot allocate device memory: their host framework's memory
pool owns all of it, or their path must never reach an allocator.
vc_draft_attn_quant_noalloc serves them with a fixed scratch array inside the
library.  These tests call it through the C ABI, twice in a row (the second
call must find the counters it needs cleared again), and compare each result
with vc_draft_attn_quant on the same inputs, within the attention tolerance
used everywhere else.  The file is collected last on purpose."""

import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import attention as A
from oracle import quant as Q
from tests.vcutil import ATTN_TOL, np32, quant_cache_to_torch, row_rel_err

pytestmark = pytest.mark.gpu
dev = "cuda"


def _inputs(seed, B=2, Hq=8, Hkv=2, D=128, T=32 * 40 + 128, R=128, bits=2, G=32):
    k, v = synth.kv_full(B, Hkv, T, D, seed=seed)
    cache = Q.build_quant_cache(np32(k), np32(v), bits, G, R)
    q = synth.normal((B, Hq, D), seed=seed + 1)
    return cache, quant_cache_to_torch(cache, dev), q.to(dev), vc.shape(B, Hq, Hkv, D)


@pytest.mark.parametrize("cfg", [dict(), dict(Hq=16, T=64 * 24 + 100, R=100, bits=4, G=64)],
                         ids=["2bit-g32-gqa4", "4bit-g64-gqa8"])
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row(cfg):
    for seed in (101, 202):
        cache, tc, q, sh = _inputs(seed, **cfg)
        qc = vc.quant_cache(tc)
        ws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qc))
        ref = torch.empty(q.shape, device=dev)
        vc.vc_draft_attn_quant(sh, qc, q, ref, ws)
        got = torch.full(q.shape, float("nan"), device=dev)
        vc.vc_draft_attn_quant_noalloc(sh, qc, q, got)
        torch.cuda.synchronize()
        assert row_rel_err(np32(got), np32(ref)) <= ATTN_TOL
        assert row_rel_err(np32(got), A.draft_attention_quant(np32(q), cache)) <= ATTN_TOL
    # no bounded wait gave up in these calls
    assert vc.vc_draft_attn_quant_noalloc_flags() == 0


def test_noalloc_calls_allocate_nothing():
    cache, tc, q, sh = _inputs(303)
    qc = vc.quant_cache(tc)
    out = torch.empty(q.shape, device=dev)
    vc.vc_draft_attn_quant_noalloc(sh, qc, q, out)  # first call: looks up the scratch array
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    reserved0 = torch.cuda.memory_reserved()
    for _ in range(20):
        vc.vc_draft_attn_quant_noalloc(sh, qc, q, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_reserved() == reserved0


def test_noalloc_refuses_a_call_larger_than_its_scratch():
    # 1600 (request, head) pairs need more split-K scratch than the fixed array
    B, Hq, Hkv, D, Lq = 200, 64, 8, 128, 64
    rec = 2 * 32 * D * 2 // 8 + 8 * D
    tc = dict(bits=2, group=32, L_q=Lq, R=0, R_cap=1,
              records=torch.zeros(B, Hkv, Lq // 32, rec, dtype=torch.uint8, device=dev),
              k_res=torch.zeros(B, Hkv, 1, D, dtype=torch.bfloat16, device=dev),
              v_res=torch.zeros(B, Hkv, 1, D, dtype=torch.bfloat16, device=dev))
    sh = vc.shape(B, Hq, Hkv, D)
    qc = vc.quant_cache(tc)
    assert vc.vc_draft_attn_quant_workspace_size(sh, qc) > (4 << 20)
    q = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device=dev)
    out = torch.zeros(B, Hq, D, device=dev)
    with pytest.raises(vc.VcError) as e:
        vc.vc_draft_attn_quant_noalloc(sh, qc, q, out)
    assert e.value.status == vc.VC_ERR_WORKSPACE
