"""The device-side failure path: a bounded on-chip wait that runs out.

Every wait of the hot-path kernels on an mbarrier (bulk-copy and tensor-core
completions) is bounded; when the limit passes, the wait returns false after
ORing VC_FLAG_WAIT_TIMEOUT into a flag word, and the kernel skips the work
that depended on it and ends.  vc_debug_wait_timeout runs that helper on an
mbarrier nothing ever completes, with a 1 ms limit; the test checks that the
kernel returned, the flag is set, and the context is still usable: a normal
draft attention call on the same stream right after it matches the oracle.
No GPU faults, traps or hangs here: the wait ends by its own limit."""

import time

import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import attention as A
from oracle import quant as Q
from tests.vcutil import ATTN_TOL, np32, quant_cache_to_torch, row_rel_err

pytestmark = pytest.mark.gpu
dev = "cuda"


def test_bounded_wait_gives_up_sets_the_flag_and_leaves_the_context_usable():
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    result = torch.zeros(1, dtype=torch.int32, device=dev)
    t0 = time.perf_counter()
    vc.vc_debug_wait_timeout(flags, result, 1_000_000)  # 1 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(result[0]) == 2, "the wait must report that it gave up"
    assert int(flags[0]) & vc.VC_FLAG_WAIT_TIMEOUT
    assert elapsed < 5.0, f"the bounded wait took {elapsed:.1f} s"

    # the same stream keeps working: a draft attention call checked against the oracle
    B, Hq, Hkv, D, T, R = 1, 8, 2, 128, 32 * 20 + 128, 128
    k, v = synth.kv_full(B, Hkv, T, D, seed=77)
    cache = Q.build_quant_cache(np32(k), np32(v), 2, 32, R)
    q = synth.normal((B, Hq, D), seed=78)
    sh = vc.shape(B, Hq, Hkv, D)
    qc = vc.quant_cache(quant_cache_to_torch(cache, dev))
    ws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qc))
    out = torch.full((B, Hq, D), float("nan"), device=dev)
    vc.vc_draft_attn_quant(sh, qc, q.to(dev), out, ws)
    torch.cuda.synchronize()
    assert row_rel_err(np32(out), A.draft_attention_quant(np32(q), cache)) <= ATTN_TOL
    assert vc.vc_workspace_flags(ws) == 0


def test_limits_outside_the_allowed_range_are_refused_on_the_host():
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    result = torch.zeros(1, dtype=torch.int32, device=dev)
    for bad in (0, 999, 200_000_000):
        with pytest.raises(vc.VcError) as e:
            vc.vc_debug_wait_timeout(flags, result, bad)
        assert e.value.status == vc.VC_ERR_INVALID_ARG


@pytest.mark.parametrize("B,Hq,Hkv,T,skip", [
    (2, 32, 8, 2000, 2),   # one row tile per block; the tile loop's wait gives up
    (2, 32, 8, 2000, 0),   # the first S's wait gives up, before the tile loop
    (1, 64, 8, 8000, 3),   # g = 8: two row tiles (two softmax warpgroups) in one block
])
def test_verify_kernel_abort_path_ends_the_call_and_leaves_the_context_usable(B, Hq, Hkv, T, skip):
    """The verification kernel's own failure path: every block's K tile
    `skip` is never requested, and the tile loop's waits give up after 20 ms.
    The wait on it raises VC_FLAG_WAIT_TIMEOUT and the block's abort flag,
    the other warps' waits give up, the block drains, releases its tensor
    memory and returns.  Then normal calls on the same stream (one of them on
    the same workspace) match the oracle."""
    D, nq = 128, 31
    g = Hq // Hkv
    k, v = synth.kv_full(B, Hkv, T, D, seed=T + 1)
    q = synth.normal((B, nq, Hq, D), seed=T + 2)
    kd, vd, qd = k.to(dev), v.to(dev), q.to(dev)
    sh = vc.shape(B, Hq, Hkv, D)
    ws = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq))
    out = torch.empty(B, nq, Hq, D, device=dev)
    lse = torch.empty(B, nq, Hq, device=dev)
    t0 = time.perf_counter()
    vc.vc_debug_verify_abort(sh, qd, kd, vd, T, nq, out, lse, ws, skip, 20_000_000)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert vc.vc_workspace_flags(ws) & vc.VC_FLAG_WAIT_TIMEOUT
    assert elapsed < 5.0, f"the aborted call took {elapsed:.1f} s"
    want, want_lse = A.verify_attention(np32(q), np32(k), np32(v))
    ws2 = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq))
    for w in (ws2, ws):  # a fresh workspace, then the one the aborted call used
        out.fill_(float("nan"))
        vc.vc_verify_attn(sh, qd, kd, vd, T, nq, out, lse, w)
        torch.cuda.synchronize()
        assert row_rel_err(np32(out), want) <= ATTN_TOL
    assert vc.vc_workspace_flags(ws2) == 0
