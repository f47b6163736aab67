"""Host-only tests of the staggering policy (simulated timeline, no GPU) and
of the argument checks of the streaming / scheduler entry points.

The simulated timeline treats the GPU and the host link as one-at-a-time
servers: a draft takes D of the GPU, a verification V of the link.  For n
equal requests and R rounds the two policies have closed forms:
  lock-step: every round is n drafts then n verifications -> R * n * (D + V)
  stagger  : link-bound (V >= D): D + R * n * V; GPU-bound: R * n * D + V
Remote prefix caching adds a fetch per request on a third one-at-a-time
server (the remote link), all fetches enqueued at the start in request
order; lock-step starts drafting only after every fetch, stagger as soon as
the request's own fetch is done.
"""

import ctypes
import random

import pytest

from lossless_draft_verify_vc_b200 import build as B
from lossless_draft_verify_vc_b200 import vc


@pytest.fixture(scope="module", autouse=True)
def _lib():
    B.build()
    vc.lib()


@pytest.mark.parametrize("n,R,D,V", [(2, 3, 10.0, 30.0), (4, 2, 10.0, 30.0), (3, 5, 7.0, 7.0)])
def test_link_bound_closed_forms(n, R, D, V):
    # (n - 1) * V >= D: another request's verification always covers a draft
    lock = vc.vc_sched_simulate([D] * n, [V] * n, R, vc.VC_SCHED_LOCKSTEP)
    stag = vc.vc_sched_simulate([D] * n, [V] * n, R, vc.VC_SCHED_STAGGER)
    assert lock == pytest.approx(R * n * (D + V))
    assert stag == pytest.approx(D + R * n * V)


def test_single_request_cannot_overlap_itself():
    # a request's next draft needs its own round to finish: both policies are serial
    for pol in (vc.VC_SCHED_LOCKSTEP, vc.VC_SCHED_STAGGER):
        assert vc.vc_sched_simulate([3.0], [11.0], 4, pol) == pytest.approx(4 * (3.0 + 11.0))


def test_gpu_bound_closed_form():
    # four requests, drafts twice as long as verifications
    n, R, D, V = 4, 2, 10.0, 5.0
    assert vc.vc_sched_simulate([D] * n, [V] * n, R, vc.VC_SCHED_LOCKSTEP) == pytest.approx(R * n * (D + V))
    assert vc.vc_sched_simulate([D] * n, [V] * n, R, vc.VC_SCHED_STAGGER) == pytest.approx(R * n * D + V)


def test_stagger_never_slower_than_lockstep():
    rng = random.Random(0)
    for _ in range(200):
        n = rng.randint(1, 6)
        R = rng.randint(1, 4)
        d = [rng.uniform(0.5, 20) for _ in range(n)]
        v = [rng.uniform(0.5, 20) for _ in range(n)]
        lock = vc.vc_sched_simulate(d, v, R, vc.VC_SCHED_LOCKSTEP)
        stag = vc.vc_sched_simulate(d, v, R, vc.VC_SCHED_STAGGER)
        assert stag <= lock + 1e-9
        # neither can beat the busiest resource
        assert stag >= max(R * sum(d), R * sum(v)) - 1e-9


def test_a_verification_that_never_completes_times_out():
    with pytest.raises(vc.VcError) as e:
        vc.vc_sched_simulate([1.0, 1.0], [2.0, 2.0], 2, vc.VC_SCHED_STAGGER, never_done=1, timeout_ms=1000.0)
    assert e.value.status == vc.VC_ERR_TIMEOUT
    with pytest.raises(vc.VcError) as e:
        vc.vc_sched_simulate([1.0], [2.0], 3, vc.VC_SCHED_LOCKSTEP, never_done=0, timeout_ms=50.0)
    assert e.value.status == vc.VC_ERR_TIMEOUT


def test_timeout_bounds_time_without_progress_not_the_whole_run():
    # every phase completes within 30 ms of simulated time, the run lasts far
    # longer than the 40 ms limit: it must finish
    n, R, D, V = 3, 6, 10.0, 30.0
    got = vc.vc_sched_simulate([D] * n, [V] * n, R, vc.VC_SCHED_STAGGER, timeout_ms=40.0)
    assert got == pytest.approx(D + R * n * V)
    assert got > 10 * 40.0
    got = vc.vc_sched_simulate([D] * n, [V] * n, R, vc.VC_SCHED_LOCKSTEP, timeout_ms=40.0)
    assert got == pytest.approx(R * n * (D + V))
    # the same run with one verification that stops completing fails
    with pytest.raises(vc.VcError) as e:
        vc.vc_sched_simulate([D] * n, [V] * n, R, vc.VC_SCHED_STAGGER, never_done=2, timeout_ms=40.0)
    assert e.value.status == vc.VC_ERR_TIMEOUT


def test_invalid_arguments_are_refused_before_any_device_call():
    L = vc.lib()
    h = ctypes.c_void_p()
    # scheduler: unknown policy, zero requests, bad timeout
    reqs = (vc.vc_sched_request * 1)()
    assert L.vc_sched_create(ctypes.byref(h), 1, reqs, 1, 4, 7, None, 1000) == vc.VC_ERR_INVALID_ARG
    assert L.vc_sched_create(ctypes.byref(h), 0, reqs, 1, 4, 1, None, 1000) == vc.VC_ERR_INVALID_ARG
    assert L.vc_sched_create(ctypes.byref(h), 1, reqs, 1, 4, 1, None, 0) == vc.VC_ERR_INVALID_ARG
    assert L.vc_sched_create(ctypes.byref(h), 1, reqs, 1, 4, 1, None, 1000) == vc.VC_ERR_INVALID_ARG  # no caches
    # streaming: null host pointers, zero bytes
    hk = (ctypes.c_void_p * 2)(None, None)
    dk = (ctypes.c_void_p * 2)(16, 32)
    assert L.vc_kvstream_create(ctypes.byref(h), 2, hk, hk, 1024, dk, dk, None) == vc.VC_ERR_INVALID_ARG
    hk2 = (ctypes.c_void_p * 2)(16, 32)
    assert L.vc_kvstream_create(ctypes.byref(h), 2, hk2, hk2, 0, dk, dk, None) == vc.VC_ERR_INVALID_ARG
    assert b"bytes" in L.vc_last_error() or len(L.vc_last_error()) > 0
    # attention entry points: impossible shapes
    sh = vc.shape(1, 3, 2, 128)
    qc = vc.vc_quant_cache()
    assert L.vc_draft_attn_quant(ctypes.byref(sh), ctypes.byref(qc), 16, 16, 16, 1 << 20, None) == vc.VC_ERR_INVALID_ARG
    sh2 = vc.shape(1, 4, 2, 96)
    assert L.vc_verify_attn_workspace_size(ctypes.byref(sh2), 100, 4) == 0
    assert L.vc_accept(16, 0, 1, 65, 10, 16, 16, 16, 16, 16, 1 << 20, None) == vc.VC_ERR_INVALID_ARG


def test_fetch_closed_forms_two_requests():
    # fetches 0-10 and 10-20; stagger: request 0 drafts 10-11, verifies 11-16,
    # request 1 drafts 20-21, verifies 21-26; lock-step: drafts 20-22, then
    # verifications 22-27 and 27-32
    f, d, v = [10.0, 10.0], [1.0, 1.0], [5.0, 5.0]
    assert vc.vc_sched_simulate(d, v, 1, vc.VC_SCHED_STAGGER, fetch_ms=f) == pytest.approx(26.0)
    assert vc.vc_sched_simulate(d, v, 1, vc.VC_SCHED_LOCKSTEP, fetch_ms=f) == pytest.approx(32.0)


@pytest.mark.parametrize("n,R,F,D,V", [(4, 3, 40.0, 2.0, 10.0), (3, 2, 100.0, 5.0, 20.0)])
def test_fetch_bound_closed_forms(n, R, F, D, V):
    # the remote link dominates (F >= R * (D + V)): with stagger, every request's
    # rounds run while the next fetch is on the link, so only the last
    # request's rounds extend past the fetches
    assert F >= R * (D + V)
    f, d, v = [F] * n, [D] * n, [V] * n
    assert vc.vc_sched_simulate(d, v, R, vc.VC_SCHED_STAGGER, fetch_ms=f) == pytest.approx(n * F + R * (D + V))
    assert vc.vc_sched_simulate(d, v, R, vc.VC_SCHED_LOCKSTEP, fetch_ms=f) == pytest.approx(n * F + R * n * (D + V))


def test_fetch_stagger_never_slower_and_no_fetch_changes_nothing():
    rng = random.Random(1)
    for _ in range(200):
        n = rng.randint(1, 5)
        R = rng.randint(1, 3)
        f = [rng.uniform(0.0, 40) for _ in range(n)]
        d = [rng.uniform(0.5, 20) for _ in range(n)]
        v = [rng.uniform(0.5, 20) for _ in range(n)]
        lock = vc.vc_sched_simulate(d, v, R, vc.VC_SCHED_LOCKSTEP, fetch_ms=f)
        stag = vc.vc_sched_simulate(d, v, R, vc.VC_SCHED_STAGGER, fetch_ms=f)
        assert stag <= lock + 1e-9
        # the remote link and the last request's own chain bound it from below
        assert stag >= sum(f) - 1e-9
        assert stag >= max(R * sum(d), R * sum(v)) - 1e-9
        for pol in (vc.VC_SCHED_LOCKSTEP, vc.VC_SCHED_STAGGER):
            assert vc.vc_sched_simulate(d, v, R, pol, fetch_ms=[0.0] * n) == pytest.approx(
                vc.vc_sched_simulate(d, v, R, pol))
