"""The C boundary's documented error behaviour, on the CPU: invalid shapes,
sizes, null or misaligned pointers return VC_ERR_INVALID_ARG with a message
naming the entry point, from host-side checks that run before any CUDA call
or launch (include/vc.h, "Conventions shared by every entry point").

The pointers below are fake device addresses: the checks only look at their
value (null, 16-byte alignment), and every case fails a check, so nothing is
dereferenced and no CUDA call is reached."""

import ctypes

import pytest

from lossless_draft_verify_vc_b200 import vc

A = 0x100000  # aligned fake device address
M = 0x100008  # 8 bytes off a 16-byte boundary
INVALID = -1
WS = 1 << 40


@pytest.fixture(scope="module")
def L():
    return vc.lib()


def _expect_invalid(L, status, who):
    assert status == INVALID, status
    msg = L.vc_last_error().decode()
    assert who in msg, msg


# ------------------------------------------------------------------ verify
@pytest.mark.parametrize("B,Hq,Hkv,D,T,nq,q,k", [
    (1, 4, 1, 128, 100, 0, A, A),        # nq < 1
    (1, 4, 1, 128, 100, 33, A, A),       # nq > 32
    (1, 4, 1, 128, 10, 31, A, A),        # T < nq
    (1, 4, 1, 128, 1 << 31, 31, A, A),   # T >= 2^31
    (1, 4, 1, 96, 100, 31, A, A),        # head dim
    (1, 6, 4, 128, 100, 31, A, A),       # Hq not a multiple of Hkv
    (1, 16, 1, 128, 100, 31, A, A),      # g > 8
    (70000, 1, 1, 128, 100, 31, A, A),   # B * Hkv > 65535
    (1, 4, 1, 128, 100, 31, 0, A),       # null q
    (1, 4, 1, 128, 100, 31, A, M),       # misaligned k
])
def test_verify_rejects(L, B, Hq, Hkv, D, T, nq, q, k):
    sh = vc.shape(B, Hq, Hkv, D)
    st = L.vc_verify_attn(ctypes.byref(sh), q, k, A, T, nq, A, 0, A, WS, 0)
    _expect_invalid(L, st, "vc_verify_attn")


def test_verify_workspace_size_is_zero_for_invalid_shapes(L):
    assert L.vc_verify_attn_workspace_size(ctypes.byref(vc.shape(1, 4, 1, 96)), 100, 31) == 0
    assert L.vc_verify_attn_workspace_size(ctypes.byref(vc.shape(1, 4, 1, 128)), 100, 40) == 0


# ------------------------------------------------------------ quantised draft
def _qc(**kw):
    f = dict(records=A, k_res=A, v_res=A, bits=2, group=32, L_q=1024, R=16, R_cap=32)
    f.update(kw)
    return vc.vc_quant_cache(f["records"], f["k_res"], f["v_res"], f["bits"], f["group"], f["L_q"], f["R"],
                             f["R_cap"])


@pytest.mark.parametrize("shape,cache,q,out", [
    ((1, 4, 1, 128), dict(bits=3), A, A),
    ((1, 4, 1, 128), dict(group=48), A, A),
    ((1, 4, 1, 128), dict(L_q=1000), A, A),            # not whole groups
    ((1, 4, 1, 128), dict(R=40), A, A),                # R > R_cap
    ((1, 4, 1, 128), dict(L_q=0, R=0), A, A),          # no token at all
    ((1, 4, 1, 128), dict(records=0), A, A),
    ((1, 4, 1, 128), dict(records=M), A, A),
    ((1, 4, 1, 128), dict(v_res=0), A, A),
    ((1, 4, 1, 96), dict(), A, A),
    ((1, 4, 1, 128), dict(), 0, A),                    # null q
    ((1, 4, 1, 128), dict(), A, M),                    # misaligned out
])
def test_quant_draft_rejects(L, shape, cache, q, out):
    sh = vc.shape(*shape)
    qc = _qc(**cache)
    st = L.vc_draft_attn_quant(ctypes.byref(sh), ctypes.byref(qc), q, out, A, WS, 0)
    _expect_invalid(L, st, "vc_draft_attn_quant")


def test_quant_noalloc_rejects_before_touching_its_scratch(L):
    sh = vc.shape(1, 4, 1, 128)
    st = L.vc_draft_attn_quant_noalloc(ctypes.byref(sh), ctypes.byref(_qc(bits=5)), A, A, 0)
    _expect_invalid(L, st, "vc_draft_attn_quant_noalloc")


# -------------------------------------------------------- token-dropped draft
@pytest.mark.parametrize("k,T_store,idx,n_keep,q", [
    (A, 100, A, 0, A),       # n_keep < 1
    (A, 0, A, 10, A),        # empty store
    (A, 100, 0, 10, A),      # null positions
    (M, 100, A, 10, A),      # misaligned K store
    (A, 100, A, 10, 0),      # null q
])
def test_sparse_draft_rejects(L, k, T_store, idx, n_keep, q):
    sh = vc.shape(1, 4, 1, 128)
    sc = vc.vc_sparse_cache(k, A, T_store, idx, n_keep)
    st = L.vc_draft_attn_sparse(ctypes.byref(sh), ctypes.byref(sc), q, A, A, WS, 0)
    _expect_invalid(L, st, "vc_draft_attn_sparse")


# ----------------------------------------------------------------- acceptance
@pytest.mark.parametrize("logits,dtype,B,K,V,target", [
    (A, vc.VC_BF16, 0, 30, 1000, A),      # B < 1
    (A, vc.VC_BF16, 1, 65, 1000, A),      # K > 64
    (A, vc.VC_BF16, 1, 30, 0, A),         # V < 1
    (A, 7, 1, 30, 1000, A),               # dtype
    (A, vc.VC_BF16, 1, 30, 1000, 0),      # null target
    (M, vc.VC_BF16, 1, 30, 1000, A),      # misaligned logits
    (A, vc.VC_BF16, 3000, 30, 1000, A),   # more than 65535 logit rows
])
def test_accept_rejects(L, logits, dtype, B, K, V, target):
    st = L.vc_accept(logits, dtype, B, K, V, A, target, A, A, A, WS, 0)
    _expect_invalid(L, st, "vc_accept")


# ------------------------------------------------------ host -> HBM streaming
def _ptrs(*xs):
    arr = (ctypes.c_void_p * len(xs))(*xs)
    return ctypes.cast(arr, ctypes.c_void_p), arr


@pytest.mark.parametrize("n_layers,nbytes,host_k,dev_k0", [
    (0, 4096, (A, A), A),      # no layer
    (2, 0, (A, A), A),         # empty layer
    (2, 4096, (A, 0), A),      # null host pointer of layer 1
    (2, 4096, (A, A), M),      # misaligned staging slot
    (2, 4096, (A, A), 0),      # null staging slot
])
def test_kvstream_create_rejects(L, n_layers, nbytes, host_k, dev_k0):
    hk, _a = _ptrs(*host_k)
    hv, _b = _ptrs(A, A)
    dk, _c = _ptrs(dev_k0, A)
    dv, _d = _ptrs(A, A)
    handle = ctypes.c_void_p(0)
    st = L.vc_kvstream_create(ctypes.byref(handle), n_layers, hk, hv, nbytes, dk, dv, 0)
    _expect_invalid(L, st, "vc_kvstream_create")
    assert not handle.value


def test_kvstream_calls_reject_a_null_object(L):
    k, v = ctypes.c_void_p(0), ctypes.c_void_p(0)
    _expect_invalid(L, L.vc_kvstream_prefetch(None, 0), "vc_kvstream_prefetch")
    _expect_invalid(L, L.vc_kvstream_acquire(None, 0, 0, ctypes.byref(k), ctypes.byref(v)), "vc_kvstream_acquire")
    _expect_invalid(L, L.vc_kvstream_release(None, 0, 0), "vc_kvstream_release")
    assert L.vc_kvstream_destroy(None) == 0  # destroying nothing is a no-op


# ------------------------------------------------------------------ scheduler
def _request(**kw):
    r = vc.vc_sched_request()
    r.shape = vc.shape(1, 4, 1, 128)
    r.draft_kind = vc.VC_DRAFT_QUANT
    r.T, r.nq, r.V = 256, 31, 1000
    r.kv_bytes_per_layer = 1 * 1 * 256 * 128 * 2
    for f in ("qcaches", "draft_q", "draft_out", "draft_ws", "host_k", "host_v", "verify_q", "verify_out",
              "verify_ws", "logits", "draft_tokens", "target", "accept_len", "correction", "accept_ws"):
        setattr(r, f, A)
    r.stage_k[0] = r.stage_k[1] = r.stage_v[0] = r.stage_v[1] = A
    r.draft_ws_bytes = r.verify_ws_bytes = r.accept_ws_bytes = WS
    r.logits_dtype = vc.VC_BF16
    for k, v in kw.items():
        setattr(r, k, v)
    return r


@pytest.mark.parametrize("n_req,policy,timeout_ms,req", [
    (0, vc.VC_SCHED_STAGGER, 1000, {}),                       # no request
    (1, 9, 1000, {}),                                         # unknown policy
    (1, vc.VC_SCHED_STAGGER, 0, {}),                          # no timeout
    (1, vc.VC_SCHED_STAGGER, 1000, {"qcaches": 0}),           # quantised draft without caches
    (1, vc.VC_SCHED_STAGGER, 1000, {"host_k": 0}),            # no host KV
    (1, vc.VC_SCHED_STAGGER, 1000, {"kv_bytes_per_layer": 12345}),
])
def test_sched_create_rejects(L, n_req, policy, timeout_ms, req):
    reqs = (vc.vc_sched_request * 1)(_request(**req))
    handle = ctypes.c_void_p(0)
    st = L.vc_sched_create(ctypes.byref(handle), n_req, reqs, 2, 30, policy, 0, timeout_ms)
    _expect_invalid(L, st, "vc_sched_create")
    assert not handle.value


@pytest.mark.parametrize("out,gbps,chunk", [
    (False, 1.2, 0),          # null output
    (True, -1.0, 0),          # negative rate
    (True, 2e4, 0),           # absurd rate
    (True, 1.2, 100),         # chunk below 4 KiB
    (True, 1.2, (1 << 32) + 16),  # chunk above 4 GiB
])
def test_link_create_rejects_before_allocating(L, out, gbps, chunk):
    handle = ctypes.c_void_p(0)
    st = L.vc_link_create(ctypes.byref(handle) if out else None, None, gbps, chunk)
    _expect_invalid(L, st, "vc_link_create")
    assert not handle.value


def test_link_and_remote_fetch_calls_reject_null_objects(L):
    _expect_invalid(L, L.vc_link_copy(None, A, A, 16), "vc_link_copy")
    flags = ctypes.c_uint32(0)
    _expect_invalid(L, L.vc_link_flags(None, ctypes.byref(flags)), "vc_link_flags")
    assert L.vc_link_destroy(None) == 0
    _expect_invalid(L, L.vc_sched_set_links(None, None, 1.2, 40.0, 0), "vc_sched_set_links")
    _expect_invalid(L, L.vc_sched_set_fetch(None, 0, 0, None, None, None), "vc_sched_set_fetch")


@pytest.mark.parametrize("shape,B,nq,T,wnull,x", [
    ((256, 512, 8, 2, 96), 1, 4, 100, False, A),     # head dim
    ((256, 512, 6, 4, 64), 1, 4, 100, False, A),     # Hq not a multiple of Hkv
    ((250, 512, 8, 2, 64), 1, 4, 100, False, A),     # d_model not a multiple of 8
    ((256, 512, 8, 2, 64), 1, 33, 100, False, A),    # nq > 32
    ((256, 512, 8, 2, 64), 1, 4, 3, False, A),       # T < nq
    ((256, 512, 8, 2, 64), 1, 4, 100, True, A),      # a null weight
    ((256, 512, 8, 2, 64), 1, 4, 100, False, M),     # misaligned x
])
def test_verify_layer_rejects_before_any_launch(L, shape, B, nq, T, wnull, x):
    ls = vc.layer_shape(*shape)
    lw = vc.vc_layer_weights(*([A] * 6))
    if wnull:
        lw.wo = None
    st = L.vc_verify_layer(ctypes.byref(ls), ctypes.byref(lw), B, nq, T, x, A, A, A, WS, None)
    _expect_invalid(L, st, "vc_verify_layer")


def test_wait_timeout_export_rejects_before_any_launch(L):
    # null pointers and limits outside 1 us .. 100 ms are refused on the host
    assert L.vc_debug_wait_timeout(None, 16, 1000000, None) == vc.VC_ERR_INVALID_ARG
    assert L.vc_debug_wait_timeout(16, None, 1000000, None) == vc.VC_ERR_INVALID_ARG
    assert L.vc_debug_wait_timeout(16, 16, 999, None) == vc.VC_ERR_INVALID_ARG
    assert L.vc_debug_wait_timeout(16, 16, 200000000, None) == vc.VC_ERR_INVALID_ARG


def test_compression_calls_reject_before_any_launch(L):
    import ctypes
    sh = vc.shape(1, 4, 2, 128)
    ws = 256
    ok = dict(k=16, v=16, T=160, bits=2, group=32, L_q=128, records=16, k_res=16, v_res=16, R_cap=32)

    def quant(**kw):
        a = dict(ok, **kw)
        return L.vc_quantize_cache(ctypes.byref(sh), a["k"], a["v"], a["T"], a["bits"], a["group"], a["L_q"],
                                   a["records"], a["k_res"], a["v_res"], a["R_cap"], ws, 256, None)
    for bad in (dict(bits=3), dict(group=48), dict(L_q=100), dict(L_q=200), dict(R_cap=16), dict(k=None),
                dict(records=None), dict(k_res=None), dict(k=17)):
        assert quant(**bad) == vc.VC_ERR_INVALID_ARG, bad
    assert L.vc_compress_workspace_size() >= 16
    # compaction: zero kept rows, null index list, misaligned pool
    assert L.vc_compact_kept(ctypes.byref(sh), 16, 16, 100, 16, 0, 16, 16, None, 0, None) == vc.VC_ERR_INVALID_ARG
    assert L.vc_compact_kept(ctypes.byref(sh), 16, 16, 100, None, 8, 16, 16, None, 0, None) == vc.VC_ERR_INVALID_ARG
    assert L.vc_compact_kept(ctypes.byref(sh), 16, 16, 100, 16, 8, 18, 16, None, 0, None) == vc.VC_ERR_INVALID_ARG


def test_cache_commit_rejects_before_any_launch(L):
    import ctypes
    sh = vc.shape(2, 8, 2, 128)

    def qc(**kw):
        c = vc.vc_quant_cache()
        c.records, c.k_res, c.v_res, c.lens = 16, 16, 16, 16
        c.bits, c.group, c.L_q, c.R, c.R_cap = 2, 32, 320, 0, 128
        for k, v in kw.items():
            setattr(c, k, v)
        return c

    def commit(c, nq=31, k_new=16, accept=16, ws=16):
        return L.vc_cache_commit(ctypes.byref(sh), ctypes.byref(c), k_new, 16, nq, accept, ws, 256, None)
    assert commit(qc(lens=None)) == vc.VC_ERR_INVALID_ARG      # needs per-request lengths
    assert commit(qc(), nq=33) == vc.VC_ERR_INVALID_ARG        # nq > group
    assert commit(qc(R_cap=40)) == vc.VC_ERR_INVALID_ARG       # R_cap < group + nq - 1
    assert commit(qc(L_q=100)) == vc.VC_ERR_INVALID_ARG        # capacity not a multiple of group
    assert commit(qc(bits=3)) == vc.VC_ERR_INVALID_ARG
    assert commit(qc(), k_new=None) == vc.VC_ERR_INVALID_ARG
    assert commit(qc(), accept=None) == vc.VC_ERR_INVALID_ARG
    assert commit(qc(), k_new=24) == vc.VC_ERR_INVALID_ARG     # misaligned block rows
