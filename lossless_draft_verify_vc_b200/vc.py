"""Python binding of the C ABI in include/vc.h (ctypes; argument marshalling
only -- every step of the hot path runs in the CUDA library).

Function names match the C entry points.  Tensor arguments are torch CUDA
tensors (or raw integer device pointers); their data pointers and the current
CUDA stream are passed through unchanged.  A non-VC_OK status raises VcError
with the library's message.  If ``libvc_b200.so`` is missing this module
raises on import of any entry point: there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, Structure, c_char_p, c_float, c_int, c_int32, c_int64, c_size_t, c_uint32, c_void_p

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvc_b200.so")

VC_OK = 0
VC_ERR_INVALID_ARG = -1
VC_ERR_UNSUPPORTED = -2
VC_ERR_CUDA = -3
VC_ERR_TIMEOUT = -4
VC_ERR_WORKSPACE = -5
VC_F32, VC_BF16, VC_F16 = 0, 1, 2
VC_FLAG_BAD_INDEX = 1
VC_FLAG_WAIT_TIMEOUT = 2
VC_FLAG_RANGE = 4
VC_FLAG_BAD_LENGTH = 8


class VcError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"vc status {status}: {msg}")
        self.status = status


class vc_attn_shape(Structure):
    _fields_ = [("B", c_int), ("Hq", c_int), ("Hkv", c_int), ("D", c_int), ("sm_scale", c_float)]


class vc_quant_cache(Structure):
    _fields_ = [("records", c_void_p), ("k_res", c_void_p), ("v_res", c_void_p),
                ("bits", c_int), ("group", c_int), ("L_q", c_int64), ("R", c_int), ("R_cap", c_int),
                ("lens", c_void_p), ("flags", c_int)]


class vc_sparse_cache(Structure):
    _fields_ = [("k", c_void_p), ("v", c_void_p), ("T_store", c_int64), ("idx", c_void_p), ("n_keep", c_int)]


class vc_sched_request(Structure):
    _fields_ = [("shape", vc_attn_shape), ("draft_kind", c_int), ("qcaches", c_void_p), ("scaches", c_void_p),
                ("draft_q", c_void_p), ("draft_out", c_void_p), ("draft_ws", c_void_p), ("draft_ws_bytes", c_size_t),
                ("host_k", c_void_p), ("host_v", c_void_p), ("kv_bytes_per_layer", c_size_t),
                ("stage_k", c_void_p * 2), ("stage_v", c_void_p * 2), ("verify_q", c_void_p),
                ("verify_out", c_void_p), ("verify_ws", c_void_p), ("verify_ws_bytes", c_size_t), ("T", c_int64),
                ("nq", c_int), ("logits", c_void_p), ("logits_dtype", c_int), ("V", c_int),
                ("draft_tokens", c_void_p), ("target", c_void_p), ("accept_len", c_void_p),
                ("correction", c_void_p), ("accept_ws", c_void_p), ("accept_ws_bytes", c_size_t),
                ("stream", c_void_p)]


class vc_sched_stats(Structure):
    _fields_ = [("elapsed_ms", ctypes.c_double), ("link_busy_ms", ctypes.c_double), ("draft_ms", ctypes.c_double),
                ("verify_ms", ctypes.c_double), ("rounds", c_int), ("requests", c_int),
                ("fetch_ms", ctypes.c_double), ("first_draft_ms", ctypes.c_double)]


class vc_layer_shape(Structure):
    _fields_ = [("d_model", c_int), ("d_ff", c_int), ("Hq", c_int), ("Hkv", c_int), ("D", c_int),
                ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float)]


class vc_layer_weights(Structure):
    _fields_ = [("w1", c_void_p), ("wqkv", c_void_p), ("wo", c_void_p), ("w2", c_void_p), ("wgu", c_void_p),
                ("wd", c_void_p)]


VC_DRAFT_QUANT, VC_DRAFT_SPARSE = 0, 1
VC_CACHE_STATIC = 1
VC_SCHED_LOCKSTEP, VC_SCHED_STAGGER = 0, 1

_lib = None


def lib() -> ctypes.CDLL:
    """Load libvc_b200.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with lossless_draft_verify_vc_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P = POINTER
        sigs = {
            "vc_last_error": (c_char_p, []),
            "vc_abi_version": (c_int, []),
            "vc_draft_attn_quant_workspace_size": (c_size_t, [P(vc_attn_shape), P(vc_quant_cache)]),
            "vc_draft_attn_quant": (c_int, [P(vc_attn_shape), P(vc_quant_cache), c_void_p, c_void_p, c_void_p,
                                            c_size_t, c_void_p]),
            "vc_draft_attn_quant_noalloc": (c_int, [P(vc_attn_shape), P(vc_quant_cache), c_void_p, c_void_p,
                                                    c_void_p]),
            "vc_draft_attn_sparse_workspace_size": (c_size_t, [P(vc_attn_shape), P(vc_sparse_cache)]),
            "vc_draft_attn_sparse": (c_int, [P(vc_attn_shape), P(vc_sparse_cache), c_void_p, c_void_p, c_void_p,
                                             c_size_t, c_void_p]),
            "vc_verify_attn_workspace_size": (c_size_t, [P(vc_attn_shape), c_int64, c_int]),
            "vc_verify_attn": (c_int, [P(vc_attn_shape), c_void_p, c_void_p, c_void_p, c_int64, c_int, c_void_p,
                                       c_void_p, c_void_p, c_size_t, c_void_p]),
            "vc_accept_workspace_size": (c_size_t, [c_int, c_int, c_int]),
            "vc_accept": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_size_t, c_void_p]),
            "vc_workspace_flags": (c_int, [c_void_p, c_size_t, P(c_uint32), c_void_p]),
            "vc_draft_attn_quant_noalloc_flags": (c_int, [P(c_uint32), c_void_p]),
            "vc_debug_dequant": (c_int, [P(vc_attn_shape), P(vc_quant_cache), c_void_p, c_void_p, c_void_p]),
            "vc_debug_wait_timeout": (c_int, [c_void_p, c_void_p, ctypes.c_int64, c_void_p]),
            "vc_debug_verify_abort": (c_int, [P(vc_attn_shape), c_void_p, c_void_p, c_void_p, c_int64, c_int,
                                              c_void_p, c_void_p, c_void_p, c_size_t, c_int, ctypes.c_int64,
                                              c_void_p]),
            "vc_compress_workspace_size": (c_size_t, []),
            "vc_cache_commit": (c_int, [P(vc_attn_shape), P(vc_quant_cache), c_void_p, c_void_p, c_int, c_void_p,
                                        c_void_p, c_size_t, c_void_p]),
            "vc_quantize_cache": (c_int, [P(vc_attn_shape), c_void_p, c_void_p, ctypes.c_int64, c_int, c_int,
                                          ctypes.c_int64, c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_size_t,
                                          c_void_p]),
            "vc_compact_kept": (c_int, [P(vc_attn_shape), c_void_p, c_void_p, ctypes.c_int64, c_void_p, c_int,
                                        c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
            "vc_debug_quant_partition": (c_int, [P(vc_attn_shape), P(vc_quant_cache), c_int, c_void_p, c_int,
                                                 P(c_int), P(c_int), P(c_int), P(c_int), P(c_int)]),
            "vc_kvstream_create": (c_int, [P(c_void_p), c_int, c_void_p, c_void_p, c_size_t, c_void_p, c_void_p,
                                           c_void_p]),
            "vc_kvstream_prefetch": (c_int, [c_void_p, c_int]),
            "vc_kvstream_acquire": (c_int, [c_void_p, c_int, c_void_p, P(c_void_p), P(c_void_p)]),
            "vc_kvstream_release": (c_int, [c_void_p, c_int, c_void_p]),
            "vc_kvstream_destroy": (c_int, [c_void_p]),
            "vc_sched_create": (c_int, [P(c_void_p), c_int, P(vc_sched_request), c_int, c_int, c_int, c_void_p,
                                        c_int]),
            "vc_sched_run_rounds": (c_int, [c_void_p, c_int, P(vc_sched_stats)]),
            "vc_sched_destroy": (c_int, [c_void_p]),
            "vc_sched_simulate": (c_int, [c_int, c_int, c_int, P(ctypes.c_double), P(ctypes.c_double),
                                          P(ctypes.c_double), c_int, ctypes.c_double, P(ctypes.c_double)]),
            "vc_sched_set_links": (c_int, [c_void_p, c_void_p, ctypes.c_double, ctypes.c_double, c_size_t]),
            "vc_sched_set_fetch": (c_int, [c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p]),
            "vc_link_create": (c_int, [P(c_void_p), c_void_p, ctypes.c_double, c_size_t]),
            "vc_verify_layer_workspace_size": (c_size_t, [P(vc_layer_shape), c_int, c_int, c_int64]),
            "vc_verify_layer": (c_int, [P(vc_layer_shape), P(vc_layer_weights), c_int, c_int, c_int64, c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
            "vc_link_copy": (c_int, [c_void_p, c_void_p, c_void_p, c_size_t]),
            "vc_link_flags": (c_int, [c_void_p, P(c_uint32)]),
            "vc_link_destroy": (c_int, [c_void_p]),
            "vc_debug_gather": (c_int, [P(vc_attn_shape), P(vc_sparse_cache), c_void_p, c_void_p, c_void_p,
                                        c_size_t, c_void_p]),
        }
        for name, (res, args) in sigs.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(st: int):
    if st != VC_OK:
        raise VcError(st, lib().vc_last_error().decode())


def _p(x) -> int:
    """Device pointer of a tensor (or pass an int / None through)."""
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    if not x.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return x.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def shape(B: int, Hq: int, Hkv: int, D: int, sm_scale: float = 0.0) -> vc_attn_shape:
    return vc_attn_shape(B, Hq, Hkv, D, sm_scale)


def quant_cache(t: dict) -> vc_quant_cache:
    """Descriptor of a quantised cache given as a dict of CUDA tensors with the
    keys records, k_res, v_res and ints bits, group, L_q, R, R_cap, and an
    optional int32 tensor lens [B, 2] of per-request (L_q, R) (the layout
    documented in vc.h) and optional int flags (VC_CACHE_STATIC).  The descriptor holds raw device pointers; it keeps
    references to the tensors so they stay allocated while it lives."""
    d = vc_quant_cache(_p(t["records"]), _p(t.get("k_res")), _p(t.get("v_res")),
                       int(t["bits"]), int(t["group"]), int(t["L_q"]), int(t["R"]), int(t["R_cap"]),
                       _p(t.get("lens")), int(t.get("flags", 0)))
    d._keep = dict(t)
    return d


def sparse_cache(k, v, idx) -> vc_sparse_cache:
    """Descriptor of a token-dropped cache (keeps references to its tensors)."""
    d = vc_sparse_cache(_p(k), _p(v), int(k.shape[2]), _p(idx), int(idx.shape[-1]))
    d._keep = (k, v, idx)
    return d


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled workspace of at least nbytes (16-byte aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


# ---- entry points (same names as the C ABI) ---------------------------------

def vc_abi_version() -> int:
    return lib().vc_abi_version()


def vc_draft_attn_quant_workspace_size(sh: vc_attn_shape, qc: vc_quant_cache) -> int:
    return lib().vc_draft_attn_quant_workspace_size(ctypes.byref(sh), ctypes.byref(qc))


def vc_draft_attn_quant(sh, qc, q, out, ws, stream=None):
    _check(lib().vc_draft_attn_quant(ctypes.byref(sh), ctypes.byref(qc), _p(q), _p(out), _p(ws),
                                     ws.numel() if hasattr(ws, "numel") else 1 << 62, _stream(stream)))


def vc_draft_attn_quant_noalloc(sh, qc, q, out, stream=None):
    """vc_draft_attn_quant without a workspace: the scratch is a fixed device
    array inside the library (for callers that cannot allocate device memory);
    calls sharing it must not overlap on the GPU."""
    _check(lib().vc_draft_attn_quant_noalloc(ctypes.byref(sh), ctypes.byref(qc), _p(q), _p(out), _stream(stream)))


def vc_draft_attn_sparse_workspace_size(sh, sc) -> int:
    return lib().vc_draft_attn_sparse_workspace_size(ctypes.byref(sh), ctypes.byref(sc))


def vc_draft_attn_sparse(sh, sc, q, out, ws, stream=None):
    _check(lib().vc_draft_attn_sparse(ctypes.byref(sh), ctypes.byref(sc), _p(q), _p(out), _p(ws),
                                      ws.numel() if hasattr(ws, "numel") else 1 << 62, _stream(stream)))


def vc_verify_attn_workspace_size(sh, T: int, nq: int) -> int:
    return lib().vc_verify_attn_workspace_size(ctypes.byref(sh), int(T), int(nq))


def vc_verify_attn(sh, q, k, v, T: int, nq: int, out, lse, ws, stream=None):
    _check(lib().vc_verify_attn(ctypes.byref(sh), _p(q), _p(k), _p(v), int(T), int(nq), _p(out), _p(lse), _p(ws),
                                ws.numel() if hasattr(ws, "numel") else 1 << 62, _stream(stream)))


def vc_accept_workspace_size(B: int, K: int, V: int) -> int:
    return lib().vc_accept_workspace_size(int(B), int(K), int(V))


def vc_accept(logits, B: int, K: int, V: int, draft, target, accept_len, correction, ws, stream=None):
    dtype = VC_BF16 if logits.dtype == torch.bfloat16 else VC_F32
    if logits.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("logits must be fp32 or bf16")
    _check(lib().vc_accept(_p(logits), dtype, int(B), int(K), int(V), _p(draft), _p(target), _p(accept_len),
                           _p(correction), _p(ws), ws.numel(), _stream(stream)))


def vc_workspace_flags(ws, stream=None) -> int:
    v = c_uint32(0)
    _check(lib().vc_workspace_flags(_p(ws), ws.numel(), ctypes.byref(v), _stream(stream)))
    return int(v.value)


def vc_draft_attn_quant_noalloc_flags(stream=None) -> int:
    """Flags set by vc_draft_attn_quant_noalloc calls on the current device
    since the last read (read and cleared)."""
    v = c_uint32(0)
    _check(lib().vc_draft_attn_quant_noalloc_flags(ctypes.byref(v), _stream(stream)))
    return int(v.value)


def vc_debug_dequant(sh, qc, k_out, v_out, stream=None):
    _check(lib().vc_debug_dequant(ctypes.byref(sh), ctypes.byref(qc), _p(k_out), _p(v_out), _stream(stream)))


def vc_compress_workspace_size() -> int:
    return lib().vc_compress_workspace_size()


def vc_quantize_cache(sh, k, v, T: int, bits: int, group: int, L_q: int, records, k_res, v_res, R_cap: int, ws,
                      stream=None):
    """Full bf16 K, V [B, Hkv, T, D] -> group records of the oldest L_q rows
    plus the residual rows (see include/vc.h)."""
    _check(lib().vc_quantize_cache(ctypes.byref(sh), _p(k), _p(v), int(T), int(bits), int(group), int(L_q),
                                   _p(records), _p(k_res), _p(v_res), int(R_cap), _p(ws), ws.numel(),
                                   _stream(stream)))


def vc_cache_commit(sh, qc, k_new, v_new, nq: int, accept_len, ws, stream=None):
    """Commit one round's accepted rows into a device-maintained quantised
    cache (qc.lens required; see include/vc.h)."""
    _check(lib().vc_cache_commit(ctypes.byref(sh), ctypes.byref(qc), _p(k_new), _p(v_new), int(nq), _p(accept_len),
                                 _p(ws), ws.numel(), _stream(stream)))


def vc_compact_kept(sh, k, v, T_store: int, idx, n_keep: int, k_out, v_out, ws=None, stream=None):
    """Kept rows of k, v into a pool [B, Hkv, n_keep, D] (see include/vc.h)."""
    _check(lib().vc_compact_kept(ctypes.byref(sh), _p(k), _p(v), int(T_store), _p(idx), int(n_keep), _p(k_out),
                                 _p(v_out), _p(ws), ws.numel() if ws is not None else 0, _stream(stream)))


def vc_debug_wait_timeout(flags, result, limit_ns: int, stream=None):
    """Bounded on-chip wait on an mbarrier that never completes (device
    uint32 flags and result; see include/vc.h)."""
    _check(lib().vc_debug_wait_timeout(_p(flags), _p(result), int(limit_ns), _stream(stream)))


def vc_debug_verify_abort(sh, q, k, v, T: int, nq: int, out, lse, ws, skip_tile: int, limit_ns: int,
                          stream=None):
    """vc_verify_attn with K tile skip_tile of every block never requested
    and the tile loop's waits giving up after limit_ns (see include/vc.h)."""
    _check(lib().vc_debug_verify_abort(ctypes.byref(sh), _p(q), _p(k), _p(v), int(T), int(nq), _p(out), _p(lse),
                                       _p(ws), ws.numel() if hasattr(ws, "numel") else 1 << 62, int(skip_tile),
                                       int(limit_ns), _stream(stream)))


def vc_debug_quant_partition(sh, qc, target_blocks: int) -> dict:
    """How vc_draft_attn_quant cuts a call into at most target_blocks blocks
    (no GPU needed): per block its units and unit-local residual tiles and
    quantised stages, plus the per-unit counts."""
    L = lib()
    nb, bpu, npu, sr, sq = (ctypes.c_int() for _ in range(5))

    def call(rows, n):
        _check(L.vc_debug_quant_partition(ctypes.byref(sh), ctypes.byref(qc), int(target_blocks), rows, n,
                                          ctypes.byref(nb), ctypes.byref(bpu), ctypes.byref(npu), ctypes.byref(sr),
                                          ctypes.byref(sq)))

    call(None, 0)
    rows = (ctypes.c_int32 * (6 * nb.value))()
    call(rows, nb.value)
    blocks = [tuple(rows[6 * k:6 * k + 6]) for k in range(nb.value)]
    return dict(blocks=blocks, n_blocks=nb.value, blocks_per_unit=bpu.value, partials_per_unit=npu.value,
                residual_tiles=sr.value, quant_stages=sq.value)


def vc_debug_gather(sh, sc, k_out, v_out, ws=None, stream=None):
    _check(lib().vc_debug_gather(ctypes.byref(sh), ctypes.byref(sc), _p(k_out), _p(v_out), _p(ws),
                                 0 if ws is None else ws.numel(), _stream(stream)))


# ---- host -> HBM layer streaming ------------------------------------------------

class KvStream:
    """Handle of a vc_kvstream (double-buffered per-layer host -> device copies).

    host_k / host_v: lists of pinned host tensors, one per layer; dev_k / dev_v:
    two device staging tensors each; copy_stream: a torch.cuda.Stream."""

    def __init__(self, host_k, host_v, dev_k, dev_v, copy_stream):
        n = len(host_k)
        self._keep = (host_k, host_v, dev_k, dev_v, copy_stream)
        self._hk = (c_void_p * n)(*[_p(t) for t in host_k])
        self._hv = (c_void_p * n)(*[_p(t) for t in host_v])
        self._dk = (c_void_p * 2)(*[_p(t) for t in dev_k])
        self._dv = (c_void_p * 2)(*[_p(t) for t in dev_v])
        nbytes = host_k[0].numel() * host_k[0].element_size()
        h = c_void_p()
        _check(lib().vc_kvstream_create(ctypes.byref(h), n, self._hk, self._hv, nbytes, self._dk, self._dv,
                                        _stream(copy_stream)))
        self.h = h

    def prefetch(self, layer: int):
        _check(lib().vc_kvstream_prefetch(self.h, int(layer)))

    def acquire(self, layer: int, stream=None):
        k, v = c_void_p(), c_void_p()
        _check(lib().vc_kvstream_acquire(self.h, int(layer), _stream(stream), ctypes.byref(k), ctypes.byref(v)))
        return k.value, v.value

    def release(self, layer: int, stream=None):
        _check(lib().vc_kvstream_release(self.h, int(layer), _stream(stream)))

    def close(self):
        if self.h:
            _check(lib().vc_kvstream_destroy(self.h))
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---- stagger scheduler ----------------------------------------------------------

class Sched:
    """Handle of a vc_sched.  `requests` is a list of vc_sched_request structs
    (see make_sched_request); keep-alive references travel with them."""

    def __init__(self, requests, n_layers: int, draft_len: int, policy: int, copy_stream, timeout_ms: int = 60000):
        n = len(requests)
        self._arr = (vc_sched_request * n)(*requests)
        self._keep = [getattr(r, "_keep", None) for r in requests] + [copy_stream]
        h = c_void_p()
        _check(lib().vc_sched_create(ctypes.byref(h), n, self._arr, int(n_layers), int(draft_len), int(policy),
                                     _stream(copy_stream), int(timeout_ms)))
        self.h = h

    def set_links(self, remote_stream, remote_gbps: float, local_gbps: float = 0.0, chunk_bytes: int = 0):
        self._keep.append(remote_stream)
        _check(lib().vc_sched_set_links(self.h, _stream(remote_stream), float(remote_gbps), float(local_gbps),
                                        int(chunk_bytes)))

    def set_fetch(self, request: int, src, dst):
        """Copies (pinned host tensor -> device tensor of the same size) that
        bring the request's compressed cache over the remote link."""
        n = len(src)
        sa = (c_void_p * n)(*[_p(t) for t in src])
        da = (c_void_p * n)(*[_p(t) for t in dst])
        ba = (c_size_t * n)(*[t.numel() * t.element_size() for t in src])
        for a, b in zip(src, dst):
            assert a.numel() * a.element_size() == b.numel() * b.element_size()
        self._keep.append((src, dst))
        _check(lib().vc_sched_set_fetch(self.h, int(request), n, ctypes.cast(sa, c_void_p), ctypes.cast(da, c_void_p),
                                        ctypes.cast(ba, c_void_p)))

    def run_rounds(self, n_rounds: int) -> dict:
        st = vc_sched_stats()
        _check(lib().vc_sched_run_rounds(self.h, int(n_rounds), ctypes.byref(st)))
        return dict(elapsed_ms=st.elapsed_ms, link_busy_ms=st.link_busy_ms, draft_ms=st.draft_ms,
                    verify_ms=st.verify_ms, rounds=st.rounds, requests=st.requests, fetch_ms=st.fetch_ms,
                    first_draft_ms=st.first_draft_ms)

    def close(self):
        if self.h:
            _check(lib().vc_sched_destroy(self.h))
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def make_sched_request(sh, kind, caches, draft_q, draft_out, draft_ws, host_k, host_v, stage_k, stage_v, verify_q,
                       verify_out, verify_ws, T, nq, logits, V, draft_tokens, target, accept_len, correction,
                       accept_ws, stream):
    """Marshal one request of the scheduler; `caches` are per-layer
    vc_quant_cache (kind VC_DRAFT_QUANT) or vc_sparse_cache descriptors."""
    n = len(caches)
    carr = ((vc_quant_cache if kind == VC_DRAFT_QUANT else vc_sparse_cache) * n)(*caches)
    hk = (c_void_p * n)(*[_p(t) for t in host_k])
    hv = (c_void_p * n)(*[_p(t) for t in host_v])
    r = vc_sched_request()
    r.shape = sh
    r.draft_kind = kind
    r.qcaches = ctypes.cast(carr, c_void_p) if kind == VC_DRAFT_QUANT else None
    r.scaches = ctypes.cast(carr, c_void_p) if kind != VC_DRAFT_QUANT else None
    r.draft_q, r.draft_out, r.draft_ws, r.draft_ws_bytes = _p(draft_q), _p(draft_out), _p(draft_ws), draft_ws.numel()
    r.host_k = ctypes.cast(hk, c_void_p)
    r.host_v = ctypes.cast(hv, c_void_p)
    r.kv_bytes_per_layer = host_k[0].numel() * host_k[0].element_size()
    r.stage_k[0], r.stage_k[1] = _p(stage_k[0]), _p(stage_k[1])
    r.stage_v[0], r.stage_v[1] = _p(stage_v[0]), _p(stage_v[1])
    r.verify_q, r.verify_out, r.verify_ws, r.verify_ws_bytes = _p(verify_q), _p(verify_out), _p(verify_ws), verify_ws.numel()
    r.T, r.nq = int(T), int(nq)
    r.logits = _p(logits)
    r.logits_dtype = VC_BF16 if logits.dtype == torch.bfloat16 else VC_F32
    r.V = int(V)
    r.draft_tokens, r.target, r.accept_len, r.correction = _p(draft_tokens), _p(target), _p(accept_len), _p(correction)
    r.accept_ws, r.accept_ws_bytes = _p(accept_ws), accept_ws.numel()
    r.stream = _stream(stream)
    r._keep = (caches, carr, hk, hv, host_k, host_v, stage_k, stage_v, draft_q, draft_out, draft_ws, verify_q,
               verify_out, verify_ws, logits, draft_tokens, target, accept_len, correction, accept_ws, stream)
    return r


def vc_sched_simulate(draft_ms, verify_ms, n_rounds: int, policy: int, never_done: int = -1,
                      timeout_ms: float = 1e9, fetch_ms=None) -> float:
    """Makespan of the scheduling policy on a simulated timeline (host only)."""
    n = len(draft_ms)
    d = (ctypes.c_double * n)(*draft_ms)
    v = (ctypes.c_double * n)(*verify_ms)
    f = (ctypes.c_double * n)(*fetch_ms) if fetch_ms is not None else None
    out = ctypes.c_double()
    _check(lib().vc_sched_simulate(n, int(n_rounds), int(policy), f, d, v, int(never_done), float(timeout_ms),
                                   ctypes.byref(out)))
    return out.value


# ---- bandwidth-limited link --------------------------------------------------------

class Link:
    """Handle of a vc_link: host -> device copies on `stream` at `gbps` GB/s
    (0: unpaced), in chunks of chunk_bytes (0: 8 MiB)."""

    def __init__(self, stream, gbps: float, chunk_bytes: int = 0):
        h = c_void_p()
        self._keep = [stream]
        _check(lib().vc_link_create(ctypes.byref(h), _stream(stream), float(gbps), int(chunk_bytes)))
        self.h = h

    def copy(self, dst, src):
        n = src.numel() * src.element_size()
        assert dst.numel() * dst.element_size() >= n
        self._keep.append((dst, src))
        _check(lib().vc_link_copy(self.h, _p(dst), _p(src), n))

    def flags(self) -> int:
        v = c_uint32(0)
        _check(lib().vc_link_flags(self.h, ctypes.byref(v)))
        return int(v.value)

    def close(self):
        if self.h:
            _check(lib().vc_link_destroy(self.h))
            self.h = None
            self._keep = []

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---- one verifier decoder layer ------------------------------------------------------

def layer_shape(d_model: int, d_ff: int, Hq: int, Hkv: int, D: int, rms_eps: float = 1e-5,
                rope_theta: float = 500000.0) -> vc_layer_shape:
    return vc_layer_shape(d_model, d_ff, Hq, Hkv, D, rms_eps, rope_theta)


def layer_weights(w: dict) -> vc_layer_weights:
    """Descriptor of a layer's bf16 weights given as a dict of CUDA tensors
    w1, wqkv, wo, w2, wgu, wd (keeps references to them)."""
    d = vc_layer_weights(*[_p(w[k]) for k in ("w1", "wqkv", "wo", "w2", "wgu", "wd")])
    d._keep = w
    return d


def vc_verify_layer_workspace_size(ls, B: int, nq: int, T: int) -> int:
    return lib().vc_verify_layer_workspace_size(ctypes.byref(ls), int(B), int(nq), int(T))


def vc_verify_layer(ls, lw, B: int, nq: int, T: int, x, k_cache, v_cache, ws, stream=None):
    _check(lib().vc_verify_layer(ctypes.byref(ls), ctypes.byref(lw), int(B), int(nq), int(T), _p(x), _p(k_cache),
                                 _p(v_cache), _p(ws), ws.numel(), _stream(stream)))
