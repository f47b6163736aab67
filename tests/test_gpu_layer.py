"""One verifier decoder layer on the GPU (vc_verify_layer) against the oracle
(oracle/layer.py) on random bf16 weights.

Both sides round every step's result to bf16 at the same points; they differ
in how each step sums before rounding (fp32 on the GPU, exact fp64 in the
oracle) and, for the attention step, by the verification kernel's own error
(up to 2e-3 of the row, its tolerance against the oracle), so a bf16
rounding can land one ulp apart and such a flip reaches later steps.
Tolerance, derived from that: per output row, the largest difference is at
most 4 bf16 ulps of the row's largest element (2^-6, relative) and the mean
difference at most 2^-9 of it (the attention tolerance).  The cache rows the
layer writes (rotated k, and v) come from the QKV projection, where a flip
is one ulp of an element; the rotation mixes each pair, so a rotated
element can move by up to two ulps of the pair's larger element: per cache
row, at most 2^-6 of the row's largest element.  Rows T - nq - 1 and older
of the cache are untouched."""

import numpy as np
import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import layer as L
from tests.vcutil import np32

pytestmark = pytest.mark.gpu
dev = "cuda"


def _weights(seed, dm, dff, Hq, Hkv, D, scale):
    g = torch.Generator().manual_seed(seed)

    def r(shape, s):
        return (torch.randn(shape, generator=g) * s).to(torch.bfloat16)

    n1 = (Hq + 2 * Hkv) * D
    return dict(w1=(1 + 0.1 * torch.randn(dm, generator=g)).to(torch.bfloat16),
                w2=(1 + 0.1 * torch.randn(dm, generator=g)).to(torch.bfloat16),
                wqkv=r((n1, dm), scale / dm ** 0.5), wo=r((dm, Hq * D), scale / (Hq * D) ** 0.5),
                wgu=r((2 * dff, dm), scale / dm ** 0.5), wd=r((dm, dff), scale / dff ** 0.5))


@pytest.mark.parametrize("B,nq,dm,dff,Hq,Hkv,D,T", [
    (2, 5, 256, 512, 8, 2, 64, 300),      # g = 4, D = 64
    (1, 31, 512, 1024, 8, 1, 128, 777),   # g = 8: two row tiles in one block
    (1, 31, 4096, 14336, 32, 8, 128, 1024),  # Llama-3.1-8B layer dimensions
])
def test_layer_matches_the_oracle(B, nq, dm, dff, Hq, Hkv, D, T):
    W = _weights(B * 1000 + dm, dm, dff, Hq, Hkv, D, 1.0)
    x = synth.normal((B, nq, dm), seed=dm + 1)
    k, v = synth.kv_full(B, Hkv, T, D, seed=dm + 2)
    ls = vc.layer_shape(dm, dff, Hq, Hkv, D)
    Wd = {n: t.to(dev) for n, t in W.items()}
    lw = vc.layer_weights(Wd)
    xd, kd, vd = x.to(dev), k.to(dev).contiguous(), v.to(dev).contiguous()
    ws = vc.workspace(vc.vc_verify_layer_workspace_size(ls, B, nq, T))
    vc.vc_verify_layer(ls, lw, B, nq, T, xd, kd, vd, ws)
    torch.cuda.synchronize()
    want, wk, wv = L.verify_layer(np32(x), {n: np32(t) for n, t in W.items()}, np32(k), np32(v), Hq, Hkv)
    got = np32(xd).astype(np.float64)
    scale = np.abs(want).max(axis=-1, keepdims=True)
    diff = np.abs(got - want)
    assert np.isfinite(got).all()
    assert (diff.max(axis=-1, keepdims=True) <= 2.0 ** -6 * scale).all(), (diff / scale).max()
    assert (diff.mean(axis=-1, keepdims=True) <= 2.0 ** -9 * scale).all(), (diff.mean(-1) / scale[..., 0]).max()
    gk, gv = np32(kd).astype(np.float64), np32(vd).astype(np.float64)
    assert np.array_equal(gk[:, :, :T - nq], wk[:, :, :T - nq])
    assert np.array_equal(gv[:, :, :T - nq], wv[:, :, :T - nq])
    for got_c, want_c in ((gk, wk), (gv, wv)):
        blk_g, blk_w = got_c[:, :, T - nq:], want_c[:, :, T - nq:]
        row_scale = np.abs(blk_w).max(axis=-1, keepdims=True)
        assert (np.abs(blk_g - blk_w) <= 2.0 ** -6 * row_scale).all()
        # most elements agree exactly: a flip needs the exact value near a rounding boundary
        assert (blk_g == blk_w).mean() >= 0.9


def test_zero_output_projections_leave_x_and_write_the_cache():
    B, nq, dm, dff, Hq, Hkv, D, T = 1, 7, 256, 256, 4, 2, 64, 100
    W = _weights(5, dm, dff, Hq, Hkv, D, 1.0)
    W["wo"] = torch.zeros_like(W["wo"])
    W["wd"] = torch.zeros_like(W["wd"])
    x = synth.normal((B, nq, dm), seed=6)
    k, v = synth.kv_full(B, Hkv, T, D, seed=7)
    ls = vc.layer_shape(dm, dff, Hq, Hkv, D)
    lw = vc.layer_weights({n: t.to(dev) for n, t in W.items()})
    xd, kd, vd = x.to(dev), k.to(dev).contiguous(), v.to(dev).contiguous()
    ws = vc.workspace(vc.vc_verify_layer_workspace_size(ls, B, nq, T))
    vc.vc_verify_layer(ls, lw, B, nq, T, xd, kd, vd, ws)
    torch.cuda.synchronize()
    assert torch.equal(xd.cpu(), x)
    assert not torch.equal(kd[:, :, T - nq:].cpu(), k[:, :, T - nq:])
