"""The GPU compression kernels against the oracle, byte for byte.

vc_quantize_cache turns one layer's full bf16 cache into the quantised draft
cache (group records + bf16 residual); the oracle's build_quant_cache does
the same in float64.  vc_compact_kept gathers kept rows into a pool; the
oracle's gather_rows is the plain definition.  Covered: every supported bit
width, group and head dim; lognormal key outliers; groups whose scale is zero;
values exactly halfway between two codes (round half to even); scales that
overflow fp16 (flagged); a full Llama-3.1-8B layer (8 x 32K) with sampled
units; kept lists with an out-of-range position (zero row, flag)."""

import numpy as np
import pytest
import torch

from lossless_draft_verify_vc_b200 import synth
from lossless_draft_verify_vc_b200 import vc
from oracle import attention as A
from oracle import quant as Q
from tests.vcutil import np32

pytestmark = pytest.mark.gpu
dev = "cuda"


def quantize_gpu(k, v, bits, G, R, R_cap=None):
    """k, v bf16 [B, Hkv, T, D] on the device -> (records, k_res, v_res, flags)."""
    B, Hkv, T, D = k.shape
    L_q = T - R
    R_cap = R_cap or max(R, 1)
    rec_bytes = 2 * G * D * bits // 8 + 8 * D
    records = torch.full((B, Hkv, L_q // G, rec_bytes), 0xAB, dtype=torch.uint8, device=dev)
    k_res = torch.full((B, Hkv, R_cap, D), float("nan"), dtype=torch.bfloat16, device=dev)
    v_res = torch.full_like(k_res, float("nan"))
    ws = vc.workspace(vc.vc_compress_workspace_size())
    vc.vc_quantize_cache(vc.shape(B, 4 * Hkv, Hkv, D), k, v, T, bits, G, L_q, records, k_res, v_res, R_cap, ws)
    torch.cuda.synchronize()
    return records, k_res, v_res, vc.vc_workspace_flags(ws)


def check_against_oracle(k, v, bits, G, R):
    records, k_res, v_res, flags = quantize_gpu(k.to(dev), v.to(dev), bits, G, R)
    want = Q.build_quant_cache(np32(k), np32(v), bits, G, R)
    assert flags == 0
    assert np.array_equal(records.cpu().numpy(), want["records"])
    if R:
        assert np.array_equal(np32(k_res[:, :, :R]), want["k_res"])
        assert np.array_equal(np32(v_res[:, :, :R]), want["v_res"])


@pytest.mark.parametrize("bits,G,D", [(2, 32, 128), (2, 64, 128), (4, 32, 128), (4, 64, 128),
                                      (2, 32, 64), (2, 64, 64), (4, 32, 64), (4, 64, 64)])
def test_records_equal_the_oracle_byte_for_byte(bits, G, D):
    B, Hkv, R = 2, 3, 37
    T = 5 * G + R
    k, v = synth.kv_full(B, Hkv, T, D, seed=bits * 100 + G + D)
    check_against_oracle(k, v, bits, G, R)


def test_zero_scales_and_exact_ties_round_half_to_even():
    B, Hkv, D, G, bits = 1, 2, 64, 32, 2
    T = 2 * G
    k, v = synth.kv_full(B, Hkv, T, D, seed=3, key_outliers=False)
    k = k.float()
    v = v.float()
    # group 0 of head 0: channel 5 constant (key scale 0), token 3 constant over
    # value group 1 (value scale 0)
    k[0, 0, :G, 5] = 0.75
    v[0, 0, 3, 32:64] = -1.25
    # group 1 of head 1, channel 9: min -1, max -0.25 -> s = 0.25 exactly; the
    # other tokens sit at halves: (x - z) / s = 0.5, 1.5, 2.5 -> codes 0, 2, 2
    col = torch.full((G,), -0.625)
    col[0], col[1] = -1.0, -0.25
    col[2:8] = torch.tensor([-0.875, -0.625, -0.375, -0.875, -0.625, -0.375])
    k[0, 1, G:2 * G, 9] = col
    # value token 7 of head 1, group 0: same construction along the channels
    row = torch.full((32,), -0.625)
    row[0], row[1] = -1.0, -0.25
    row[2:5] = torch.tensor([-0.875, -0.625, -0.375])
    v[0, 1, 7, 0:32] = row
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    check_against_oracle(k, v, bits, G, 0)
    kc, sk, zk, vc_, sv, zv = Q.cache_parts(Q.build_quant_cache(np32(k), np32(v), bits, G, 0))
    assert sk[0, 0, 0, 5] == 0 and (kc[0, 0, :G, 5] == 0).all()
    assert sk[0, 1, 1, 9] == 0.25 and list(kc[0, 1, G + 2:G + 8, 9]) == [0, 2, 2, 0, 2, 2]
    assert list(vc_[0, 1, 7, 2:5]) == [0, 2, 2]


def test_tie_whose_fp32_difference_is_inexact():
    """x - z not exact in fp32 next to a tie: z = -1000, s = 400 (max 200),
    x = 2^-30, so (x - z) / s = 2.5 + 2^-30 / 400 rounds up to 3, while the
    fp32 difference (1000) would sit exactly on the tie and round to even (2).
    Keys (channel 3 of group 0) and values (token 5, value group 0)."""
    B, Hkv, D, G, bits = 1, 1, 64, 32, 2
    k, v = synth.kv_full(B, Hkv, G, D, seed=8, key_outliers=False)
    k = k.float()
    v = v.float()
    k[0, 0, :, 3] = torch.linspace(-900.0, 100.0, G)
    k[0, 0, 0, 3], k[0, 0, 1, 3], k[0, 0, 2, 3] = -1000.0, 200.0, 2.0 ** -30
    v[0, 0, 5, 0:32] = torch.linspace(-900.0, 100.0, 32)
    v[0, 0, 5, 0], v[0, 0, 5, 1], v[0, 0, 5, 2] = -1000.0, 200.0, 2.0 ** -30
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    assert k[0, 0, 2, 3].item() == 2.0 ** -30 and v[0, 0, 5, 2].item() == 2.0 ** -30
    check_against_oracle(k, v, bits, G, 0)
    kc, sk, zk, vc_, sv, zv = Q.cache_parts(Q.build_quant_cache(np32(k), np32(v), bits, G, 0))
    assert sk[0, 0, 0, 3] == 400.0 and zk[0, 0, 0, 3] == -1000.0 and kc[0, 0, 2, 3] == 3
    assert vc_[0, 0, 5, 2] == 3


def test_scale_outside_fp16_is_flagged():
    B, Hkv, D, G = 1, 1, 64, 32
    k, v = synth.kv_full(B, Hkv, G, D, seed=4)
    k = k.float()
    k[0, 0, 0, 0] = -1.0e5  # zero (the group minimum) overflows fp16
    _, _, _, flags = quantize_gpu(k.to(torch.bfloat16).to(dev), v.to(dev), 2, G, 0)
    assert flags & vc.VC_FLAG_RANGE


def test_full_layer_llama_shape_sampled_units():
    B, Hkv, D, T, R, G, bits = 8, 8, 128, 32768, 128, 32, 2
    k, v = synth.kv_full(B, Hkv, T, D, seed=11, device=dev)
    records, k_res, v_res, flags = quantize_gpu(k, v, bits, G, R, R_cap=128)
    assert flags == 0
    for u in (0, 29, 63):
        b, h = divmod(u, Hkv)
        want = Q.build_quant_cache(np32(k[b:b + 1, h:h + 1]), np32(v[b:b + 1, h:h + 1]), bits, G, R)
        assert np.array_equal(records[b, h].cpu().numpy(), want["records"][0, 0]), u
        assert np.array_equal(np32(k_res[b, h]), want["k_res"][0, 0]), u
    del k, v, records
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,Hkv,D,T,n_keep", [(1, 2, 64, 512, 128), (2, 8, 128, 100000, 25000), (3, 1, 128, 77, 77)])
def test_compaction_equals_the_gather(B, Hkv, D, T, n_keep):
    k, v = synth.kv_full(B, Hkv, T, D, seed=T, device=dev)
    idx = synth.kept_positions(B, Hkv, T, n_keep, seed=T + 1, device=dev)
    ko = torch.full((B, Hkv, n_keep, D), float("nan"), dtype=torch.bfloat16, device=dev)
    vo = torch.full_like(ko, float("nan"))
    ws = vc.workspace(vc.vc_compress_workspace_size())
    vc.vc_compact_kept(vc.shape(B, Hkv, Hkv, D), k, v, T, idx, n_keep, ko, vo, ws)
    torch.cuda.synchronize()
    assert vc.vc_workspace_flags(ws) == 0
    want_k = A.gather_rows(np32(k), idx.cpu().numpy())
    want_v = A.gather_rows(np32(v), idx.cpu().numpy())
    assert np.array_equal(np32(ko), want_k) and np.array_equal(np32(vo), want_v)


def test_compaction_out_of_range_position_writes_zeros_and_flags():
    B, Hkv, D, T, n_keep = 1, 2, 64, 256, 16
    k, v = synth.kv_full(B, Hkv, T, D, seed=9, device=dev)
    idx = synth.kept_positions(B, Hkv, T, n_keep, seed=10, device=dev)
    idx[0, 1, 4] = T + 3
    idx[0, 0, 0] = -1
    ko = torch.empty((B, Hkv, n_keep, D), dtype=torch.bfloat16, device=dev)
    vo = torch.empty_like(ko)
    ws = vc.workspace(vc.vc_compress_workspace_size())
    vc.vc_compact_kept(vc.shape(B, Hkv, Hkv, D), k, v, T, idx, n_keep, ko, vo, ws)
    torch.cuda.synchronize()
    assert vc.vc_workspace_flags(ws) & vc.VC_FLAG_BAD_INDEX
    assert (np32(ko[0, 1, 4]) == 0).all() and (np32(vo[0, 0, 0]) == 0).all()
    good = idx.clone()
    good[0, 1, 4] = 0
    good[0, 0, 0] = 0
    want = A.gather_rows(np32(k), good.cpu().numpy())
    assert np.array_equal(np32(ko[0, 1, 5:]), want[0, 1, 5:])
