"""Pins for the oracle's quantiser / dequantiser (CPU only).

The oracle's rule is a reading of the pages (see oracle/quant.py); these
tests pin it to values worked by hand, to the bit layout written out by hand,
to exact reconstruction when the data sit on the quantisation grid, and to
the error bound of round-to-nearest."""

import json
import os

import numpy as np
import pytest

from oracle import quant


def _load(golden_dir):
    with open(os.path.join(golden_dir, "quant_hand_examples.json")) as f:
        return json.load(f)


def test_hand_examples_as_key_groups(golden_dir):
    for ex in _load(golden_dir)["groups"]:
        x = np.array(ex["x"], np.float64)[:, None]            # G tokens, 1 channel
        codes, s, z = quant.quantize_keys(x, ex["bits"], len(ex["x"]))
        assert codes[:, 0].tolist() == ex["codes"], ex["why"]
        assert float(s[0, 0]) == ex["scale"] and float(z[0, 0]) == ex["zero"], ex["why"]
        deq = quant.dequantize_keys(codes, s, z, len(ex["x"]))
        assert deq[:, 0].tolist() == ex["dequant"], ex["why"]


def test_hand_examples_as_value_groups(golden_dir):
    for ex in _load(golden_dir)["groups"]:
        x = np.array(ex["x"], np.float64)[None, :]            # 1 token, G channels
        codes, s, z = quant.quantize_values(x, ex["bits"], len(ex["x"]))
        assert codes[0].tolist() == ex["codes"], ex["why"]
        assert float(s[0, 0]) == ex["scale"] and float(z[0, 0]) == ex["zero"]
        deq = quant.dequantize_values(codes, s, z, len(ex["x"]))
        assert deq[0].tolist() == ex["dequant"], ex["why"]


def test_hand_packing(golden_dir):
    for ex in _load(golden_dir)["packing"]:
        codes = np.array(ex["codes"], np.uint8)
        packed = quant.pack_codes(codes, ex["bits"])
        assert packed.tolist() == ex["bytes"], ex["why"]
        assert quant.unpack_codes(packed, ex["bits"]).tolist() == ex["codes"]


@pytest.mark.parametrize("bits", [2, 4])
def test_pack_matches_bitstring(bits):
    """Packing against an independent bit-string construction: the row's bits,
    least significant first, are the codes' bits least significant first."""
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 1 << bits, size=(5, 64)).astype(np.uint8)
    packed = quant.pack_codes(codes, bits)
    for r in range(codes.shape[0]):
        stream = "".join(format(int(c), f"0{bits}b")[::-1] for c in codes[r])
        want = [int(stream[8 * i:8 * i + 8][::-1], 2) for i in range(len(stream) // 8)]
        assert packed[r].tolist() == want


@pytest.mark.parametrize("bits,G", [(2, 32), (4, 64), (2, 16)])
def test_grid_data_reconstruct_exactly(bits, G):
    """Data built as z + code * s with s a power of two and every group using
    both extreme codes quantise back to the same codes and dequantise exactly."""
    rng = np.random.default_rng(bits * 100 + G)
    levels = (1 << bits) - 1
    T, D = 4 * G, 2 * G
    codes = rng.integers(0, levels + 1, size=(T, D))
    codes[0::G, :] = 0
    codes[1::G, :] = levels            # every key group (per channel) spans the grid
    vcodes = rng.integers(0, levels + 1, size=(T, D))
    vcodes[:, 0::G] = 0
    vcodes[:, 1::G] = levels           # every value group (per token) spans the grid
    s_exp = rng.integers(-6, 2, size=(T // G, D))
    s = 2.0 ** s_exp
    z = -rng.integers(0, 8, size=(T // G, D)) * s
    x = z.repeat(G, 0) + codes * s.repeat(G, 0)
    kc, ks, kz = quant.quantize_keys(x, bits, G)
    assert np.array_equal(kc, codes)
    assert np.array_equal(quant.dequantize_keys(kc, ks, kz, G).astype(np.float64), x)
    # values: the grid runs along channels
    sv = 2.0 ** rng.integers(-6, 2, size=(T, D // G))
    zv = -rng.integers(0, 8, size=(T, D // G)) * sv
    xv = zv.repeat(G, 1) + vcodes * sv.repeat(G, 1)
    vc, vs, vz = quant.quantize_values(xv, bits, G)
    assert np.array_equal(vc, vcodes)
    assert np.array_equal(quant.dequantize_values(vc, vs, vz, G).astype(np.float64), xv)


@pytest.mark.parametrize("bits,G", [(2, 32), (4, 64)])
def test_round_to_nearest_error_bound(bits, G):
    """|x_hat - x| is at most half a step plus the fp16 rounding of s and z
    (relative 2**-11 each, scaled by the number of levels)."""
    rng = np.random.default_rng(7)
    levels = (1 << bits) - 1
    x = (rng.standard_normal((2 * G, 64)) * np.exp(rng.standard_normal(64))).astype(np.float32)
    codes, s, z = quant.quantize_keys(x, bits, G)
    assert codes.max() <= levels
    xh = quant.dequantize_keys(codes, s, z, G)
    s_t = np.repeat(s.astype(np.float64), G, 0)
    rng_t = np.repeat((x.reshape(2, G, 64).max(1) - x.reshape(2, G, 64).min(1)).astype(np.float64), G, 0)
    bound = 0.5 * s_t + 2.0 ** -10 * rng_t * (levels + 1) + 1e-30
    assert np.all(np.abs(xh - x) <= bound)


def test_block_positions_worked_by_hand(golden_dir):
    with open(os.path.join(golden_dir, "code_block_positions.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        fn = quant.key_code_positions if c["kind"] == "key" else quant.value_code_positions
        byte, shift = fn(c["bits"], c["group"], c["D"])
        assert (int(byte[c["token"], c["channel"]]), int(shift[c["token"], c["channel"]])) == (c["byte"], c["shift"]), c["why"]


@pytest.mark.parametrize("bits,G,D", [(2, 32, 128), (2, 64, 128), (4, 64, 128), (4, 32, 128), (2, 32, 64), (4, 64, 64)])
@pytest.mark.parametrize("values", [False, True])
def test_block_order_is_a_permutation(bits, G, D, values):
    """Every code of a group gets its own bits, the block is exactly G*D*b/8
    bytes, and pack/unpack round-trip."""
    byte, shift = quant._block_positions(bits, G, D, values)
    slots = byte * 8 + shift
    assert len(np.unique(slots)) == G * D
    assert np.all(shift % bits == 0) and byte.max() == G * D * bits // 8 - 1
    rng = np.random.default_rng(bits + G + D)
    c = rng.integers(0, 1 << bits, size=(2, 3 * G, D)).astype(np.uint8)
    blk = quant.pack_group_blocks(c, bits, G, values)
    assert np.array_equal(quant.unpack_group_blocks(blk, bits, G, D, values), c)


def test_pair_interleave():
    p = np.arange(2 * 6 * 4).reshape(2, 6, 4)
    q = quant.pair_interleave(p)
    assert q.shape == (2, 3, 4, 2)
    assert q[1, 2, 3].tolist() == [p[1, 4, 3], p[1, 5, 3]]
    assert np.array_equal(quant.pair_deinterleave(q), p)


def test_build_cache_layout():
    rng = np.random.default_rng(0)
    B, H, T, D, R, G = 2, 3, 96, 64, 32, 32
    k = rng.standard_normal((B, H, T, D)).astype(np.float32)
    v = rng.standard_normal((B, H, T, D)).astype(np.float32)
    c = quant.build_quant_cache(k, v, 2, G, R)
    assert c["k_codes"].shape == (B, H, (T - R) // G, G * D // 4)
    assert c["k_scale"].shape == (B, H, (T - R) // G, D)
    assert c["v_scale"].shape == (B, H, (T - R) // 2, D // G, 2)
    kh, vh = quant.dequantize_cache(c)
    assert kh.shape == (B, H, T, D)
    assert np.array_equal(kh[:, :, T - R:], k[:, :, T - R:])
    with pytest.raises(ValueError):
        quant.build_quant_cache(k, v, 2, G, 33)


def test_fp16_overflow_refused():
    x = np.array([[0.0], [3e5]])
    with pytest.raises(ValueError):
        quant.quantize_keys(x, 2, 2)
