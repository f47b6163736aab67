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


def _records(golden_dir):
    with open(os.path.join(golden_dir, "record_positions.json")) as f:
        return json.load(f)


def test_key_param_slots_worked_by_hand(golden_dir):
    for c in _records(golden_dir)["key_param_slots"]:
        assert int(quant.key_param_positions(c["D"])[c["channel"]]) == c["slot"], c["why"]


@pytest.mark.parametrize("D", [64, 128])
def test_key_param_order_gives_each_tig_one_run(D):
    """Permutation of the D slots; lane tig's channel pairs are the words
    [tig*2KT, (tig+1)*2KT) in the order (kt, h) -- one contiguous run."""
    pos = quant.key_param_positions(D)
    assert sorted(pos.tolist()) == list(range(D))
    KT = D // 16
    for tig in range(4):
        chans = [16 * kt + 8 * h + 2 * tig + e for kt in range(KT) for h in (0, 1) for e in (0, 1)]
        assert pos[chans].tolist() == list(range(tig * 4 * KT, (tig + 1) * 4 * KT))


def test_record_sizes_worked_by_hand(golden_dir):
    for c in _records(golden_dir)["record_size"]:
        assert quant.record_layout(c["bits"], c["group"], c["D"])["size"] == c["size"]


def test_planted_parameters_land_on_hand_worked_bytes(golden_dir):
    """Quantise data whose scales / zeros are known, then read the fp16 at the
    byte offset worked by hand."""
    for c in _records(golden_dir)["record_bytes"]:
        bits, G, D = c["bits"], c["group"], c["D"]
        levels = (1 << bits) - 1
        rng = np.random.default_rng(1)
        x = rng.integers(0, levels + 1, size=(1, 1, G, D)).astype(np.float64)
        if c["part"] in ("key_scale", "key_zero"):
            ch = c["channel"]
            x[..., ch] = 0.25
            x[..., 1, ch] = 0.25 + 0.5 * levels                         # zero 0.25, scale 0.5
            want = 0.5 if c["part"] == "key_scale" else 0.25
            cache = quant.build_quant_cache(x, np.zeros_like(x), bits, G, 0)
        else:
            t, vg = c["token"], c["vgroup"]
            v = np.zeros_like(x)
            v[..., t, vg * G:(vg + 1) * G] = -0.75
            v[..., t, vg * G + 1] = -0.75 + 0.125 * levels                  # zero -0.75, scale 0.125
            want = 0.125 if c["part"] == "value_scale" else -0.75
            cache = quant.build_quant_cache(x, v, bits, G, 0)
        rec = cache["records"][0, 0, 0]
        got = float(rec[c["byte"]:c["byte"] + 2].view(np.float16)[0])
        assert got == want, c["why"]


@pytest.mark.parametrize("bits,G,D", [(2, 32, 128), (4, 64, 128), (2, 64, 64), (4, 32, 64)])
def test_records_round_trip_and_match_direct_quantisation(bits, G, D):
    rng = np.random.default_rng(bits * G + D)
    B, H, T, R = 2, 3, 3 * G + 5, 5
    k = (rng.standard_normal((B, H, T, D)) * np.exp(rng.standard_normal((B, H, 1, D)))).astype(np.float32)
    v = rng.standard_normal((B, H, T, D)).astype(np.float32)
    c = quant.build_quant_cache(k, v, bits, G, R)
    assert c["records"].shape == (B, H, (T - R) // G, quant.record_layout(bits, G, D)["size"])
    kc, sk, zk, vc, sv, zv = quant.cache_parts(c)
    kc0, sk0, zk0 = quant.quantize_keys(k[..., :T - R, :], bits, G)
    vc0, sv0, zv0 = quant.quantize_values(v[..., :T - R, :], bits, G)
    for a, b in ((kc, kc0), (sk, sk0), (zk, zk0), (vc, vc0), (sv, sv0), (zv, zv0)):
        assert np.array_equal(a, b)
    parts = quant.unpack_group_records(c["records"], bits, G, D)
    again = quant.pack_group_records(*parts, bits, G)
    assert np.array_equal(again, c["records"])


def test_build_cache_layout():
    rng = np.random.default_rng(0)
    B, H, T, D, R, G = 2, 3, 96, 64, 32, 32
    k = rng.standard_normal((B, H, T, D)).astype(np.float32)
    v = rng.standard_normal((B, H, T, D)).astype(np.float32)
    c = quant.build_quant_cache(k, v, 2, G, R)
    assert c["records"].shape == (B, H, (T - R) // G, 2 * G * D // 4 + 8 * D)
    kh, vh = quant.dequantize_cache(c)
    assert kh.shape == (B, H, T, D)
    assert np.array_equal(kh[:, :, T - R:], k[:, :, T - R:])
    with pytest.raises(ValueError):
        quant.build_quant_cache(k, v, 2, G, 33)


def test_fp16_overflow_refused():
    x = np.array([[0.0], [3e5]])
    with pytest.raises(ValueError):
        quant.quantize_keys(x, 2, 2)
