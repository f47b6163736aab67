"""Reference KV-cache quantisation (oracle; test infrastructure only).

What the pages fix
------------------
[P2] "Key Contributions": a compressor is known to the system only through
the positions it drops and the bit width it stores; KIVI and KVQuant are
among the quantising drafters it wraps.  [P2] "Limitations": a single bit
width is shared by every layer and token.  [P1] "The Tradeoff VeriCache Is
Trying to Escape": quantisation keeps all positions and lowers the precision
of each stored number.

Readings taken where the pages are silent
-----------------------------------------
* Uniform asymmetric min/max quantisation, b in {2, 4} bits.
* Keys are grouped per channel over G consecutive tokens; values are grouped
  per token over G consecutive channels (the KIVI split).
* Per group: s = fp16((max - min) / (2**b - 1)), z = fp16(min), both rounded
  to nearest-even from the exact float64 quotient / minimum.
* code = clamp(round_half_even((x - z) / s), 0, 2**b - 1) with the *stored*
  fp16 s and z; a group with s == 0 stores code 0.
* Dequantised value = fp32(code * s + z) with ONE rounding (an fp32 fused
  multiply-add).  In float64 the product and sum below are exact (code < 2**4,
  s and z are fp16), so rounding the float64 result to float32 once is exactly
  that single rounding.
* Storage (a choice of this library, the pages fix none): everything one
  group of G quantised tokens needs is one contiguous RECORD (record_layout
  below): the key-code block, the value-code block, the key scales and
  zeros of the group's D channels, and the value scales and zeros of its G
  tokens.  Code blocks are in the "fragment-native" order defined in
  key_code_positions / value_code_positions -- the order in which a warp of
  the draft kernel feeds them to its tensor-core tiles.  Key scales and
  zeros are in the fragment order of key_param_positions.  Value scales and
  zeros are pair-interleaved: for tokens (2p, 2p+1) the CPG = D / G groups
  hold (s[2p][cg], s[2p+1][cg]) next to each other.  pack_codes /
  unpack_codes (the plain row order: channel c of a token at bits
  [(c mod (8/b)) * b, +b) of byte c * b / 8) remain as the reference from
  which the block order is a fixed permutation.
* The oldest L_q = T - R tokens are quantised; the newest R stay bf16
  (the "recent-token residual window").
"""

from __future__ import annotations

import numpy as np

FP16_MAX = 65504.0


def _fp16(x: np.ndarray) -> np.ndarray:
    """Round float64 to IEEE fp16, nearest-even; refuse values that overflow."""
    x = np.asarray(x, dtype=np.float64)
    if np.any(np.abs(x) > FP16_MAX):
        raise ValueError("scale or zero outside the fp16 range")
    return x.astype(np.float16)


def group_scale_zero(xmin: np.ndarray, xmax: np.ndarray, bits: int):
    """Scale and zero of one quantisation group (reading stated in the module
    docstring).  Returns (s, z) as float16 arrays."""
    levels = (1 << bits) - 1
    s = _fp16((np.asarray(xmax, np.float64) - np.asarray(xmin, np.float64)) / levels)
    z = _fp16(xmin)
    return s, z


def quantize_group_codes(x: np.ndarray, s: np.ndarray, z: np.ndarray, bits: int) -> np.ndarray:
    """code = clamp(rint((x - z) / s), 0, 2**b - 1) with the stored fp16 s, z.

    ``x``, ``s``, ``z`` broadcast against each other.  np.rint rounds half to
    even.  Entries whose group scale is zero get code 0."""
    levels = (1 << bits) - 1
    x = np.asarray(x, np.float64)
    s64 = np.asarray(s, np.float64)
    z64 = np.asarray(z, np.float64)
    safe = np.where(s64 == 0.0, 1.0, s64)
    q = np.rint((x - z64) / safe)
    q = np.where(s64 == 0.0, 0.0, q)
    return np.clip(q, 0, levels).astype(np.uint8)


def quantize_keys(k: np.ndarray, bits: int, group: int):
    """Per-channel key quantisation over groups of ``group`` tokens.

    k: [..., L, D] real values (bf16 values held in float32/float64), L a
    multiple of ``group``.  Returns (codes uint8 [..., L, D], s [..., L/G, D],
    z [..., L/G, D]) with s, z float16."""
    k = np.asarray(k, np.float64)
    *lead, L, D = k.shape
    if L % group:
        raise ValueError("quantised length must be a multiple of the group size")
    kg = k.reshape(*lead, L // group, group, D)
    s, z = group_scale_zero(kg.min(axis=-2), kg.max(axis=-2), bits)
    codes = quantize_group_codes(kg, s[..., None, :], z[..., None, :], bits)
    return codes.reshape(*lead, L, D), s, z


def quantize_values(v: np.ndarray, bits: int, group: int):
    """Per-token value quantisation over groups of ``group`` channels.

    v: [..., L, D].  Returns (codes uint8 [..., L, D], s [..., L, D/G],
    z [..., L, D/G])."""
    v = np.asarray(v, np.float64)
    *lead, L, D = v.shape
    if D % group:
        raise ValueError("head dim must be a multiple of the group size")
    vg = v.reshape(*lead, L, D // group, group)
    s, z = group_scale_zero(vg.min(axis=-1), vg.max(axis=-1), bits)
    codes = quantize_group_codes(vg, s[..., None], z[..., None], bits)
    return codes.reshape(*lead, L, D), s, z


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack [..., D] codes into [..., D*bits/8] bytes, layout in the module
    docstring."""
    codes = np.asarray(codes, np.uint8)
    per = 8 // bits
    *lead, D = codes.shape
    if D % per:
        raise ValueError("row length must fill whole bytes")
    c = codes.reshape(*lead, D // per, per).astype(np.uint16)
    out = np.zeros((*lead, D // per), np.uint16)
    for j in range(per):
        out |= c[..., j] << (j * bits)
    return out.astype(np.uint8)


def unpack_codes(packed: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of :func:`pack_codes`: [..., D*bits/8] bytes -> [..., D] codes."""
    packed = np.asarray(packed, np.uint8)
    per = 8 // bits
    mask = (1 << bits) - 1
    parts = [(packed >> (j * bits)) & mask for j in range(per)]
    return np.stack(parts, axis=-1).reshape(*packed.shape[:-1], packed.shape[-1] * per)


# ---------------------------------------------------------------------------
# Fragment-native block order of the codes of one group.
#
# Keys (a G x D block C[t][c], t token in the group, c channel): tokens in
# tiles of 16 (t = 16 mt + r), channels in tiles of 16 (c = 16 kt + j).
# Lane L = 4 gid + tig (gid 0..7, tig 0..3) of a 32-lane warp owns, per
# (mt, kt), four registers of two codes each (first code = even slot):
#   reg0 = C[16mt+gid  ][16kt+2tig+{0,1}]    reg1 = C[16mt+gid+8][16kt+2tig+{0,1}]
#   reg2 = C[16mt+gid  ][16kt+2tig+8+{0,1}]  reg3 = C[16mt+gid+8][16kt+2tig+8+{0,1}]
# The lane's 32-bit words, per mt, are X_0, Y_0, X_1, Y_1, ... where X_j holds
# (reg0, reg1) and Y_j holds (reg2, reg3) of the TPW = 8 / b tiles
# kt = TPW j + i.  Inside a word, for local tile i and the pair
# (first register F, second register S):
#   F.code0 at bits [b i, +b)        F.code1 at bits [16 + b i, +b)
#   S.code0 at bits [8 + b i, +b)    S.code1 at bits [24 + b i, +b)
# Word w of lane L in token tile mt is the 32-bit word number
# (mt * 32 + L) * NW + w of the block (little-endian), NW = 2 (D/16) / TPW.
#
# Values (a G x D block C[t][c]): tokens in tiles of 16 (t = 16 kk + k),
# channels in tiles of 16 (c = 16 mc + r); per (kk, mc) lane L owns
#   reg0 = C[16kk+2tig+{0,1}][16mc+gid]      reg1 = C[16kk+2tig+{0,1}][16mc+gid+8]
#   reg2 = C[16kk+2tig+8+{0,1}][16mc+gid]    reg3 = C[16kk+2tig+8+{0,1}][16mc+gid+8]
# X_j holds (reg0, reg2), Y_j holds (reg1, reg3) of tiles mc = TPW j + i, with
# the same bit rule and word numbering (token tile kk in place of mt).
# ---------------------------------------------------------------------------

def _block_positions(bits: int, G: int, D: int, values: bool):
    """(byte index, bit shift) of every code of a G x D group block."""
    tpw = 8 // bits
    ntile_c = D // 16
    nw = 2 * ntile_c // tpw
    byte = np.full((G, D), -1, np.int64)
    shift = np.zeros((G, D), np.int64)
    for tt in range(G // 16):
        for L in range(32):
            gid, tig = L // 4, L % 4
            for ct in range(ntile_c):
                j, i = divmod(ct, tpw)
                if not values:
                    # (token, channel) of reg0..reg3, code0/code1
                    regs = [[(16 * tt + gid, 16 * ct + 2 * tig + e) for e in (0, 1)],
                            [(16 * tt + gid + 8, 16 * ct + 2 * tig + e) for e in (0, 1)],
                            [(16 * tt + gid, 16 * ct + 2 * tig + 8 + e) for e in (0, 1)],
                            [(16 * tt + gid + 8, 16 * ct + 2 * tig + 8 + e) for e in (0, 1)]]
                    words = [(2 * j, regs[0], regs[1]), (2 * j + 1, regs[2], regs[3])]
                else:
                    regs = [[(16 * tt + 2 * tig + e, 16 * ct + gid) for e in (0, 1)],
                            [(16 * tt + 2 * tig + e, 16 * ct + gid + 8) for e in (0, 1)],
                            [(16 * tt + 2 * tig + 8 + e, 16 * ct + gid) for e in (0, 1)],
                            [(16 * tt + 2 * tig + 8 + e, 16 * ct + gid + 8) for e in (0, 1)]]
                    words = [(2 * j, regs[0], regs[2]), (2 * j + 1, regs[1], regs[3])]
                for w, F, S in words:
                    word_index = (tt * 32 + L) * nw + w
                    for (t, c), bit in ((F[0], bits * i), (F[1], 16 + bits * i),
                                        (S[0], 8 + bits * i), (S[1], 24 + bits * i)):
                        byte[t, c] = word_index * 4 + bit // 8
                        shift[t, c] = bit % 8
    assert (byte >= 0).all(), "every code must have a place"
    return byte, shift


def key_code_positions(bits: int, G: int, D: int):
    return _block_positions(bits, G, D, values=False)


def value_code_positions(bits: int, G: int, D: int):
    return _block_positions(bits, G, D, values=True)


def pack_group_blocks(codes: np.ndarray, bits: int, G: int, values: bool) -> np.ndarray:
    """[..., L, D] codes -> [..., L/G, G*D*bits/8] bytes in block order."""
    codes = np.asarray(codes, np.uint8)
    *lead, L, D = codes.shape
    byte, shift = _block_positions(bits, G, D, values)
    c = codes.reshape(*lead, L // G, G, D).astype(np.uint32)
    out = np.zeros((*lead, L // G, G * D * bits // 8), np.uint32)
    flat_out = out.reshape(-1, out.shape[-1])
    flat_c = c.reshape(-1, G, D)
    for n in range(flat_c.shape[0]):
        np.bitwise_or.at(flat_out[n], byte.ravel(), (flat_c[n] << shift).ravel())
    return out.astype(np.uint8)


def unpack_group_blocks(blocks: np.ndarray, bits: int, G: int, D: int, values: bool) -> np.ndarray:
    """Inverse of pack_group_blocks: [..., L/G, G*D*bits/8] -> [..., L, D]."""
    blocks = np.asarray(blocks, np.uint8)
    byte, shift = _block_positions(bits, G, D, values)
    mask = (1 << bits) - 1
    out = (blocks[..., byte] >> shift) & mask
    *lead, ng, _, _ = out.shape
    return out.reshape(*lead, ng * G, D).astype(np.uint8)


def pair_interleave(params: np.ndarray) -> np.ndarray:
    """Value scales or zeros [..., L, CPG] -> [..., L/2, CPG, 2]: the two tokens
    of a pair sit next to each other for every value group."""
    p = np.asarray(params)
    *lead, L, cpg = p.shape
    return np.ascontiguousarray(p.reshape(*lead, L // 2, 2, cpg).swapaxes(-1, -2))


def pair_deinterleave(params: np.ndarray) -> np.ndarray:
    p = np.asarray(params)
    *lead, P, cpg, two = p.shape
    return np.ascontiguousarray(p.swapaxes(-1, -2)).reshape(*lead, 2 * P, cpg)


def dequantize_keys(codes: np.ndarray, s: np.ndarray, z: np.ndarray, group: int) -> np.ndarray:
    """k_hat[t, c] = fp32(code[t, c] * s[t // G, c] + z[t // G, c]) (single rounding)."""
    codes = np.asarray(codes, np.float64)
    s_t = np.repeat(np.asarray(s, np.float64), group, axis=-2)
    z_t = np.repeat(np.asarray(z, np.float64), group, axis=-2)
    return (codes * s_t + z_t).astype(np.float32)


def dequantize_values(codes: np.ndarray, s: np.ndarray, z: np.ndarray, group: int) -> np.ndarray:
    """v_hat[t, c] = fp32(code[t, c] * s[t, c // G] + z[t, c // G]) (single rounding)."""
    codes = np.asarray(codes, np.float64)
    s_c = np.repeat(np.asarray(s, np.float64), group, axis=-1)
    z_c = np.repeat(np.asarray(z, np.float64), group, axis=-1)
    return (codes * s_c + z_c).astype(np.float32)


# ---------------------------------------------------------------------------
# Key scales / zeros of a group in fragment order.  A lane with tig (0..3)
# multiplies, for every 16-channel tile kt, the channel pairs
# (16kt + 2tig, +1) and (16kt + 8 + 2tig, +1); the row of D fp16 entries is
# stored so that those pairs are one run of 2 * (D/16) 32-bit words per tig:
#   channel c = 16 kt + 8 h + 2 tig + e   (h, e in {0, 1})
#   -> 32-bit word tig * 2 (D/16) + 2 kt + h, fp16 slot e of that word.
# ---------------------------------------------------------------------------

def key_param_positions(D: int) -> np.ndarray:
    """fp16 index, inside a group's key-scale (or key-zero) row, of channel c."""
    KT = D // 16
    pos = np.empty(D, np.int64)
    for c in range(D):
        kt, r = divmod(c, 16)
        h, r2 = divmod(r, 8)
        tig, e = divmod(r2, 2)
        pos[c] = 2 * (tig * 2 * KT + 2 * kt + h) + e
    return pos


def record_layout(bits: int, G: int, D: int) -> dict:
    """Byte offsets of the parts of one group record and its size.
      kc  key codes,   G*D*bits/8 bytes (fragment-native block)
      vc  value codes, G*D*bits/8 bytes (fragment-native block)
      sk  key scales,  D fp16 (key_param_positions order)
      zk  key zeros,   D fp16 (same order)
      sv  value scales of the G tokens, [G/2][D/G][2] fp16 (pair-interleaved)
      zv  value zeros, same shape"""
    cb = G * D * bits // 8
    off = dict(kc=0, vc=cb, sk=2 * cb, zk=2 * cb + 2 * D, sv=2 * cb + 4 * D, zv=2 * cb + 6 * D)
    off["size"] = 2 * cb + 8 * D
    return off


def pack_group_records(kc_blocks, vc_blocks, sk, zk, sv_pairs, zv_pairs, bits: int, G: int) -> np.ndarray:
    """Assemble records [..., L/G, size] from code blocks [..., L/G, CB], key
    scales/zeros [..., L/G, D] (natural channel order) and pair-interleaved
    value scales/zeros [..., L/2, D/G, 2]."""
    kc_blocks = np.asarray(kc_blocks, np.uint8)
    *lead, ng, _ = kc_blocks.shape
    D = np.asarray(sk).shape[-1]
    lay = record_layout(bits, G, D)
    out = np.zeros((*lead, ng, lay["size"]), np.uint8)
    pos = key_param_positions(D)

    def put(name, arr16):
        b = np.ascontiguousarray(arr16.astype(np.float16)).view(np.uint8)
        out[..., lay[name]:lay[name] + b.shape[-1]] = b

    out[..., lay["kc"]:lay["vc"]] = kc_blocks
    out[..., lay["vc"]:lay["sk"]] = np.asarray(vc_blocks, np.uint8)
    for name, row in (("sk", sk), ("zk", zk)):
        perm = np.empty_like(np.asarray(row, np.float16))
        perm[..., pos] = np.asarray(row, np.float16)
        put(name, perm)
    for name, pr in (("sv", sv_pairs), ("zv", zv_pairs)):
        pr = np.asarray(pr, np.float16)
        put(name, pr.reshape(*lead, ng, (G // 2) * pr.shape[-2] * 2))
    return out


def unpack_group_records(records, bits: int, G: int, D: int):
    """Inverse of pack_group_records: (kc_blocks, vc_blocks, sk, zk, sv_pairs,
    zv_pairs) with key parameters back in natural channel order."""
    rec = np.asarray(records, np.uint8)
    *lead, ng, size = rec.shape
    lay = record_layout(bits, G, D)
    if size != lay["size"]:
        raise ValueError("record size does not match bits, group and head dim")
    pos = key_param_positions(D)

    def get16(name, n):
        return np.ascontiguousarray(rec[..., lay[name]:lay[name] + 2 * n]).view(np.float16)

    sk = get16("sk", D)[..., pos]
    zk = get16("zk", D)[..., pos]
    cpg = D // G
    sv = get16("sv", D).reshape(*lead, ng * G // 2, cpg, 2)
    zv = get16("zv", D).reshape(*lead, ng * G // 2, cpg, 2)
    return (rec[..., lay["kc"]:lay["vc"]].copy(), rec[..., lay["vc"]:lay["sk"]].copy(), sk, zk, sv, zv)


def build_quant_cache(k: np.ndarray, v: np.ndarray, bits: int, group: int, residual: int) -> dict:
    """Compress one layer's full cache into the quantised draft cache.

    k, v: [B, Hkv, T, D] bf16 values (as float32).  The oldest
    L_q = T - residual tokens are quantised, the newest ``residual`` stay bf16.
    Returns a dict in the library's storage layout:
      records     uint8 [B, Hkv, L_q/G, size]  (record_layout)
      k_res, v_res bf16 values [B, Hkv, residual, D]
    plus bits, group, L_q, R, D."""
    k = np.asarray(k, np.float32)
    v = np.asarray(v, np.float32)
    T, D = k.shape[-2], k.shape[-1]
    L_q = T - residual
    if L_q < 0 or L_q % group:
        raise ValueError("T - residual must be a non-negative multiple of the group size")
    kc, sk, zk = quantize_keys(k[..., :L_q, :], bits, group)
    vc, sv, zv = quantize_values(v[..., :L_q, :], bits, group)
    records = pack_group_records(pack_group_blocks(kc, bits, group, values=False),
                                 pack_group_blocks(vc, bits, group, values=True),
                                 sk, zk, pair_interleave(sv), pair_interleave(zv), bits, group)
    return dict(bits=bits, group=group, L_q=L_q, R=residual, D=D, records=records,
                k_res=k[..., L_q:, :].copy(), v_res=v[..., L_q:, :].copy())


def cache_parts(cache: dict):
    """Codes and parameters of a quantised cache in natural order:
    (k_codes [.., L_q, D], k_scale, k_zero [.., L_q/G, D],
     v_codes [.., L_q, D], v_scale, v_zero [.., L_q, D/G])."""
    bits, G, D = cache["bits"], cache["group"], cache["D"]
    kb, vb, sk, zk, sv, zv = unpack_group_records(cache["records"], bits, G, D)
    return (unpack_group_blocks(kb, bits, G, D, values=False), sk, zk,
            unpack_group_blocks(vb, bits, G, D, values=True), pair_deinterleave(sv), pair_deinterleave(zv))


def dequantize_cache(cache: dict):
    """Full-length (K_hat, V_hat) of a quantised cache: dequantised rows
    followed by the bf16 residual rows.  Float32 arrays [B, Hkv, L_q + R, D]."""
    G = cache["group"]
    kc, sk, zk, vc, sv, zv = cache_parts(cache)
    kh = dequantize_keys(kc, sk, zk, G)
    vh = dequantize_values(vc, sv, zv, G)
    R = cache["R"]
    kr = np.asarray(cache["k_res"], np.float32)[..., :R, :]
    vr = np.asarray(cache["v_res"], np.float32)[..., :R, :]
    return np.concatenate([kh, kr], axis=-2), np.concatenate([vh, vr], axis=-2)
