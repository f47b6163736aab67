"""Reference KV-cache quantisation (oracle; test infrastructure only).

What the pages fix
------------------
[P2] "Key Contributions": a compressor is known to the system only through
the positions it drops and the bit width it stores; KIVI and KVQuant are
among the quantising drafters it wraps.  [P2] "Limitations": a single bit
width is shared by every layer and token.  [P1] "The Tradeoff VeriCache Is
Trying to Escape": quantisation keeps all positions and lowers the precision
of each stored number.

Readings taken where the pages are silent (all listed in the design doc)
------------------------------------------------------------------
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
* Packing: code of channel c of a token occupies bits
  [(c mod (8/b)) * b, +b) of byte floor(c * b / 8) of that token's row
  (little-endian within the byte, channels contiguous along the row).
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


def build_quant_cache(k: np.ndarray, v: np.ndarray, bits: int, group: int, residual: int) -> dict:
    """Compress one layer's full cache into the quantised draft cache.

    k, v: [B, Hkv, T, D] bf16 values (as float32).  The oldest
    L_q = T - residual tokens are quantised, the newest ``residual`` stay bf16.
    Returns a dict with the packed codes, fp16 scales/zeros and the residual
    rows, in the layouts the library's quantised-cache descriptor names."""
    k = np.asarray(k, np.float32)
    v = np.asarray(v, np.float32)
    T = k.shape[-2]
    L_q = T - residual
    if L_q < 0 or L_q % group:
        raise ValueError("T - residual must be a non-negative multiple of the group size")
    kc, sk, zk = quantize_keys(k[..., :L_q, :], bits, group)
    vc, sv, zv = quantize_values(v[..., :L_q, :], bits, group)
    return dict(
        bits=bits, group=group, L_q=L_q, R=residual,
        k_codes=pack_codes(kc, bits), v_codes=pack_codes(vc, bits),
        k_scale=sk, k_zero=zk, v_scale=sv, v_zero=zv,
        k_res=k[..., L_q:, :].copy(), v_res=v[..., L_q:, :].copy(),
    )


def dequantize_cache(cache: dict):
    """Full-length (K_hat, V_hat) of a quantised cache: dequantised rows
    followed by the bf16 residual rows.  Float32 arrays [B, Hkv, L_q + R, D]."""
    bits, G = cache["bits"], cache["group"]
    kc = unpack_codes(cache["k_codes"], bits)
    vc = unpack_codes(cache["v_codes"], bits)
    kh = dequantize_keys(kc, cache["k_scale"], cache["k_zero"], G)
    vh = dequantize_values(vc, cache["v_scale"], cache["v_zero"], G)
    R = cache["R"]
    kr = np.asarray(cache["k_res"], np.float32)[..., :R, :]
    vr = np.asarray(cache["v_res"], np.float32)[..., :R, :]
    return np.concatenate([kh, kr], axis=-2), np.concatenate([vh, vr], axis=-2)
