// vc_compress.cu -- building the compressed draft caches on the GPU:
//   vc_quantize_cache   full bf16 K, V -> group records (KIVI-style uniform
//                       quantisation, keys per channel, values per token) +
//                       the bf16 residual window;
//   vc_compact_kept     full bf16 K, V + kept positions -> a kept-row pool.
//
// A compressor is known to the system only through the positions it drops
// and the bit width it stores ("VeriCache: Turning Lossy KV Cache into
// Lossless LLM Inference", menfem.com, "Key Contributions"); these two
// kernels produce exactly those two kinds of cache in the layouts the draft
// kernels read (include/vc.h).
//
// Quantisation rule (the library's reading, identical to the oracle's):
// per group, s = fp16(round-to-nearest((max - min) / (2^b - 1))),
// z = fp16(min), code = clamp(rint((x - z) / s), 0, 2^b - 1) with the STORED
// s and z, half to even; s == 0 gives code 0.  Every code equals the one the
// float64 quotient gives: the quotient is first taken in fp32 as
// (x - z) * (1 / s), whose error is below 2^-18 for the quotients that are
// not clamped (|q| <= 16); only when that lands within 2^-17 of a rounding
// tie (k + 1/2) is it recomputed as an IEEE float64 division of the exact
// float64 difference.
#include "vc_common.cuh"

namespace vc {
namespace {

constexpr uint32_t kRangeFlag = VC_FLAG_RANGE;

// fp16 bits of v rounded to nearest even, or a range flag when |v| > 65504
__device__ __forceinline__ uint16_t to_half_checked(double v, uint32_t* flags) {
  if (!(fabs(v) <= 65504.0)) {
    if (flags) atomicOr(flags, kRangeFlag);
  }
  const __half h = __double2half(v);
  return __half_as_ushort(h);
}

// Codes of a pair of elements (one bf16x2 register): clamp(rint((x - z) / s),
// 0, levels), returned as code(lo) | code(hi) << 16.  Fast form: the
// quotient in fp32 as (x - z) * (1 / s), both halves in one packed fp32x2
// instruction each; its error is at most 3 * 2^-24 * |q| < 2^-18 where
// 0 <= q <= 15.5, so a quotient farther than 2^-17 from a rounding tie
// rounds as the exact one does, and `near` is set for the others (exact
// ties are common: bf16 data, fp16 scale and zero).  Rounding adds
// 1.5 * 2^23, which leaves rint(q) in the low mantissa bits.  Clamping
// before rounding gives the same codes as clamping after it; a NaN quotient
// (zero or scale outside fp16) gives code 0.
template <int BITS>
__device__ __forceinline__ uint32_t codes2_fast(uint32_t xb, float2 negz, float2 inv, bool& near) {
  constexpr float levels = static_cast<float>((1 << BITS) - 1);
  constexpr float kMagic = 12582912.0f;                // 1.5 * 2^23
  constexpr float kTie = 0.5f - 7.62939453125e-6f;     // 0.5 - 2^-17
  const float2 x = unpack_bf2(xb);
  const float2 q = __fmul2_rn(__fadd2_rn(x, negz), inv);
  const float2 qc = make_float2(fminf(fmaxf(q.x, 0.f), levels), fminf(fmaxf(q.y, 0.f), levels));
  const float2 m = __fadd2_rn(qc, make_float2(kMagic, kMagic));
  const float2 e = __ffma2_rn(__fadd2_rn(m, make_float2(-kMagic, -kMagic)), make_float2(-1.f, -1.f), qc);
  near = fabsf(e.x) > kTie || fabsf(e.y) > kTie;
  return __byte_perm(__float_as_uint(m.x), __float_as_uint(m.y), 0x5410);
}

// Code of one element as the float64 rule gives it: rint of the float64
// quotient of the float64 difference by the stored scale (out of line: it
// runs only where x - z is not exact in fp32, which needs exponents ~2^24
// apart).
template <int BITS>
__device__ __noinline__ uint32_t code_f64(float x, float negz, float s) {
  const double r = rint((static_cast<double>(x) + static_cast<double>(negz)) / static_cast<double>(s));
  return static_cast<uint32_t>(fmin(fmax(r, 0.0), static_cast<double>((1 << BITS) - 1)));
}

// Code of one element whose fp32 quotient may sit on the wrong side of a
// tie T = k + 1/2.  When d = fp32(x - z) is exact (its two-sum error is
// zero), d and T s are exact fp32 numbers, and the sign of d - T s (one
// fused multiply-add, so the sign is exact) tells whether (x - z) / s lies
// above, below or on T; on T the even neighbour wins.  Any other quotient is
// at least ~2^-24 T from T, so the float64 quotient falls on the same side.
template <int BITS>
__device__ __forceinline__ uint32_t code_near(float x, float negz, float inv, float s) {
  constexpr float levels = static_cast<float>((1 << BITS) - 1);
  if (s == 0.f) return 0u;
  const float d = __fadd_rn(x, negz);
  const float bv = __fsub_rn(d, x), av = __fsub_rn(d, bv);
  const float err = __fadd_rn(__fsub_rn(x, av), __fsub_rn(negz, bv));
  if (err != 0.f) return code_f64<BITS>(x, negz, s);
  const float qc = fminf(fmaxf(__fmul_rn(d, inv), 0.f), levels);
  const float r = rintf(qc);
  if (fabsf(qc - r) <= 0.25f) return static_cast<uint32_t>(r);  // not near a tie
  const float T = qc > r ? r + 0.5f : r - 0.5f;
  const float t = fmaf(-T, s, d);
  const float lo = T - 0.5f;
  float c = t > 0.f ? T + 0.5f : (t < 0.f ? lo : ((static_cast<int>(lo) & 1) == 0 ? lo : T + 0.5f));
  c = fminf(fmaxf(c, 0.f), levels);
  return static_cast<uint32_t>(c);
}

// Both codes of a register pair with code_near (out of line: it runs only
// for the rare pairs near a tie, and inlined in every tile it would cost the
// common path registers and code size).
template <int BITS>
__device__ __noinline__ uint32_t codes2_near(uint32_t xb, float2 negz, float2 inv, float2 sc) {
  const float2 x = unpack_bf2(xb);
  return code_near<BITS>(x.x, negz.x, inv.x, sc.x) | (code_near<BITS>(x.y, negz.y, inv.y, sc.y) << 16);
}

template <int BITS, int G, int D>
struct QuantLayout {
  static constexpr int CB = G * D * BITS / 8;
  static constexpr int REC = 2 * CB + 8 * D;
  static constexpr int KT = D / 16;
  static constexpr int TPW = 8 / BITS;
  static constexpr int NW = 2 * KT / TPW;  // words per lane per 16-token tile
  static constexpr int NJ = KT / TPW;      // word pairs (X, Y) per lane per 16-token tile
  static constexpr int CPG = D / G;
};

// One block of 128 threads per (group, unit).  The group's K and V rows are
// staged in shared memory (bf16, rows padded by 16 bytes so that the eight
// 16-byte rows of an ldmatrix hit distinct banks).  Parameters: keys per
// channel by one thread each, values per (token, value group) by one warp
// per token row with shuffles.  Codes: a warp takes one (16-token tile,
// word pair) of K or V at a time; ldmatrix (transposed for V) hands every
// lane the elements of its fragment-native code words directly (the order in
// which the draft kernel's lanes consume them), so each lane computes and
// packs whole words and stores them.
template <int BITS, int G, int D>
__device__ __forceinline__ void quantize_group(const __nv_bfloat16* __restrict__ kgp,
                                               const __nv_bfloat16* __restrict__ vgp, uint8_t* __restrict__ rec,
                                               uint32_t* flags) {
  using L = QuantLayout<BITS, G, D>;
  constexpr int levels = (1 << BITS) - 1;
  constexpr int RS = 2 * D + 16;  // bytes per staged row
  constexpr int TT = G / 16, TPW = L::TPW, NJ = L::NJ, NW = L::NW, CPG = L::CPG;
  constexpr int EPL = D / 32;     // channels per lane in a row
  constexpr int LPG = G / EPL;    // lanes per value group
  __shared__ __align__(16) unsigned char ks[G * RS];
  __shared__ __align__(16) unsigned char vs[G * RS];
  __shared__ __align__(8) float kzn[D], kin[D], ksc[D];             // -zero, 1 / scale (0 if 0), scale
  __shared__ __align__(8) float vzn[CPG][G], vin[CPG][G], vsc[CPG][G];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint4* kg = reinterpret_cast<const uint4*>(kgp);
  const uint4* vg = reinterpret_cast<const uint4*>(vgp);
  for (int e = tid; e < G * D / 8; e += 128) {  // stage the group's rows, 16-byte streaming loads
    const int t = e / (D / 8), c8 = e - t * (D / 8);
    *reinterpret_cast<uint4*>(ks + t * RS + c8 * 16) = __ldcs(kg + e);
    *reinterpret_cast<uint4*>(vs + t * RS + c8 * 16) = __ldcs(vg + e);
  }
  __syncthreads();
  auto Kf = [&](int t, int c) { return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(ks + t * RS + 2 * c)); };
  uint16_t* sk = reinterpret_cast<uint16_t*>(rec + 2 * L::CB);
  uint16_t* zk = sk + D;
  uint16_t* sv = zk + D;
  uint16_t* zv = sv + D;

  // key parameters: channel c over the group's G tokens; stored in fragment
  // order, channel c = 16 kt + 8 h + 2 t + e at fp16 slot 2 (t * 2 (D/16) + 2 kt + h) + e
  for (int c = tid; c < D; c += 128) {
    float mn = Kf(0, c), mx = mn;
    for (int t = 1; t < G; ++t) mn = fminf(mn, Kf(t, c)), mx = fmaxf(mx, Kf(t, c));
    const uint16_t sb = to_half_checked((static_cast<double>(mx) - static_cast<double>(mn)) / levels, flags);
    const uint16_t zb = to_half_checked(static_cast<double>(mn), flags);
    const int kt = c >> 4, h = (c >> 3) & 1, tq = (c >> 1) & 3, e = c & 1;
    const int slot = 2 * (tq * 2 * L::KT + 2 * kt + h) + e;
    sk[slot] = sb;
    zk[slot] = zb;
    const float sf = __half2float(__ushort_as_half(sb));
    kzn[c] = -__half2float(__ushort_as_half(zb));
    kin[c] = sf != 0.f ? 1.f / sf : 0.f;
    ksc[c] = sf;
  }
  // value parameters: token t, value group cg over its G channels; the
  // minimum and maximum by one warp per token row (lane l holds channels
  // EPL l ..), then one thread per (token, value group) forms the
  // parameters; stored pair-interleaved [G/2][CPG][2]
  for (int t = warp; t < G; t += 4) {
    float mn, mx;
    if constexpr (EPL == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(vs + t * RS + 8 * lane);
      const float2 a = unpack_bf2(w.x), b = unpack_bf2(w.y);
      mn = fminf(fminf(a.x, a.y), fminf(b.x, b.y));
      mx = fmaxf(fmaxf(a.x, a.y), fmaxf(b.x, b.y));
    } else {
      const float2 a = unpack_bf2(*reinterpret_cast<const uint32_t*>(vs + t * RS + 4 * lane));
      mn = fminf(a.x, a.y);
      mx = fmaxf(a.x, a.y);
    }
#pragma unroll
    for (int m = 1; m < LPG; m <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    }
    if (lane % LPG == 0) {
      vsc[lane / LPG][t] = mn;  // staged here until the parameters replace them
      vin[lane / LPG][t] = mx;
    }
  }
  __syncthreads();
  for (int e = tid; e < G * CPG; e += 128) {
    const int cg = e / G, t = e - cg * G;
    const float mn = vsc[cg][t], mx = vin[cg][t];
    const uint16_t sb = to_half_checked((static_cast<double>(mx) - static_cast<double>(mn)) / levels, flags);
    const uint16_t zb = to_half_checked(static_cast<double>(mn), flags);
    const int slot = ((t >> 1) * CPG + cg) * 2 + (t & 1);
    sv[slot] = sb;
    zv[slot] = zb;
    const float sf = __half2float(__ushort_as_half(sb));
    vzn[cg][t] = -__half2float(__ushort_as_half(zb));
    vin[cg][t] = sf != 0.f ? 1.f / sf : 0.f;
    vsc[cg][t] = sf;
  }
  __syncthreads();

  // code words: word index = (tt * 32 + lane) * NW + w, w = 2 j + (0: X, 1: Y);
  // local tile i of pair j covers channel (key) / channel-row (value) tile
  // TPW j + i; first register's codes at bits [b i] and [16 + b i], second's
  // at [8 + b i], [24 + b i].  ldmatrix row providers: lane 8 mi + ri.
  const int tig = lane & 3, mi = lane >> 3, ri = lane & 7;
  uint32_t* kw = reinterpret_cast<uint32_t*>(rec);
  uint32_t* vw = reinterpret_cast<uint32_t*>(rec + L::CB);
  for (int item = warp; item < 2 * TT * NJ; item += 4) {  // warp-uniform
    const bool isv = item >= TT * NJ;
    const int it = isv ? item - TT * NJ : item;
    const int tt = it / NJ, j = it - tt * NJ;
    uint32_t X = 0u, Y = 0u;
    // keys: r0 / r1 = tokens gid / gid + 8 at channels 16 ct + 2 tig (+1), r2 /
    // r3 the same at channels + 8: X = r0 | r1 << 8, Y = r2 | r3 << 8.
    // values (transposed): r0 / r1 = channel gid / gid + 8 at tokens
    // 16 tt + 2 tig (+1), r2 / r3 the same at tokens + 8: X = r0 | r2 << 8,
    // Y = r1 | r3 << 8.  Register k goes to word (k >> wsh) & 1 of (X, Y) at
    // offset 8 ((k >> osh) & 1); its parameters are those of the first (k < 2:
    // keys channel c, values tokens t0) or the second pair (c + 8, t0 + 8).
    const int wsh = isv ? 0 : 1, osh = isv ? 1 : 0;
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      const int ct = TPW * j + i;
      uint32_t r[4];
      const float *zp, *ip;
      int o0;
      if (!isv) {
        ldsm_x4(r, ks + (16 * tt + 8 * (mi & 1) + ri) * RS + (16 * ct + 8 * (mi >> 1)) * 2);
        zp = kzn, ip = kin, o0 = 16 * ct + 2 * tig;
      } else {
        ldsm_x4_t(r, vs + (16 * tt + 8 * (mi >> 1) + ri) * RS + (16 * ct + 8 * (mi & 1)) * 2);
        const int cg = 16 * ct / G;
        zp = &vzn[cg][0], ip = &vin[cg][0], o0 = 16 * tt + 2 * tig;
      }
      const float2 za = *reinterpret_cast<const float2*>(zp + o0), ia = *reinterpret_cast<const float2*>(ip + o0);
      const float2 zb = *reinterpret_cast<const float2*>(zp + o0 + 8), ib = *reinterpret_cast<const float2*>(ip + o0 + 8);
      uint32_t nmi = 0u;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        bool nr;
        const uint32_t p = codes2_fast<BITS>(r[k], k < 2 ? za : zb, k < 2 ? ia : ib, nr);
        nmi |= (nr ? 1u : 0u) << k;
        const uint32_t placed = p << (8 * ((k >> osh) & 1) + BITS * i);
        if ((k >> wsh) & 1)
          Y |= placed;
        else
          X |= placed;
      }
      // pairs of this tile near a tie (rare per pair, but some lane meets one
      // in most word pairs): their codes again, exactly
      if (__any_sync(0xffffffffu, nmi != 0u) && nmi != 0u) {
        const float* sp = isv ? &vsc[16 * ct / G][0] : ksc;
        const float2 sa = *reinterpret_cast<const float2*>(sp + o0), sb = *reinterpret_cast<const float2*>(sp + o0 + 8);
        for (int k = 0; k < 4; ++k) {
          if (!((nmi >> k) & 1u)) continue;
          const uint32_t p = codes2_near<BITS>(r[k], k < 2 ? za : zb, k < 2 ? ia : ib, k < 2 ? sa : sb);
          const int sh = 8 * ((k >> osh) & 1) + BITS * i;
          const uint32_t field = static_cast<uint32_t>(levels | (levels << 16)) << sh;
          if ((k >> wsh) & 1)
            Y = (Y & ~field) | (p << sh);
          else
            X = (X & ~field) | (p << sh);
        }
      }
    }
    uint32_t* dst = (isv ? vw : kw) + (tt * 32 + lane) * NW + 2 * j;
    *reinterpret_cast<uint2*>(dst) = make_uint2(X, Y);
  }
}

template <int BITS, int G, int D>
__global__ void __launch_bounds__(128) quantize_kernel(const __nv_bfloat16* __restrict__ k,
                                                       const __nv_bfloat16* __restrict__ v, int64_t T,
                                                       int64_t ng, uint8_t* __restrict__ records, uint32_t* flags) {
  using L = QuantLayout<BITS, G, D>;
  const int64_t grp = blockIdx.x, unit = blockIdx.y;
  quantize_group<BITS, G, D>(k + (unit * T + grp * G) * D, v + (unit * T + grp * G) * D,
                             records + (unit * ng + grp) * L::REC, flags);
}

// The newest R rows of every unit into the residual buffers (rows 0..R-1 of R_cap).
__global__ void copy_residual_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, int64_t T, int64_t L_q,
                                     int R, int R_cap, int D, uint4* __restrict__ kr, uint4* __restrict__ vr,
                                     int64_t units) {
  const int vec = D / 8;  // uint4 per row
  const int64_t n = units * R * vec;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t u = e / (static_cast<int64_t>(R) * vec);
    const int64_t rem = e - u * R * vec;
    const int64_t r = rem / vec, x = rem - r * vec;
    kr[(u * R_cap + r) * vec + x] = k[(u * T + L_q + r) * vec + x];
    vr[(u * R_cap + r) * vec + x] = v[(u * T + L_q + r) * vec + x];
  }
}

// Kept rows into the pool: one warp per (unit, kept row); lanes 0-15 copy the
// K row, lanes 16-31 the V row, 16 bytes each per step.  An index outside
// [0, T_store) writes a zero row and raises VC_FLAG_BAD_INDEX.
__global__ void compact_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                               int64_t T_store, const int32_t* __restrict__ idx, int n_keep, int D, int64_t units,
                               __nv_bfloat16* __restrict__ ko, __nv_bfloat16* __restrict__ vo, uint32_t* flags) {
  const int lane = threadIdx.x & 31;
  const int vec = D / 8;
  const int64_t rows = units * n_keep;
  for (int64_t rw = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) / 32; rw < rows;
       rw += static_cast<int64_t>(gridDim.x) * blockDim.x / 32) {
    const int64_t u = rw / n_keep;
    const int32_t p = idx[rw];
    const bool okp = p >= 0 && p < T_store;
    if (!okp && lane == 0 && flags) atomicOr(flags, VC_FLAG_BAD_INDEX);
    const bool isv = lane >= 16;
    const int l = lane & 15;
    const uint4* src = reinterpret_cast<const uint4*>((isv ? v : k) + (u * T_store + (okp ? p : 0)) * D);
    uint4* dst = reinterpret_cast<uint4*>((isv ? vo : ko) + rw * D);
    for (int x = l; x < vec; x += 16) dst[x] = okp ? src[x] : make_uint4(0u, 0u, 0u, 0u);
  }
}

// ---- cache maintenance after a round (vc_cache_commit) -----------------------
// Per request b: a = accept_len[b] accepted drafts, n = a + 1 rows of the
// verifier's block (x, d_1 .. d_a) are committed.  lens[b] = (L_q, R) of the
// request's quantised cache.  If R + n > R_cap the oldest `group` residual
// rows become record L_q / group and the residual keeps rows group .. R - 1;
// the n rows are appended after the residual.  Three launches in stream
// order, all deciding from the same (lens, accept_len): re-quantise, rewrite
// the residual, update lens.  A request whose accepted length is outside
// [0, nq) or whose records would exceed the capacity is left unchanged and
// raises VC_FLAG_BAD_LENGTH.
struct CommitDecision {
  bool valid, requant;
  int L_q, R, n;
};

__device__ __forceinline__ CommitDecision commit_decision(const int32_t* lens, const int32_t* accept, int b, int nq,
                                                          int R_cap, int G, int64_t ng_cap) {
  CommitDecision d;
  d.L_q = lens[2 * b];
  d.R = lens[2 * b + 1];
  const int a = accept[b];
  d.n = a + 1;
  d.requant = d.R + d.n > R_cap;
  d.valid = a >= 0 && a < nq && d.R >= 0 && d.R <= R_cap && d.L_q >= 0 && d.L_q % G == 0 &&
            (!d.requant || (d.R >= G && d.L_q / G < ng_cap));
  return d;
}

template <int BITS, int G, int D>
__global__ void __launch_bounds__(128) commit_requant_kernel(const __nv_bfloat16* __restrict__ k_res,
                                                             const __nv_bfloat16* __restrict__ v_res, int R_cap,
                                                             uint8_t* __restrict__ records, int64_t ng_cap,
                                                             const int32_t* __restrict__ lens,
                                                             const int32_t* __restrict__ accept, int Hkv, int nq,
                                                             uint32_t* flags) {
  using L = QuantLayout<BITS, G, D>;
  const int64_t u = blockIdx.x;
  const int b = static_cast<int>(u / Hkv);
  const CommitDecision d = commit_decision(lens, accept, b, nq, R_cap, G, ng_cap);
  if (!d.valid) {
    if (threadIdx.x == 0 && u % Hkv == 0 && flags) atomicOr(flags, VC_FLAG_BAD_LENGTH);
    return;
  }
  if (!d.requant) return;
  quantize_group<BITS, G, D>(k_res + u * R_cap * D, v_res + u * R_cap * D,
                             records + (u * ng_cap + d.L_q / G) * L::REC, flags);
}

// Residual rewrite of one unit: rows kept (group .. R - 1 after a re-quantisation,
// else none move) are staged in shared memory and written back from row 0,
// then the n committed rows follow.
__global__ void __launch_bounds__(256) commit_residual_kernel(__nv_bfloat16* __restrict__ k_res,
                                                              __nv_bfloat16* __restrict__ v_res, int R_cap, int D,
                                                              const __nv_bfloat16* __restrict__ k_new,
                                                              const __nv_bfloat16* __restrict__ v_new, int nq,
                                                              const int32_t* __restrict__ lens,
                                                              const int32_t* __restrict__ accept, int Hkv, int G,
                                                              int64_t ng_cap) {
  extern __shared__ __align__(16) uint4 stage[];
  const int64_t u = blockIdx.x;
  const int b = static_cast<int>(u / Hkv);
  const CommitDecision d = commit_decision(lens, accept, b, nq, R_cap, G, ng_cap);
  if (!d.valid) return;
  const int vec = D / 8;  // uint4 per row
  uint4* kr = reinterpret_cast<uint4*>(k_res + u * R_cap * D);
  uint4* vr = reinterpret_cast<uint4*>(v_res + u * R_cap * D);
  int dst = d.R;
  if (d.requant) {
    const int kept = d.R - G;
    for (int e = threadIdx.x; e < kept * vec; e += blockDim.x) {
      stage[e] = kr[G * vec + e];
      stage[kept * vec + e] = vr[G * vec + e];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kept * vec; e += blockDim.x) {
      kr[e] = stage[e];
      vr[e] = stage[kept * vec + e];
    }
    dst = kept;
  }
  const uint4* kn = reinterpret_cast<const uint4*>(k_new + u * nq * D);
  const uint4* vn = reinterpret_cast<const uint4*>(v_new + u * nq * D);
  for (int e = threadIdx.x; e < d.n * vec; e += blockDim.x) {
    kr[dst * vec + e] = kn[e];
    vr[dst * vec + e] = vn[e];
  }
}

__global__ void commit_lens_kernel(int32_t* lens, const int32_t* accept, int B, int nq, int R_cap, int G,
                                   int64_t ng_cap) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) {
    const CommitDecision d = commit_decision(lens, accept, b, nq, R_cap, G, ng_cap);
    if (!d.valid) continue;
    if (d.requant) {
      lens[2 * b] = d.L_q + G;
      lens[2 * b + 1] = d.R + d.n - G;
    } else {
      lens[2 * b + 1] = d.R + d.n;
    }
  }
}

template <typename F>
bool dispatch_q(int bits, int group, int D, F&& f) {
#define VC_QQ_CASE(BI, GR, DD)                                                                                \
  if (bits == BI && group == GR && D == DD) {                                                                 \
    f(std::integral_constant<int, BI>{}, std::integral_constant<int, GR>{}, std::integral_constant<int, DD>{}); \
    return true;                                                                                              \
  }
  VC_QQ_CASE(2, 32, 128) VC_QQ_CASE(2, 64, 128) VC_QQ_CASE(4, 32, 128) VC_QQ_CASE(4, 64, 128)
  VC_QQ_CASE(2, 32, 64) VC_QQ_CASE(2, 64, 64) VC_QQ_CASE(4, 32, 64) VC_QQ_CASE(4, 64, 64)
#undef VC_QQ_CASE
  return false;
}

}  // namespace
}  // namespace vc

extern "C" {

size_t vc_compress_workspace_size(void) { return vc::align_up(sizeof(vc::WsHeader), 256); }

vc_status vc_quantize_cache(const vc_attn_shape* shape, const void* k, const void* v, int64_t T, int bits, int group,
                            int64_t L_q, void* records, void* k_res, void* v_res, int R_cap, void* ws,
                            size_t ws_bytes, void* stream) {
  VC_REQUIRE(shape, "vc_quantize_cache: null shape");
  const vc_attn_shape& sh = *shape;
  VC_REQUIRE(sh.B >= 1 && sh.Hkv >= 1, "vc_quantize_cache: need B >= 1 and Hkv >= 1");
  VC_REQUIRE(sh.D == 64 || sh.D == 128, "vc_quantize_cache: head dim must be 64 or 128 (got %d)", sh.D);
  VC_REQUIRE(bits == 2 || bits == 4, "vc_quantize_cache: bits must be 2 or 4 (got %d)", bits);
  VC_REQUIRE(group == 32 || group == 64, "vc_quantize_cache: group must be 32 or 64 (got %d)", group);
  VC_REQUIRE(L_q >= 0 && L_q % group == 0 && L_q <= T, "vc_quantize_cache: need 0 <= L_q <= T, L_q a multiple of group");
  VC_REQUIRE(T >= 1, "vc_quantize_cache: T must be >= 1");
  const int64_t R = T - L_q;
  VC_REQUIRE(R <= R_cap, "vc_quantize_cache: the %lld newest rows do not fit the residual (R_cap %d)",
             static_cast<long long>(R), R_cap);
  VC_REQUIRE(k && v && ws, "vc_quantize_cache: null k, v or workspace");
  VC_REQUIRE(L_q == 0 || records, "vc_quantize_cache: null records");
  VC_REQUIRE(R == 0 || (k_res && v_res), "vc_quantize_cache: null residual buffers");
  VC_REQUIRE(vc::aligned16(k) && vc::aligned16(v) && vc::aligned16(records) && vc::aligned16(k_res) &&
                 vc::aligned16(v_res) && vc::aligned16(ws),
             "vc_quantize_cache: pointers must be 16-byte aligned");
  VC_REQUIRE(ws_bytes >= vc_compress_workspace_size(), "vc_quantize_cache: workspace too small");
  VC_REQUIRE(L_q / group <= 2147483647 && static_cast<int64_t>(sh.B) * sh.Hkv <= 65535,
             "vc_quantize_cache: too many groups or units");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* flags = static_cast<uint32_t*>(ws);
  const int64_t ng = L_q / group;
  const int64_t units = static_cast<int64_t>(sh.B) * sh.Hkv;
  if (ng > 0) {
    vc::dispatch_q(bits, group, sh.D, [&](auto BI, auto GR, auto DD) {
      dim3 grid(static_cast<unsigned>(ng), static_cast<unsigned>(units));
      vc::quantize_kernel<decltype(BI)::value, decltype(GR)::value, decltype(DD)::value><<<grid, 128, 0, s>>>(
          static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), T, ng,
          static_cast<uint8_t*>(records), flags);
    });
  }
  if (R > 0) {
    const int64_t n = units * R * (sh.D / 8);
    const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, 148 * 8));
    vc::copy_residual_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(k), static_cast<const uint4*>(v), T,
                                                     L_q, static_cast<int>(R), R_cap, sh.D, static_cast<uint4*>(k_res),
                                                     static_cast<uint4*>(v_res), units);
  }
  return vc::launch_status("vc_quantize_cache");
}

vc_status vc_compact_kept(const vc_attn_shape* shape, const void* k, const void* v, int64_t T_store,
                          const int32_t* idx, int n_keep, void* k_out, void* v_out, void* ws, size_t ws_bytes,
                          void* stream) {
  VC_REQUIRE(shape, "vc_compact_kept: null shape");
  const vc_attn_shape& sh = *shape;
  VC_REQUIRE(sh.B >= 1 && sh.Hkv >= 1, "vc_compact_kept: need B >= 1 and Hkv >= 1");
  VC_REQUIRE(sh.D == 64 || sh.D == 128, "vc_compact_kept: head dim must be 64 or 128 (got %d)", sh.D);
  VC_REQUIRE(T_store >= 1 && n_keep >= 1, "vc_compact_kept: need T_store >= 1 and n_keep >= 1");
  VC_REQUIRE(k && v && idx && k_out && v_out, "vc_compact_kept: null pointer");
  VC_REQUIRE(vc::aligned16(k) && vc::aligned16(v) && vc::aligned16(k_out) && vc::aligned16(v_out),
             "vc_compact_kept: K/V pointers must be 16-byte aligned");
  VC_REQUIRE(ws == nullptr || ws_bytes >= vc_compress_workspace_size(), "vc_compact_kept: workspace too small");
  const int64_t units = static_cast<int64_t>(sh.B) * sh.Hkv;
  const int64_t rows = units * n_keep;
  const int blocks = static_cast<int>(std::min<int64_t>((rows * 32 + 255) / 256, 148 * 16));
  vc::compact_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), T_store, idx, n_keep, sh.D, units,
      static_cast<__nv_bfloat16*>(k_out), static_cast<__nv_bfloat16*>(v_out), static_cast<uint32_t*>(ws));
  return vc::launch_status("vc_compact_kept");
}

vc_status vc_cache_commit(const vc_attn_shape* shape, const vc_quant_cache* cache, const void* k_new,
                          const void* v_new, int nq, const int32_t* accept_len, void* ws, size_t ws_bytes,
                          void* stream) {
  VC_REQUIRE(shape && cache, "vc_cache_commit: null shape or cache");
  const vc_attn_shape& sh = *shape;
  const vc_quant_cache& c = *cache;
  VC_REQUIRE(sh.B >= 1 && sh.Hkv >= 1 && static_cast<int64_t>(sh.B) * sh.Hkv <= 65535,
             "vc_cache_commit: need 1 <= B * Hkv <= 65535");
  VC_REQUIRE(sh.D == 64 || sh.D == 128, "vc_cache_commit: head dim must be 64 or 128 (got %d)", sh.D);
  VC_REQUIRE(c.bits == 2 || c.bits == 4, "vc_cache_commit: bits must be 2 or 4 (got %d)", c.bits);
  VC_REQUIRE(c.group == 32 || c.group == 64, "vc_cache_commit: group must be 32 or 64 (got %d)", c.group);
  VC_REQUIRE(c.lens != nullptr, "vc_cache_commit: the cache needs per-request lengths (lens)");
  VC_REQUIRE(c.L_q >= 0 && c.L_q % c.group == 0, "vc_cache_commit: record capacity L_q must be a multiple of group");
  VC_REQUIRE(nq >= 1 && nq <= c.group, "vc_cache_commit: need 1 <= nq <= group (got nq %d)", nq);
  VC_REQUIRE(c.R_cap >= c.group + nq - 1,
             "vc_cache_commit: R_cap must be >= group + nq - 1 so an overflowing residual holds a whole group");
  VC_REQUIRE(c.records && c.k_res && c.v_res && k_new && v_new && accept_len && ws,
             "vc_cache_commit: null pointer");
  VC_REQUIRE(vc::aligned16(c.records) && vc::aligned16(c.k_res) && vc::aligned16(c.v_res) &&
                 vc::aligned16(k_new) && vc::aligned16(v_new),
             "vc_cache_commit: cache and block pointers must be 16-byte aligned");
  VC_REQUIRE(ws_bytes >= vc_compress_workspace_size(), "vc_cache_commit: workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* flags = static_cast<uint32_t*>(ws);
  const int64_t units = static_cast<int64_t>(sh.B) * sh.Hkv;
  const int64_t ng_cap = c.L_q / c.group;
  int32_t* lens = const_cast<int32_t*>(c.lens);
  const auto* kres = static_cast<const __nv_bfloat16*>(c.k_res);
  const auto* vres = static_cast<const __nv_bfloat16*>(c.v_res);
  vc::dispatch_q(c.bits, c.group, sh.D, [&](auto BI, auto GR, auto DD) {
    vc::commit_requant_kernel<decltype(BI)::value, decltype(GR)::value, decltype(DD)::value>
        <<<static_cast<unsigned>(units), 128, 0, s>>>(kres, vres, c.R_cap, static_cast<uint8_t*>(const_cast<void*>(c.records)),
                                                      ng_cap, lens, accept_len, sh.Hkv, nq, flags);
  });
  const size_t smem = static_cast<size_t>(c.R_cap) * sh.D * 2 * 2;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(vc::commit_residual_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
  vc::commit_residual_kernel<<<static_cast<unsigned>(units), 256, smem, s>>>(
      static_cast<__nv_bfloat16*>(const_cast<void*>(c.k_res)), static_cast<__nv_bfloat16*>(const_cast<void*>(c.v_res)),
      c.R_cap, sh.D, static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new), nq, lens,
      accept_len, sh.Hkv, c.group, ng_cap);
  vc::commit_lens_kernel<<<1, 128, 0, s>>>(lens, accept_len, sh.B, nq, c.R_cap, c.group, ng_cap);
  return vc::launch_status("vc_cache_commit");
}

}  // extern "C"
