// vc_draft_quant.cu -- single-token draft attention over a quantised KV cache
// (KIVI-style 2-bit or KVQuant-style 4-bit codes with per-channel key groups,
// per-token value groups, fp16 scales/zeros, bf16 recent-token residual).
//
// Pages: drafting decodes one token at a time against the compressed cache
// in HBM and is bound by HBM bandwidth ("VeriCache: Turning Lossy KV Cache
// into Lossless LLM Inference", menfem.com, "Key Contributions"; devshah.ca
// page, "Verifying Without Giving Back the Speedup").  The pages give no
// kernel; everything below is this library's design.
//
// Arithmetic.  With k_hat = code * s + z per key group (s, z per channel) and
// v_hat = code * s + z per value group (s, z per token):
//   q . k_hat[t]        = sum_c (q_c s_c) code[t][c] + sum_c q_c z_c
//   sum_t p_t v_hat[t]c = sum_t (p_t s_t) code[t][c] + sum_t p_t z_t
// so the codes enter the tensor cores as exact small integers (fp16), and the
// scales are folded into the other operand once per group.  The folded
// operands q*s and p*s are split into an fp16 high part and an fp16 low
// part (two MMA columns each), which keeps ~22 significant bits; the zero
// terms are separate small MMAs with exact fp16 products.  Accumulation is
// fp32.  The result equals attention over fp32-dequantised values up to fp32
// rounding (the oracle dequantises with one fp32 FMA per element).
//
// Work layout.  The job is one axis of STAGES: first every (request, KV
// head) unit's bf16 residual, 16 rows per stage, then every unit's quantised
// groups, NG consecutive group records per stage.  A persistent grid of
// (SMs x resident blocks) blocks cuts that axis into equal-cost contiguous
// ranges (Partition); inside a block the 4 warps take the range's stages
// round-robin.  A quantised stage is ONE bulk copy of contiguous records into
// the warp's private ring (NST stages deep, completed on mbarriers, waits
// bounded).  Wherever the range crosses from one unit's segment to the next,
// the block merges its warps' online-softmax states into one partial of that
// segment; a second launch (combine_kernel, one block per (unit, head))
// merges each unit's partials into the output.  All g query heads of a GQA
// group share each record (they are the MMA's N columns).
//
// MMA arrangement (mma.sync m16n8k16, fp16 x fp16 -> fp32):
//   scores:  D[token][col] = codes[token][chan] x qfold[chan][col]
//            col = 2 * head + part (part 0 = high, 1 = low), 4 heads per n-tile
//   values:  D[chan][col]  = codes^T[chan][token] x pfold[token][col]
// Code bits reach the tensor cores as fp16 subnormals (one AND per two codes,
// see Frag); the record layout puts each lane's codes at fixed bit positions
// and each lane's key scales in one contiguous run.
#include <mutex>

#include "vc_common.cuh"

namespace vc {
namespace {

constexpr int kQNW = 4;          // warps per block
constexpr int kResRows = 16;     // residual rows per stage
constexpr int kResCostWeight = 2;  // residual stages are not pipelined: count their bytes twice

template <int BITS, int G, int D, int NT>
struct QCfg {
  static constexpr int CB = G * D * BITS / 8;  // one code block (keys or values) of a group
  static constexpr int REC = 2 * CB + 8 * D;   // group record: kc | vc | sk | zk | sv | zv
  static constexpr int OFF_VC = CB;
  static constexpr int OFF_SK = 2 * CB;
  static constexpr int OFF_ZK = 2 * CB + 2 * D;
  static constexpr int OFF_SV = 2 * CB + 4 * D;
  static constexpr int OFF_ZV = 2 * CB + 6 * D;
  static constexpr int NG = REC >= 3072 ? 1 : 3072 / REC;  // records per stage
  static constexpr int STAGE = NG * REC;
  static constexpr int NST0 = (NT == 1 ? 9216 : 18432) / STAGE;
  static constexpr int NST = NST0 < 2 ? 2 : (NST0 > 4 ? 4 : NST0);  // ring depth
  static constexpr int RSTAGE = 2 * kResRows * D * 2;                // 16 K + 16 V bf16 rows
  static constexpr int RING0 = NST * STAGE > RSTAGE ? NST * STAGE : RSTAGE;
  static constexpr int RING = (RING0 + 127) / 128 * 128;
  static constexpr int HEADS = 4 * NT;
  static constexpr int RP_B = HEADS * kResRows * 4;  // residual tile scores, fp32 [HEADS][16]
  static constexpr int WARP_B = RING + RP_B;
  static constexpr int STATE_OFF = kQNW * WARP_B;                       // fp32 [kQNW][HEADS][D]
  static constexpr int ML_OFF = STATE_OFF + kQNW * HEADS * D * 4;       // fp32 [kQNW][HEADS][2]
  static constexpr int MW_OFF = ML_OFF + kQNW * HEADS * 2 * 4;          // merge weights + (M, L)
  static constexpr int MW_FLOATS = kQNW * HEADS + 2 * HEADS;
  static constexpr int BAR_OFF = (MW_OFF + MW_FLOATS * 4 + 15) / 16 * 16;
  static constexpr int SMEM_B = BAR_OFF + kQNW * (NST + 1) * 8;
  static constexpr int KT = D / 16;   // channel tiles
  static constexpr int CPG = D / G;   // value groups per token
  static_assert(G % 32 == 0, "group must be a multiple of 32");
  static_assert(REC % 16 == 0 && STAGE % 16 == 0, "bulk copies need 16-byte multiples");
  static_assert(WARP_B % 128 == 0, "warp areas stay 128-byte aligned");
};

// The stage axis and its cut into blocks; the same arithmetic runs on the
// host (planning, workspace size) and on the device.
//   stage s <  RZ : residual stage s % sr of unit s / sr            (cost cr)
//   stage s >= RZ : quantised stage (s - RZ) % sq of unit (s - RZ) / sq (cost cq)
// The residual zone comes first so that a unit's last partial (whose block
// finishes the unit) comes from the quantised zone, spread over many blocks.
// Block k owns the stages whose start cost c_s satisfies
// ceil(k C / n) <= c_s < ceil((k + 1) C / n); equivalently the block of stage
// s is floor(c_s n / C).  The host keeps n <= C / max(cq, cr), so every block
// owns at least one stage.  Segments along the axis: the residual part of
// unit u (id u), then the quantised part of unit u (id U + u).
struct Partition {
  int64_t ng;      // groups per unit
  int64_t RZ;      // stages in the residual zone = U * sr
  int64_t S_tot;   // all stages = RZ + U * sq
  int64_t cq, cr;  // cost of one quantised / residual stage
  int64_t C;       // total cost
  int U, sq, sr, nblk;

  __host__ __device__ int64_t cost(int64_t s) const { return s < RZ ? s * cr : RZ * cr + (s - RZ) * cq; }
  __host__ __device__ int64_t first(int k) const {
    if (k <= 0) return 0;
    if (k >= nblk) return S_tot;
    const int64_t T = (static_cast<int64_t>(k) * C + nblk - 1) / nblk;
    if (RZ > 0 && T <= (RZ - 1) * cr) return (T + cr - 1) / cr;
    const int64_t base = RZ * cr;
    if (T <= base) return RZ;
    const int64_t s = RZ + (T - base + cq - 1) / cq;
    return s < S_tot ? s : S_tot;
  }
  __host__ __device__ int block_of(int64_t s) const {
    const int64_t k = cost(s) * nblk / C;
    return k < nblk ? static_cast<int>(k) : nblk - 1;
  }
  __host__ __device__ int seg_of(int64_t s) const {
    return s < RZ ? static_cast<int>(s / sr) : U + static_cast<int>((s - RZ) / sq);
  }
  __host__ __device__ int64_t seg_begin(int seg) const {
    return seg < U ? static_cast<int64_t>(seg) * sr : RZ + static_cast<int64_t>(seg - U) * sq;
  }
  __host__ __device__ int64_t seg_end(int seg) const { return seg_begin(seg) + (seg < U ? sr : sq); }
};

struct QArgs {
  const uint8_t* rec;  // [U][ng][REC] group records
  const __nv_bfloat16* kr;
  const __nv_bfloat16* vr;
  const __nv_bfloat16* q;
  Partition P;
  int R, R_cap;
  int Hq, Hkv, g;
  int MAXS;  // partial slots per block
  float scale_log2;
  uint32_t* flags;
  float* part_o;      // [nblk * MAXS][g][D]
  float* part_ml;     // [nblk * MAXS][g][2]
  float* out;         // [B][Hq][D]
};

// ---- code extraction shared by the attention kernel and vc_debug_dequant
//
// Storage: the codes of a group of G tokens form one block in fragment-native
// order (include/vc.h): for each 16-token tile, lane L of the warp finds its
// NW 32-bit words at word (tile * 32 + L) * NW.  Words come in pairs (X_j,
// Y_j) covering TPW = 8 / bits channel tiles; a word holds two MMA registers
// ("first" in the low byte of each 16-bit half, "second" in the high byte),
// each register two codes (one per half), local tile i at bit position
// bits * i.
//
// A code reaches the tensor core as an fp16 SUBNORMAL: AND-ing a word with a
// mask that keeps one code per half at bit position pos (< 10) yields the
// fp16 value code * 2^(pos - 24) exactly, and the tensor cores multiply
// subnormal inputs exactly.  So a register costs one AND (the second
// register of a word also shares one shift).  The factors 2^(pos - 24) are
// folded into the query operand (keys) or undone per output row (values).
template <int BITS>
struct Frag {
  static constexpr int TPW = 8 / BITS;  // channel (key) or row (value) tiles per word
  static constexpr uint32_t BASE = BITS == 2 ? 0x00030003u : 0x000F000Fu;
  __device__ __forceinline__ static uint32_t mask(int i) { return BASE << (BITS * i); }
};

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

template <int N>
__device__ __forceinline__ void load_words(const uint32_t* p, uint32_t (&w)[N]) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int v = 0; v < N / 4; ++v) {
      const uint4 x = reinterpret_cast<const uint4*>(p)[v];
      w[4 * v] = x.x, w[4 * v + 1] = x.y, w[4 * v + 2] = x.z, w[4 * v + 3] = x.w;
    }
  } else {
    static_assert(N == 2, "two or a multiple of four words");
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    w[0] = x.x, w[1] = x.y;
  }
}

// the CPG words (one per value group) of a token pair
template <int CPG>
__device__ __forceinline__ void load_cpg(const uint32_t* p, uint32_t (&w)[CPG]) {
  if constexpr (CPG == 4) {
    const uint4 x = *reinterpret_cast<const uint4*>(p);
    w[0] = x.x, w[1] = x.y, w[2] = x.z, w[3] = x.w;
  } else if constexpr (CPG == 2) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    w[0] = x.x, w[1] = x.y;
  } else {
    w[0] = p[0];
  }
}

// Where this warp's next quantised stage to fetch lives: unit u, stage ls of
// that unit (both < 2^31: units are capped at 2^24, groups per unit at 2^30).
// Advancing by kQNW stages needs no division.
struct IssuePtr {
  int u, ls;
  __device__ void start(const Partition& P, int64_t s) {
    u = static_cast<int>(s / P.sq);
    ls = static_cast<int>(s - static_cast<int64_t>(u) * P.sq);
  }
  __device__ void advance(const Partition& P) {
    ls += kQNW;
    while (ls >= P.sq) {
      ls -= P.sq;
      ++u;
    }
  }
};

// One bulk copy of this warp's next quantised stage (at ip) into ring slot `slot`.
template <typename C>
__device__ __forceinline__ void issue_stage(const QArgs& a, unsigned char* ring, uint64_t* bars, int lane, int slot,
                                            const IssuePtr& ip) {
  const int64_t g0 = static_cast<int64_t>(ip.ls) * C::NG;
  const int64_t left = a.P.ng - g0;
  const uint32_t bytes = static_cast<uint32_t>((left < C::NG ? left : C::NG) * C::REC);
  if (lane == 0) {
    mbar_arrive_expect_tx(&bars[slot], bytes);
    bulk_g2s(ring + slot * C::STAGE, a.rec + (static_cast<int64_t>(ip.u) * a.P.ng + g0) * C::REC, bytes,
             &bars[slot]);
  }
}

// ----------------------------------------------------------- quantised part
//
// Two arrangements of the same arithmetic, chosen by the GQA group size g:
//
//   TokM (g <= 4): scores D[token][col] = codes[token][chan] x qfold[chan][col]
//     with col = 2 * head + part (part 0 = high, 1 = low fp16 part of q*s),
//     so the 4 heads' two parts fill the MMA's N = 8.  The softmax weights
//     of a lane (one head, four tokens) are moved into the value MMA's B
//     layout with movmatrix (8x8 transposes in registers).
//   HeadM (4 < g <= 8): scores D[row][token] = qfold[row][chan] x
//     codes[chan][token] with row = head (high part) or 8 + head (low part),
//     so the 8 heads' two parts fill M = 16; a lane ends up holding the
//     weights of one head for the token pairs the value MMA's B operand
//     needs, and no data moves between lanes.
//
// Both: values D[chan][col] = codes^T[chan][token] x pfold[token][col].
// The softmax weights p (<= 2^kLazyLog2 by the lazy running maximum) are
// rounded once to fp16 (p~) for the value side; the softmax denominator
// sums the fp32 p.  p~ * s is split into an fp16 high part and the exact
// fp16 remainder (one fma), so the value operand carries ~22 bits.

constexpr float kLazy = 8.f;  // raise the running max only when a score exceeds it by > 2^8

__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(x));
  return d;
}

// a * b - c, f16x2
__device__ __forceinline__ uint32_t hfms2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("{\n\t.reg .b32 t;\n\tneg.f16x2 t, %3;\n\tfma.rn.f16x2 %0, %1, %2, t;\n\t}\n"
      : "=r"(d)
      : "r"(a), "r"(b), "r"(c));
  return d;
}

template <int BITS>
__device__ __forceinline__ uint32_t zscale(uint32_t z, int i) {
  // z * 2^(bits i) in fp16 (exact while |z| 2^(bits i) stays below 65504)
  if (i == 0) return z;
  const uint32_t f2 = static_cast<uint32_t>(15 + BITS * i) << 10;
  return hmul2(z, f2 | (f2 << 16));
}

template <int BITS, int G, int D>
struct TokM {
  using F = Frag<BITS>;
  static constexpr int KT = D / 16, TPW = F::TPW, NW = 2 * KT / TPW, MT = G / 16, CPG = D / G;
  static constexpr int HEADS = 4;
  uint32_t qs[KT][2];  // q * 2^-(bits i), negated in low-part lanes
  uint32_t qm[KT][2];  // q * 2^-(bits i) in low-part lanes, 0 in high-part lanes
  float acc[KT][4];    // D[channel][col]
  float vb[4];         // value zero-point term: D[value group][col]
  float m_run, m_lim, l_run;

  __device__ __forceinline__ void init(const QArgs& a, int b, int h, int lane) {
    const int gid = lane >> 2, tig = lane & 3, part = gid & 1;
    const int hh = gid >> 1;
    const bool hv = hh < a.g;
    const __nv_bfloat16* qp = a.q + (static_cast<size_t>(b) * a.Hq + h * a.g + (hv ? hh : 0)) * D;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
      const float f = pow2i(-BITS * (kt % TPW));
      const float2 lo = unpack_bf2(*reinterpret_cast<const uint32_t*>(qp + kt * 16 + 2 * tig));
      const float2 hi = unpack_bf2(*reinterpret_cast<const uint32_t*>(qp + kt * 16 + 8 + 2 * tig));
      const uint32_t q0 = hv ? pack_h2(lo.x * f, lo.y * f) : 0u;
      const uint32_t q1 = hv ? pack_h2(hi.x * f, hi.y * f) : 0u;
      qs[kt][0] = part ? q0 ^ 0x80008000u : q0;
      qs[kt][1] = part ? q1 ^ 0x80008000u : q1;
      qm[kt][0] = part ? q0 : 0u;
      qm[kt][1] = part ? q1 : 0u;
    }
#pragma unroll
    for (int mc = 0; mc < KT; ++mc) acc[mc][0] = acc[mc][1] = acc[mc][2] = acc[mc][3] = 0.f;
    vb[0] = vb[1] = vb[2] = vb[3] = 0.f;
    m_run = -INFINITY;
    m_lim = -INFINITY;
    l_run = 0.f;
  }

  // One group record at rs (shared memory).
  __device__ __forceinline__ void group(const unsigned char* rs, int lane, float scl, float sl2) {
    constexpr unsigned FULL = 0xffffffffu;
    using C = QCfg<BITS, G, D, 1>;
    const int gid = lane >> 2, tig = lane & 3;
    const uint32_t* kcw = reinterpret_cast<const uint32_t*>(rs);
    const uint32_t* vcw = reinterpret_cast<const uint32_t*>(rs + C::OFF_VC);
    const uint4* skw = reinterpret_cast<const uint4*>(rs + C::OFF_SK) + tig * (KT / 2);
    const uint4* zkw = reinterpret_cast<const uint4*>(rs + C::OFF_ZK) + tig * (KT / 2);
    const uint32_t* sv32 = reinterpret_cast<const uint32_t*>(rs + C::OFF_SV);  // [G/2][CPG] token pairs
    const uint32_t* zv32 = reinterpret_cast<const uint32_t*>(rs + C::OFF_ZV);

    // (1) scores: per channel tile kt the key scales are folded into q right
    //     before use (high part in part-0 columns, low part in part-1
    //     columns); the zero-point term sum_c q_c z_c is an MMA of the zeros
    //     (times 2^(bits i), exact) against the signed q in the high columns.
    float sc[MT][4], kb[4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
    kb[0] = kb[1] = kb[2] = kb[3] = 0.f;
#pragma unroll
    for (int j = 0; j < NW / 2; ++j) {
      uint32_t X[MT], Y[MT], XS[MT], YS[MT];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const uint2 w = *reinterpret_cast<const uint2*>(kcw + (mt * 32 + lane) * NW + 2 * j);
        X[mt] = w.x, Y[mt] = w.y, XS[mt] = w.x >> 8, YS[mt] = w.y >> 8;
      }
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        const int kt = TPW * j + i;
        const uint4 s4 = skw[kt >> 1];
        const uint32_t sA = (kt & 1) ? s4.z : s4.x, sC = (kt & 1) ? s4.w : s4.y;
        const uint32_t fa = hfma2(qm[kt][0], sA, hmul2(qs[kt][0], sA));
        const uint32_t fc = hfma2(qm[kt][1], sC, hmul2(qs[kt][1], sC));
        const uint32_t m = F::mask(i);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const uint32_t af[4] = {X[mt] & m, XS[mt] & m, Y[mt] & m, YS[mt] & m};
          mma_f16(sc[mt], af, fa, fc);
        }
        const uint4 z4 = zkw[kt >> 1];
        const uint32_t z0 = zscale<BITS>((kt & 1) ? z4.z : z4.x, i);
        const uint32_t z8 = zscale<BITS>((kt & 1) ? z4.w : z4.y, i);
        const uint32_t za[4] = {z0, z0, z8, z8};
        mma_f16(kb, za, qs[kt][0], qs[kt][1]);
      }
    }

    // (2) softmax of head tig over the lane's tokens 16 mt + gid (+8); the
    //     scores sit in the 2^-24 domain of the code encoding
    const float kzs = kb[0] * sl2;
    float x[MT][2];
    float t = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      x[mt][0] = fmaf(sc[mt][0] + sc[mt][1], scl, kzs);
      x[mt][1] = fmaf(sc[mt][2] + sc[mt][3], scl, kzs);
      t = fmaxf(t, fmaxf(x[mt][0], x[mt][1]));
    }
    t = warp_max_xor(t, 4);
    t = warp_max_xor(t, 8);
    t = warp_max_xor(t, 16);
    if (__any_sync(FULL, t > m_lim)) {
      const float m_new = fmaxf(m_run, t);
      const float alpha = ex2(m_run - m_new);
      m_run = m_new;
      m_lim = m_new + kLazy;
      l_run *= alpha;
#pragma unroll
      for (int mc = 0; mc < KT; ++mc) {
        acc[mc][0] *= alpha;
        acc[mc][1] *= alpha;
        acc[mc][2] *= alpha;
        acc[mc][3] *= alpha;
      }
      vb[0] *= alpha;
      vb[1] *= alpha;
      vb[2] *= alpha;
      vb[3] *= alpha;
    }
    // p~ into the value MMA's B layout: an 8x8 block [token][col] holds
    // (p, -p) in a head's (high, low) columns for PA and (0, p) for PB;
    // after the transpose lane (gid, tig) holds its column's entries for
    // tokens 2 tig, 2 tig + 1 of the block.
    uint32_t PA[MT][2], PB[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float p = ex2(x[mt][hf] - m_run);
        l_run += p;
        PA[mt][hf] = movm_t(pack_h2(p, -p));
        PB[mt][hf] = movm_t(pack_h2(0.f, p));
      }
    }

    // (3) P . V: per 16-token tile, the folded operand of value group cg is
    //     high (part 0 columns: 0 + fp16(p~ s)) or low (part 1 columns:
    //     p~ s - fp16(p~ s), exact) -- the same two instructions in every lane
#pragma unroll
    for (int ktt = 0; ktt < MT; ++ktt) {
      uint32_t s01[CPG], s89[CPG];
      load_cpg<CPG>(sv32 + (ktt * 8 + tig) * CPG, s01);
      load_cpg<CPG>(sv32 + (ktt * 8 + 4 + tig) * CPG, s89);
      {
        // value zero-point term: A = z_v^T (row = value group gid), B = p~ (low columns)
        uint32_t za[4] = {0u, 0u, 0u, 0u};
        if (gid < CPG) {
          za[0] = zv32[(ktt * 8 + tig) * CPG + gid];
          za[2] = zv32[(ktt * 8 + 4 + tig) * CPG + gid];
        }
        mma_f16(vb, za, PB[ktt][0], PB[ktt][1]);
      }
      uint32_t pf0 = 0u, pf1 = 0u;
#pragma unroll
      for (int j = 0; j < NW / 2; ++j) {
        const uint2 w = *reinterpret_cast<const uint2*>(vcw + (ktt * 32 + lane) * NW + 2 * j);
        const uint32_t X = w.x, Y = w.y, XS = w.x >> 8, YS = w.y >> 8;
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
          const int mc = TPW * j + i;
          const int cg = mc * 16 / G;
          if (mc == 0 || (mc - 1) * 16 / G != cg) {
            pf0 = hfma2(PB[ktt][0], s01[cg], hmul2(PA[ktt][0], s01[cg]));
            pf1 = hfma2(PB[ktt][1], s89[cg], hmul2(PA[ktt][1], s89[cg]));
          }
          const uint32_t m = F::mask(i);
          const uint32_t af[4] = {X & m, Y & m, XS & m, YS & m};
          mma_f16(acc[mc], af, pf0, pf1);
        }
      }
    }
  }

  // This warp's state -> its slot (natural channel order, unnormalised).
  __device__ __forceinline__ void store(const QArgs& a, int warp, int lane, bool ok, float* st_o, float* st_ml) {
    constexpr unsigned FULL = 0xffffffffu;
    const int gid = lane >> 2, tig = lane & 3;
    const int hh = tig;
    float l = l_run;
    l += __shfl_xor_sync(FULL, l, 4);
    l += __shfl_xor_sync(FULL, l, 8);
    l += __shfl_xor_sync(FULL, l, 16);
    const float vbs = vb[1];  // value-zero term of group gid, head tig (low column)
#pragma unroll
    for (int mc = 0; mc < KT; ++mc) {
      const int cg = mc * 16 / G;
      const float zb = __shfl_sync(FULL, vbs, cg * 4 + tig);
      const float uf = pow2i(24 - BITS * (mc % TPW));  // undo the code encoding of this tile
      if (hh < a.g) {
        float* wo = st_o + (warp * HEADS + hh) * D + mc * 16 + gid;
        wo[0] = (acc[mc][0] + acc[mc][1]) * uf + zb;
        wo[8] = (acc[mc][2] + acc[mc][3]) * uf + zb;
      }
    }
    if (hh < a.g && gid == 0) {
      st_ml[(warp * HEADS + hh) * 2] = ok ? m_run : -INFINITY;
      st_ml[(warp * HEADS + hh) * 2 + 1] = ok ? l : 0.f;
    }
  }
};

template <int BITS, int G, int D>
struct HeadM {
  using F = Frag<BITS>;
  static constexpr int KT = D / 16, TPW = F::TPW, NW = 2 * KT / TPW, MT = G / 16, CPG = D / G;
  static constexpr int HEADS = 8;
  uint32_t q2[KT][2];  // head gid: q * 2^-(bits i), channel pairs (2 tig, +1), (2 tig + 8, +9)
  float acc[KT][4];    // D[channel][head]: (channel gid, heads 2 tig, 2 tig + 1), channel + 8
  float vb[4];         // D[value group][head]
  float m_run, m_lim, l_run;  // head gid

  __device__ __forceinline__ void init(const QArgs& a, int b, int h, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
    const bool hv = gid < a.g;
    const __nv_bfloat16* qp = a.q + (static_cast<size_t>(b) * a.Hq + h * a.g + (hv ? gid : 0)) * D;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
      const float f = pow2i(-BITS * (kt % TPW));
      const float2 lo = unpack_bf2(*reinterpret_cast<const uint32_t*>(qp + kt * 16 + 2 * tig));
      const float2 hi = unpack_bf2(*reinterpret_cast<const uint32_t*>(qp + kt * 16 + 8 + 2 * tig));
      q2[kt][0] = hv ? pack_h2(lo.x * f, lo.y * f) : 0u;
      q2[kt][1] = hv ? pack_h2(hi.x * f, hi.y * f) : 0u;
    }
#pragma unroll
    for (int mc = 0; mc < KT; ++mc) acc[mc][0] = acc[mc][1] = acc[mc][2] = acc[mc][3] = 0.f;
    vb[0] = vb[1] = vb[2] = vb[3] = 0.f;
    m_run = -INFINITY;
    m_lim = -INFINITY;
    l_run = 0.f;
  }

  __device__ __forceinline__ void group(const unsigned char* rs, int lane, float scl, float sl2) {
    constexpr unsigned FULL = 0xffffffffu;
    using C = QCfg<BITS, G, D, 2>;
    const int gid = lane >> 2, tig = lane & 3;
    const uint32_t* kcw = reinterpret_cast<const uint32_t*>(rs);
    const uint32_t* vcw = reinterpret_cast<const uint32_t*>(rs + C::OFF_VC);
    const uint4* skw = reinterpret_cast<const uint4*>(rs + C::OFF_SK) + tig * (KT / 2);
    const uint4* zkw = reinterpret_cast<const uint4*>(rs + C::OFF_ZK) + tig * (KT / 2);
    const uint32_t* sv32 = reinterpret_cast<const uint32_t*>(rs + C::OFF_SV);
    const uint32_t* zv32 = reinterpret_cast<const uint32_t*>(rs + C::OFF_ZV);

    // (1) scores, n-tile nt = tokens 8 nt .. 8 nt + 7: rows gid (high part of
    //     head gid's q*s) and gid + 8 (its low part); zero-point term from
    //     rows = q (unfolded) against the zeros broadcast over the columns
    float sc[2 * MT][4], kb[4];
#pragma unroll
    for (int n = 0; n < 2 * MT; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
    kb[0] = kb[1] = kb[2] = kb[3] = 0.f;
#pragma unroll
    for (int j = 0; j < NW / 2; ++j) {
      uint32_t fa[TPW][4];
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        const int kt = TPW * j + i;
        const uint4 s4 = skw[kt >> 1];
        const uint32_t sA = (kt & 1) ? s4.z : s4.x, sC = (kt & 1) ? s4.w : s4.y;
        fa[i][0] = hmul2(q2[kt][0], sA);
        fa[i][1] = hfms2(q2[kt][0], sA, fa[i][0]);
        fa[i][2] = hmul2(q2[kt][1], sC);
        fa[i][3] = hfms2(q2[kt][1], sC, fa[i][2]);
        const uint4 z4 = zkw[kt >> 1];
        const uint32_t z0 = zscale<BITS>((kt & 1) ? z4.z : z4.x, i);
        const uint32_t z8 = zscale<BITS>((kt & 1) ? z4.w : z4.y, i);
        const uint32_t qa[4] = {q2[kt][0], 0u, q2[kt][1], 0u};
        mma_f16(kb, qa, z0, z8);
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const uint2 w = *reinterpret_cast<const uint2*>(kcw + (mt * 32 + lane) * NW + 2 * j);
        const uint32_t X = w.x, Y = w.y, XS = w.x >> 8, YS = w.y >> 8;
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
          const uint32_t m = F::mask(i);
          mma_f16(sc[2 * mt], fa[i], X & m, Y & m);
          mma_f16(sc[2 * mt + 1], fa[i], XS & m, YS & m);
        }
      }
    }

    // (2) softmax of head gid over tokens 8 n + 2 tig, +1
    const float kzs = kb[0] * sl2;
    float y[2 * MT][2];
    float t = -INFINITY;
#pragma unroll
    for (int n = 0; n < 2 * MT; ++n) {
      y[n][0] = sc[n][0] + sc[n][2];
      y[n][1] = sc[n][1] + sc[n][3];
      t = fmaxf(t, fmaxf(y[n][0], y[n][1]));
    }
    t = fmaxf(t, __shfl_xor_sync(FULL, t, 1));
    t = fmaxf(t, __shfl_xor_sync(FULL, t, 2));
    t = fmaf(t, scl, kzs);
    if (__any_sync(FULL, t > m_lim)) {
      const float m_new = fmaxf(m_run, t);
      const float alpha = ex2(m_run - m_new);
      m_run = m_new;
      m_lim = m_new + kLazy;
      l_run *= alpha;
      // acc and vb columns are heads 2 tig, 2 tig + 1: fetch their factors
      const float a0 = __shfl_sync(FULL, alpha, 8 * tig);
      const float a1 = __shfl_sync(FULL, alpha, 8 * tig + 4);
#pragma unroll
      for (int mc = 0; mc < KT; ++mc) {
        acc[mc][0] *= a0;
        acc[mc][1] *= a1;
        acc[mc][2] *= a0;
        acc[mc][3] *= a1;
      }
      vb[0] *= a0;
      vb[1] *= a1;
      vb[2] *= a0;
      vb[3] *= a1;
    }
    const float off = kzs - m_run;
    uint32_t P[2 * MT];
#pragma unroll
    for (int n = 0; n < 2 * MT; ++n) {
      const float p0 = ex2(fmaf(y[n][0], scl, off)), p1 = ex2(fmaf(y[n][1], scl, off));
      l_run += p0 + p1;
      P[n] = pack_h2(p0, p1);
    }

    // (3) P . V: B = p~ * s of head gid for tokens (2 tig, +1) and (2 tig + 8, +9),
    //     high part and exact low part as two MMAs into the same accumulator
#pragma unroll
    for (int ktt = 0; ktt < MT; ++ktt) {
      uint32_t s01[CPG], s89[CPG];
      load_cpg<CPG>(sv32 + (ktt * 8 + tig) * CPG, s01);
      load_cpg<CPG>(sv32 + (ktt * 8 + 4 + tig) * CPG, s89);
      {
        uint32_t za[4] = {0u, 0u, 0u, 0u};
        if (gid < CPG) {
          za[0] = zv32[(ktt * 8 + tig) * CPG + gid];
          za[2] = zv32[(ktt * 8 + 4 + tig) * CPG + gid];
        }
        mma_f16(vb, za, P[2 * ktt], P[2 * ktt + 1]);
      }
      uint32_t h0 = 0u, h1 = 0u, l0 = 0u, l1 = 0u;
#pragma unroll
      for (int j = 0; j < NW / 2; ++j) {
        const uint2 w = *reinterpret_cast<const uint2*>(vcw + (ktt * 32 + lane) * NW + 2 * j);
        const uint32_t X = w.x, Y = w.y, XS = w.x >> 8, YS = w.y >> 8;
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
          const int mc = TPW * j + i;
          const int cg = mc * 16 / G;
          if (mc == 0 || (mc - 1) * 16 / G != cg) {
            h0 = hmul2(P[2 * ktt], s01[cg]);
            l0 = hfms2(P[2 * ktt], s01[cg], h0);
            h1 = hmul2(P[2 * ktt + 1], s89[cg]);
            l1 = hfms2(P[2 * ktt + 1], s89[cg], h1);
          }
          const uint32_t m = F::mask(i);
          const uint32_t af[4] = {X & m, Y & m, XS & m, YS & m};
          mma_f16(acc[mc], af, h0, h1);
          mma_f16(acc[mc], af, l0, l1);
        }
      }
    }
  }

  __device__ __forceinline__ void store(const QArgs& a, int warp, int lane, bool ok, float* st_o, float* st_ml) {
    constexpr unsigned FULL = 0xffffffffu;
    const int gid = lane >> 2, tig = lane & 3;
    float l = l_run;
    l += __shfl_xor_sync(FULL, l, 1);
    l += __shfl_xor_sync(FULL, l, 2);
    const int h0 = 2 * tig, h1 = 2 * tig + 1;
#pragma unroll
    for (int mc = 0; mc < KT; ++mc) {
      const int cg = mc * 16 / G;
      const float zb0 = __shfl_sync(FULL, vb[0], cg * 4 + tig);
      const float zb1 = __shfl_sync(FULL, vb[1], cg * 4 + tig);
      const float uf = pow2i(24 - BITS * (mc % TPW));
      if (h0 < a.g) {
        float* wo = st_o + (warp * HEADS + h0) * D + mc * 16 + gid;
        wo[0] = acc[mc][0] * uf + zb0;
        wo[8] = acc[mc][2] * uf + zb0;
      }
      if (h1 < a.g) {
        float* wo = st_o + (warp * HEADS + h1) * D + mc * 16 + gid;
        wo[0] = acc[mc][1] * uf + zb1;
        wo[8] = acc[mc][3] * uf + zb1;
      }
    }
    if (gid < a.g && tig == 0) {
      st_ml[(warp * HEADS + gid) * 2] = ok ? m_run : -INFINITY;
      st_ml[(warp * HEADS + gid) * 2 + 1] = ok ? l : 0.f;
    }
  }
};

// Processes this warp's stages of unit u's quantised segment (the prefetch
// pipeline runs on across segments) and leaves the warp's state in its slot.
template <int BITS, int G, int D, int NT>
__device__ __forceinline__ void quant_seg(const QArgs& a, unsigned char* ring, uint64_t* bars, int u, int64_t qs0,
                                          int my_nq, int& iq, int& issued, IssuePtr& ip, int& islot, int& cslot,
                                          uint32_t& cphase, bool& ok, float* st_o, float* st_ml) {
  using C = QCfg<BITS, G, D, NT>;
  using Body = std::conditional_t<NT == 1, TokM<BITS, G, D>, HeadM<BITS, G, D>>;
  constexpr unsigned FULL = 0xffffffffu;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = u / a.Hkv, h = u - b * a.Hkv;
  // the score MMAs accumulate scores * 2^-24; undo it together with the softmax scale
  const float scl = a.scale_log2 * 16777216.0f;
  Body body;
  body.init(a, b, h, lane);

  // this warp's stages of the segment: local stages ls0, ls0 + kQNW, ...
  // (qs: index inside the quantised zone; this warp's i-th one is qs0 + kQNW i)
  int n_seg = 0, ls0 = 0;
  {
    const int64_t seg_lo = static_cast<int64_t>(u) * a.P.sq, seg_hi = seg_lo + a.P.sq;
    const int64_t s_first = qs0 + static_cast<int64_t>(iq) * kQNW;
    if (iq < my_nq && s_first < seg_hi) {
      const int64_t n = (seg_hi - s_first + kQNW - 1) / kQNW;
      n_seg = n < my_nq - iq ? static_cast<int>(n) : my_nq - iq;
      ls0 = static_cast<int>(s_first - seg_lo);
    }
  }
#pragma unroll 1
  for (int kk = 0; kk < n_seg; ++kk, ++iq) {
    if (!ok) continue;
    if (issued < my_nq && issued <= iq + C::NST - 1) {
      fence_proxy_async_smem();
      __syncwarp();
      issue_stage<C>(a, ring, bars, lane, islot, ip);
      ip.advance(a.P);
      ++issued;
      islot = islot + 1 == C::NST ? 0 : islot + 1;
    }
    const int slot = cslot;  // = iq mod NST, with phase cphase = (iq / NST) mod 2
    cslot = cslot + 1 == C::NST ? 0 : cslot + 1;
    const uint32_t phase = cphase;
    cphase ^= cslot == 0 ? 1u : 0u;
    if (!__all_sync(FULL, mbar_wait_bounded(&bars[slot], phase, a.flags))) {  // warp-uniform
      ok = false;
      for (int k = iq; k < issued; ++k) mbar_wait_bounded(&bars[k % C::NST], (k / C::NST) & 1, nullptr, 100000000ull);
      continue;
    }
    if constexpr (C::NG == 1) {
      body.group(ring + slot * C::STAGE, lane, scl, a.scale_log2);
    } else {
      const int64_t g0 = static_cast<int64_t>(ls0 + kk * kQNW) * C::NG;
      const int n_here = a.P.ng - g0 < C::NG ? static_cast<int>(a.P.ng - g0) : C::NG;
#pragma unroll 1
      for (int gi = 0; gi < n_here; ++gi) body.group(ring + slot * C::STAGE + gi * C::REC, lane, scl, a.scale_log2);
    }
    __syncwarp();
  }
  body.store(a, warp, lane, ok, st_o, st_ml);
}

// -------------------------------------------------------- bf16 residual part
// This warp's residual stages of unit u (16 rows each, one bulk copy per row,
// not pipelined; the residual is a few percent of the bytes).  Leaves the
// warp's state in its slot.
template <int D, int NT, int HEADS>
__device__ __forceinline__ void residual_seg(const QArgs& a, unsigned char* ring, float* P_s, uint64_t* bar, int& rph, int u,
                             int64_t first_s, int64_t end_s, int64_t seg_b, bool& ok, float* st_o, float* st_ml) {
  constexpr int KT = D / 16;
  constexpr int ROW_B = D * 2;
  constexpr unsigned FULL = 0xffffffffu;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int part = gid & 1;
  const int b = u / a.Hkv, h = u - b * a.Hkv;
  const __nv_bfloat16* kr = a.kr + static_cast<size_t>(u) * a.R_cap * D;
  const __nv_bfloat16* vr = a.vr + static_cast<size_t>(u) * a.R_cap * D;

  // query B fragments (bf16, natural channels): high columns = q, low = 0
  uint32_t qb[KT][NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hh = nt * 4 + (gid >> 1);
    const bool hv = hh < a.g && part == 0;
    const __nv_bfloat16* qp = a.q + (static_cast<size_t>(b) * a.Hq + h * a.g + (hh < a.g ? hh : 0)) * D;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
      qb[kt][nt][0] = hv ? *reinterpret_cast<const uint32_t*>(qp + kt * 16 + 2 * tig) : 0u;
      qb[kt][nt][1] = hv ? *reinterpret_cast<const uint32_t*>(qp + kt * 16 + 8 + 2 * tig) : 0u;
    }
  }
  float acc[KT][NT][4];
  float m_run[NT], l_run[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt] = -INFINITY;
    l_run[nt] = 0.f;
#pragma unroll
    for (int mc = 0; mc < KT; ++mc) acc[mc][nt][0] = acc[mc][nt][1] = acc[mc][nt][2] = acc[mc][nt][3] = 0.f;
  }
  for (int64_t s = first_s; s < end_s && ok; s += kQNW) {
    const int t0 = static_cast<int>(s - seg_b) * kResRows;
    const int nv = a.R - t0 < kResRows ? a.R - t0 : kResRows;  // rows of this tile inside the window
    fence_proxy_async_smem();
    __syncwarp();
    if (nv < kResRows) {
      // V rows the copy does not fill must read as zeros (their p is 0, but
      // whatever a buffer holds past the window must not reach the MMA)
      uint4* vz = reinterpret_cast<uint4*>(ring + (kResRows + nv) * ROW_B);
      for (int e = lane; e < (kResRows - nv) * ROW_B / 16; e += 32) vz[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    // the tile's K rows and V rows are contiguous: two bulk copies
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, 2u * nv * ROW_B);
      bulk_g2s(ring, kr + static_cast<size_t>(t0) * D, nv * ROW_B, bar);
      bulk_g2s(ring + kResRows * ROW_B, vr + static_cast<size_t>(t0) * D, nv * ROW_B, bar);
    }
    __syncwarp();
    if (!__all_sync(FULL, mbar_wait_bounded(bar, rph & 1, a.flags))) {  // warp-uniform
      ok = false;
      mbar_wait_bounded(bar, rph & 1, nullptr, 100000000ull);
      ++rph;
      break;
    }
    ++rph;
    const unsigned char* Ks = ring;
    const unsigned char* Vs = ring + kResRows * ROW_B;
    const int mi = lane >> 3, ri = lane & 7;
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
      // A = K rows (tokens x channels): matrices (rows 0-7,k 0-7) (8-15,0-7) (0-7,8-15) (8-15,8-15)
      uint32_t af[4];
      ldsm_x4(af, Ks + (ri + (mi & 1) * 8) * ROW_B + (kt * 16 + (mi >> 1) * 8) * 2);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16(sc[nt], af, qb[kt][nt][0], qb[kt][nt][1]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const bool v0 = t0 + gid < a.R, v1 = t0 + gid + 8 < a.R;
      float x[2] = {v0 ? (sc[nt][0] + sc[nt][1]) * a.scale_log2 : -INFINITY,
                    v1 ? (sc[nt][2] + sc[nt][3]) * a.scale_log2 : -INFINITY};
      float t = fmaxf(x[0], x[1]);
      t = warp_max_xor(t, 4);
      t = warp_max_xor(t, 8);
      t = warp_max_xor(t, 16);
      const float m_new = fmaxf(m_run[nt], t);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = ex2(m_run[nt] - m_use);
      x[0] = ex2(x[0] - m_use);
      x[1] = ex2(x[1] - m_use);
      l_run[nt] = l_run[nt] * alpha + x[0] + x[1];
      m_run[nt] = m_new;
#pragma unroll
      for (int mc = 0; mc < KT; ++mc) {
        acc[mc][nt][0] *= alpha;
        acc[mc][nt][1] *= alpha;
        acc[mc][nt][2] *= alpha;
        acc[mc][nt][3] *= alpha;
      }
      float* ps = P_s + (nt * 4 + tig) * 16 + gid;
      ps[0] = x[0];
      ps[8] = x[1];
    }
    __syncwarp();
    // B = P as bf16 high/low columns; A = V^T via transposed ldmatrix
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float* pp = P_s + (nt * 4 + (gid >> 1)) * 16 + 2 * tig;
      const float2 p01 = *reinterpret_cast<const float2*>(pp);
      const float2 p89 = *reinterpret_cast<const float2*>(pp + 8);
      const uint32_t h01 = pack_bf2(p01.x, p01.y), h89 = pack_bf2(p89.x, p89.y);
      const float2 f01 = unpack_bf2(h01), f89 = unpack_bf2(h89);
      pb[nt][0] = part ? pack_bf2(p01.x - f01.x, p01.y - f01.y) : h01;
      pb[nt][1] = part ? pack_bf2(p89.x - f89.x, p89.y - f89.y) : h89;
    }
#pragma unroll
    for (int mc = 0; mc < KT; ++mc) {
      // A[chan][token]: matrices (ch 0-7, tok 0-7) (ch 8-15, tok 0-7) (ch 0-7, tok 8-15) (ch 8-15, tok 8-15)
      uint32_t af[4];
      ldsm_x4_t(af, Vs + (ri + (mi >> 1) * 8) * ROW_B + (mc * 16 + (mi & 1) * 8) * 2);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[mc][nt], af, pb[nt][0], pb[nt][1]);
    }
    __syncwarp();
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hh = nt * 4 + tig;
    float l = l_run[nt];
    l += __shfl_xor_sync(FULL, l, 4);
    l += __shfl_xor_sync(FULL, l, 8);
    l += __shfl_xor_sync(FULL, l, 16);
    if (hh < a.g) {
#pragma unroll
      for (int mc = 0; mc < KT; ++mc) {
        float* wo = st_o + (warp * HEADS + hh) * D + mc * 16 + gid;
        wo[0] = acc[mc][nt][0] + acc[mc][nt][1];
        wo[8] = acc[mc][nt][2] + acc[mc][nt][3];
      }
      if (gid == 0) {
        st_ml[(warp * HEADS + hh) * 2] = ok ? m_run[nt] : -INFINITY;
        st_ml[(warp * HEADS + hh) * 2 + 1] = ok ? l : 0.f;
      }
    }
  }
}

// Number of block partials of unit u and the slot of partial p of it.  A
// unit's partials are those of its residual segment (blocks block_of(begin)
// .. block_of(end - 1)) followed by those of its quantised segment.  Every
// block after the first one of a segment starts inside it, so its local
// segment index is 0; only the first block's index needs computing.
struct UnitPartials {
  int seg[2];
  int kb[2];
  int cnt[2];
  int loc0[2];
  __device__ void init(const Partition& P, int u) {
    int n = 0;
    if (P.sr > 0) seg[n++] = u;
    if (P.sq > 0) seg[n++] = P.U + u;
    for (int i = 0; i < 2; ++i) {
      if (i < n) {
        kb[i] = P.block_of(P.seg_begin(seg[i]));
        cnt[i] = P.block_of(P.seg_end(seg[i]) - 1) - kb[i] + 1;
        loc0[i] = seg[i] - P.seg_of(P.first(kb[i]));
      } else {
        seg[i] = 0, kb[i] = 0, cnt[i] = 0, loc0[i] = 0;
      }
    }
  }
  __device__ int total() const { return cnt[0] + cnt[1]; }
  __device__ int64_t slot(int maxs, int p) const {
    const int i = p < cnt[0] ? 0 : 1;
    const int pl = i ? p - cnt[0] : p;
    return static_cast<int64_t>(kb[i] + pl) * maxs + (pl == 0 ? loc0[i] : 0);
  }
};

// Block-wide: merges the kQNW warp states of segment `seg` (local index j of
// block k) into the block's partial of that segment.
template <int D, int HEADS>
__device__ __forceinline__ void merge_segment(const QArgs& a, int k, int j, const float* st_o, const float* st_ml,
                                           float* mw) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int g = a.g;
  float* wts = mw;               // [kQNW][HEADS]
  float* ML = mw + kQNW * HEADS;  // [HEADS][2]
  for (int r = tid; r < g; r += nthr) {
    float M = -INFINITY;
    for (int w = 0; w < kQNW; ++w) M = fmaxf(M, st_ml[(w * HEADS + r) * 2]);
    float L = 0.f;
    for (int w = 0; w < kQNW; ++w) {
      const float mw_ = st_ml[(w * HEADS + r) * 2];
      const float sc = (mw_ == -INFINITY) ? 0.f : ex2(mw_ - M);
      wts[w * HEADS + r] = sc;
      L += sc * st_ml[(w * HEADS + r) * 2 + 1];
    }
    ML[2 * r] = M;
    ML[2 * r + 1] = L;
  }
  __syncthreads();
  const int64_t slot = static_cast<int64_t>(k) * a.MAXS + j;
  float* po = a.part_o + slot * g * D;
  float* pml = a.part_ml + slot * g * 2;
  for (int e = tid; e < g * D; e += nthr) {
    const int r = e / D, d = e - r * D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kQNW; ++w) acc += wts[w * HEADS + r] * st_o[(w * HEADS + r) * D + d];
    po[e] = acc;
  }
  for (int r = tid; r < g; r += nthr) {
    pml[2 * r] = ML[2 * r];
    pml[2 * r + 1] = ML[2 * r + 1];
  }
  __syncthreads();  // the warp slots are reused by the next segment
}

// Merges every unit's block partials into out.  One block of 128 threads per
// (unit, head r): warp w takes partials w, w + 4, ...; each lane keeps a
// running online-softmax merge (M, L, D/32 channels) of them, loading a
// partial's (m, l) and its channel slice together (independent loads, one
// round trip); the four warp states are then merged through shared memory.
struct CArgs {
  Partition P;
  int MAXS, g, Hq, Hkv;
  const float* part_o;
  const float* part_ml;
  float* out;
};

template <int D>
__global__ void __launch_bounds__(128) combine_kernel(CArgs a) {
  __shared__ float wsum[4][D];
  __shared__ float wml[4][2];
  // launched as a programmatic dependent of draft_quant_kernel: wait until that
  // grid has completed and its partials are visible
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int u = blockIdx.x, r = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = a.g;
  UnitPartials up;
  up.init(a.P, u);
  const int np = up.total();
  constexpr int PER = D / 32;  // channels per lane
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float M = -INFINITY, L = 0.f;
  for (int p0 = warp; p0 < np; p0 += 8) {  // two partials of this warp per trip
    float v[2][PER];
    float2 ml[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int p = p0 + 4 * t;
      if (p < np) {
        const int64_t slot = up.slot(a.MAXS, p);
        ml[t] = *reinterpret_cast<const float2*>(a.part_ml + slot * g * 2 + 2 * r);
        const float* src = a.part_o + (slot * g + r) * D + lane * PER;
        if constexpr (PER == 4) {
          const float4 x = *reinterpret_cast<const float4*>(src);
          v[t][0] = x.x, v[t][1] = x.y, v[t][2] = x.z, v[t][3] = x.w;
        } else {
          const float2 x = *reinterpret_cast<const float2*>(src);
          v[t][0] = x.x, v[t][1] = x.y;
        }
      } else {
        ml[t] = make_float2(-INFINITY, 0.f);
#pragma unroll
        for (int i = 0; i < PER; ++i) v[t][i] = 0.f;
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (ml[t].x == -INFINITY) continue;
      const float Mn = fmaxf(M, ml[t].x);
      const float ro = M == -INFINITY ? 0.f : ex2(M - Mn);
      const float rn = ex2(ml[t].x - Mn);
      L = L * ro + ml[t].y * rn;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = acc[i] * ro + v[t][i] * rn;
      M = Mn;
    }
  }
  if (lane == 0) {
    wml[warp][0] = M;
    wml[warp][1] = L;
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) wsum[warp][lane * PER + i] = acc[i];
  __syncthreads();
  float Mb = -INFINITY;
#pragma unroll
  for (int w = 0; w < 4; ++w) Mb = fmaxf(Mb, wml[w][0]);
  float f[4], Lb = 0.f;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    f[w] = wml[w][0] == -INFINITY ? 0.f : ex2(wml[w][0] - Mb);
    Lb += f[w] * wml[w][1];
  }
  const int b = u / a.Hkv, h = u - b * a.Hkv;
  float* o = a.out + (static_cast<size_t>(b) * a.Hq + h * g + r) * D;
  for (int d = tid; d < D; d += 128) {
    const float t = (f[0] * wsum[0][d] + f[1] * wsum[1][d]) + (f[2] * wsum[2][d] + f[3] * wsum[3][d]);
    o[d] = Lb > 0.f ? t / Lb : 0.f;
  }
}

template <int BITS, int G, int D, int NT>
__global__ void __launch_bounds__(kQNW * 32, (NT == 1 ? 4 : 3)) draft_quant_kernel(QArgs a) {
  using C = QCfg<BITS, G, D, NT>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x;
  const Partition& P = a.P;
  // let the combine grid be scheduled as this grid's blocks retire (it waits
  // for this grid's completion before reading anything)
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int64_t B0 = P.first(k), B1 = P.first(k + 1);
  if (B0 >= B1) return;  // the host sizes the grid so that this never happens
  const int seg0 = P.seg_of(B0), seg1 = P.seg_of(B1 - 1);
  unsigned char* ring = smem + warp * C::WARP_B;
  float* P_res = reinterpret_cast<float*>(ring + C::RING);  // residual tile scores
  float* st_o = reinterpret_cast<float*>(smem + C::STATE_OFF);
  float* st_ml = reinterpret_cast<float*>(smem + C::ML_OFF);
  float* mw = reinterpret_cast<float*>(smem + C::MW_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF) + warp * (C::NST + 1);

  // this warp's quantised stages: s = sQ0 + kQNW i (s >= RZ), i < my_nq
  const int64_t lo_q = B0 > P.RZ ? B0 : P.RZ;
  const int64_t off_q = lo_q - B0;
  const int64_t sQ0 = B0 + warp + (off_q <= warp ? 0 : (off_q - warp + kQNW - 1) / kQNW) * kQNW;
  const int my_nq = sQ0 < B1 ? static_cast<int>((B1 - sQ0 + kQNW - 1) / kQNW) : 0;
  if (lane == 0)
    for (int s = 0; s <= C::NST; ++s) mbar_init(&bars[s], 1);
  fence_mbar_init();
  __syncwarp();
  bool ok = true, primed = false;
  int iq = 0, issued = 0, rph = 0, islot = 0, cslot = 0;
  uint32_t cphase = 0;
  IssuePtr ip;
  for (int seg = seg0; seg <= seg1; ++seg) {
    if (seg >= P.U) {
      if (!primed) {  // the ring is free of residual tiles from here on
        primed = true;
        fence_proxy_async_smem();
        __syncwarp();
        if (my_nq > 0) ip.start(P, sQ0 - P.RZ);
        while (issued < my_nq && issued < C::NST - 1) {
          issue_stage<C>(a, ring, bars, lane, islot, ip);
          ip.advance(P);
          ++issued;
          islot = islot + 1 == C::NST ? 0 : islot + 1;
        }
      }
      quant_seg<BITS, G, D, NT>(a, ring, bars, seg - P.U, sQ0 - P.RZ, my_nq, iq, issued, ip, islot, cslot, cphase,
                                ok, st_o, st_ml);
    } else {
      const int64_t sb = P.seg_begin(seg), se = P.seg_end(seg);
      const int64_t lo = sb > B0 ? sb : B0;
      const int64_t off = lo - B0;
      const int64_t i0 = off <= warp ? 0 : (off - warp + kQNW - 1) / kQNW;
      residual_seg<D, NT, C::HEADS>(a, ring, P_res, &bars[C::NST], rph, seg,
                                    B0 + warp + i0 * kQNW, se < B1 ? se : B1, sb, ok, st_o, st_ml);
    }
    __syncthreads();
    merge_segment<D, C::HEADS>(a, k, seg - seg0, st_o, st_ml, mw);
  }
}

// vc_debug_dequant: one warp per (group, unit).  The codes are extracted with
// the same word layout, masks and subnormal encoding the attention kernel
// uses (Frag), then dequantised with one fp32 FMA each and stored at their
// natural positions.
template <int BITS, int G, int D>
__global__ void __launch_bounds__(32) debug_dequant_kernel(const uint8_t* recs, int64_t ng, float* ko, float* vo) {
  using F = Frag<BITS>;
  using C = QCfg<BITS, G, D, 1>;
  constexpr int CPG = D / G, KT = D / 16, NW = 2 * KT / F::TPW;
  const int lane = threadIdx.x, gid = lane >> 2, tig = lane & 3;
  const int unit = blockIdx.y;
  const int64_t j = blockIdx.x;
  const uint8_t* rs = recs + (static_cast<size_t>(unit) * ng + j) * C::REC;
  const uint32_t* kc = reinterpret_cast<const uint32_t*>(rs);
  const uint32_t* vcw = reinterpret_cast<const uint32_t*>(rs + C::OFF_VC);
  const __half* sk = reinterpret_cast<const __half*>(rs + C::OFF_SK);
  const __half* zk = reinterpret_cast<const __half*>(rs + C::OFF_ZK);
  const __half* sv = reinterpret_cast<const __half*>(rs + C::OFF_SV);  // pair-interleaved
  const __half* zv = reinterpret_cast<const __half*>(rs + C::OFF_ZV);
  float* kou = ko + (static_cast<size_t>(unit) * ng + j) * G * D;
  float* vou = vo + (static_cast<size_t>(unit) * ng + j) * G * D;
  auto code = [](uint32_t reg, int half, float undo) {
    const float2 f = unpack_h2(reg);
    return (half ? f.y : f.x) * undo;
  };
  // fp16 slot of channel c in the key-parameter row: word tig*2KT + 2kt + h
  auto kslot = [](int c) {
    const int kt = c >> 4, h = (c >> 3) & 1, t = (c >> 1) & 3, e = c & 1;
    return 2 * (t * 2 * KT + 2 * kt + h) + e;
  };
  for (int tt = 0; tt < G / 16; ++tt) {
    for (int jw = 0; jw < NW / 2; ++jw) {
      const uint32_t X = kc[(tt * 32 + lane) * NW + 2 * jw], Y = kc[(tt * 32 + lane) * NW + 2 * jw + 1];
      for (int i = 0; i < F::TPW; ++i) {
        const int kt = F::TPW * jw + i;
        const uint32_t m = F::mask(i);
        const float undo = pow2i(24 - BITS * i);
        // reg0: token gid, channels 2tig+{0,1}; reg1: token gid+8; reg2/3: channels +8
        const uint32_t regs[4] = {X & m, (X >> 8) & m, Y & m, (Y >> 8) & m};
        for (int r = 0; r < 4; ++r)
          for (int e = 0; e < 2; ++e) {
            const int t = tt * 16 + gid + ((r & 1) ? 8 : 0);
            const int c = kt * 16 + 2 * tig + ((r & 2) ? 8 : 0) + e;
            kou[t * D + c] =
                __fmaf_rn(code(regs[r], e, undo), __half2float(sk[kslot(c)]), __half2float(zk[kslot(c)]));
          }
      }
    }
    for (int jw = 0; jw < NW / 2; ++jw) {
      const uint32_t X = vcw[(tt * 32 + lane) * NW + 2 * jw], Y = vcw[(tt * 32 + lane) * NW + 2 * jw + 1];
      for (int i = 0; i < F::TPW; ++i) {
        const int mc = F::TPW * jw + i;
        const uint32_t m = F::mask(i);
        const float undo = pow2i(24 - BITS * i);
        // reg0: channel gid, tokens 2tig+{0,1}; reg1: channel gid+8; reg2/3: tokens +8
        const uint32_t regs[4] = {X & m, Y & m, (X >> 8) & m, (Y >> 8) & m};
        for (int r = 0; r < 4; ++r)
          for (int e = 0; e < 2; ++e) {
            const int t = tt * 16 + 2 * tig + ((r & 2) ? 8 : 0) + e;
            const int c = mc * 16 + gid + ((r & 1) ? 8 : 0);
            const int cg = c / G;
            const int pi = ((t >> 1) * CPG + cg) * 2 + (t & 1);
            vou[t * D + c] = __fmaf_rn(code(regs[r], e, undo), __half2float(sv[pi]), __half2float(zv[pi]));
          }
      }
    }
  }
}

struct QPlan {
  Partition P;
  int MAXS;
  size_t off_ml, off_o, total;
};

// Blocks per SM for one kernel instance (cached per device).
template <int BITS, int G, int D, int NT>
int quant_occupancy() {
  using C = QCfg<BITS, G, D, NT>;
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    cudaFuncSetAttribute(draft_quant_kernel<BITS, G, D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_B);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, draft_quant_kernel<BITS, G, D, NT>, kQNW * 32,
                                                      C::SMEM_B) != cudaSuccess ||
        n < 1)
      n = 1;
    cache[dev] = n;
  }
  return cache[dev];
}

// The stage axis of one call and its cut into at most `target_blocks` blocks.
QPlan make_plan(const vc_attn_shape& sh, const vc_quant_cache& c, int ng_per_stage, int rec_bytes,
                int64_t target_blocks) {
  QPlan p{};
  Partition& P = p.P;
  P.U = sh.B * sh.Hkv;
  P.ng = c.L_q / c.group;
  P.sq = static_cast<int>((P.ng + ng_per_stage - 1) / ng_per_stage);
  P.sr = (c.R + kResRows - 1) / kResRows;
  P.RZ = static_cast<int64_t>(P.U) * P.sr;
  P.S_tot = P.RZ + static_cast<int64_t>(P.U) * P.sq;
  P.cq = P.sq > 0 ? static_cast<int64_t>(ng_per_stage) * rec_bytes : 1;
  P.cr = P.sr > 0 ? static_cast<int64_t>(kResRows) * 4 * sh.D * kResCostWeight : 1;
  P.C = P.RZ * P.cr + (P.S_tot - P.RZ) * P.cq;
  const int64_t mx = P.sq > 0 && P.sr > 0 ? (P.cq > P.cr ? P.cq : P.cr) : (P.sq > 0 ? P.cq : P.cr);
  int64_t n = target_blocks;
  if (n > P.S_tot) n = P.S_tot;
  if (n > P.C / mx) n = P.C / mx;
  if (n < 1) n = 1;
  P.nblk = static_cast<int>(n);
  int maxs = 1;
  for (int k = 0; k < P.nblk; ++k) {
    const int64_t b0 = P.first(k), b1 = P.first(k + 1);
    const int segs = P.seg_of(b1 - 1) - P.seg_of(b0) + 1;
    if (segs > maxs) maxs = segs;
  }
  p.MAXS = maxs;
  const int g = sh.Hq / sh.Hkv;
  const size_t slots = static_cast<size_t>(P.nblk) * maxs;
  p.off_ml = align_up(sizeof(WsHeader), 256);
  p.off_o = align_up(p.off_ml + slots * g * 2 * 4, 256);
  p.total = align_up(p.off_o + slots * g * sh.D * 4, 256);
  return p;
}

template <int BITS, int G, int D, int NT>
QPlan plan_t(const vc_attn_shape& sh, const vc_quant_cache& c, int64_t target_blocks) {
  using C = QCfg<BITS, G, D, NT>;
  if (target_blocks <= 0) target_blocks = static_cast<int64_t>(quant_occupancy<BITS, G, D, NT>()) * sm_count();
  return make_plan(sh, c, C::NG, C::REC, target_blocks);
}

template <int BITS, int G, int D, int NT>
void launch_t(const QArgs& a, const QPlan& p, cudaStream_t s) {
  using C = QCfg<BITS, G, D, NT>;
  quant_occupancy<BITS, G, D, NT>();  // sets the shared-memory attribute once per device
  draft_quant_kernel<BITS, G, D, NT><<<p.P.nblk, kQNW * 32, C::SMEM_B, s>>>(a);
  CArgs c{};
  c.P = p.P;
  c.MAXS = p.MAXS;
  c.g = a.g;
  c.Hq = a.Hq;
  c.Hkv = a.Hkv;
  c.part_o = a.part_o;
  c.part_ml = a.part_ml;
  c.out = a.out;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.P.U), static_cast<unsigned>(a.g));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, combine_kernel<D>, c);
}

template <int BITS, int G, int D>
void debug_t(const vc_quant_cache& c, const vc_attn_shape& sh, float* ko, float* vo, cudaStream_t s) {
  const int64_t n_groups = c.L_q / G;
  if (n_groups == 0) return;
  dim3 grid(static_cast<unsigned>(n_groups), sh.B * sh.Hkv);
  debug_dequant_kernel<BITS, G, D><<<grid, 32, 0, s>>>(static_cast<const uint8_t*>(c.records), n_groups, ko, vo);
}

// Dispatch over the compiled instances: bits {2,4} x group {32,64} x D
// {64,128} x n-tiles {1 (g <= 4), 2 (g <= 8)}.
template <typename F>
bool dispatch(int bits, int group, int D, int nt, F&& f) {
#define VC_Q_CASE(BI, GR, DD, NN)                                               \
  if (bits == BI && group == GR && D == DD && nt == NN) {                       \
    f(std::integral_constant<int, BI>{}, std::integral_constant<int, GR>{},      \
      std::integral_constant<int, DD>{}, std::integral_constant<int, NN>{});     \
    return true;                                                                \
  }
  VC_Q_CASE(2, 32, 128, 1) VC_Q_CASE(2, 32, 128, 2) VC_Q_CASE(2, 64, 128, 1) VC_Q_CASE(2, 64, 128, 2)
  VC_Q_CASE(4, 32, 128, 1) VC_Q_CASE(4, 32, 128, 2) VC_Q_CASE(4, 64, 128, 1) VC_Q_CASE(4, 64, 128, 2)
  VC_Q_CASE(2, 32, 64, 1) VC_Q_CASE(2, 32, 64, 2) VC_Q_CASE(2, 64, 64, 1) VC_Q_CASE(2, 64, 64, 2)
  VC_Q_CASE(4, 32, 64, 1) VC_Q_CASE(4, 32, 64, 2) VC_Q_CASE(4, 64, 64, 1) VC_Q_CASE(4, 64, 64, 2)
#undef VC_Q_CASE
  return false;
}

vc_status check_quant(const vc_attn_shape* sh, const vc_quant_cache* c, const char* who) {
  VC_REQUIRE(sh && c, "%s: null shape or cache", who);
  VC_REQUIRE(sh->B >= 1 && sh->Hkv >= 1 && sh->Hq >= 1 && sh->Hq % sh->Hkv == 0 && sh->Hq / sh->Hkv <= 8,
             "%s: need B >= 1, Hq a multiple of Hkv, Hq/Hkv <= 8", who);
  VC_REQUIRE(sh->D == 64 || sh->D == 128, "%s: head dim must be 64 or 128 (got %d)", who, sh->D);
  VC_REQUIRE(c->bits == 2 || c->bits == 4, "%s: bits must be 2 or 4 (got %d)", who, c->bits);
  VC_REQUIRE(c->group == 32 || c->group == 64, "%s: group must be 32 or 64 (got %d)", who, c->group);
  VC_REQUIRE(c->L_q >= 0 && c->L_q % c->group == 0, "%s: L_q must be a non-negative multiple of group", who);
  VC_REQUIRE(c->L_q / c->group < (int64_t(1) << 30), "%s: L_q too large", who);
  VC_REQUIRE(c->R >= 0 && c->R <= c->R_cap, "%s: need 0 <= R <= R_cap", who);
  VC_REQUIRE(c->L_q + c->R >= 1, "%s: the cache holds no token", who);
  VC_REQUIRE(static_cast<int64_t>(sh->B) * sh->Hkv <= (int64_t(1) << 24), "%s: too many (request, head) pairs",
             who);
  if (c->L_q > 0) {
    VC_REQUIRE(c->records, "%s: null group-record pointer", who);
    VC_REQUIRE(aligned16(c->records), "%s: group records must be 16-byte aligned", who);
  }
  if (c->R > 0) {
    VC_REQUIRE(c->k_res && c->v_res, "%s: null residual pointer", who);
    VC_REQUIRE(aligned16(c->k_res) && aligned16(c->v_res), "%s: residual arrays must be 16-byte aligned", who);
  }
  return VC_OK;
}

QArgs make_args(const vc_attn_shape& sh, const vc_quant_cache& c, const void* q) {
  QArgs a{};
  a.rec = static_cast<const uint8_t*>(c.records);
  a.kr = static_cast<const __nv_bfloat16*>(c.k_res);
  a.vr = static_cast<const __nv_bfloat16*>(c.v_res);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.R = c.R;
  a.R_cap = c.R_cap;
  a.Hq = sh.Hq;
  a.Hkv = sh.Hkv;
  a.g = sh.Hq / sh.Hkv;
  const float sm = sh.sm_scale > 0.f ? sh.sm_scale : 1.0f / sqrtf(static_cast<float>(sh.D));
  a.scale_log2 = sm * 1.4426950408889634f;
  return a;
}

bool quant_plan(const vc_attn_shape& sh, const vc_quant_cache& c, QPlan* out, int64_t target_blocks = 0) {
  const int nt = (sh.Hq / sh.Hkv) <= 4 ? 1 : 2;
  return dispatch(c.bits, c.group, sh.D, nt, [&](auto BI, auto GR, auto DD, auto NN) {
    *out = plan_t<decltype(BI)::value, decltype(GR)::value, decltype(DD)::value, decltype(NN)::value>(
        sh, c, target_blocks);
  });
}

void bind_scratch(QArgs& a, const QPlan& p, void* scratch, float* out) {
  char* w = static_cast<char*>(scratch);
  a.P = p.P;
  a.MAXS = p.MAXS;
  a.flags = reinterpret_cast<uint32_t*>(w);
  a.part_ml = reinterpret_cast<float*>(w + p.off_ml);
  a.part_o = reinterpret_cast<float*>(w + p.off_o);
  a.out = out;
}

void launch_quant(const vc_attn_shape& sh, const vc_quant_cache& c, const QArgs& a, const QPlan& p, cudaStream_t s) {
  const int nt = a.g <= 4 ? 1 : 2;
  dispatch(c.bits, c.group, sh.D, nt, [&](auto BI, auto GR, auto DD, auto NN) {
    launch_t<decltype(BI)::value, decltype(GR)::value, decltype(DD)::value, decltype(NN)::value>(a, p, s);
  });
}

}  // namespace
}  // namespace vc

extern "C" {

size_t vc_draft_attn_quant_workspace_size(const vc_attn_shape* shape, const vc_quant_cache* cache) {
  if (vc::check_quant(shape, cache, "vc_draft_attn_quant_workspace_size") != VC_OK) return 0;
  vc::QPlan p{};
  if (!vc::quant_plan(*shape, *cache, &p)) return 0;
  return p.total;
}

vc_status vc_draft_attn_quant(const vc_attn_shape* shape, const vc_quant_cache* cache, const void* q, float* out,
                              void* ws, size_t ws_bytes, void* stream) {
  vc_status st = vc::check_quant(shape, cache, "vc_draft_attn_quant");
  if (st != VC_OK) return st;
  VC_REQUIRE(q && out && ws, "vc_draft_attn_quant: null q, out or workspace");
  VC_REQUIRE(vc::aligned16(q) && vc::aligned16(out) && vc::aligned16(ws),
             "vc_draft_attn_quant: q, out and workspace must be 16-byte aligned");
  vc::QPlan p{};
  if (!vc::quant_plan(*shape, *cache, &p))
    return vc::set_error(VC_ERR_UNSUPPORTED, "vc_draft_attn_quant: no kernel for this configuration");
  VC_REQUIRE(ws_bytes >= p.total, "vc_draft_attn_quant: workspace too small (%zu < %zu)", ws_bytes, p.total);
  vc::QArgs a = vc::make_args(*shape, *cache, q);
  vc::bind_scratch(a, p, ws, out);
  vc::launch_quant(*shape, *cache, a, p, static_cast<cudaStream_t>(stream));
  return vc::launch_status("vc_draft_attn_quant");
}

vc_status vc_debug_dequant(const vc_attn_shape* shape, const vc_quant_cache* cache, float* k_out, float* v_out,
                           void* stream) {
  vc_status st = vc::check_quant(shape, cache, "vc_debug_dequant");
  if (st != VC_OK) return st;
  VC_REQUIRE(k_out && v_out, "vc_debug_dequant: null output");
  VC_REQUIRE(cache->L_q / cache->group <= 2147483647, "vc_debug_dequant: too many groups");
  VC_REQUIRE(static_cast<int64_t>(shape->B) * shape->Hkv <= 65535, "vc_debug_dequant: too many units");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  vc::dispatch(cache->bits, cache->group, shape->D, 1, [&](auto BI, auto GR, auto DD, auto) {
    vc::debug_t<decltype(BI)::value, decltype(GR)::value, decltype(DD)::value>(*cache, *shape, k_out, v_out, s);
  });
  return vc::launch_status("vc_debug_dequant");
}

vc_status vc_debug_quant_partition(const vc_attn_shape* shape, const vc_quant_cache* cache, int target_blocks,
                                   int64_t* first_stage, int max_blocks, int* n_blocks, int* max_segments,
                                   int64_t* n_stages, int64_t* n_quant_stages) {
  vc_status st = vc::check_quant(shape, cache, "vc_debug_quant_partition");
  if (st != VC_OK) return st;
  VC_REQUIRE(target_blocks >= 1, "vc_debug_quant_partition: target_blocks must be >= 1");
  VC_REQUIRE(n_blocks && max_segments && n_stages && n_quant_stages, "vc_debug_quant_partition: null output");
  vc::QPlan p{};
  if (!vc::quant_plan(*shape, *cache, &p, target_blocks))
    return vc::set_error(VC_ERR_UNSUPPORTED, "vc_debug_quant_partition: no kernel for this configuration");
  *n_blocks = p.P.nblk;
  *max_segments = p.MAXS;
  *n_stages = p.P.S_tot;
  *n_quant_stages = p.P.S_tot - p.P.RZ;
  if (first_stage) {
    VC_REQUIRE(max_blocks >= p.P.nblk + 1, "vc_debug_quant_partition: first_stage needs %d entries",
               p.P.nblk + 1);
    for (int k = 0; k <= p.P.nblk; ++k) first_stage[k] = p.P.first(k);
  }
  return VC_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of vc_draft_attn_quant.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code
// that runs inside a host framework whose memory pool owns every byte of
// device memory, or latency-critical paths that must never reach an
// allocator (cudaMalloc may implicitly synchronise the device).  For them
// this entry point keeps the split-K scratch (flag word, partials)
// in a file-scope device array of fixed size, VC_NOALLOC_SCRATCH_BYTES, that
// every GPU which loads the library holds until the process exits.
//
// The array's address is looked up once per device, with that device
// current, on the first call made on it (cudaGetSymbolAddress); make that
// first call before any stream capture.  Every call shares the one array,
// and calls that overlap on the GPU (other streams, other host threads) race
// on it.  Only its flag word must start at zero: a device array is zero when
// the module loads, kernels only OR bits into the word, and
// vc_draft_attn_quant_noalloc_flags reads and clears it, so a timed-out call
// stays visible until the caller asks.  The block partials need no clearing.
namespace vc {
namespace {

constexpr size_t kNoAllocScratchBytes = VC_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device (nullptr + error
// status on failure).  Host code must not use the symbol's name as an
// address: it is a host-side stand-in.
vc_status noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(VC_ERR_CUDA, "vc_draft_attn_quant_noalloc: no usable current device");
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return set_error(VC_ERR_CUDA, "vc_draft_attn_quant_noalloc: cudaGetSymbolAddress failed: %s",
                       cudaGetErrorString(e));
    addr[dev] = p;
  }
  *out = addr[dev];
  return VC_OK;
}

}  // namespace
}  // namespace vc

extern "C" {

vc_status vc_draft_attn_quant_noalloc(const vc_attn_shape* shape, const vc_quant_cache* cache, const void* q,
                                      float* out, void* stream) {
  vc_status st = vc::check_quant(shape, cache, "vc_draft_attn_quant_noalloc");
  if (st != VC_OK) return st;
  VC_REQUIRE(q && out, "vc_draft_attn_quant_noalloc: null q or out");
  VC_REQUIRE(vc::aligned16(q) && vc::aligned16(out), "vc_draft_attn_quant_noalloc: q and out must be 16-byte aligned");
  vc::QPlan p{};
  if (!vc::quant_plan(*shape, *cache, &p))
    return vc::set_error(VC_ERR_UNSUPPORTED, "vc_draft_attn_quant_noalloc: no kernel for this configuration");
  if (p.total > vc::kNoAllocScratchBytes)
    return vc::set_error(VC_ERR_WORKSPACE,
                         "vc_draft_attn_quant_noalloc: this call needs %zu bytes of scratch, more than the fixed "
                         "%zu-byte device array; use vc_draft_attn_quant with a caller workspace",
                         p.total, vc::kNoAllocScratchBytes);
  void* scratch = nullptr;
  st = vc::noalloc_scratch(&scratch);
  if (st != VC_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  vc::QArgs a = vc::make_args(*shape, *cache, q);
  vc::bind_scratch(a, p, scratch, out);
  vc::launch_quant(*shape, *cache, a, p, s);
  return vc::launch_status("vc_draft_attn_quant_noalloc");
}

vc_status vc_draft_attn_quant_noalloc_flags(uint32_t* host_flags, void* stream) {
  VC_REQUIRE(host_flags != nullptr, "vc_draft_attn_quant_noalloc_flags: null output");
  void* scratch = nullptr;
  vc_status st = vc::noalloc_scratch(&scratch);
  if (st != VC_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, scratch, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemsetAsync(scratch, 0, sizeof(uint32_t), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
    return vc::set_error(VC_ERR_CUDA, "vc_draft_attn_quant_noalloc_flags: %s",
                         cudaGetErrorString(cudaGetLastError()));
  *host_flags = v;
  vc::clear_error();
  return VC_OK;
}

}  // extern "C"
