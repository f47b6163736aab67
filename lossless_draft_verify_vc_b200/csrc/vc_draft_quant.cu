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
// Work layout.  grid (S, B * Hkv): block x < units-with-residual ... see
// plan_quant(); a block owns a contiguous run of groups (G tokens each) of one
// (request, KV head), or that head's bf16 residual rows.  Each of its 4 warps
// takes groups round-robin and streams them through a private ring of
// shared-memory stages filled by 1-D bulk copies (codes, scales, zeros of a
// group are contiguous in HBM, so one group = 6 bulk copies) completed on
// mbarriers; waits are bounded.  All g query heads of the GQA group share each
// group read (they are the MMA's N columns).
//
// MMA arrangement (mma.sync m16n8k16, fp16 x fp16 -> fp32):
//   scores:  D[token][col] = codes[token][chan] x qfold[chan][col]
//            col = 2 * head + part (part 0 = high, 1 = low), 4 heads per n-tile
//   values:  D[chan][col]  = codes^T[chan][token] x pfold[token][col]
// Code bits reach the tensor cores as fp16 subnormals (one AND per two codes,
// see KLane / VLane); the assignment of MMA k-slots / rows to channels is
// chosen so that each lane's codes sit at fixed bit positions.
#include <mutex>

#include "vc_splitk.cuh"

namespace vc {
namespace {

constexpr int kQNW = 4;  // warps per block

template <int BITS, int G, int D, int NT>
struct QCfg {
  static constexpr int RB = D * BITS / 8;           // bytes per packed token row
  static constexpr int WPR = RB / 4;                // 32-bit words per row
  static constexpr int KC_B = G * RB;               // key (or value) codes per group
  static constexpr int SC_B = 2 * D;                // each of sk, zk, sv, zv per group
  static constexpr int QSTAGE = 2 * KC_B + 4 * SC_B;
  static constexpr int NST = QSTAGE <= 4096 ? 4 : 2;
  static constexpr int RS = D * 2 + 16;             // residual smem row stride
  static constexpr int RSTAGE = 32 * RS;            // 16 K + 16 V residual rows
  static constexpr int RING = (NST * QSTAGE > RSTAGE) ? NST * QSTAGE : RSTAGE;
  static constexpr int PS_B = 2 * (4 * NT * G) * 2;  // p high/low parts, fp16 [heads][G] each
  static constexpr int WARP_B = RING + PS_B;
  static constexpr int BAR_OFF = kQNW * WARP_B;
  static constexpr int SMEM_B = BAR_OFF + kQNW * NST * 8 + 16;
  static constexpr int KT = D / 16;                 // channel tiles
  static constexpr int CPG = D / G;                 // value groups per token
  static_assert(G % 32 == 0, "group must be a multiple of 32");
};

struct QArgs {
  const uint8_t* kc;
  const uint8_t* vc;
  const __half* sk;
  const __half* zk;
  const __half* sv;
  const __half* zv;
  const __nv_bfloat16* kr;
  const __nv_bfloat16* vr;
  const __nv_bfloat16* q;
  int64_t L_q;
  int R, R_cap;
  int Hq, Hkv, g;
  int S, Sq, GPC, res_first;  // chunks; quant chunks; groups per chunk; residual blocks lead
  float scale_log2;
  uint32_t* flags;
  SplitKOut o;
};

// Online-softmax update of one head state with 4 new (already scaled) scores.
__device__ __forceinline__ float softmax_step(float (&x)[4], float& m_run, float& l_run, int xor0) {
  float tmax = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
  tmax = warp_max_xor(tmax, xor0);
  tmax = warp_max_xor(tmax, xor0 * 2);
  tmax = warp_max_xor(tmax, xor0 * 4);
  const float m_new = fmaxf(m_run, tmax);
  const float m_use = m_new == -INFINITY ? 0.f : m_new;
  const float alpha = ex2(m_run - m_use);
  float ps = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[j] = ex2(x[j] - m_use);
    ps += x[j];
  }
  l_run = l_run * alpha + ps;
  m_run = m_new;
  return alpha;
}

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

// ----------------------------------------------------------- quantised part
template <int BITS, int G, int D, int NT>
__device__ void quant_role(const QArgs& a, unsigned char* smem, int unit, int b, int h, int qchunk,
                           float* wst_ml, bool& ok) {
  using C = QCfg<BITS, G, D, NT>;
  using F = Frag<BITS>;
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int NW = 2 * C::KT / F::TPW;  // words per lane per 16-token tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int part = gid & 1;
  unsigned char* ring = smem + warp * C::WARP_B;
  __half* Ph = reinterpret_cast<__half*>(ring + C::RING);  // [4 * NT][G] fp16 high parts of p
  __half* Pl = Ph + 4 * NT * G;                            // low parts
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF) + warp * C::NST;

  const int64_t n_groups = a.L_q / G;
  const int64_t g_begin = static_cast<int64_t>(qchunk) * a.GPC;
  const int64_t g_end = min(n_groups, g_begin + a.GPC);
  const int ngr = static_cast<int>(g_end - g_begin);
  const int my_n = ngr > warp ? (ngr - warp + kQNW - 1) / kQNW : 0;

  const uint8_t* kc_u = a.kc + static_cast<size_t>(unit) * a.L_q * C::RB;
  const uint8_t* vc_u = a.vc + static_cast<size_t>(unit) * a.L_q * C::RB;
  const __half* sk_u = a.sk + static_cast<size_t>(unit) * n_groups * D;
  const __half* zk_u = a.zk + static_cast<size_t>(unit) * n_groups * D;
  const __half* sv_u = a.sv + static_cast<size_t>(unit) * a.L_q * C::CPG;
  const __half* zv_u = a.zv + static_cast<size_t>(unit) * a.L_q * C::CPG;

  auto issue = [&](int i) {
    const int s = i % C::NST;
    const int64_t j = g_begin + warp + static_cast<int64_t>(i) * kQNW;
    unsigned char* st = ring + s * C::QSTAGE;
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[s], C::QSTAGE);
      bulk_g2s(st, kc_u + j * C::KC_B, C::KC_B, &bars[s]);
      bulk_g2s(st + C::KC_B, vc_u + j * C::KC_B, C::KC_B, &bars[s]);
      bulk_g2s(st + 2 * C::KC_B, sk_u + j * D, C::SC_B, &bars[s]);
      bulk_g2s(st + 2 * C::KC_B + C::SC_B, zk_u + j * D, C::SC_B, &bars[s]);
      bulk_g2s(st + 2 * C::KC_B + 2 * C::SC_B, sv_u + j * G * C::CPG, C::SC_B, &bars[s]);
      bulk_g2s(st + 2 * C::KC_B + 3 * C::SC_B, zv_u + j * G * C::CPG, C::SC_B, &bars[s]);
    }
  };

  const uint32_t lomask = part ? 0xffffffffu : 0u;  // low-part columns

  // ---- query registers (fp16, exact from bf16), column head = nt*4 + gid/2,
  //      natural channel pairs (16kt + 2tig, +1) and (16kt + 2tig + 8, +9)
  //   q2s: scaled by 2^-(bits * (kt % TPW)) of the code encoding
  //   qb : unscaled, high columns only (zero-point MMA)
  uint32_t q2s[C::KT][NT][2], qb[C::KT][NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hh = nt * 4 + (gid >> 1);
    const bool hv = hh < a.g;
    const __nv_bfloat16* qp = a.q + (static_cast<size_t>(b) * a.Hq + h * a.g + (hv ? hh : 0)) * D;
#pragma unroll
    for (int kt = 0; kt < C::KT; ++kt) {
      const float f = pow2i(-BITS * (kt % F::TPW));
      const float2 lo = unpack_bf2(*reinterpret_cast<const uint32_t*>(qp + kt * 16 + 2 * tig));
      const float2 hi = unpack_bf2(*reinterpret_cast<const uint32_t*>(qp + kt * 16 + 8 + 2 * tig));
      q2s[kt][nt][0] = hv ? pack_h2(lo.x * f, lo.y * f) : 0u;
      q2s[kt][nt][1] = hv ? pack_h2(hi.x * f, hi.y * f) : 0u;
      qb[kt][nt][0] = (hv && !part) ? pack_h2(lo.x, lo.y) : 0u;
      qb[kt][nt][1] = (hv && !part) ? pack_h2(hi.x, hi.y) : 0u;
    }
  }
  // the score MMAs accumulate scores * 2^-24; undo it together with the softmax scale
  const float scl = a.scale_log2 * 16777216.0f;

  float acc[C::KT][NT][4];
  float vb[NT][4];
  float m_run[NT], l_run[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt] = -INFINITY;
    l_run[nt] = 0.f;
    vb[nt][0] = vb[nt][1] = vb[nt][2] = vb[nt][3] = 0.f;
#pragma unroll
    for (int mc = 0; mc < C::KT; ++mc) acc[mc][nt][0] = acc[mc][nt][1] = acc[mc][nt][2] = acc[mc][nt][3] = 0.f;
  }

  if (lane == 0)
    for (int s = 0; s < C::NST; ++s) mbar_init(&bars[s], 1);
  fence_mbar_init();
  __syncwarp();
  const int pre = my_n < C::NST - 1 ? my_n : C::NST - 1;
  for (int i = 0; i < pre; ++i) issue(i);

  for (int i = 0; i < my_n; ++i) {
    if (i + C::NST - 1 < my_n) {
      fence_proxy_async_smem();
      __syncwarp();
      issue(i + C::NST - 1);
    }
    const int s = i % C::NST;
    if (!__all_sync(FULL, mbar_wait_bounded(&bars[s], (i / C::NST) & 1, a.flags))) {  // warp-uniform
      ok = false;
      for (int k = i; k < my_n && k < i + C::NST; ++k)
        mbar_wait_bounded(&bars[k % C::NST], (k / C::NST) & 1, nullptr, 100000000ull);
      break;
    }
    const unsigned char* st = ring + s * C::QSTAGE;
    const uint32_t* kcw = reinterpret_cast<const uint32_t*>(st);
    const uint32_t* vcw = reinterpret_cast<const uint32_t*>(st + C::KC_B);
    const __half* sk = reinterpret_cast<const __half*>(st + 2 * C::KC_B);
    const __half* zk = sk + D;
    const uint32_t* sv32 = reinterpret_cast<const uint32_t*>(zk + D);      // [G/2][CPG] token pairs
    const uint32_t* zv32 = sv32 + G / 2 * C::CPG;

    // (1) fold the key scales into q (fp16 high part in part-0 columns, low
    //     part in part-1 columns) and the zero-point term sum_c q_c z_c
    uint32_t qf[C::KT][NT][2];
    float kb[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) kb[nt][0] = kb[nt][1] = kb[nt][2] = kb[nt][3] = 0.f;
#pragma unroll
    for (int kt = 0; kt < C::KT; ++kt) {
      const uint32_t sA = *reinterpret_cast<const uint32_t*>(sk + kt * 16 + 2 * tig);
      const uint32_t sC = *reinterpret_cast<const uint32_t*>(sk + kt * 16 + 8 + 2 * tig);
      const uint32_t z0 = *reinterpret_cast<const uint32_t*>(zk + kt * 16 + 2 * tig);
      const uint32_t z8 = *reinterpret_cast<const uint32_t*>(zk + kt * 16 + 8 + 2 * tig);
      const uint32_t za[4] = {z0, z0, z8, z8};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t qa = q2s[kt][nt][0], qc = q2s[kt][nt][1];
        qf[kt][nt][0] = hfma2(qa, sA, hmul2((qa ^ 0x80008000u) & lomask, sA));
        qf[kt][nt][1] = hfma2(qc, sC, hmul2((qc ^ 0x80008000u) & lomask, sC));
        mma_f16(kb[nt], za, qb[kt][nt][0], qb[kt][nt][1]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) kb[nt][e] *= 5.9604644775390625e-8f;  // 2^-24

    // (2) 32-token sub-blocks: scores, softmax, P . V
#pragma unroll 1
    for (int sb = 0; sb < G / 32; ++sb) {
      float sc[2][NT][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[mt][nt][e] = kb[nt][e];
        uint32_t w[NW];
        load_words(kcw + ((sb * 2 + mt) * 32 + lane) * NW, w);
#pragma unroll
        for (int j = 0; j < NW / 2; ++j) {
          const uint32_t X = w[2 * j], Y = w[2 * j + 1], xs = X >> 8, ys = Y >> 8;
#pragma unroll
          for (int i = 0; i < F::TPW; ++i) {
            const int kt = F::TPW * j + i;
            const uint32_t m = F::mask(i);
            const uint32_t af[4] = {X & m, xs & m, Y & m, ys & m};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_f16(sc[mt][nt], af, qf[kt][nt][0], qf[kt][nt][1]);
          }
        }
      }
      // softmax per head nt*4 + tig over tokens sb*32 + {gid, gid+8, gid+16, gid+24}
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float x[4] = {(sc[0][nt][0] + sc[0][nt][1]) * scl, (sc[0][nt][2] + sc[0][nt][3]) * scl,
                      (sc[1][nt][0] + sc[1][nt][1]) * scl, (sc[1][nt][2] + sc[1][nt][3]) * scl};
        const float alpha = softmax_step(x, m_run[nt], l_run[nt], 4);
#pragma unroll
        for (int mc = 0; mc < C::KT; ++mc) {
          acc[mc][nt][0] *= alpha;
          acc[mc][nt][1] *= alpha;
          acc[mc][nt][2] *= alpha;
          acc[mc][nt][3] *= alpha;
        }
        vb[nt][0] *= alpha;
        vb[nt][1] *= alpha;
        vb[nt][2] *= alpha;
        vb[nt][3] *= alpha;
        // p as fp16 high + low parts, split once here for the value side
        const uint32_t h01 = pack_h2(x[0], x[1]), h23 = pack_h2(x[2], x[3]);
        const float2 f01 = unpack_h2(h01), f23 = unpack_h2(h23);
        const uint32_t l01 = pack_h2(x[0] - f01.x, x[1] - f01.y), l23 = pack_h2(x[2] - f23.x, x[3] - f23.y);
        unsigned short* ph = reinterpret_cast<unsigned short*>(Ph + (nt * 4 + tig) * G + sb * 32 + gid);
        unsigned short* pl = reinterpret_cast<unsigned short*>(Pl + (nt * 4 + tig) * G + sb * 32 + gid);
        ph[0] = static_cast<unsigned short>(h01);
        ph[8] = static_cast<unsigned short>(h01 >> 16);
        ph[16] = static_cast<unsigned short>(h23);
        ph[24] = static_cast<unsigned short>(h23 >> 16);
        pl[0] = static_cast<unsigned short>(l01);
        pl[8] = static_cast<unsigned short>(l01 >> 16);
        pl[16] = static_cast<unsigned short>(l23);
        pl[24] = static_cast<unsigned short>(l23 >> 16);
      }
      __syncwarp();
#pragma unroll
      for (int ktt = 0; ktt < 2; ++ktt) {
        const int t0 = sb * 32 + ktt * 16 + 2 * tig;  // tokens t0, t0+1, t0+8, t0+9
        uint32_t ph01[NT], ph89[NT], plm01[NT], plm89[NT], phn01[NT], phn89[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int hh = nt * 4 + (gid >> 1);
          ph01[nt] = *reinterpret_cast<const uint32_t*>(Ph + hh * G + t0);
          ph89[nt] = *reinterpret_cast<const uint32_t*>(Ph + hh * G + t0 + 8);
          const uint32_t pl01 = *reinterpret_cast<const uint32_t*>(Pl + hh * G + t0);
          const uint32_t pl89 = *reinterpret_cast<const uint32_t*>(Pl + hh * G + t0 + 8);
          plm01[nt] = pl01 & lomask;
          plm89[nt] = pl89 & lomask;
          phn01[nt] = (ph01[nt] ^ 0x80008000u) & lomask;
          phn89[nt] = (ph89[nt] ^ 0x80008000u) & lomask;
          // value zero-point term: A = z_v^T (row = value group gid), B = p (high or low column)
          uint32_t za[4] = {0u, 0u, 0u, 0u};
          if (gid < C::CPG) {
            za[0] = zv32[(t0 >> 1) * C::CPG + gid];
            za[2] = zv32[((t0 + 8) >> 1) * C::CPG + gid];
          }
          mma_f16(vb[nt], za, part ? pl01 : ph01[nt], part ? pl89 : ph89[nt]);
        }
        // folded p*s for every value group: high part (part 0) or low part (part 1)
        uint32_t pf[C::CPG][NT][2];
        {
          uint32_t s01[C::CPG], s89[C::CPG];
          load_cpg<C::CPG>(sv32 + (t0 >> 1) * C::CPG, s01);
          load_cpg<C::CPG>(sv32 + ((t0 + 8) >> 1) * C::CPG, s89);
#pragma unroll
          for (int cg = 0; cg < C::CPG; ++cg)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              pf[cg][nt][0] = hfma2(plm01[nt], s01[cg], hfma2(ph01[nt], s01[cg], hmul2(phn01[nt], s01[cg])));
              pf[cg][nt][1] = hfma2(plm89[nt], s89[cg], hfma2(ph89[nt], s89[cg], hmul2(phn89[nt], s89[cg])));
            }
        }
        uint32_t w[NW];
        load_words(vcw + ((sb * 2 + ktt) * 32 + lane) * NW, w);
#pragma unroll
        for (int j = 0; j < NW / 2; ++j) {
          const uint32_t X = w[2 * j], Y = w[2 * j + 1], xs = X >> 8, ys = Y >> 8;
#pragma unroll
          for (int i = 0; i < F::TPW; ++i) {
            const int mc = F::TPW * j + i;  // 16-channel tile
            const int cg = mc * 16 / G;
            const uint32_t m = F::mask(i);
            const uint32_t af[4] = {X & m, Y & m, xs & m, ys & m};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_f16(acc[mc][nt], af, pf[cg][nt][0], pf[cg][nt][1]);
          }
        }
      }
      __syncwarp();
    }
  }

  // ---- this warp's state -> its own (finished) ring, natural channel order
  __syncwarp();
  float* my_o = reinterpret_cast<float*>(ring);  // [g][D]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hh = nt * 4 + tig;
    float l = l_run[nt];
    l += __shfl_xor_sync(FULL, l, 4);
    l += __shfl_xor_sync(FULL, l, 8);
    l += __shfl_xor_sync(FULL, l, 16);
    const float vbs = vb[nt][0] + vb[nt][1];  // value-zero term of group gid, head hh
#pragma unroll
    for (int mc = 0; mc < C::KT; ++mc) {
      const int cg = mc * 16 / G;
      const float zb = __shfl_sync(FULL, vbs, cg * 4 + tig);
      const float u = pow2i(24 - BITS * (mc % F::TPW));  // undo the code encoding of this tile
      if (hh < a.g) {
        float* wo = my_o + hh * D + mc * 16 + gid;
        wo[0] = (acc[mc][nt][0] + acc[mc][nt][1]) * u + zb;
        wo[8] = (acc[mc][nt][2] + acc[mc][nt][3]) * u + zb;
      }
    }
    if (hh < a.g && gid == 0) {
      wst_ml[(warp * a.g + hh) * 2] = ok ? m_run[nt] : -INFINITY;
      wst_ml[(warp * a.g + hh) * 2 + 1] = ok ? l : 0.f;
    }
  }
}

// -------------------------------------------------------- bf16 residual part
template <int D, int NT, int RSTRIDE, int WARPB>
__device__ void residual_role(const QArgs& a, unsigned char* smem, int unit, int b, int h, float* wst_ml,
                              bool& ok, int bar_off) {
  constexpr int KT = D / 16;
  constexpr int ROW_B = D * 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int part = gid & 1;
  unsigned char* ring = smem + warp * WARPB;  // one stage: 16 K rows + 16 V rows
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + bar_off) + warp;
  float* P_s = reinterpret_cast<float*>(ring + 32 * RSTRIDE);  // [4*NT][16]
  const int ntiles = (a.R + 15) / 16;
  const int my_n = ntiles > warp ? (ntiles - warp + kQNW - 1) / kQNW : 0;
  const __nv_bfloat16* kr = a.kr + static_cast<size_t>(unit) * a.R_cap * D;
  const __nv_bfloat16* vr = a.vr + static_cast<size_t>(unit) * a.R_cap * D;

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
  if (lane == 0) mbar_init(bar, 1);
  fence_mbar_init();
  __syncwarp();
  for (int i = 0; i < my_n; ++i) {
    const int t0 = (warp + i * kQNW) * 16;
    const int r = lane & 15;
    const bool valid = t0 + r < a.R;
    if (lane == 0) mbar_arrive_expect_tx(bar, 32u * ROW_B);
    __syncwarp();
    const __nv_bfloat16* src = (lane < 16 ? kr : vr) + static_cast<size_t>(valid ? t0 + r : 0) * D;
    bulk_g2s(ring + lane * RSTRIDE, src, ROW_B, bar);
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar, i & 1, a.flags))) {  // warp-uniform
      ok = false;
      break;
    }
    const unsigned char* Ks = ring;
    const unsigned char* Vs = ring + 16 * RSTRIDE;
    const int mi = lane >> 3, ri = lane & 7;
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
      // A = K rows (tokens x channels): matrices (rows 0-7,k 0-7) (8-15,0-7) (0-7,8-15) (8-15,8-15)
      uint32_t af[4];
      ldsm_x4(af, Ks + (ri + (mi & 1) * 8) * RSTRIDE + (kt * 16 + (mi >> 1) * 8) * 2);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16(sc[nt], af, qb[kt][nt][0], qb[kt][nt][1]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const bool v0 = t0 + gid < a.R, v1 = t0 + gid + 8 < a.R;
      float x[4] = {v0 ? (sc[nt][0] + sc[nt][1]) * a.scale_log2 : -INFINITY,
                    v1 ? (sc[nt][2] + sc[nt][3]) * a.scale_log2 : -INFINITY, -INFINITY, -INFINITY};
      const float alpha = softmax_step(x, m_run[nt], l_run[nt], 4);
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
      ldsm_x4_t(af, Vs + (ri + (mi >> 1) * 8) * RSTRIDE + (mc * 16 + (mi & 1) * 8) * 2);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[mc][nt], af, pb[nt][0], pb[nt][1]);
    }
    __syncwarp();
  }
  __syncwarp();
  float* my_o = reinterpret_cast<float*>(ring);  // [g][D]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hh = nt * 4 + tig;
    float l = l_run[nt];
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    if (hh < a.g) {
#pragma unroll
      for (int mc = 0; mc < KT; ++mc) {
        float* wo = my_o + hh * D + mc * 16 + gid;
        wo[0] = acc[mc][nt][0] + acc[mc][nt][1];
        wo[8] = acc[mc][nt][2] + acc[mc][nt][3];
      }
      if (gid == 0) {
        wst_ml[(warp * a.g + hh) * 2] = ok ? m_run[nt] : -INFINITY;
        wst_ml[(warp * a.g + hh) * 2 + 1] = ok ? l : 0.f;
      }
    }
  }
}


template <int BITS, int G, int D, int NT>
__global__ void __launch_bounds__(kQNW * 32, (NT == 1 ? 4 : 2)) draft_quant_kernel(QArgs a) {
  using C = QCfg<BITS, G, D, NT>;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float wst_ml[kQNW * 8 * 2];
  __shared__ float smem_w[kQNW * 8 + 2 * 8];
  const int unit = blockIdx.y;
  const int b = unit / a.Hkv, h = unit - b * a.Hkv;
  const int chunk = blockIdx.x;
  bool ok = true;
  // chunk numbering: the residual block (if any) first, then quantised chunks
  if (a.res_first && chunk == 0)
    residual_role<D, NT, C::RS, C::WARP_B>(a, smem, unit, b, h, wst_ml, ok, C::BAR_OFF);
  else
    quant_role<BITS, G, D, NT>(a, smem, unit, b, h, chunk - a.res_first, wst_ml, ok);
  __syncthreads();
  const int hq0 = b * a.Hq + h * a.g;
  splitk_finish<D>(
      reinterpret_cast<const float*>(smem), C::WARP_B / 4, wst_ml, kQNW, a.g, a.g, a.S, chunk, unit, a.o,
      [&](int r) { return static_cast<size_t>(hq0 + r) * D; }, [&](int r) { return static_cast<size_t>(hq0 + r); },
      smem_w);
}

// vc_debug_dequant: one warp per (group, unit).  The codes are extracted with
// the same word layout, masks and subnormal encoding the attention kernel
// uses (Frag), then dequantised with one fp32 FMA each and stored at their
// natural positions.
template <int BITS, int G, int D>
__global__ void __launch_bounds__(32) debug_dequant_kernel(QArgs a, float* ko, float* vo) {
  using F = Frag<BITS>;
  constexpr int RB = D * BITS / 8, CPG = D / G, KT = D / 16, NW = 2 * KT / F::TPW;
  const int lane = threadIdx.x, gid = lane >> 2, tig = lane & 3;
  const int unit = blockIdx.y;
  const int64_t j = blockIdx.x;
  const int64_t n_groups = a.L_q / G;
  const uint32_t* kc = reinterpret_cast<const uint32_t*>(a.kc + (static_cast<size_t>(unit) * a.L_q + j * G) * RB);
  const uint32_t* vcw = reinterpret_cast<const uint32_t*>(a.vc + (static_cast<size_t>(unit) * a.L_q + j * G) * RB);
  const __half* sk = a.sk + (static_cast<size_t>(unit) * n_groups + j) * D;
  const __half* zk = a.zk + (static_cast<size_t>(unit) * n_groups + j) * D;
  const __half* sv = a.sv + (static_cast<size_t>(unit) * a.L_q + j * G) * CPG;  // pair-interleaved
  const __half* zv = a.zv + (static_cast<size_t>(unit) * a.L_q + j * G) * CPG;
  float* kou = ko + (static_cast<size_t>(unit) * a.L_q + j * G) * D;
  float* vou = vo + (static_cast<size_t>(unit) * a.L_q + j * G) * D;
  auto code = [](uint32_t reg, int half, float undo) {
    const float2 f = unpack_h2(reg);
    return (half ? f.y : f.x) * undo;
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
            kou[t * D + c] = __fmaf_rn(code(regs[r], e, undo), __half2float(sk[c]), __half2float(zk[c]));
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
  int S, Sq, GPC, res;
  size_t off_tick, off_ml, off_o, total;
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

QPlan make_plan(const vc_attn_shape& sh, const vc_quant_cache& c, int occ) {
  QPlan p{};
  const int units = sh.B * sh.Hkv;
  const int64_t n_groups = c.L_q / c.group;
  p.res = c.R > 0 ? 1 : 0;
  if (n_groups > 0) {
    const int64_t slots = static_cast<int64_t>(occ) * sm_count();
    int64_t sq = (slots - static_cast<int64_t>(units) * p.res) / units;
    if (sq < 1) sq = 1;
    int64_t gpc = (n_groups + sq - 1) / sq;
    if (gpc < 4) gpc = 4;
    p.GPC = static_cast<int>(gpc);
    p.Sq = static_cast<int>((n_groups + gpc - 1) / gpc);
  }
  p.S = p.Sq + p.res;
  const int g = sh.Hq / sh.Hkv;
  p.off_tick = sizeof(WsHeader);
  p.off_ml = align_up(p.off_tick + static_cast<size_t>(units) * 4, 256);
  p.off_o = align_up(p.off_ml + static_cast<size_t>(units) * p.S * g * 2 * 4, 256);
  p.total = align_up(p.off_o + static_cast<size_t>(units) * p.S * g * sh.D * 4, 256);
  return p;
}

template <int BITS, int G, int D, int NT>
QPlan plan_t(const vc_attn_shape& sh, const vc_quant_cache& c) {
  return make_plan(sh, c, quant_occupancy<BITS, G, D, NT>());
}

template <int BITS, int G, int D, int NT>
void launch_t(const QArgs& a, const QPlan& p, const vc_attn_shape& sh, cudaStream_t s) {
  using C = QCfg<BITS, G, D, NT>;
  quant_occupancy<BITS, G, D, NT>();  // sets the shared-memory attribute once per device
  dim3 grid(p.S, sh.B * sh.Hkv);
  draft_quant_kernel<BITS, G, D, NT><<<grid, kQNW * 32, C::SMEM_B, s>>>(a);
}

template <int BITS, int G, int D>
void debug_t(const QArgs& a, const vc_attn_shape& sh, float* ko, float* vo, cudaStream_t s) {
  const int64_t n_groups = a.L_q / G;
  if (n_groups == 0) return;
  dim3 grid(static_cast<unsigned>(n_groups), sh.B * sh.Hkv);
  debug_dequant_kernel<BITS, G, D><<<grid, 32, 0, s>>>(a, ko, vo);
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
  VC_REQUIRE(static_cast<int64_t>(sh->B) * sh->Hkv <= 65535, "%s: too many (request, head) pairs", who);
  if (c->L_q > 0) {
    VC_REQUIRE(c->k_codes && c->v_codes && c->k_scale && c->k_zero && c->v_scale && c->v_zero,
               "%s: null quantised-cache pointer", who);
    VC_REQUIRE(aligned16(c->k_codes) && aligned16(c->v_codes) && aligned16(c->k_scale) && aligned16(c->k_zero) &&
                   aligned16(c->v_scale) && aligned16(c->v_zero),
               "%s: quantised-cache arrays must be 16-byte aligned", who);
  }
  if (c->R > 0) {
    VC_REQUIRE(c->k_res && c->v_res, "%s: null residual pointer", who);
    VC_REQUIRE(aligned16(c->k_res) && aligned16(c->v_res), "%s: residual arrays must be 16-byte aligned", who);
  }
  return VC_OK;
}

QArgs make_args(const vc_attn_shape& sh, const vc_quant_cache& c, const void* q) {
  QArgs a{};
  a.kc = static_cast<const uint8_t*>(c.k_codes);
  a.vc = static_cast<const uint8_t*>(c.v_codes);
  a.sk = static_cast<const __half*>(c.k_scale);
  a.zk = static_cast<const __half*>(c.k_zero);
  a.sv = static_cast<const __half*>(c.v_scale);
  a.zv = static_cast<const __half*>(c.v_zero);
  a.kr = static_cast<const __nv_bfloat16*>(c.k_res);
  a.vr = static_cast<const __nv_bfloat16*>(c.v_res);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.L_q = c.L_q;
  a.R = c.R;
  a.R_cap = c.R_cap;
  a.Hq = sh.Hq;
  a.Hkv = sh.Hkv;
  a.g = sh.Hq / sh.Hkv;
  const float sm = sh.sm_scale > 0.f ? sh.sm_scale : 1.0f / sqrtf(static_cast<float>(sh.D));
  a.scale_log2 = sm * 1.4426950408889634f;
  return a;
}

bool quant_plan(const vc_attn_shape& sh, const vc_quant_cache& c, QPlan* out) {
  const int nt = (sh.Hq / sh.Hkv) <= 4 ? 1 : 2;
  return dispatch(c.bits, c.group, sh.D, nt, [&](auto BI, auto GR, auto DD, auto NN) {
    *out = plan_t<decltype(BI)::value, decltype(GR)::value, decltype(DD)::value, decltype(NN)::value>(sh, c);
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
  char* w = static_cast<char*>(ws);
  a.S = p.S;
  a.Sq = p.Sq;
  a.GPC = p.GPC;
  a.res_first = p.res;
  a.flags = reinterpret_cast<uint32_t*>(w);
  a.o.out = out;
  a.o.lse = nullptr;
  a.o.tickets = reinterpret_cast<uint32_t*>(w + p.off_tick);
  a.o.part_ml = reinterpret_cast<float*>(w + p.off_ml);
  a.o.part_o = reinterpret_cast<float*>(w + p.off_o);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nt = a.g <= 4 ? 1 : 2;
  vc::dispatch(cache->bits, cache->group, shape->D, nt, [&](auto BI, auto GR, auto DD, auto NN) {
    vc::launch_t<decltype(BI)::value, decltype(GR)::value, decltype(DD)::value, decltype(NN)::value>(a, p, *shape,
                                                                                                     s);
  });
  return vc::launch_status("vc_draft_attn_quant");
}

vc_status vc_debug_dequant(const vc_attn_shape* shape, const vc_quant_cache* cache, float* k_out, float* v_out,
                           void* stream) {
  vc_status st = vc::check_quant(shape, cache, "vc_debug_dequant");
  if (st != VC_OK) return st;
  VC_REQUIRE(k_out && v_out, "vc_debug_dequant: null output");
  VC_REQUIRE(cache->L_q / cache->group <= 2147483647, "vc_debug_dequant: too many groups");
  vc::QArgs a = vc::make_args(*shape, *cache, nullptr);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  vc::dispatch(cache->bits, cache->group, shape->D, 1, [&](auto BI, auto GR, auto DD, auto) {
    vc::debug_t<decltype(BI)::value, decltype(GR)::value, decltype(DD)::value>(a, *shape, k_out, v_out, s);
  });
  return vc::launch_status("vc_debug_dequant");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of vc_draft_attn_quant.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code
// that runs inside a host framework whose memory pool owns every byte of
// device memory, or latency-critical paths that must never reach an
// allocator (cudaMalloc may implicitly synchronise the device).  For them
// this entry point keeps the split-K scratch (flag word, tickets, partials)
// in a file-scope device array of fixed size, VC_NOALLOC_SCRATCH_BYTES, that
// every GPU which loads the library holds until the process exits.
//
// The array's address is looked up once per device, with that device
// current, on the first call made on it (cudaGetSymbolAddress); make that
// first call before any stream capture.  Every call shares the one array:
// each call clears the words that must start at zero, and calls that
// overlap on the GPU (other streams, other host threads) race on it.
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
  // flag word and tickets must start at zero; partials need no clearing
  if (cudaMemsetAsync(scratch, 0, p.off_ml, s) != cudaSuccess)
    return vc::set_error(VC_ERR_CUDA, "vc_draft_attn_quant_noalloc: clearing the scratch failed: %s",
                         cudaGetErrorString(cudaGetLastError()));
  vc::QArgs a = vc::make_args(*shape, *cache, q);
  char* w = static_cast<char*>(scratch);
  a.S = p.S;
  a.Sq = p.Sq;
  a.GPC = p.GPC;
  a.res_first = p.res;
  a.flags = reinterpret_cast<uint32_t*>(w);
  a.o.out = out;
  a.o.lse = nullptr;
  a.o.tickets = reinterpret_cast<uint32_t*>(w + p.off_tick);
  a.o.part_ml = reinterpret_cast<float*>(w + p.off_ml);
  a.o.part_o = reinterpret_cast<float*>(w + p.off_o);
  const int nt = a.g <= 4 ? 1 : 2;
  vc::dispatch(cache->bits, cache->group, shape->D, nt, [&](auto BI, auto GR, auto DD, auto NN) {
    vc::launch_t<decltype(BI)::value, decltype(GR)::value, decltype(DD)::value, decltype(NN)::value>(a, p, *shape,
                                                                                                     s);
  });
  return vc::launch_status("vc_draft_attn_quant_noalloc");
}

}  // extern "C"
