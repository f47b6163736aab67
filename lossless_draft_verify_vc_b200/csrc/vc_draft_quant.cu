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
// operands q*s and p~*s are split into an fp16 high part and an fp16 low
// part (two MMA columns each), which keeps ~22 significant bits; p~ is the
// softmax weight rounded once to fp16 (the denominator sums the fp32
// weights); the zero terms are separate small MMAs with exact fp16
// products.  Accumulation is fp32.
//
// Work layout.  Every (request, KV head) unit is an axis of residual tiles
// (16 bf16 rows) followed by quantised stages (NG consecutive group records,
// ONE bulk copy).  A persistent grid of (SMs x resident blocks) blocks takes
// the units in equal-cost pieces (UPart): with fewer units than blocks each
// unit is cut into bpu contiguous pieces, otherwise each block owns whole
// units.  Inside a block the 4 warps take the piece's stages round-robin,
// each through its own shared-memory ring (NST stages deep, completed on
// mbarriers, waits bounded); at the end of each segment (the residual tiles,
// then the quantised stages) the block merges its warps' online-softmax
// states into one partial of the unit.  The block that finishes a unit's
// last partial (a per-unit ticket) merges the unit's partials into the
// output, so a call is one launch (a programmatic dependent launch: its
// prologue overlaps the previous kernel's tail).  All g query heads of a GQA
// group share each record (they are MMA columns or rows).
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
// A residual tile (16 bf16 K and V rows, fetched without a pipeline, so its
// time is mostly one memory round trip) costs about 4/3 of its bytes in
// quantised-stage bytes (measured on B200: a tile takes the time of ~3.6
// 2-bit group-32 records)
constexpr int kResCostNum = 4, kResCostDen = 3;
constexpr int kMergeFloats = 512;  // shared-memory area of the final per-unit merge (2 KB)
constexpr int kMinWarpStages = 8;  // measured on B200: 1 x 32K keys 26.0 -> 22.8 us per call, larger shapes unchanged

template <int BITS, int G, int D, int NT>
struct QCfg {
  static constexpr int CB = G * D * BITS / 8;  // one code block (keys or values) of a group
  static constexpr int REC = 2 * CB + 8 * D;   // group record: kc | vc | sk | zk | sv | zv
  static constexpr int OFF_VC = CB;
  static constexpr int OFF_SK = 2 * CB;
  static constexpr int OFF_ZK = 2 * CB + 2 * D;
  static constexpr int OFF_SV = 2 * CB + 4 * D;
  static constexpr int OFF_ZV = 2 * CB + 6 * D;
  static constexpr int HEADS = 4 * NT;
  static constexpr int STATE_W = HEADS * D * 4;  // one warp's unnormalised o, fp32 [HEADS][D]
  static constexpr int NG0 = REC >= 3072 ? 1 : 3072 / REC;
  // records per stage (a stage slot also holds a warp's state at a segment end)
  static constexpr int NG = NG0 * REC >= STATE_W ? NG0 : (STATE_W + REC - 1) / REC;
  static constexpr int STAGE = NG * REC;
  static constexpr bool PIPE = NT == 1 && NG == 1;  // software-pipelined group loop (TokM)
  static constexpr int NST0 = (PIPE ? 12288 : 18432) / STAGE;
  static constexpr int NMIN = PIPE ? 3 : 2;
  static constexpr int NST = NST0 < NMIN ? NMIN : (NST0 > 4 ? 4 : NST0);  // ring depth
  static constexpr int RSTAGE = 2 * kResRows * D * 2;                      // 16 K + 16 V bf16 rows
  // the ring also holds a residual tile; a warp's residual state is written over
  // its last tile once that is consumed
  static constexpr int RING0 = NST * STAGE > RSTAGE ? NST * STAGE : RSTAGE;
  static constexpr int RING = (RING0 + 127) / 128 * 128;
  static constexpr int RP_B = HEADS * kResRows * 4;  // residual tile scores, fp32 [HEADS][16]
  static constexpr int WARP_B = RING + RP_B;
  static constexpr int ML_OFF = kQNW * WARP_B;                  // fp32 [kQNW][HEADS][2]
  static constexpr int SO_OFF = ML_OFF + kQNW * HEADS * 2 * 4;  // int [kQNW]: where each warp's state is
  static constexpr int MW_OFF = SO_OFF + kQNW * 4;              // merge weights + (M, L)
  static constexpr int MW_FLOATS = kQNW * HEADS + 2 * HEADS;
  static constexpr int MA_OFF = (MW_OFF + MW_FLOATS * 4 + 15) / 16 * 16;  // unit merge area
  // block-shared query fragments of TokM (all warps of a block work on one
  // unit at a time): uint4 [KT][32 lanes]
  static constexpr int QSM_OFF = MA_OFF + kMergeFloats * 4;
  static constexpr int QSM_B = NT == 1 ? (D / 16) * 32 * 16 : 0;
  static constexpr int FLAG_OFF = QSM_OFF + QSM_B;
  static constexpr int BAR_OFF = (FLAG_OFF + 4 + 15) / 16 * 16;
  static constexpr int SMEM_B = BAR_OFF + kQNW * (NST + 1) * 8;
  static constexpr int KT = D / 16;   // channel tiles
  static constexpr int CPG = D / G;   // value groups per token
  static_assert(G % 32 == 0, "group must be a multiple of 32");
  static_assert(REC % 16 == 0 && STAGE % 16 == 0, "bulk copies need 16-byte multiples");
  static_assert(STAGE >= STATE_W, "a stage slot holds a warp state");
  static_assert(RSTAGE >= STATE_W, "a residual tile area holds a warp state");
  static_assert(WARP_B % 128 == 0, "warp areas stay 128-byte aligned");
};

// The work of one call and its cut into blocks; the same arithmetic runs on
// the host (planning, workspace size) and on the device.  Unit u (one
// request's KV head) is an axis of sr residual tiles (16 bf16 rows each,
// cost cr) followed by sq quantised stages (NG group records each, cost cq).
//  * bpu >= 1 (at most as many units as blocks): every unit is cut into bpu
//    contiguous pieces of equal cost (piece j starts at axis index A(j),
//    the first index whose start cost is >= ceil(j Cu / bpu)); block k owns
//    piece k % bpu of unit k / bpu.  The host keeps bpu <= Cu / max(cq, cr),
//    so no piece is empty.
//  * bpu == 0 (more units than blocks): block k owns the whole units
//    [k U / nblk, (k + 1) U / nblk).
// A block's work on one unit is at most two segments, its residual tiles and
// its quantised stages, each ending in one block partial.  Every unit has
// the same partials: with bpu >= 1, the residual partials of pieces
// 0 .. jr - 1 and the quantised partials of pieces jq .. bpu - 1
// (np = jr + bpu - jq); with bpu == 0, one of each kind.
struct UPart {
  int64_t ng;      // groups per unit
  int64_t cq, cr;  // cost of one quantised stage / residual tile
  int U, sq, sr;   // units, quantised stages and residual tiles per unit
  int bpu;         // blocks per unit (0: units per block >= 1)
  int nblk;        // blocks in the grid
  int upb;         // most units of one block (1 when bpu >= 1)
  int jr, jq, np;  // pieces with residual / first piece with quantised stages / partials per unit

  __host__ __device__ int64_t ucost() const { return static_cast<int64_t>(sr) * cr + static_cast<int64_t>(sq) * cq; }
  // first unit-axis index of piece j (bpu >= 1)
  __host__ __device__ int axis_first(int j) const {
    if (j <= 0) return 0;
    if (j >= bpu) return sr + sq;
    const int64_t T = (static_cast<int64_t>(j) * ucost() + bpu - 1) / bpu;
    if (sr > 0 && T <= static_cast<int64_t>(sr - 1) * cr) return static_cast<int>((T + cr - 1) / cr);
    const int64_t base = static_cast<int64_t>(sr) * cr;
    if (T <= base) return sr;
    const int64_t s = sr + (T - base + cq - 1) / cq;
    return s < sr + sq ? static_cast<int>(s) : sr + sq;
  }
  // units [u0, u1) and unit-local residual tiles [r0, r1) / quantised stages [q0, q1) of block k
  __host__ __device__ void block_range(int k, int& u0, int& u1, int& r0, int& r1, int& q0, int& q1) const {
    if (bpu > 0) {
      u0 = k / bpu;
      u1 = u0 + 1;
      const int j = k - u0 * bpu;
      const int a0 = axis_first(j), a1 = axis_first(j + 1);
      r0 = a0 < sr ? a0 : sr;
      r1 = a1 < sr ? a1 : sr;
      q0 = a0 > sr ? a0 - sr : 0;
      q1 = a1 > sr ? a1 - sr : 0;
    } else {
      u0 = static_cast<int>(static_cast<int64_t>(k) * U / nblk);
      u1 = static_cast<int>(static_cast<int64_t>(k + 1) * U / nblk);
      r0 = 0, r1 = sr, q0 = 0, q1 = sq;
    }
  }
  // slot of partial p (0 <= p < np) of unit u; a block's slots are
  // k * 2 upb + 2 (unit - u0) + (0 residual, 1 quantised)
  __host__ __device__ int64_t partial_slot(int u, int p) const {
    if (bpu > 0) {
      const int j = p < jr ? p : jq + (p - jr);
      return 2 * (static_cast<int64_t>(u) * bpu + j) + (p < jr ? 0 : 1);
    }
    const int k = static_cast<int>((static_cast<int64_t>(u + 1) * nblk + U - 1) / U) - 1;
    const int u0 = static_cast<int>(static_cast<int64_t>(k) * U / nblk);
    const int kind = (sr > 0 && p == 0) ? 0 : 1;
    return static_cast<int64_t>(k) * 2 * upb + 2 * (u - u0) + kind;
  }
};

struct QArgs {
  const uint8_t* rec;  // [U][ng][REC] group records
  const __nv_bfloat16* kr;
  const __nv_bfloat16* vr;
  const __nv_bfloat16* q;
  UPart P;
  int R, R_cap, group;
  int Hq, Hkv, g;
  int MAXS;  // partial slots per block
  float scale_log2;
  uint32_t* flags;
  uint32_t* tickets;  // [U] partials of each unit written so far in this call (back to 0 after it)
  const int32_t* lens;  // optional [B][2] per-request (L_q, R); NULL: P.ng groups and R rows everywhere
  int cache_flags;      // VC_CACHE_STATIC: the first stages may be fetched before the stream dependency
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

// Groups and residual rows of unit u's request (per-request lengths when the
// cache carries them; the planned capacity is then an upper bound).
// Clamped to the planned capacity, so a length the host did not validate can
// never make a kernel read past the buffers.
__device__ __forceinline__ int64_t unit_groups(const QArgs& a, int u) {
  if (!a.lens) return a.P.ng;
  const int64_t g = a.lens[2 * (u / a.Hkv)] / a.group;
  return g < 0 ? 0 : (g > a.P.ng ? a.P.ng : g);
}
__device__ __forceinline__ int unit_res_rows(const QArgs& a, int u) {
  if (!a.lens) return a.R;
  const int r = a.lens[2 * (u / a.Hkv) + 1];
  return r < 0 ? 0 : (r > a.R_cap ? a.R_cap : r);
}

// Where this warp's next quantised stage to fetch lives: unit u, unit-local
// stage ls.  Warp w takes the stages q0 + w, q0 + w + kQNW, ... < q1 of each
// of its block's units in turn.
struct IssuePtr {
  int u, ls;
  int qend;            // end of unit u's quantised stages in this block
  const uint8_t* src;  // record of group ls * NG of unit u
};

// End of unit u's quantised stages in a block whose planned range ends at q1:
// with per-request lengths, a request's own stage count can be smaller.
template <typename C>
__device__ __forceinline__ int unit_qend(const QArgs& a, int u, int q1) {
  if (!a.lens) return q1;
  const int sq_u = static_cast<int>((unit_groups(a, u) + C::NG - 1) / C::NG);
  return sq_u < q1 ? sq_u : q1;
}

// This warp's stage count in unit u: stages q_first, q_first + kQNW, ... < qend.
__device__ __forceinline__ int warp_stage_count(int q_first, int qend) {
  return qend > q_first ? (qend - q_first + kQNW - 1) / kQNW : 0;
}

template <typename C>
__device__ __forceinline__ void issue_start(const QArgs& a, IssuePtr& ip, int u, int ls, int q1) {
  ip.u = u;
  ip.ls = ls;
  ip.qend = unit_qend<C>(a, u, q1);
  ip.src = a.rec + (static_cast<int64_t>(u) * a.P.ng + static_cast<int64_t>(ls) * C::NG) * C::REC;
}

// Next stage of this warp: the next one in the unit, else the first one of
// the next unit of the block that holds any (a unit with none is skipped).
template <typename C>
__device__ __forceinline__ void issue_advance(const QArgs& a, IssuePtr& ip, int q_first, int u_end, int q1) {
  ip.ls += kQNW;
  ip.src += kQNW * C::STAGE;
  if (ip.ls >= ip.qend) {
    int u = ip.u + 1;
    while (u < u_end && warp_stage_count(q_first, unit_qend<C>(a, u, q1)) == 0) ++u;
    if (u < u_end) issue_start<C>(a, ip, u, q_first, q1);
    else ip.u = u;
  }
}

// One bulk copy of this warp's next quantised stage (at ip) into ring slot
// `slot`; the records are read once per call (evict-first in L2).
template <typename C>
__device__ __forceinline__ void issue_stage(const QArgs& a, unsigned char* ring, uint64_t* bars, int lane, int slot,
                                            const IssuePtr& ip) {
  uint32_t bytes = C::STAGE;
  if constexpr (C::NG > 1) {  // a unit's last stage may hold fewer groups
    const int64_t left = a.P.ng - static_cast<int64_t>(ip.ls) * C::NG;
    if (left < C::NG) bytes = static_cast<uint32_t>(left * C::REC);
  }
  if (lane == 0) {
    mbar_arrive_expect_tx(&bars[slot], bytes);
    bulk_g2s_once(ring + slot * C::STAGE, ip.src, bytes, &bars[slot]);
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
// The softmax weights p (<= 2^kLazy by the lazy running maximum) are
// rounded once to fp16 (p~) for the value side; the softmax denominator
// sums the fp32 p.  p~ * s is split into an fp16 high part and the exact
// fp16 remainder (one fma), so the value operand carries ~22 bits.
//
// Each body has three steps per group: keys() (scores of the group into
// registers), softmax() (running max and sum, weights in the value MMA's
// operand layout) and values() (P . V into the accumulators).  TokM runs
// them software-pipelined: values() of group j and keys() of group j + 1
// form one straight-line block, so the long MMA and load latencies of one
// overlap the other's independent work.

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
  using C = QCfg<BITS, G, D, 1>;
  static constexpr int KT = D / 16, TPW = F::TPW, NW = 2 * KT / TPW, MT = G / 16, CPG = D / G;
  static constexpr int HEADS = 4;
  // per (kt, lane) in block-shared memory: (qs0, qs1, qm0, qm1) with
  //   qs = q * 2^-(bits i), negated in low-part lanes,
  //   qm = q * 2^-(bits i) in low-part lanes, 0 in high-part lanes
  const uint4* qsm;
  float acc[KT][4];    // D[channel][col]
  float vb[4];         // value zero-point term: D[value group][col]
  float m_run, m_lim, l_run;
  float sc[MT][4], kb[4];          // scores of the group keys() read last
  uint32_t PA[MT][2], PB[MT][2];  // its weights, after softmax()

  // Query fragments of unit (b, h) into the block-shared area (one warp).
  __device__ __forceinline__ static void write_q(const QArgs& a, int b, int h, int lane, uint4* q_sm) {
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
      q_sm[kt * 32 + lane] = make_uint4(part ? q0 ^ 0x80008000u : q0, part ? q1 ^ 0x80008000u : q1,
                                        part ? q0 : 0u, part ? q1 : 0u);
    }
  }

  __device__ __forceinline__ void init(const QArgs& a, int b, int h, int lane, const uint4* q_sm) {
    (void)a, (void)b, (void)h, (void)lane;
    qsm = q_sm;
#pragma unroll
    for (int mc = 0; mc < KT; ++mc) acc[mc][0] = acc[mc][1] = acc[mc][2] = acc[mc][3] = 0.f;
    vb[0] = vb[1] = vb[2] = vb[3] = 0.f;
    m_run = -INFINITY;
    m_lim = -INFINITY;
    l_run = 0.f;
  }

  // (1) scores: per channel tile kt the key scales are folded into q right
  //     before use (high part in part-0 columns, low part in part-1
  //     columns); the zero-point term sum_c q_c z_c is an MMA of the zeros
  //     (times 2^(bits i), exact) against the signed q in the high columns.
  __device__ __forceinline__ void keys(const unsigned char* rs, int lane) {
    const int tig = lane & 3;
    const uint32_t* kcw = reinterpret_cast<const uint32_t*>(rs);
    const uint4* skw = reinterpret_cast<const uint4*>(rs + C::OFF_SK) + tig * (KT / 2);
    const uint4* zkw = reinterpret_cast<const uint4*>(rs + C::OFF_ZK) + tig * (KT / 2);
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
        const uint4 qq = qsm[kt * 32 + lane];  // (qs0, qs1, qm0, qm1)
        const uint32_t fa = hfma2(qq.z, sA, hmul2(qq.x, sA));
        const uint32_t fc = hfma2(qq.w, sC, hmul2(qq.y, sC));
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
        mma_f16(kb, za, qq.x, qq.y);
      }
    }
  }

  // (2) softmax of head tig over the lane's tokens 16 mt + gid (+8); the
  //     scores sit in the 2^-24 domain of the code encoding
  __device__ __forceinline__ void softmax(float scl, float sl2) {
    constexpr unsigned FULL = 0xffffffffu;
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
  }

  // (3) P . V: per 16-token tile, the folded operand of value group cg is
  //     high (part 0 columns: 0 + fp16(p~ s)) or low (part 1 columns:
  //     p~ s - fp16(p~ s), exact) -- the same two instructions in every lane
  __device__ __forceinline__ void values(const unsigned char* rs, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
    const uint32_t* vcw = reinterpret_cast<const uint32_t*>(rs + C::OFF_VC);
    const uint32_t* sv32 = reinterpret_cast<const uint32_t*>(rs + C::OFF_SV);  // [G/2][CPG] token pairs
    const uint32_t* zv32 = reinterpret_cast<const uint32_t*>(rs + C::OFF_ZV);
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

  // This warp's state -> wst [HEADS][D] (natural channel order, unnormalised)
  // and wml [HEADS][2].
  __device__ __forceinline__ void store(const QArgs& a, int lane, bool ok, float* wst, float* wml) {
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
        float* wo = wst + hh * D + mc * 16 + gid;
        wo[0] = (acc[mc][0] + acc[mc][1]) * uf + zb;
        wo[8] = (acc[mc][2] + acc[mc][3]) * uf + zb;
      }
    }
    if (hh < a.g && gid == 0) {
      wml[hh * 2] = ok ? m_run : -INFINITY;
      wml[hh * 2 + 1] = ok ? l : 0.f;
    }
  }
};

template <int BITS, int G, int D>
struct HeadM {
  using F = Frag<BITS>;
  using C = QCfg<BITS, G, D, 2>;
  static constexpr int KT = D / 16, TPW = F::TPW, NW = 2 * KT / TPW, MT = G / 16, CPG = D / G;
  static constexpr int HEADS = 8;
  uint32_t q2[KT][2];  // head gid: q * 2^-(bits i), channel pairs (2 tig, +1), (2 tig + 8, +9)
  float acc[KT][4];    // D[channel][head]: (channel gid, heads 2 tig, 2 tig + 1), channel + 8
  float vb[4];         // D[value group][head]
  float m_run, m_lim, l_run;  // head gid
  float sc[2 * MT][4], kb[4];  // n-tile n: tokens 8 n .. 8 n + 7
  uint32_t P[2 * MT];          // p~ of head gid, tokens 8 n + 2 tig, +1

  __device__ __forceinline__ void init(const QArgs& a, int b, int h, int lane, const uint4* q_sm) {
    (void)q_sm;
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

  // (1) scores: rows gid (high part of head gid's q*s) and gid + 8 (its low
  //     part); zero-point term from rows = q (unfolded) against the zeros
  //     broadcast over the columns
  __device__ __forceinline__ void keys(const unsigned char* rs, int lane) {
    const int tig = lane & 3;
    const uint32_t* kcw = reinterpret_cast<const uint32_t*>(rs);
    const uint4* skw = reinterpret_cast<const uint4*>(rs + C::OFF_SK) + tig * (KT / 2);
    const uint4* zkw = reinterpret_cast<const uint4*>(rs + C::OFF_ZK) + tig * (KT / 2);
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
  }

  // (2) softmax of head gid over tokens 8 n + 2 tig, +1
  __device__ __forceinline__ void softmax(float scl, float sl2) {
    constexpr unsigned FULL = 0xffffffffu;
    const int tig = threadIdx.x & 3;
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
#pragma unroll
    for (int n = 0; n < 2 * MT; ++n) {
      const float p0 = ex2(fmaf(y[n][0], scl, off)), p1 = ex2(fmaf(y[n][1], scl, off));
      l_run += p0 + p1;
      P[n] = pack_h2(p0, p1);
    }
  }

  // (3) P . V: B = p~ * s of head gid for tokens (2 tig, +1) and (2 tig + 8, +9),
  //     high part and exact low part as two MMAs into the same accumulator
  __device__ __forceinline__ void values(const unsigned char* rs, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
    const uint32_t* vcw = reinterpret_cast<const uint32_t*>(rs + C::OFF_VC);
    const uint32_t* sv32 = reinterpret_cast<const uint32_t*>(rs + C::OFF_SV);
    const uint32_t* zv32 = reinterpret_cast<const uint32_t*>(rs + C::OFF_ZV);
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

  __device__ __forceinline__ void store(const QArgs& a, int lane, bool ok, float* wst, float* wml) {
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
        float* wo = wst + h0 * D + mc * 16 + gid;
        wo[0] = acc[mc][0] * uf + zb0;
        wo[8] = acc[mc][2] * uf + zb0;
      }
      if (h1 < a.g) {
        float* wo = wst + h1 * D + mc * 16 + gid;
        wo[0] = acc[mc][1] * uf + zb1;
        wo[8] = acc[mc][3] * uf + zb1;
      }
    }
    if (gid < a.g && tig == 0) {
      wml[gid * 2] = ok ? m_run : -INFINITY;
      wml[gid * 2 + 1] = ok ? l : 0.f;
    }
  }
};

// A warp's ring of NST stage slots.  Stage i (the warp's i-th quantised
// stage) lives in slot i mod NST and completes phase (i / NST) mod 2 of that
// slot's mbarrier.  A slot is refilled (the stage NST later is issued into
// it) only once the stage it holds is released.
struct WarpRing {
  int issued;     // stages issued
  int head;       // next stage to wait for
  int tail;       // next stage to release
  int hslot;
  uint32_t hphase;
  int q_first, q_end;  // this warp's first quantised stage in a unit, and the block's planned end
  int u_end;           // end of the block's units
  IssuePtr ip;
};

template <typename C>
__device__ __forceinline__ void ring_issue_next(const QArgs& a, unsigned char* ring, uint64_t* bars, int lane,
                                                WarpRing& r, int slot, int my_nq) {
  if (r.issued < my_nq) {
    fence_proxy_async_smem();
    __syncwarp();
    issue_stage<C>(a, ring, bars, lane, slot, r.ip);
    issue_advance<C>(a, r.ip, r.q_first, r.u_end, r.q_end);
    ++r.issued;
  }
}

// Waits for stage r.head; returns its slot or -1 if the bounded wait gave up
// (then every stage still in flight is drained and the warp stops).
template <typename C>
__device__ __forceinline__ int ring_wait(const QArgs& a, uint64_t* bars, WarpRing& r, bool& ok) {
  constexpr unsigned FULL = 0xffffffffu;
  const int slot = r.hslot;
  if (!__all_sync(FULL, mbar_wait_bounded(&bars[slot], r.hphase, a.flags))) {  // warp-uniform
    ok = false;
    for (int k = r.head; k < r.issued; ++k)
      mbar_wait_bounded(&bars[k % C::NST], (k / C::NST) & 1, nullptr, 100000000ull);
    return -1;
  }
  ++r.head;
  r.hslot = slot + 1 == C::NST ? 0 : slot + 1;
  r.hphase ^= r.hslot == 0 ? 1u : 0u;
  return slot;
}

// Processes this warp's stages of unit u's quantised segment and leaves the
// warp's state in the slot of its last stage of the segment (that slot is
// released, and refilled, only after the block has merged the warp states:
// *state_slot returns it, -1 if the warp had no stage here).
template <int BITS, int G, int D, int NT>
__device__ __forceinline__ void quant_seg(const QArgs& a, unsigned char* ring, uint64_t* bars, int u, int n_seg,
                                          int my_nq, WarpRing& r, bool& ok, float* wml, int& state_slot,
                                          const uint4* q_sm) {
  using C = QCfg<BITS, G, D, NT>;
  using Body = std::conditional_t<NT == 1, TokM<BITS, G, D>, HeadM<BITS, G, D>>;
  const int lane = threadIdx.x & 31;
  const int b = u / a.Hkv, h = u - b * a.Hkv;
  // the score MMAs accumulate scores * 2^-24; undo it together with the softmax scale
  const float scl = a.scale_log2 * 16777216.0f;
  const float sl2 = a.scale_log2;
  Body body;
  body.init(a, b, h, lane, q_sm);
  state_slot = -1;

  // this warp's stages of the segment: r.head .. r.head + n_seg - 1, unit-local
  // stages r.q_first + kQNW kk
  auto stage_ptr = [&](int slot) { return ring + slot * C::STAGE; };
  if (n_seg > 0 && ok) {
    if constexpr (C::PIPE) {
      static_assert(C::NG == 1, "the pipelined loop takes one group per stage");
      int s_cur = ring_wait<C>(a, bars, r, ok);
      if (s_cur >= 0) {
        body.keys(stage_ptr(s_cur), lane);
        body.softmax(scl, sl2);
#pragma unroll 1
        for (int kk = 1; kk < n_seg; ++kk) {
          const int s_nxt = ring_wait<C>(a, bars, r, ok);
          if (s_nxt < 0) break;
          body.values(stage_ptr(s_cur), lane);
          body.keys(stage_ptr(s_nxt), lane);
          __syncwarp();
          ring_issue_next<C>(a, ring, bars, lane, r, s_cur, my_nq);  // stage tail + NST into the freed slot
          ++r.tail;
          body.softmax(scl, sl2);
          s_cur = s_nxt;
        }
        if (ok) {
          body.values(stage_ptr(s_cur), lane);
          __syncwarp();
          state_slot = s_cur;
        }
      }
    } else {
#pragma unroll 1
      for (int kk = 0; kk < n_seg; ++kk) {
        const int s_cur = ring_wait<C>(a, bars, r, ok);
        if (s_cur < 0) break;
        const unsigned char* rs = stage_ptr(s_cur);
        if constexpr (C::NG == 1) {
          body.keys(rs, lane);
          body.softmax(scl, sl2);
          body.values(rs, lane);
        } else {
          const int64_t gs = static_cast<int64_t>(r.q_first + kQNW * kk) * C::NG;
          const int64_t ng_u = unit_groups(a, u);
          const int n_here = ng_u - gs < C::NG ? static_cast<int>(ng_u - gs) : C::NG;
#pragma unroll 1
          for (int gi = 0; gi < n_here; ++gi) {
            body.keys(rs + gi * C::REC, lane);
            body.softmax(scl, sl2);
            body.values(rs + gi * C::REC, lane);
          }
        }
        __syncwarp();
        if (kk + 1 < n_seg) {
          ring_issue_next<C>(a, ring, bars, lane, r, s_cur, my_nq);
          ++r.tail;
        } else {
          state_slot = s_cur;
        }
      }
    }
  }
  if (state_slot >= 0) {
    body.store(a, lane, ok, reinterpret_cast<float*>(stage_ptr(state_slot)), wml);
  } else if (lane < C::HEADS) {
    wml[lane * 2] = -INFINITY;  // no state from this warp
    wml[lane * 2 + 1] = 0.f;
  }
}

// -------------------------------------------------------- bf16 residual part
// This warp's residual stages of unit u (16 rows each, one bulk copy per row,
// not pipelined; the residual is a few percent of the bytes).  Leaves the
// warp's state in its slot.
template <int D, int NT, int HEADS>
__device__ __forceinline__ void residual_seg(const QArgs& a, unsigned char* ring, float* P_s, uint64_t* bar,
                                             int& rph, int u, int t_first, int t_end, bool& ok, float* wst,
                                             float* wml) {
  constexpr int KT = D / 16;
  constexpr int ROW_B = D * 2;
  constexpr unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
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
  const int R_u = unit_res_rows(a, u);
  for (int t = t_first; t < t_end && ok; t += kQNW) {
    const int t0 = t * kResRows;
    if (t0 >= R_u) break;  // (per-request lengths) past this request's residual
    const int nv = R_u - t0 < kResRows ? R_u - t0 : kResRows;  // rows of this tile inside the window
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
      bulk_g2s_once(ring, kr + static_cast<size_t>(t0) * D, nv * ROW_B, bar);
      bulk_g2s_once(ring + kResRows * ROW_B, vr + static_cast<size_t>(t0) * D, nv * ROW_B, bar);
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
      const bool v0 = t0 + gid < R_u, v1 = t0 + gid + 8 < R_u;
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
        float* wo = wst + hh * D + mc * 16 + gid;
        wo[0] = acc[mc][nt][0] + acc[mc][nt][1];
        wo[8] = acc[mc][nt][2] + acc[mc][nt][3];
      }
      if (gid == 0) {
        wml[hh * 2] = ok ? m_run[nt] : -INFINITY;
        wml[hh * 2 + 1] = ok ? l : 0.f;
      }
    }
  }
}

// Block-wide: merges the kQNW warp states of a segment into the block's
// partial of that segment (partial slot `slot`).  Warp w's state is at
// byte offset st_off[w] of shared memory (-1: that warp had nothing here).
template <int D, int HEADS>
__device__ __forceinline__ void merge_segment(const QArgs& a, int64_t slot, const unsigned char* smem,
                                              const int* st_off, const float* st_ml, float* mw) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int g = a.g;
  float* wts = mw;                // [kQNW][HEADS]
  float* ML = mw + kQNW * HEADS;  // [HEADS][2]
  for (int r = tid; r < g; r += nthr) {
    float M = -INFINITY;
    for (int w = 0; w < kQNW; ++w)
      if (st_off[w] >= 0) M = fmaxf(M, st_ml[(w * HEADS + r) * 2]);
    float L = 0.f;
    for (int w = 0; w < kQNW; ++w) {
      const float mw_ = st_ml[(w * HEADS + r) * 2];
      const float sc = (st_off[w] < 0 || mw_ == -INFINITY) ? 0.f : ex2(mw_ - M);
      wts[w * HEADS + r] = sc;
      L += sc > 0.f ? sc * st_ml[(w * HEADS + r) * 2 + 1] : 0.f;
    }
    ML[2 * r] = M;
    ML[2 * r + 1] = L;
  }
  __syncthreads();
  float* po = a.part_o + slot * g * D;
  float* pml = a.part_ml + slot * g * 2;
  for (int e = tid; e < g * D; e += nthr) {
    const int r = e / D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kQNW; ++w) {
      const float wt = wts[w * HEADS + r];
      if (wt > 0.f) acc += wt * reinterpret_cast<const float*>(smem + st_off[w])[e];
    }
    po[e] = acc;
  }
  for (int r = tid; r < g; r += nthr) {
    pml[2 * r] = ML[2 * r];
    pml[2 * r + 1] = ML[2 * r + 1];
  }
  fence_proxy_async_smem();  // the state slots are refilled by bulk copies after this
  __syncthreads();
}

// After the block wrote its partial of unit u: the block that writes the
// unit's last partial (a per-unit ticket counts them) merges all of them
// into the output and resets the ticket for the next call.  Partials come
// from other SMs, so they are read past L1 (ld.global.cg).  The merge is on
// the kernel's tail, so it is latency-bound: the partials' slots and merge
// weights are staged in shared memory once, then each thread owns output
// float4s and keeps up to 16 partial loads in flight.
// After the block wrote its partial of unit u (and passed the barrier that
// follows those writes): the block that writes the unit's last partial (a
// per-unit ticket counts them) merges all of them into the output and resets
// the ticket for the next call.  Partials come from other SMs, so they are
// read past L1 (ld.global.cg).  The merge sits on the kernel's tail and is
// latency-bound, so it takes two rounds of loads: (1) lane p of warp r reads
// partial p's (max, sum) of head r, the warp reduces the maximum and the sum
// and stages the weights; (2) each thread owns output float4s and keeps up to
// 16 partial loads in flight.
template <int D>
__device__ __forceinline__ void unit_finish(const QArgs& a, int u, float* ma, int* s_flag) {
  constexpr unsigned FULL = 0xffffffffu;
  const int np = a.P.np;
  if (threadIdx.x == 1) {
    // lane 1 of warp 0 issues no bulk copies, so its fence waits on no copy
    // in flight; it orders the block's partial writes (seen through the
    // barrier) before the ticket
    __threadfence();
    const unsigned old = atomicAdd(a.tickets + u, 1u);
    const int last = old + 1u == static_cast<unsigned>(np) ? 1 : 0;
    if (last) {
      __threadfence();    // the other blocks' partials are visible past this point
      a.tickets[u] = 0u;  // every partial of u is in; no other block touches it in this call
    }
    *s_flag = last;
  }
  __syncthreads();
  if (!*s_flag) return;
  const int g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // merge area: (M, L) of 8 heads | slot of each partial | weights [np][g]
  float* MLs = ma;
  int* SL = reinterpret_cast<int*>(ma + 16);
  float* W = ma + 16 + np;
  const bool staged = 16 + np * (g + 1) <= kMergeFloats;
  if (staged)
    for (int p = threadIdx.x; p < np; p += blockDim.x) SL[p] = static_cast<int>(a.P.partial_slot(u, p));
  __syncthreads();
  auto slot_of = [&](int p) -> int64_t { return staged ? static_cast<int64_t>(SL[p]) : a.P.partial_slot(u, p); };
  // (1) per head: online max and sum over the partials, one load per lane and pass
  for (int r = warp; r < g; r += kQNW) {
    float M = -INFINITY, L = 0.f;
    for (int p = lane; p < np; p += 32) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(a.part_ml + (slot_of(p) * g + r) * 2));
      if (ml.x != -INFINITY) {
        const float Mn = fmaxf(M, ml.x);
        L = (M == -INFINITY ? 0.f : L * ex2(M - Mn)) + ml.y * ex2(ml.x - Mn);
        M = Mn;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float Mo = __shfl_xor_sync(FULL, M, o), Lo = __shfl_xor_sync(FULL, L, o);
      const float Mn = fmaxf(M, Mo);
      L = (M == -INFINITY ? 0.f : L * ex2(M - Mn)) + (Mo == -INFINITY ? 0.f : Lo * ex2(Mo - Mn));
      M = Mn;
    }
    if (staged)
      for (int p = lane; p < np; p += 32) {
        const float m = __ldcg(a.part_ml + (slot_of(p) * g + r) * 2);
        W[p * g + r] = (M == -INFINITY || m == -INFINITY) ? 0.f : ex2(m - M);
      }
    if (lane == 0) {
      MLs[2 * r] = M;
      MLs[2 * r + 1] = L;
    }
  }
  __syncthreads();
  // (2) weighted sum of the partials' o
  const int b = u / a.Hkv, h = u - b * a.Hkv;
  float4* out = reinterpret_cast<float4*>(a.out + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(h) * g) * D);
  constexpr int UNR = 16;
  for (int e4 = threadIdx.x; e4 < g * D / 4; e4 += blockDim.x) {
    const int r = e4 / (D / 4);
    const float M = MLs[2 * r], L = MLs[2 * r + 1];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = 0; p0 < np; p0 += UNR) {
      float4 v[UNR];
      float w[UNR];
#pragma unroll
      for (int i = 0; i < UNR; ++i) {
        const int p = p0 + i;
        v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        w[i] = 0.f;
        if (p < np) {
          const int64_t sl = slot_of(p);
          if (staged) {
            w[i] = W[p * g + r];
          } else {
            const float m = __ldcg(a.part_ml + (sl * g + r) * 2);
            w[i] = (M == -INFINITY || m == -INFINITY) ? 0.f : ex2(m - M);
          }
          if (w[i] > 0.f) v[i] = __ldcg(reinterpret_cast<const float4*>(a.part_o + sl * g * D) + e4);
        }
      }
#pragma unroll
      for (int i = 0; i < UNR; ++i) {
        acc.x += w[i] * v[i].x;
        acc.y += w[i] * v[i].y;
        acc.z += w[i] * v[i].z;
        acc.w += w[i] * v[i].w;
      }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    out[e4] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
  __syncthreads();  // the merge area and flag are reused by the next unit
}

template <int BITS, int G, int D, int NT>
__global__ void __launch_bounds__(kQNW * 32, (NT == 1 ? 4 : 2)) draft_quant_kernel(QArgs a) {
  using C = QCfg<BITS, G, D, NT>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x;
  const UPart& P = a.P;
  unsigned char* ring = smem + warp * C::WARP_B;
  float* P_res = reinterpret_cast<float*>(ring + C::RING);  // residual tile scores
  float* st_ml = reinterpret_cast<float*>(smem + C::ML_OFF);
  int* st_off = reinterpret_cast<int*>(smem + C::SO_OFF);
  float* mw = reinterpret_cast<float*>(smem + C::MW_OFF);
  float* ma = reinterpret_cast<float*>(smem + C::MA_OFF);
  int* s_flag = reinterpret_cast<int*>(smem + C::FLAG_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF) + warp * (C::NST + 1);
  if (lane == 0)
    for (int s = 0; s <= C::NST; ++s) mbar_init(&bars[s], 1);
  fence_mbar_init();
  __syncwarp();
  int u0, u1, r0, r1, q0, q1;
  P.block_range(k, u0, u1, r0, r1, q0, q1);
  bool ok = true;
  int rph = 0;
  float* wml = st_ml + warp * C::HEADS * 2;
  const int64_t slot0 = static_cast<int64_t>(k) * 2 * P.upb;
  // this warp's quantised stages: q0 + warp + kQNW i < q1 of every unit of the
  // block (< the request's own stage count with per-request lengths)
  WarpRing r;
  int my_nq = 0;
  auto prime = [&]() {
    for (int u = u0; u < u1; ++u) my_nq += warp_stage_count(q0 + warp, unit_qend<C>(a, u, q1));
    r.issued = 0, r.head = 0, r.tail = 0, r.hslot = 0, r.hphase = 0u;
    r.q_first = q0 + warp, r.q_end = q1, r.u_end = u1;
    int uf = u0;  // first unit where this warp has a stage
    while (uf < u1 && warp_stage_count(q0 + warp, unit_qend<C>(a, uf, q1)) == 0) ++uf;
    issue_start<C>(a, r.ip, uf < u1 ? uf : u0, q0 + warp, q1);
    fence_proxy_async_smem();
    __syncwarp();
    while (r.issued < my_nq && r.issued < C::NST) {
      issue_stage<C>(a, ring, bars, lane, r.issued, r.ip);
      issue_advance<C>(a, r.ip, r.q_first, r.u_end, r.q_end);
      ++r.issued;
    }
  };
  // Launched as a programmatic dependent of the previous kernel in the
  // stream: nothing global is read or written before that grid completed,
  // except, when the caller declares the cache static (VC_CACHE_STATIC: the
  // previous kernel does not write it), the first NST stages of group
  // records of a block without residual tiles, whose copies then overlap the
  // previous kernel's tail.  (A block with residual tiles stages them in its
  // ring first and primes the ring after them.)  The next kernel may be
  // scheduled as this grid's blocks retire (it waits the same way).
  const bool early = (a.cache_flags & VC_CACHE_STATIC) != 0 && r1 <= r0;
  if (early && q1 > q0) prime();
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // residual tiles of each unit (the ring is not primed yet)
  if (r1 > r0) {
    for (int u = u0; u < u1; ++u) {
      residual_seg<D, NT, C::HEADS>(a, ring, P_res, &bars[C::NST], rph, u, r0 + warp, r1, ok,
                                    reinterpret_cast<float*>(ring), wml);
      if (lane == 0) st_off[warp] = static_cast<int>(ring - smem);
      __syncthreads();
      merge_segment<D, C::HEADS>(a, slot0 + 2 * (u - u0), smem, st_off, st_ml, mw);
      unit_finish<D>(a, u, ma, s_flag);
    }
  }
  if (!early && q1 > q0) prime();

  if (q1 > q0) {
    uint4* q_sm = reinterpret_cast<uint4*>(smem + C::QSM_OFF);
    for (int u = u0; u < u1; ++u) {
      if constexpr (NT == 1) {  // the unit's query fragments, shared by the block's warps
        if (warp == 0) TokM<BITS, G, D>::write_q(a, u / a.Hkv, u - (u / a.Hkv) * a.Hkv, lane, q_sm);
        __syncthreads();
      }
      int state_slot = -1;
      const int n_u = warp_stage_count(q0 + warp, unit_qend<C>(a, u, q1));
      quant_seg<BITS, G, D, NT>(a, ring, bars, u, n_u, my_nq, r, ok, wml, state_slot, q_sm);
      if (lane == 0) st_off[warp] = state_slot >= 0 ? static_cast<int>(ring + state_slot * C::STAGE - smem) : -1;
      __syncthreads();
      merge_segment<D, C::HEADS>(a, slot0 + 2 * (u - u0) + 1, smem, st_off, st_ml, mw);
      if (state_slot >= 0) {  // the deferred slot is free again: refill it
        ring_issue_next<C>(a, ring, bars, lane, r, state_slot, my_nq);
        ++r.tail;
      }
      unit_finish<D>(a, u, ma, s_flag);
    }
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
  UPart P;
  int MAXS;
  size_t off_tk, off_ml, off_o, total;
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
  UPart& P = p.P;
  P.U = sh.B * sh.Hkv;
  P.ng = c.L_q / c.group;
  P.sq = static_cast<int>((P.ng + ng_per_stage - 1) / ng_per_stage);
  const int Rp = c.lens ? c.R_cap : c.R;  // per-request lengths: plan for the capacity
  P.sr = (Rp + kResRows - 1) / kResRows;
  P.cq = P.sq > 0 ? static_cast<int64_t>(ng_per_stage) * rec_bytes : 1;
  P.cr = P.sr > 0 ? static_cast<int64_t>(kResRows) * 4 * sh.D * kResCostNum / kResCostDen : 1;
  if (target_blocks < 1) target_blocks = 1;
  if (P.U <= target_blocks) {
    const int64_t mx = P.sq > 0 && P.sr > 0 ? (P.cq > P.cr ? P.cq : P.cr) : (P.sq > 0 ? P.cq : P.cr);
    int64_t bpu = target_blocks / P.U;
    if (bpu > P.ucost() / mx) bpu = P.ucost() / mx;  // every piece holds at least one tile or stage
    // every warp gets at least kMinWarpStages quantised stages: the last
    // block of a unit merges all of the unit's partials at the call's end,
    // so more blocks than that shorten the stages but lengthen the merge
    const int64_t cap = P.sq / (static_cast<int64_t>(kQNW) * kMinWarpStages);
    if (P.sq > 0 && bpu > cap) bpu = cap;
    if (bpu < 1) bpu = 1;
    P.bpu = static_cast<int>(bpu);
    P.nblk = P.U * P.bpu;
    P.upb = 1;
    int jr = 0, jq = P.bpu;
    for (int j = 0; j < P.bpu; ++j) {
      if (P.axis_first(j) < P.sr) jr = j + 1;
      if (jq == P.bpu && P.axis_first(j + 1) > P.sr) jq = j;
    }
    P.jr = jr, P.jq = jq;
    P.np = jr + (P.bpu - jq);
  } else {
    P.bpu = 0;
    P.nblk = static_cast<int>(target_blocks);
    P.upb = static_cast<int>((P.U + target_blocks - 1) / target_blocks);
    P.jr = P.jq = 0;
    P.np = (P.sr > 0 ? 1 : 0) + (P.sq > 0 ? 1 : 0);
  }
  p.MAXS = 2 * P.upb;
  const int g = sh.Hq / sh.Hkv;
  const size_t slots = static_cast<size_t>(P.nblk) * p.MAXS;
  p.off_tk = align_up(sizeof(WsHeader), 256);
  p.off_ml = align_up(p.off_tk + static_cast<size_t>(P.U) * 4, 256);
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
  // programmatic dependent launch: the grid may be scheduled while the
  // previous kernel of the stream drains; it waits for it before reading
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.P.nblk));
  cfg.blockDim = dim3(kQNW * 32);
  cfg.dynamicSmemBytes = C::SMEM_B;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, draft_quant_kernel<BITS, G, D, NT>, a);
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
  if (c->lens == nullptr) {
    VC_REQUIRE(c->R >= 0 && c->R <= c->R_cap, "%s: need 0 <= R <= R_cap", who);
    VC_REQUIRE(c->L_q + c->R >= 1, "%s: the cache holds no token", who);
  } else {
    VC_REQUIRE(c->R_cap >= 0 && c->L_q + c->R_cap >= 1, "%s: the cache has no capacity", who);
    VC_REQUIRE(reinterpret_cast<uintptr_t>(c->lens) % 8 == 0, "%s: lens must be 8-byte aligned", who);
  }
  VC_REQUIRE(static_cast<int64_t>(sh->B) * sh->Hkv <= (int64_t(1) << 24), "%s: too many (request, head) pairs",
             who);
  if (c->L_q > 0) {
    VC_REQUIRE(c->records, "%s: null group-record pointer", who);
    VC_REQUIRE(aligned16(c->records), "%s: group records must be 16-byte aligned", who);
  }
  if ((c->lens ? c->R_cap : c->R) > 0) {
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
  a.group = c.group;
  a.lens = c.lens;
  a.cache_flags = c.flags;
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
  a.tickets = reinterpret_cast<uint32_t*>(w + p.off_tk);
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
                                   int32_t* block_ranges, int max_blocks, int* n_blocks, int* blocks_per_unit,
                                   int* partials_per_unit, int* residual_tiles, int* quant_stages) {
  vc_status st = vc::check_quant(shape, cache, "vc_debug_quant_partition");
  if (st != VC_OK) return st;
  VC_REQUIRE(target_blocks >= 1, "vc_debug_quant_partition: target_blocks must be >= 1");
  VC_REQUIRE(n_blocks && blocks_per_unit && partials_per_unit && residual_tiles && quant_stages,
             "vc_debug_quant_partition: null output");
  vc::QPlan p{};
  if (!vc::quant_plan(*shape, *cache, &p, target_blocks))
    return vc::set_error(VC_ERR_UNSUPPORTED, "vc_debug_quant_partition: no kernel for this configuration");
  *n_blocks = p.P.nblk;
  *blocks_per_unit = p.P.bpu;
  *partials_per_unit = p.P.np;
  *residual_tiles = p.P.sr;
  *quant_stages = p.P.sq;
  if (block_ranges) {
    VC_REQUIRE(max_blocks >= p.P.nblk, "vc_debug_quant_partition: block_ranges needs %d rows", p.P.nblk);
    for (int k = 0; k < p.P.nblk; ++k) {
      int u0, u1, r0, r1, q0, q1;
      p.P.block_range(k, u0, u1, r0, r1, q0, q1);
      int32_t* row = block_ranges + 6 * static_cast<size_t>(k);
      row[0] = u0, row[1] = u1, row[2] = r0, row[3] = r1, row[4] = q0, row[5] = q1;
    }
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
