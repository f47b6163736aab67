// vc_verify.cu -- block verification attention on the sm_100a tensor cores.
//
// The verifier checks every drafted position in one pass over the full KV
// cache and yields one prediction more than there are drafted tokens
// (devshah.ca page "VeriCache: making lossy KV compression exact", section
// "The Core Idea"); verification is bound by the interconnect and by FLOPs
// ("VeriCache: Turning Lossy KV Cache into Lossless LLM Inference",
// menfem.com, "Key Contributions").  The pages give no kernel.
//
// Design.  For one (request, KV head) the nq query rows of all g heads of the
// GQA group form the MMA's M dimension (row r = position i * g + head), so each
// K/V tile is read from HBM once for the whole group.  When nq * g exceeds
// 128 rows (g = 5 or 8 with 31 rows), the rows form two row tiles of <= 128
// rows, and ONE block computes both against each K/V tile it loads: two
// softmax warpgroups, two S double buffers and two O accumulators fill the
// 512 TMEM columns.  Blocks split the context (split-K) and merge through
// the workspace.  Per block:
//   * Q (<= 128 rows per row tile) is staged once into shared memory in the 128-byte
//     swizzled K-major layout by tiled TMA (a 3-D map over positions x heads
//     x channels: the g heads of nqt positions are the tile's rows), the
//     first request of the block so that it does not queue behind K and V;
//   * K and V tiles of BN = 64 keys stream in through 2-slot rings of tiled
//     TMA loads (3-D tensor maps, rows past T read as zeros, no multicast,
//     evict-first in L2), K and V on barriers of their own: a K slot is
//     refilled as soon as the S that read it is done, a V slot once its P.V
//     is done;
//   * a loader warp issues the TMA loads, an MMA warp issues tcgen05.mma:
//     S = Q K^T into tensor memory (TMEM), and P.V; the MMA warp blocks on
//     the tensor pipe's queue while the softmax warps work, so no row waits
//     for it.  S is double buffered: S of tile i + 1 is computed while the
//     softmax of tile i runs;
//   * each softmax thread owns one row of its warpgroup's row tile: it reads its scores from TMEM,
//     applies the causal mask (row i sees keys 0 .. T - nq + i), updates an
//     online softmax with lazy rescaling (O is rescaled only when the running
//     maximum grows by more than 8 in log2 units), and writes P back to TMEM
//     over its own S as a bf16 high part and a bf16 low part (P keeps ~16
//     bits); each softmax warp then arrives on that S buffer's "P stored"
//     mbarrier and goes straight on to the next tile -- the MMA thread waits
//     on the barrier, the softmax warps never wait for the MMA thread;
//   * O += P_hi V + P_lo V as tcgen05.mma with A read from TMEM and V from
//     shared memory (MN-major), accumulating in TMEM;
//   * at the end each softmax thread moves its O row from TMEM to the output
//     (one chunk) or, through shared memory and a TMA store, to its chunk's
//     partial, which splitk_combine_kernel merges in a programmatic-dependent
//     launch.
// All waits are bounded; TMEM is always released.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <type_traits>

#include "vc_splitk.cuh"
#include "vc_tc.cuh"

namespace vc {
namespace {

constexpr int kVBN = 64;        // keys per tile
constexpr int kVThreads = 128;  // one softmax warpgroup: thread r owns row r of its row tile
// Block of RTC row tiles: RTC softmax warpgroups, then the MMA warp and the
// loader warp.
template <int RTC>
struct VBlk {
  static constexpr int SOFTMAX = RTC * kVThreads;
  static constexpr int THREADS = SOFTMAX + 64;
  static constexpr int ISSUER = SOFTMAX;       // the MMA warp's elected thread
  static constexpr int LOADER = SOFTMAX + 32;  // the loader warp's elected thread
  static constexpr uint32_t TMEM_COLS = RTC * 256;
};
// TMEM column map of row tile rt (base rt * 256): two S buffers of kVBN fp32
// columns (tile i in buffer i & 1), each overwritten by its P -- high part in
// the first kVBN / 2 columns, low part in the next (bf16 pairs) -- then O,
// D fp32 columns.
constexpr uint32_t kColS = 0;
constexpr uint32_t kColPlo = kVBN / 2;  // offset of P's low part inside a buffer
constexpr uint32_t kColO = 2 * kVBN;
constexpr uint32_t kColTile = 256;      // columns of one row tile
// One box of a partial's O rows in shared memory for the TMA store: 32 fp32
// channels (128 bytes) x up to 128 rows.
constexpr int kOBox = 128 * 128;

template <int D, int RTC>
struct VCfg {
  static constexpr int HALVES = D / 64;              // 128-byte swizzle atoms across D
  static constexpr int QT_B = 128 * D * 2;           // one row tile: 128 rows
  static constexpr int Q_B = RTC * QT_B;
  static constexpr int KV_B = kVBN * D * 2;          // one of K or V per stage
  static constexpr int STAGE_B = 2 * KV_B;
  // K/V stages in flight per block (measured on B200: 4 stages for the
  // two-row-tile block were no faster than 2)
  static constexpr int NS = 2;
  static constexpr int Q_OFF = 0;
  static constexpr int ST_OFF = Q_B;
  static constexpr int BAR_OFF = ST_OFF + NS * STAGE_B;
  // barriers: K full / K free / V full / V free per stage, S, P and P.V per
  // S buffer, Q, drain; then the TMEM address slot and the abort flag
  static constexpr int NBAR = 4 * NS + 8;
  static constexpr int SMEM_B = BAR_OFF + NBAR * 8 + 16 + 1024;  // + alignment slack
  // the partials' O boxes reuse the Q and K/V area after the tile loop
  static_assert(RTC * (D / 32) * kOBox <= BAR_OFF, "O boxes must fit below the barriers");
};

struct VArgs {
  const __nv_bfloat16* q;
  int64_t T;
  int nq, Hq, Hkv, g, nqt, RT, C, tiles_per_chunk;
  float scale_log2;
  uint32_t* flags;
  SplitKOut o;
  // failure-path test only (vc_debug_verify_abort): the block-local K tile
  // that is never requested (-1: none) and the give-up limit of the tile
  // loop's waits
  int skip_k;
  uint64_t wait_ns;
};

template <int D, int RTC>
__global__ void __launch_bounds__(VBlk<RTC>::THREADS) verify_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                     const __grid_constant__ CUtensorMap tm_k,
                                                                     const __grid_constant__ CUtensorMap tm_v,
                                                                     const __grid_constant__ CUtensorMap tm_o,
                                                                     VArgs a) {
  using C = VCfg<D, RTC>;
  using K = VBlk<RTC>;
  // the chunk-merge launch that follows may be scheduled as this grid's blocks
  // retire; it waits for this grid's completion before reading the partials
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_s = smem + C::Q_OFF;
  unsigned char* st_s = smem + C::ST_OFF;
  constexpr int NS = C::NS;
  uint64_t* bar_k = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);  // [NS] K stage landed
  uint64_t* bar_kf = bar_k + NS;                                      // [NS] K stage read by its S MMAs
  uint64_t* bar_v = bar_kf + NS;                                      // [NS] V stage landed
  uint64_t* bar_vf = bar_v + NS;                                      // [NS] V stage read by its P.V MMAs
  uint64_t* bar_s = bar_vf + NS;                                      // [2] S buffer computed
  uint64_t* bar_p = bar_s + 2;                                        // [2] P of that buffer stored
  uint64_t* bar_pv = bar_p + 2;                                       // [2] P.V of that buffer done
  uint64_t* bar_q = bar_pv + 2;                                       // Q staged
  uint64_t* bar_dr = bar_q + 1;                                       // drain after a give-up
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_dr + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);  // a wait gave up

  const int tid = threadIdx.x, warp = tid >> 5;
  const int chunk = blockIdx.x;
  const int unit = blockIdx.y;  // b * Hkv + h
  // row tile of this thread: blockIdx.z when a block takes one row tile, its
  // warpgroup when the block takes all of them (RTC == 2)
  const int wg = RTC == 1 ? 0 : (tid < K::SOFTMAX ? tid / kVThreads : 0);
  const int rt = RTC == 1 ? static_cast<int>(blockIdx.z) : wg;
  const int b = unit / a.Hkv, h = unit - b * a.Hkv;
  const int i0 = rt * a.nqt;
  const int nq_t = max(0, min(a.nqt, a.nq - i0));
  const int M = nq_t * a.g;  // valid rows of this thread's row tile
  const int64_t k_begin = static_cast<int64_t>(chunk) * a.tiles_per_chunk * kVBN;
  const int64_t k_end = min(a.T, k_begin + static_cast<int64_t>(a.tiles_per_chunk) * kVBN);
  const int ntiles = static_cast<int>((k_end - k_begin + kVBN - 1) / kVBN);
  const bool softmax_thread = tid < K::SOFTMAX;
  bool fail = false;

  // K (v = 0) or V (v = 1) of tile i into stage i % NS; loader only.  K and
  // V are read once: their lines go first when L2 needs room.
  const uint64_t kv_policy = tc::l2_evict_first();
  auto issue_load = [&](int i, int v) {
    unsigned char* dst = st_s + (i % NS) * C::STAGE_B + v * C::KV_B;
    uint64_t* bar = v ? &bar_v[i % NS] : &bar_k[i % NS];
    const int y = static_cast<int>(k_begin + static_cast<int64_t>(i) * kVBN);
    if (v == 0 && i == a.skip_k) return;  // failure-path test: this tile never lands
    mbar_arrive_expect_tx(bar, C::KV_B);
#pragma unroll
    for (int hf = 0; hf < C::HALVES; ++hf)
      tc::tma_load_3d_hint(dst + hf * kVBN * 128, v ? &tm_v : &tm_k, hf * 64, y, unit, bar, kv_policy);
  };

  // The loader owns the barriers' initialisation and requests Q (every row
  // tile of the block), then the first NS tiles; nobody else touches a
  // barrier before the block-wide barrier below.
  if (tid == K::LOADER) {
    for (int j = 0; j < C::NBAR; ++j) mbar_init(&bar_k[j], 1);
    mbar_init(&bar_p[0], K::SOFTMAX / 32);  // one arrival per softmax warp
    mbar_init(&bar_p[1], K::SOFTMAX / 32);
    *s_abort = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar_q, RTC * C::HALVES * 128 * a.g * a.nqt);
#pragma unroll
    for (int t = 0; t < RTC; ++t) {
      const int rtq = RTC == 1 ? rt : t;
#pragma unroll
      for (int hf = 0; hf < C::HALVES; ++hf)
        tc::tma_load_3d(q_s + t * C::QT_B + hf * (128 * 128), &tm_q, hf * 64, h * a.g, b * a.nq + rtq * a.nqt, bar_q);
    }
    for (int j = 0; j < NS && j < ntiles; ++j) {
      issue_load(j, 0);
      issue_load(j, 1);
    }
  }
  if (warp == 0) tc::alloc(tmem_slot, K::TMEM_COLS);

  // ---- Q rows past the TMA tile's g * nqt rows are zeros (rows of the tile
  //      whose position is past nq hold finite data and are never stored)
  const int r = tid - wg * kVThreads;  // row of this softmax thread in its row tile
  unsigned char* q_t = q_s + wg * C::QT_B;
  if (softmax_thread && r >= a.g * a.nqt) {
#pragma unroll
    for (int c = 0; c < D / 8; ++c)
      *reinterpret_cast<uint4*>(q_t + (c >> 3) * (128 * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4)) =
          make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  constexpr uint32_t IDESC_QK = tc::idesc_bf16_f32(128, kVBN, false);
  constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(128, D, true);
  const uint32_t q_base = smem_addr(q_s);
  // this warp's TMEM lanes and its row tile's columns
  const uint32_t lane_off = (static_cast<uint32_t>((warp & 3) * 32) << 16) + static_cast<uint32_t>(wg) * kColTile;

  // row state
  const int i_row = i0 + (r < M ? r / a.g : 0);
  const int64_t vis_end = a.T - a.nq + i_row + 1;  // keys [0, vis_end) visible to this row
  float m_run = -INFINITY, l_run = 0.f;

  // Bounded wait that also gives up as soon as another thread of the block
  // has given up (*s_abort), so that a failure ends the block promptly.
  auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
      if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
      if (*s_abort != 0) return false;
      if (global_timer_ns() - t0 > a.wait_ns) {
        atomicOr(a.flags, VC_FLAG_WAIT_TIMEOUT);
        return false;
      }
    }
  };

  // S = Q K^T of tile i into buffer i & 1 of every row tile: MMA thread, once
  // tile i's K has landed; when those MMAs complete, the S buffer is ready
  // for the softmax and the K stage free for the loader
  auto issue_s = [&](int i) -> bool {
    const uint32_t ks_addr = smem_addr(st_s + (i % NS) * C::STAGE_B);
    if (!wait_or_abort(&bar_k[i % NS], (i / NS) & 1)) return false;
    tc::fence_after_sync();
#pragma unroll
    for (int t = 0; t < RTC; ++t)
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int hf = kk >> 2, ko = (kk & 3) * 32;
        const uint64_t ad = tc::smem_desc_sw128(q_base + t * C::QT_B + hf * (128 * 128) + ko, 16, 1024);
        const uint64_t bd = tc::smem_desc_sw128(ks_addr + hf * (kVBN * 128) + ko, 16, 1024);
        tc::mma_ss(tmem + t * kColTile + kColS + (i & 1) * kVBN, ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
      }
    tc::commit(&bar_s[i & 1]);
    tc::commit(&bar_kf[i % NS]);
    return true;
  };

  if (tid == K::ISSUER) {
    if (!mbar_wait_bounded(bar_q, 0, a.flags)) fail = true;
    if (!fail && ntiles > 0 && !issue_s(0)) fail = true;
    if (!fail && ntiles > 1 && !issue_s(1)) fail = true;
    if (fail) *s_abort = 1;
  }

  // Failure handling: every wait is bounded; a thread that sees a timeout sets
  // its sticky `fail` and the block's abort flag, and every other wait gives
  // up once it sees the flag.  tcgen05.ld / st are warp-collective, so each
  // warp decides them with __any_sync; a softmax warp that gives up still
  // arrives on its P barrier (after setting the flag), so the MMA thread does
  // not wait for it.  All meet again after the loop.
  constexpr unsigned FULL = 0xffffffffu;
  int nk = ntiles < NS ? ntiles : NS, nv = nk;  // K / V tiles issued so far (loader)
  if (warp == K::LOADER / 32) {
    // ---- loader: K of tile j once the S MMAs of tile j - NS released its
    //      stage, V of tile j once the P.V MMAs of tile j - NS did, in the
    //      order those happen (K runs a tile ahead of V).  A stage's "free"
    //      barrier completes once per tile that used the stage, and its next
    //      completion needs this very load, so its phase cannot run ahead of
    //      the wait.
    if (tid == K::LOADER) {
      while (nk < ntiles || nv < ntiles) {
        const bool is_k = nk < ntiles && nk <= nv + 1;
        const int j = is_k ? nk : nv;
        if (!wait_or_abort(is_k ? &bar_kf[j % NS] : &bar_vf[j % NS], (j / NS - 1) & 1)) {
          fail = true;
          *s_abort = 1;
          break;
        }
        issue_load(j, is_k ? 0 : 1);
        if (is_k)
          nk = j + 1;
        else
          nv = j + 1;
      }
    }
    __syncwarp();  // the other lanes wait here, not in a barrier poll
  } else if (softmax_thread) {
    // ---- softmax warps: S of tile i -> P of tile i (over S), then one
    //      arrival per warp on the buffer's "P stored" barrier; they go on
    //      to tile i + 1 without waiting for the MMA warp
    for (int i = 0; i < ntiles; ++i) {
      const int s = i & 1;
      if (__any_sync(FULL, *s_abort != 0)) {
        fail = true;
        break;
      }
      if (!fail && !wait_or_abort(&bar_s[s], (i >> 1) & 1)) fail = true;
      tc::fence_after_sync();
      bool wfail = __any_sync(FULL, fail);
      uint32_t sr[2][32];
      if (!wfail) {
        tc::ld32(tmem + lane_off + kColS + s * kVBN, sr[0]);
        tc::ld32(tmem + lane_off + kColS + s * kVBN + 32, sr[1]);
        tc::wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) sr[0][j] = sr[1][j] = 0u;
      }
      const int64_t t0 = k_begin + static_cast<int64_t>(i) * kVBN;
      const int64_t lim = min(vis_end, k_end) - t0;  // keys [t0, t0 + lim) are live
      // raw scores; the scale (> 0) is applied in the exponent's FMA below
      float tmax = -INFINITY;
      if (__all_sync(FULL, lim >= kVBN)) {  // whole tile visible to the warp's rows: no mask
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j) tmax = fmaxf(tmax, __uint_as_float(sr[c][j]));
      } else {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float x = (c * 32 + j < lim) ? __uint_as_float(sr[c][j]) : -INFINITY;
            sr[c][j] = __float_as_uint(x);
            tmax = fmaxf(tmax, x);
          }
      }
      tmax *= a.scale_log2;
      // lazy rescale: keep the stale maximum unless the new one exceeds it by > 8
      float m_use = m_run;
      float alpha = 1.f;
      if (tmax > m_run + 8.f || (m_run == -INFINITY && tmax != -INFINITY)) {
        m_use = tmax;
        if (m_run != -INFINITY) alpha = ex2(m_run - m_use);
        m_run = m_use;
      }
      const float m_sub = m_use == -INFINITY ? 0.f : m_use;
      uint32_t phi[32], plo[32];
      float psum = 0.f;
      // pairs of columns in packed fp32x2 arithmetic (each half rounds as the
      // scalar instruction would)
      const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(-m_sub, -m_sub);
      const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 e = __ffma2_rn(make_float2(__uint_as_float(sr[c][j]), __uint_as_float(sr[c][j + 1])), sc2, nm2);
          const float p0 = ex2(e.x), p1 = ex2(e.y);
          psum += p0 + p1;
          const uint32_t hw = pack_bf2(p0, p1);
          const float2 lo = __ffma2_rn(unpack_bf2(hw), neg1, make_float2(p0, p1));  // p - bf16(p), exact
          phi[c * 16 + j / 2] = hw;
          plo[c * 16 + j / 2] = pack_bf2(lo.x, lo.y);
        }
      l_run = l_run * alpha + psum;
      // O is rescaled only when a row of the warp raised its maximum (rare
      // with the lazy rule); only then must the previous P.V be done first.
      // P goes over this tile's own S buffer, which no MMA in flight reads,
      // so storing it needs no wait: the softmax of tile i overlaps P.V of
      // tile i - 1.
      const bool rescale = __any_sync(FULL, alpha != 1.f);  // warp-uniform
      if (rescale) {
        if (i > 0 && !fail && !wait_or_abort(&bar_pv[(i - 1) & 1], ((i - 1) >> 1) & 1)) fail = true;
        tc::fence_after_sync();
      }
      wfail = __any_sync(FULL, fail);
      if (!wfail && rescale) {  // lanes without a new max scale by 1
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tc::ld32(tmem + lane_off + kColO + c0, o);
          tc::wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tc::st32(tmem + lane_off + kColO + c0, o);
        }
      }
      if (!wfail) {  // P over this tile's S, read above
        tc::st32(tmem + lane_off + kColS + s * kVBN, phi);
        tc::st32(tmem + lane_off + kColS + s * kVBN + kColPlo, plo);
        tc::wait_st();
      }
      tc::fence_before_sync();
      __syncwarp();
      if (wfail) {
        if ((tid & 31) == 0) *s_abort = 1;  // seen by the MMA thread after its wait below
        __syncwarp();
      }
      if ((tid & 31) == 0) mbar_arrive(&bar_p[s]);
      if (wfail) {
        fail = true;
        break;
      }
    }
  } else if (warp == K::ISSUER / 32) {
    if (tid == K::ISSUER) {
      // ---- MMA thread: P.V of tile i once every softmax warp stored P (and
      //      any rescale of O); once that P.V is done, S of tile i + 2 into the
      //      same buffer
      for (int i = 0; i < ntiles; ++i) {
        const int s = i & 1;
        const uint32_t vs_addr = smem_addr(st_s + (i % NS) * C::STAGE_B) + C::KV_B;
        if (!wait_or_abort(&bar_p[s], (i >> 1) & 1) || *s_abort != 0) fail = true;
        tc::fence_after_sync();
        if (!fail && !wait_or_abort(&bar_v[i % NS], (i / NS) & 1)) fail = true;
        if (!fail) {
#pragma unroll
          for (int t = 0; t < RTC; ++t) {
            const uint32_t pcol = t * kColTile + kColS + s * kVBN;
            const uint32_t ocol = t * kColTile + kColO;
#pragma unroll
            for (int j = 0; j < kVBN / 16; ++j) {
              const uint64_t vd = tc::smem_desc_sw128(vs_addr + j * 2048, kVBN * 128, 1024);
              tc::mma_ts(tmem + ocol, tmem + pcol + 8 * j, vd, IDESC_PV, (i > 0 || j > 0) ? 1u : 0u);
            }
#pragma unroll
            for (int j = 0; j < kVBN / 16; ++j) {
              const uint64_t vd = tc::smem_desc_sw128(vs_addr + j * 2048, kVBN * 128, 1024);
              tc::mma_ts(tmem + ocol, tmem + pcol + kColPlo + 8 * j, vd, IDESC_PV, 1u);
            }
          }
          tc::commit(&bar_pv[s]);
          tc::commit(&bar_vf[i % NS]);
        }
        if (!fail && i + 2 < ntiles) {
          // P.V of tile i done: its S buffers take tile i + 2
          if (!wait_or_abort(&bar_pv[s], (i >> 1) & 1) || !issue_s(i + 2)) fail = true;
        }
        if (fail) {
          *s_abort = 1;
          break;
        }
      }
    }
    __syncwarp();
  }

  // ---- drain, read O, release TMEM
  if (!fail && ntiles > 0 && !wait_or_abort(&bar_pv[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1)) fail = true;
  tc::fence_after_sync();
  const bool aborted = __syncthreads_or(fail) != 0;
  if (aborted && tid == K::ISSUER) {
    // let MMAs already issued finish before TMEM is released: a commit
    // arrives once every earlier MMA of this thread is done (bounded wait)
    tc::commit(bar_dr);
    mbar_wait_bounded(bar_dr, 0, nullptr, 100000000ull);
  }
  if (aborted && tid == K::LOADER) {
    // and the loads still in flight: Q, and the last tile issued into each
    // stage (earlier ones into it were consumed, hence landed)
    mbar_wait_bounded(bar_q, 0, nullptr, 100000000ull);
    for (int v = 0; v < 2; ++v) {
      const int n = v ? nv : nk;
      for (int j = n - NS; j < n; ++j)
        if (j >= 0) mbar_wait_bounded(v ? &bar_v[j % NS] : &bar_k[j % NS], (j / NS) & 1, nullptr, 100000000ull);
    }
  }
  __syncthreads();
  const bool ok = !aborted;
  // ---- O rows from TMEM: with one chunk the normalised output rows (and
  //      lse) straight to global memory; otherwise this chunk's partial
  //      (unnormalised O, m, l) for splitk_combine_kernel.  A partial's O
  //      rows are contiguous in the workspace, so the softmax threads write
  //      them into shared memory (free once the last P.V is done) in the
  //      128-byte-swizzled layout of the partials' tensor map -- one box of
  //      32 channels x the row tile's rows per 16 KB, bank-conflict free --
  //      and the loader thread stores the boxes with TMA: coalesced full
  //      lines instead of one 512-byte row per lane.  Rows past M are never
  //      read back.
  if (softmax_thread && ok) {
    const bool live = r < M;
    const bool any = ntiles > 0;
    const int rows_cap = a.nqt * a.g;
    const float m_out = any ? m_run : -INFINITY;
    const float l_out = any ? l_run : 0.f;
    if (a.C == 1) {
      const size_t orow = (static_cast<size_t>(b) * a.nq + i0 + r / a.g) * a.Hq + h * a.g + r % a.g;
      float* dst = a.o.out + orow * D;
      const float sc = (any && l_run > 0.f) ? 1.f / l_run : 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (any) {
          tc::ld32(tmem + lane_off + kColO + c0, o);  // warp-collective: every lane
          tc::wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = 0u;
        }
        if (live) {
          float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            d4[j / 4] = make_float4(__uint_as_float(o[j]) * sc, __uint_as_float(o[j + 1]) * sc,
                                    __uint_as_float(o[j + 2]) * sc, __uint_as_float(o[j + 3]) * sc);
        }
      }
      if (live && a.o.lse) a.o.lse[orow] = lse_from(m_out, l_out);
    } else {
      unsigned char* ob = smem + wg * (D / 32) * kOBox + r * 128;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (any) {
          tc::ld32(tmem + lane_off + kColO + c0, o);  // warp-collective: every lane
          tc::wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = 0u;
        }
        if (r < rows_cap) {
          unsigned char* row = ob + (c0 / 32) * kOBox;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(row + ((q ^ (r & 7)) << 4)) =
                make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        }
      }
      fence_proxy_async_smem();  // the boxes are read by the TMA store (async proxy)
      if (live) {
        const size_t slot = (static_cast<size_t>(unit) * a.RT + rt) * a.C + chunk;
        a.o.part_ml[(slot * rows_cap + r) * 2] = m_out;
        a.o.part_ml[(slot * rows_cap + r) * 2 + 1] = l_out;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::dealloc(tmem, K::TMEM_COLS);
  }
  if (a.C > 1 && ok && tid == K::LOADER) {
#pragma unroll 1
    for (int t = 0; t < RTC; ++t) {
      const int rts = RTC == 1 ? rt : t;
      const int slot = (unit * a.RT + rts) * a.C + chunk;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tc::tma_store_3d(&tm_o, smem + (t * (D / 32) + c) * kOBox, c * 32, 0, slot);
    }
    tc::bulk_commit();
    tc::bulk_wait_read();  // the shared memory must outlive the stores' reads
  }
}

// Output row of flattened partial row fr = ((unit * RT + rt) * rows_cap + r),
// for splitk_combine_kernel: row r of row tile rt is query i = rt * nqt + r / g
// of head h * g + r % g.
struct VerifyRowMap {
  int rows_cap, RT, Hkv, nq, nqt, g, Hq, D;
  __device__ bool locate(int64_t fr, int& unit_rt, int& r, size_t& out_off, size_t& lse_off) const {
    const int64_t uu = fr / rows_cap;
    r = static_cast<int>(fr - uu * rows_cap);
    const int rt = static_cast<int>(uu % RT);
    const int64_t unit = uu / RT;
    const int i = rt * nqt + r / g;
    if (r / g >= nqt || i >= nq) return false;
    const int b = static_cast<int>(unit / Hkv), h = static_cast<int>(unit % Hkv);
    const size_t row = (static_cast<size_t>(b) * nq + i) * Hq + h * g + r % g;
    out_off = row * D;
    lse_off = row;
    unit_rt = static_cast<int>(uu);
    return true;
  }
};

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D map over [units][T][D] bf16 with a box of 64 channels x kVBN keys x 1.
bool make_kv_map(CUtensorMap* m, const void* base, int64_t T, int D, int units) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(units)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(T) * D * 2};
  cuuint32_t box[3] = {64, kVBN, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the chunk partials' O [slots][rows_cap][D] fp32 with a box of
// 32 channels x rows_cap rows x 1 slot, 128-byte swizzle (the kernel's
// shared-memory layout of a box).
bool make_part_map(CUtensorMap* m, float* base, int rows_cap, int D, int64_t slots) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows_cap), static_cast<cuuint64_t>(slots)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4, static_cast<cuuint64_t>(rows_cap) * D * 4};
  cuuint32_t box[3] = {32, static_cast<cuuint32_t>(rows_cap), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over Q [B * nq][Hq][D] bf16 with a box of 64 channels x g heads x
// nqt positions: one box is the 128-byte-swizzled rows (position, head) of a
// row tile, for one half of the channels.
bool make_q_map(CUtensorMap* m, const void* base, int64_t positions, int Hq, int D, int g, int nqt) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hq), static_cast<cuuint64_t>(positions)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(Hq) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(g), static_cast<cuuint32_t>(nqt)};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct VPlan {
  int nqt, RT, C, tiles_per_chunk;
  int RTC;  // row tiles per block (RT when two row tiles share each K/V tile, else 1)
  size_t off_ml, off_o, total;
};

// Resident blocks per SM of one instance (cached per device; also sets the
// kernel's shared-memory attribute on that device).
template <int D, int RTC>
int verify_occupancy() {
  using C = VCfg<D, RTC>;
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    cudaFuncSetAttribute(verify_kernel<D, RTC>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_B);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, verify_kernel<D, RTC>, VBlk<RTC>::THREADS, C::SMEM_B) !=
            cudaSuccess ||
        n < 1)
      n = 1;
    cache[dev] = n;
  }
  return cache[dev];
}

// Split of the context into C chunks per unit: the C that
// minimises waves x (tiles per chunk + 2), where a wave is SMs x resident
// blocks and the 2 stands for a block's fixed cost (its query load, pipeline
// fill and partial write).
VPlan plan_verify(const vc_attn_shape& sh, int64_t T, int nq) {
  VPlan p{};
  const int g = sh.Hq / sh.Hkv;
  p.nqt = 128 / g;
  if (p.nqt > nq) p.nqt = nq;
  p.RT = (nq + p.nqt - 1) / p.nqt;  // 1 or 2 (nq <= 32, g <= 8)
  const int units = sh.B * sh.Hkv;
  // Two row tiles: one block per unit computes both against each K/V tile it
  // loads (K/V read once), or one block per row tile (two blocks per SM).
  // Measured on B200 at 31 rows: with 8 (request, KV head) units the shared
  // block is 16% faster (g = 8 at 131K keys, g = 5 at 100K), with 32 units
  // (4 x 32K, g = 8) it is 5-8% slower -- its tile loop is bound by the
  // tensor pipe's round trips, not by HBM, so it pays off only when the
  // separate blocks' second read of K/V is what limits them.
  p.RTC = (p.RT == 2 && units <= 16) ? 2 : 1;
  const int64_t tiles = (T + kVBN - 1) / kVBN;
  const int occ = p.RTC == 2 ? (sh.D == 128 ? verify_occupancy<128, 2>() : verify_occupancy<64, 2>())
                             : (sh.D == 128 ? verify_occupancy<128, 1>() : verify_occupancy<64, 1>());
  const int64_t slots = static_cast<int64_t>(occ) * sm_count();
  const int64_t n = static_cast<int64_t>(units) * (p.RT / p.RTC);
  int64_t c = 1, best = -1;
  for (int64_t cc = 1; cc <= tiles && cc <= 256; ++cc) {
    const int64_t waves = (n * cc + slots - 1) / slots;
    const int64_t cost = waves * ((tiles + cc - 1) / cc + 2);
    if (best < 0 || cost < best) {
      best = cost;
      c = cc;
    }
  }
  int64_t tpc = (tiles + c - 1) / c;
  p.tiles_per_chunk = static_cast<int>(tpc);
  p.C = static_cast<int>((tiles + tpc - 1) / tpc);
  const int rows = p.nqt * g;
  const size_t nunit = static_cast<size_t>(units) * p.RT;
  p.off_ml = align_up(sizeof(WsHeader), 256);
  p.off_o = align_up(p.off_ml + nunit * p.C * rows * 2 * 4, 256);
  p.total = align_up(p.off_o + nunit * p.C * rows * sh.D * 4, 256);
  return p;
}

vc_status check_verify(const vc_attn_shape* sh, int64_t T, int nq, const char* who) {
  VC_REQUIRE(sh, "%s: null shape", who);
  VC_REQUIRE(sh->B >= 1 && sh->Hkv >= 1 && sh->Hq >= 1 && sh->Hq % sh->Hkv == 0 && sh->Hq / sh->Hkv <= 8,
             "%s: need B >= 1, Hq a multiple of Hkv, Hq/Hkv <= 8", who);
  VC_REQUIRE(sh->D == 64 || sh->D == 128, "%s: head dim must be 64 or 128 (got %d)", who, sh->D);
  VC_REQUIRE(nq >= 1 && nq <= 32, "%s: need 1 <= nq <= 32 (got %d)", who, nq);
  VC_REQUIRE(T >= nq && T < (int64_t(1) << 31), "%s: need nq <= T < 2^31", who);
  VC_REQUIRE(static_cast<int64_t>(sh->B) * sh->Hkv <= 65535, "%s: too many (request, head) pairs", who);
  return VC_OK;
}

}  // namespace
}  // namespace vc

extern "C" {

size_t vc_verify_attn_workspace_size(const vc_attn_shape* shape, int64_t T, int nq) {
  if (vc::check_verify(shape, T, nq, "vc_verify_attn_workspace_size") != VC_OK) return 0;
  return vc::plan_verify(*shape, T, nq).total;
}

}  // extern "C"

namespace vc {
namespace {
vc_status verify_launch(const vc_attn_shape* shape, const void* q, const void* k, const void* v, int64_t T, int nq,
                        float* out, float* lse, void* ws, size_t ws_bytes, void* stream, int skip_k,
                        uint64_t wait_ns) {
  vc_status st = vc::check_verify(shape, T, nq, "vc_verify_attn");
  if (st != VC_OK) return st;
  VC_REQUIRE(q && k && v && out && ws, "vc_verify_attn: null pointer argument");
  VC_REQUIRE(vc::aligned16(q) && vc::aligned16(k) && vc::aligned16(v) && vc::aligned16(out) && vc::aligned16(ws),
             "vc_verify_attn: q, k, v, out and workspace must be 16-byte aligned");
  const vc::VPlan p = vc::plan_verify(*shape, T, nq);
  VC_REQUIRE(ws_bytes >= p.total, "vc_verify_attn: workspace too small (%zu < %zu)", ws_bytes, p.total);
  const int units = shape->B * shape->Hkv;
  CUtensorMap tq, tk, tv;
  if (!vc::make_kv_map(&tk, k, T, shape->D, units) || !vc::make_kv_map(&tv, v, T, shape->D, units) ||
      !vc::make_q_map(&tq, q, static_cast<int64_t>(shape->B) * nq, shape->Hq, shape->D, shape->Hq / shape->Hkv, p.nqt))
    return vc::set_error(VC_ERR_CUDA, "vc_verify_attn: could not encode the Q/K/V tensor maps");
  char* w = static_cast<char*>(ws);
  vc::VArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.T = T;
  a.nq = nq;
  a.Hq = shape->Hq;
  a.Hkv = shape->Hkv;
  a.g = shape->Hq / shape->Hkv;
  a.nqt = p.nqt;
  a.RT = p.RT;
  a.C = p.C;
  a.tiles_per_chunk = p.tiles_per_chunk;
  const float sm = shape->sm_scale > 0.f ? shape->sm_scale : 1.0f / sqrtf(static_cast<float>(shape->D));
  a.scale_log2 = sm * 1.4426950408889634f;
  a.flags = reinterpret_cast<uint32_t*>(w);
  a.skip_k = skip_k;
  a.wait_ns = wait_ns;
  a.o.out = out;
  a.o.lse = lse;
  a.o.part_ml = reinterpret_cast<float*>(w + p.off_ml);
  a.o.part_o = reinterpret_cast<float*>(w + p.off_o);
  CUtensorMap to;
  memset(&to, 0, sizeof(to));
  if (p.C > 1 && !vc::make_part_map(&to, a.o.part_o, p.nqt * a.g, shape->D, static_cast<int64_t>(units) * p.RT * p.C))
    return vc::set_error(VC_ERR_CUDA, "vc_verify_attn: could not encode the partials' tensor map");
  dim3 grid(p.C, units, p.RT / p.RTC);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto go = [&](auto DD, auto RR) {
    constexpr int Dv = decltype(DD)::value, Rv = decltype(RR)::value;
    vc::verify_occupancy<Dv, Rv>();  // sets the shared-memory attribute once per device
    vc::verify_kernel<Dv, Rv><<<grid, vc::VBlk<Rv>::THREADS, vc::VCfg<Dv, Rv>::SMEM_B, s>>>(tq, tk, tv, to, a);
  };
  using I128 = std::integral_constant<int, 128>;
  using I64 = std::integral_constant<int, 64>;
  using R1 = std::integral_constant<int, 1>;
  using R2 = std::integral_constant<int, 2>;
  if (shape->D == 128) {
    if (p.RTC == 2) go(I128{}, R2{}); else go(I128{}, R1{});
  } else {
    if (p.RTC == 2) go(I64{}, R2{}); else go(I64{}, R1{});
  }
  if (p.C > 1) {  // chunk partials -> output rows (and lse)
    const int rows_cap = p.nqt * a.g;
    const vc::VerifyRowMap map{rows_cap, p.RT, shape->Hkv, nq, p.nqt, a.g, shape->Hq, shape->D};
    const int64_t n_rows = static_cast<int64_t>(units) * p.RT * rows_cap;
    // many chunks (long contexts, few units): one block per row
    const bool wide = p.C >= 16 && p.C <= vc::kWideMaxS;
    if (shape->D == 128) {
      if (wide)
        vc::launch_splitk_combine_wide<128>(a.o, p.C, rows_cap, n_rows, map, s);
      else
        vc::launch_splitk_combine<128>(a.o, p.C, rows_cap, n_rows, map, s);
    } else {
      if (wide)
        vc::launch_splitk_combine_wide<64>(a.o, p.C, rows_cap, n_rows, map, s);
      else
        vc::launch_splitk_combine<64>(a.o, p.C, rows_cap, n_rows, map, s);
    }
  }
  return vc::launch_status("vc_verify_attn");
}
}  // namespace
}  // namespace vc

extern "C" {

vc_status vc_verify_attn(const vc_attn_shape* shape, const void* q, const void* k, const void* v, int64_t T, int nq,
                         float* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  return vc::verify_launch(shape, q, k, v, T, nq, out, lse, ws, ws_bytes, stream, -1, 2000000000ull);
}

vc_status vc_debug_verify_abort(const vc_attn_shape* shape, const void* q, const void* k, const void* v, int64_t T,
                                int nq, float* out, float* lse, void* ws, size_t ws_bytes, int skip_tile,
                                int64_t limit_ns, void* stream) {
  VC_REQUIRE(skip_tile >= 0, "vc_debug_verify_abort: skip_tile must be >= 0 (got %d)", skip_tile);
  VC_REQUIRE(limit_ns >= 1000 && limit_ns <= 100000000,
             "vc_debug_verify_abort: limit must be 1 us .. 100 ms (got %lld ns)", static_cast<long long>(limit_ns));
  return vc::verify_launch(shape, q, k, v, T, nq, out, lse, ws, ws_bytes, stream, skip_tile,
                           static_cast<uint64_t>(limit_ns));
}

}  // extern "C"
