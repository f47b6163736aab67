// vc_draft_sparse.cu -- single-token draft attention over a token-dropped
// KV cache (kept-position lists with the same count for every head).
//
// Pages: the compressed cache drafts one token per step from HBM
// ("VeriCache: Turning Lossy KV Cache into Lossless LLM Inference",
// menfem.com, "Key Contributions"); a dropping compressor is described by its
// kept positions, with equal counts per layer and head ("Limitations").
//
// Design (sm_100a, HBM-bound): grid (S chunks, B * Hkv), one wave of the
// resident blocks (plan_sparse).  A block owns CH
// consecutive kept positions of one (request, KV head); its warps take
// 16-row tiles round-robin.  Each warp gathers its tile's K and V rows with
// one 1-D bulk copy per row (lane l copies K row l, lane 16 + l V row l) into
// a private NST-deep shared-memory ring completed by mbarriers, so the
// gathers of later tiles overlap the math of the current one.  The math is
// warp-level tensor-core MMA in the FA2 arrangement: S = Q K^T with the g
// query heads of the group as MMA rows (the GQA group shares one K/V read),
// an online softmax per head in registers, and O += P V with P split into a
// bf16 high part (rows 0..7) and a bf16 low part (rows 8..15) so that P
// keeps ~16 significant bits.  Per-warp states merge in shared memory; blocks
// merge through the workspace (vc_splitk.cuh).
#include "vc_splitk.cuh"

namespace vc {
namespace {

constexpr int kSpNW = 4;   // warps per block
constexpr int kSpNST = 2;  // ring stages per warp (3 blocks per SM)

template <int D>
struct SpCfg {
  static constexpr int ROW_B = D * 2;            // bytes of one bf16 row
  static constexpr int RS = ROW_B + 16;          // padded smem row stride
  static constexpr int STAGE_B = 32 * RS;        // 16 K rows + 16 V rows
  static constexpr int KT = D / 16;              // k-tiles over channels
  static constexpr int NTO = D / 8;              // output n-tiles over channels
  static constexpr int WARP_B = kSpNST * STAGE_B;
  static constexpr int RING_B = kSpNW * WARP_B;
  static constexpr int BAR_OFF = RING_B;                         // kSpNW * kSpNST mbarriers
  static constexpr int MASK_OFF = BAR_OFF + kSpNW * kSpNST * 8;  // valid masks
  static constexpr int SMEM_B = MASK_OFF + kSpNW * kSpNST * 4 + 16;
};

struct SpArgs {
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* idx;
  const __nv_bfloat16* q;
  int64_t T_store;
  int n_keep, Hq, Hkv, g, S, CH;
  float scale_log2;
  uint32_t* flags;
  SplitKOut o;
};

template <int D>
__global__ void __launch_bounds__(kSpNW * 32) draft_sparse_kernel(SpArgs a) {
  using C = SpCfg<D>;
  // the chunk-merge launch that follows may be scheduled as this grid's blocks
  // retire; it waits for this grid's completion before reading the partials
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  extern __shared__ __align__(128) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int unit = blockIdx.y;  // b * Hkv + h
  const int b = unit / a.Hkv, h = unit - b * a.Hkv;
  const int chunk = blockIdx.x;
  const int t_begin = chunk * a.CH;
  const int t_end = min(a.n_keep, t_begin + a.CH);
  const int ntiles = (t_end - t_begin + 15) / 16;

  unsigned char* ring = smem + warp * C::WARP_B;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF) + warp * kSpNST;
  uint32_t* masks = reinterpret_cast<uint32_t*>(smem + C::MASK_OFF) + warp * kSpNST;
  if (lane == 0)
    for (int s = 0; s < kSpNST; ++s) mbar_init(&bars[s], 1);
  fence_mbar_init();
  __syncwarp();

  const size_t head_off = static_cast<size_t>(unit) * a.T_store * D;
  const __nv_bfloat16* kh = a.k + head_off;
  const __nv_bfloat16* vh = a.v + head_off;
  const int32_t* ih = a.idx + static_cast<size_t>(unit) * a.n_keep;

  // my tiles: j = warp, warp + NW, ...
  const int my_n = ntiles > warp ? (ntiles - warp + kSpNW - 1) / kSpNW : 0;

  auto issue = [&](int i) {  // issue the gathers of my i-th tile into stage i % NST
    const int s = i % kSpNST;
    const int t0 = t_begin + (warp + i * kSpNW) * 16;
    const int r = lane & 15;
    const int t = t0 + r;
    bool valid = t < t_end;
    int pos = valid ? __ldg(ih + t) : 0;
    if (valid && (pos < 0 || static_cast<int64_t>(pos) >= a.T_store)) {
      if (lane < 16 && a.flags) atomicOr(a.flags, VC_FLAG_BAD_INDEX);
      valid = false;
      pos = 0;
    }
    if (!valid) pos = 0;  // copy a real row; its score is masked below
    const uint32_t m = __ballot_sync(0xffffffffu, valid) & 0xffffu;
    if (lane == 0) {
      masks[s] = m;
      mbar_arrive_expect_tx(&bars[s], 32u * C::ROW_B);
    }
    __syncwarp();
    const __nv_bfloat16* src = (lane < 16 ? kh : vh) + static_cast<size_t>(pos) * D;
    bulk_g2s_once(ring + s * C::STAGE_B + lane * C::RS, src, C::ROW_B, &bars[s]);
  };

  // Q fragments: rows 0..7 = query heads of this group (zero beyond g),
  // rows 8..15 = 0.  a0a1 / a4a5 per k-tile.
  uint32_t qf[C::KT][2];
  {
    const int hq = h * a.g + gid;
    const __nv_bfloat16* qp = a.q + (static_cast<size_t>(b) * a.Hq + hq) * D;
#pragma unroll
    for (int kt = 0; kt < C::KT; ++kt) {
      if (gid < a.g) {
        qf[kt][0] = *reinterpret_cast<const uint32_t*>(qp + kt * 16 + 2 * tig);
        qf[kt][1] = *reinterpret_cast<const uint32_t*>(qp + kt * 16 + 8 + 2 * tig);
      } else {
        qf[kt][0] = qf[kt][1] = 0u;
      }
    }
  }

  float acc[C::NTO][4];
#pragma unroll
  for (int n = 0; n < C::NTO; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  bool ok = true;

  const int pre = my_n < kSpNST - 1 ? my_n : kSpNST - 1;
  for (int i = 0; i < pre; ++i) issue(i);

  for (int i = 0; i < my_n && ok; ++i) {
    if (i + kSpNST - 1 < my_n) {
      fence_proxy_async_smem();
      issue(i + kSpNST - 1);
    }
    const int s = i % kSpNST;
    ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[s], (i / kSpNST) & 1, a.flags));  // warp-uniform
    if (!ok) break;
    const unsigned char* Ks = ring + s * C::STAGE_B;
    const unsigned char* Vs = Ks + 16 * C::RS;
    const uint32_t vmask = masks[s];

    // ---- S = Q K^T over 16 tokens (two n-tiles of 8)
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int kt = 0; kt < C::KT; kt += 2) {
        uint32_t bf[4];
        const int mi = lane >> 3, ri = lane & 7;
        ldsm_x4(bf, Ks + (nt * 8 + ri) * C::RS + (kt * 16 + mi * 8) * 2);
        const uint32_t a0[4] = {qf[kt][0], 0u, qf[kt][1], 0u};
        mma_bf16(sc[nt], a0, bf[0], bf[1]);
        const uint32_t a1[4] = {qf[kt + 1][0], 0u, qf[kt + 1][1], 0u};
        mma_bf16(sc[nt], a1, bf[2], bf[3]);
      }
    }
    // ---- online softmax for head row gid (tokens 2tig, 2tig+1, 8+2tig, 9+2tig)
    float p[4];
    {
      float x[4] = {sc[0][0], sc[0][1], sc[1][0], sc[1][1]};
      const int tok[4] = {2 * tig, 2 * tig + 1, 8 + 2 * tig, 9 + 2 * tig};
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[j] = ((vmask >> tok[j]) & 1u) ? x[j] * a.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, x[j]);
      }
      tmax = warp_max_xor(tmax, 1);
      tmax = warp_max_xor(tmax, 2);
      const float m_new = fmaxf(m_run, tmax);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = ex2(m_run - m_use);
      float ps = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        p[j] = ex2(x[j] - m_use);
        ps += p[j];
      }
      l_run = l_run * alpha + ps;
      m_run = m_new;
#pragma unroll
      for (int n = 0; n < C::NTO; ++n) {
        acc[n][0] *= alpha;
        acc[n][1] *= alpha;
        acc[n][2] *= alpha;
        acc[n][3] *= alpha;
      }
    }
    // ---- P as the A operand: rows 0..7 high bf16 part, rows 8..15 low part
    uint32_t pa[4];
    {
      const uint32_t hi01 = pack_bf2(p[0], p[1]);
      const uint32_t hi23 = pack_bf2(p[2], p[3]);
      const float2 h01 = unpack_bf2(hi01), h23 = unpack_bf2(hi23);
      pa[0] = hi01;
      pa[1] = pack_bf2(p[0] - h01.x, p[1] - h01.y);
      pa[2] = hi23;
      pa[3] = pack_bf2(p[2] - h23.x, p[3] - h23.y);
    }
    // ---- O += P V (V^T fragments via transposed ldmatrix)
#pragma unroll
    for (int n = 0; n < C::NTO; n += 2) {
      uint32_t bf[4];
      const int mi = lane >> 3, ri = lane & 7;
      ldsm_x4_t(bf, Vs + (ri + (mi & 1) * 8) * C::RS + (n * 8 + (mi >> 1) * 8) * 2);
      mma_bf16(acc[n], pa, bf[0], bf[1]);
      mma_bf16(acc[n + 1], pa, bf[2], bf[3]);
    }
    __syncwarp();
  }
  if (!ok) {
    // drain my copies still in flight (bounded) before the ring is reused
    for (int i = 0; i < my_n; ++i) mbar_wait_bounded(&bars[i % kSpNST], (i / kSpNST) & 1, nullptr, 100000000ull);
    m_run = -INFINITY;
    l_run = 0.f;
  }

  // ---- per-warp state -> this warp's own (finished) ring region
  __shared__ float wst_ml[kSpNW * 8 * 2];
  __shared__ float smem_w[kSpNW * 8 + 2 * 8];
  float* my_o = reinterpret_cast<float*>(ring);  // [g][D]
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  if (gid < a.g) {
    float* wo = my_o + gid * D;
#pragma unroll
    for (int n = 0; n < C::NTO; ++n) {
      wo[n * 8 + 2 * tig] = acc[n][0] + acc[n][2];
      wo[n * 8 + 2 * tig + 1] = acc[n][1] + acc[n][3];
    }
    if (tig == 0) {
      wst_ml[(warp * a.g + gid) * 2] = ok ? m_run : -INFINITY;
      wst_ml[(warp * a.g + gid) * 2 + 1] = ok ? l_run : 0.f;
    }
  }
  __syncthreads();
  const int hq0 = b * a.Hq + h * a.g;
  splitk_store<D>(
      reinterpret_cast<const float*>(smem), C::WARP_B / 4, wst_ml, kSpNW, a.g, a.g, a.S, chunk, unit, a.o,
      [&](int r) { return static_cast<size_t>(hq0 + r) * D; }, [&](int r) { return static_cast<size_t>(hq0 + r); },
      smem_w);
}

// Output row of flattened partial row fr = unit * g + r (query head h * g + r).
struct SparseRowMap {
  int g, Hq, Hkv, D;
  __device__ bool locate(int64_t fr, int& unit, int& r, size_t& out_off, size_t& lse_off) const {
    unit = static_cast<int>(fr / g);
    r = static_cast<int>(fr - static_cast<int64_t>(unit) * g);
    const int b = unit / Hkv, h = unit - b * Hkv;
    out_off = (static_cast<size_t>(b) * Hq + h * g + r) * D;
    lse_off = 0;
    return true;
  }
};

struct SpPlan {
  int S, CH;
  size_t off_ml, off_o, total;
};

// Resident blocks per SM of one instance (cached per device; also sets the
// kernel's shared-memory attribute on that device).
template <int D>
int sparse_occupancy() {
  using C = SpCfg<D>;
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    cudaFuncSetAttribute(draft_sparse_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_B);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, draft_sparse_kernel<D>, kSpNW * 32, C::SMEM_B) !=
            cudaSuccess ||
        n < 1)
      n = 1;
    cache[dev] = n;
  }
  return cache[dev];
}

// Chunks of CH kept rows per block, sized so that the grid is one wave of
// the resident blocks (SMs x occupancy).
SpPlan plan_sparse(const vc_attn_shape& sh, int n_keep) {
  SpPlan p{};
  const int units = sh.B * sh.Hkv;
  const int64_t rows = static_cast<int64_t>(units) * n_keep;
  const int occ = sh.D == 128 ? sparse_occupancy<128>() : sparse_occupancy<64>();
  const int64_t target_blocks = static_cast<int64_t>(sm_count()) * occ;
  // smallest multiple of 16 rows that keeps units * ceil(n_keep / ch) <= target_blocks
  int64_t ch = (rows + target_blocks - 1) / target_blocks;
  ch = (ch + 15) / 16 * 16;
  if (ch < 64) ch = 64;
  while (units * ((n_keep + ch - 1) / ch) > target_blocks && ch < n_keep) ch += 16;
  p.CH = static_cast<int>(ch);
  p.S = static_cast<int>((n_keep + p.CH - 1) / p.CH);
  const int g = sh.Hq / sh.Hkv;
  p.off_ml = align_up(sizeof(WsHeader), 256);
  p.off_o = align_up(p.off_ml + static_cast<size_t>(units) * p.S * g * 2 * 4, 256);
  p.total = align_up(p.off_o + static_cast<size_t>(units) * p.S * g * sh.D * 4, 256);
  return p;
}

vc_status check_sparse(const vc_attn_shape* sh, const vc_sparse_cache* c, const char* who) {
  VC_REQUIRE(sh && c, "%s: null shape or cache", who);
  VC_REQUIRE(sh->B >= 1 && sh->Hkv >= 1 && sh->Hq >= 1 && sh->Hq % sh->Hkv == 0 && sh->Hq / sh->Hkv <= 8,
             "%s: need B >= 1, Hq a multiple of Hkv, Hq/Hkv <= 8", who);
  VC_REQUIRE(sh->D == 64 || sh->D == 128, "%s: head dim must be 64 or 128 (got %d)", who, sh->D);
  VC_REQUIRE(c->n_keep >= 1 && c->T_store >= 1 && c->T_store <= INT32_MAX, "%s: need n_keep >= 1, 1 <= T_store < 2^31",
             who);
  VC_REQUIRE(c->k && c->v && c->idx, "%s: null cache pointer", who);
  VC_REQUIRE(aligned16(c->k) && aligned16(c->v), "%s: K/V store must be 16-byte aligned", who);
  VC_REQUIRE(static_cast<int64_t>(sh->B) * sh->Hkv <= 65535, "%s: too many (request, head) pairs", who);
  return VC_OK;
}

__global__ void gather_kernel(const __nv_bfloat16* k, const __nv_bfloat16* v, const int32_t* idx, int64_t T_store,
                              int n_keep, int D, __nv_bfloat16* ko, __nv_bfloat16* vo, uint32_t* flags) {
  const int unit = blockIdx.y;
  const int j = blockIdx.x;
  const int pos = __ldg(idx + static_cast<size_t>(unit) * n_keep + j);
  const bool ok = pos >= 0 && static_cast<int64_t>(pos) < T_store;
  if (!ok && threadIdx.x == 0 && flags) atomicOr(flags, VC_FLAG_BAD_INDEX);
  const size_t src = (static_cast<size_t>(unit) * T_store + (ok ? pos : 0)) * D;
  const size_t dst = (static_cast<size_t>(unit) * n_keep + j) * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    ko[dst + d] = ok ? k[src + d] : __float2bfloat16(0.f);
    vo[dst + d] = ok ? v[src + d] : __float2bfloat16(0.f);
  }
}

}  // namespace
}  // namespace vc

extern "C" {

size_t vc_draft_attn_sparse_workspace_size(const vc_attn_shape* shape, const vc_sparse_cache* cache) {
  if (!shape || !cache || shape->Hkv < 1 || shape->Hq % shape->Hkv || cache->n_keep < 1) return 0;
  return vc::plan_sparse(*shape, cache->n_keep).total;
}

vc_status vc_draft_attn_sparse(const vc_attn_shape* shape, const vc_sparse_cache* cache, const void* q, float* out,
                               void* ws, size_t ws_bytes, void* stream) {
  vc_status st = vc::check_sparse(shape, cache, "vc_draft_attn_sparse");
  if (st != VC_OK) return st;
  VC_REQUIRE(q && out && ws, "vc_draft_attn_sparse: null q, out or workspace");
  VC_REQUIRE(vc::aligned16(q) && vc::aligned16(out) && vc::aligned16(ws),
             "vc_draft_attn_sparse: q, out and workspace must be 16-byte aligned");
  const vc::SpPlan pl = vc::plan_sparse(*shape, cache->n_keep);
  VC_REQUIRE(ws_bytes >= pl.total, "vc_draft_attn_sparse: workspace too small (%zu < %zu)", ws_bytes, pl.total);
  char* w = static_cast<char*>(ws);
  vc::SpArgs a{};
  a.k = static_cast<const __nv_bfloat16*>(cache->k);
  a.v = static_cast<const __nv_bfloat16*>(cache->v);
  a.idx = cache->idx;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.T_store = cache->T_store;
  a.n_keep = cache->n_keep;
  a.Hq = shape->Hq;
  a.Hkv = shape->Hkv;
  a.g = shape->Hq / shape->Hkv;
  a.S = pl.S;
  a.CH = pl.CH;
  const float sm = shape->sm_scale > 0.f ? shape->sm_scale : 1.0f / sqrtf(static_cast<float>(shape->D));
  a.scale_log2 = sm * 1.4426950408889634f;
  a.flags = reinterpret_cast<uint32_t*>(w);
  a.o.out = out;
  a.o.lse = nullptr;
  a.o.part_ml = reinterpret_cast<float*>(w + pl.off_ml);
  a.o.part_o = reinterpret_cast<float*>(w + pl.off_o);
  dim3 grid(pl.S, shape->B * shape->Hkv);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (shape->D == 128) {
    vc::sparse_occupancy<128>();  // sets the shared-memory attribute once per device
    vc::draft_sparse_kernel<128><<<grid, vc::kSpNW * 32, vc::SpCfg<128>::SMEM_B, s>>>(a);
  } else {
    vc::sparse_occupancy<64>();
    vc::draft_sparse_kernel<64><<<grid, vc::kSpNW * 32, vc::SpCfg<64>::SMEM_B, s>>>(a);
  }
  if (pl.S > 1) {  // chunk partials -> output rows
    const vc::SparseRowMap map{a.g, shape->Hq, shape->Hkv, shape->D};
    const int64_t n_rows = static_cast<int64_t>(shape->B) * shape->Hkv * a.g;
    // tens of chunks per row: one block per row keeps each thread's loads
    // few and independent (one warp per row above kWideMaxS chunks)
    const bool wide = pl.S >= 16 && pl.S <= vc::kWideMaxS;
    if (shape->D == 128) {
      if (wide)
        vc::launch_splitk_combine_wide<128>(a.o, pl.S, a.g, n_rows, map, s);
      else
        vc::launch_splitk_combine<128>(a.o, pl.S, a.g, n_rows, map, s);
    } else {
      if (wide)
        vc::launch_splitk_combine_wide<64>(a.o, pl.S, a.g, n_rows, map, s);
      else
        vc::launch_splitk_combine<64>(a.o, pl.S, a.g, n_rows, map, s);
    }
  }
  return vc::launch_status("vc_draft_attn_sparse");
}

vc_status vc_debug_gather(const vc_attn_shape* shape, const vc_sparse_cache* cache, void* k_out, void* v_out, void* ws,
                          size_t ws_bytes, void* stream) {
  vc_status st = vc::check_sparse(shape, cache, "vc_debug_gather");
  if (st != VC_OK) return st;
  VC_REQUIRE(k_out && v_out, "vc_debug_gather: null output");
  VC_REQUIRE(cache->n_keep <= 2147483647, "vc_debug_gather: n_keep too large");
  uint32_t* flags = (ws && ws_bytes >= sizeof(vc::WsHeader)) ? static_cast<uint32_t*>(ws) : nullptr;
  dim3 grid(cache->n_keep, shape->B * shape->Hkv);
  vc::gather_kernel<<<grid, 64, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(cache->k), static_cast<const __nv_bfloat16*>(cache->v), cache->idx,
      cache->T_store, cache->n_keep, shape->D, static_cast<__nv_bfloat16*>(k_out), static_cast<__nv_bfloat16*>(v_out),
      flags);
  return vc::launch_status("vc_debug_gather");
}

}  // extern "C"
