// vc_splitk.cuh -- split-K bookkeeping of the attention kernels: the
// in-block merge of per-warp online-softmax states into a per-chunk partial
// (splitk_store; the token-dropped draft -- verification stores its one
// state per row straight from tensor memory), and the cross-chunk merge as a
// separate launch with one warp per output row (splitk_combine_kernel; both)
// or, for many chunks and few rows, one block per row
// (splitk_combine_wide_kernel; the token-dropped draft).
//
// A partial of one (unit, chunk) holds, per query row r < rows:
//   o[r][0..D)  unnormalised sum_j 2^(s_j - m) v_j
//   ml[r]       (m, l) with l = sum_j 2^(s_j - m); m = -inf for "no keys"
// where s_j are scores already multiplied by sm_scale * log2(e).
#pragma once

#include "vc_common.cuh"

namespace vc {

// Where the merged rows go: the final output rows (a single chunk) or the
// per-(unit, chunk) partials that splitk_combine_kernel merges.
struct SplitKOut {
  float* out;          // final output rows, row r at out + out_row_off(r)
  float* lse;          // optional natural-log lse per row (nullptr if unused)
  float* part_o;       // [units][S][rows][D]
  float* part_ml;      // [units][S][rows][2]
};

__device__ __forceinline__ float lse_from(float m, float l) {
  // m, l in base 2 -> natural log of sum exp(s_nat)
  return (m + log2f(l)) * 0.6931471805599453f;
}

// Block-wide (every thread of the block calls it): merges the per-warp
// states of one (unit, chunk) -- wst_o: warp w's rows at wst_o + w * o_wstride
// (floats), row r at + r * D; wst_ml [nw][rows][2] -- and stores, with S == 1,
// the normalised output rows (row_out(r) / row_lse(r) give element offsets),
// otherwise the chunk's partial (rows_cap rows reserved per (unit, chunk)),
// which splitk_combine_kernel merges later.
template <int D, typename RowOff, typename RowLse>
__device__ void splitk_store(const float* wst_o, int o_wstride, const float* wst_ml, int nw, int rows, int rows_cap,
                             int S, int chunk, int unit, const SplitKOut& o, RowOff row_out, RowLse row_lse,
                             float* smem_w) {
  const int tid = threadIdx.x;
  const int nthr = blockDim.x;
  for (int r = tid; r < rows; r += nthr) {
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, wst_ml[(w * rows + r) * 2]);
    float L = 0.f;
    for (int w = 0; w < nw; ++w) {
      const float mw = wst_ml[(w * rows + r) * 2];
      const float sc = (mw == -INFINITY) ? 0.f : ex2(mw - M);
      smem_w[w * rows + r] = sc;
      L += sc * wst_ml[(w * rows + r) * 2 + 1];
    }
    smem_w[nw * rows + 2 * r] = M;
    smem_w[nw * rows + 2 * r + 1] = L;
  }
  __syncthreads();
  const int total = rows * D;
  if (S == 1) {
    for (int e = tid; e < total; e += nthr) {
      const int r = e / D, d = e - r * D;
      float acc = 0.f;
      for (int w = 0; w < nw; ++w) acc += smem_w[w * rows + r] * wst_o[w * o_wstride + r * D + d];
      const float L = smem_w[nw * rows + 2 * r + 1];
      o.out[row_out(r) + d] = L > 0.f ? acc / L : 0.f;
    }
    if (o.lse)
      for (int r = tid; r < rows; r += nthr)
        o.lse[row_lse(r)] = lse_from(smem_w[nw * rows + 2 * r], smem_w[nw * rows + 2 * r + 1]);
    return;
  }
  float* po = o.part_o + (static_cast<size_t>(unit) * S + chunk) * rows_cap * D;
  float* pml = o.part_ml + (static_cast<size_t>(unit) * S + chunk) * rows_cap * 2;
  for (int e = tid; e < total; e += nthr) {
    const int r = e / D, d = e - r * D;
    float acc = 0.f;
    for (int w = 0; w < nw; ++w) acc += smem_w[w * rows + r] * wst_o[w * o_wstride + r * D + d];
    po[e] = acc;
  }
  for (int r = tid; r < rows; r += nthr) {
    pml[2 * r] = smem_w[nw * rows + 2 * r];
    pml[2 * r + 1] = smem_w[nw * rows + 2 * r + 1];
  }
}

// Cross-chunk merge as its own launch: warp w of block b merges row
// (b * 4 + w) of the flattened (unit, row) list over the S chunk partials.
// Each lane owns D/32 consecutive channels; the S (m, l) pairs are reduced by
// warp shuffles; the S partial loads of a lane are independent.  Map gives,
// for a flattened row, its unit, its row inside the unit's partials, whether
// it exists, and its output / lse element offsets.  Launched as a
// programmatic dependent of the attention kernel: it waits for that grid.
template <int D, typename Map>
__global__ void __launch_bounds__(128) splitk_combine_kernel(SplitKOut o, int S, int rows_cap, int64_t n_rows,
                                                             Map map) {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t fr = static_cast<int64_t>(blockIdx.x) * 4 + warp;
  if (fr >= n_rows) return;
  int unit, r;
  size_t out_off, lse_off;
  if (!map.locate(fr, unit, r, out_off, lse_off)) return;
  const float* pml = o.part_ml + static_cast<size_t>(unit) * S * rows_cap * 2 + 2 * r;
  float M = -INFINITY;
  for (int s = lane; s < S; s += 32) M = fmaxf(M, pml[static_cast<size_t>(s) * rows_cap * 2]);
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
  float L = 0.f;
  for (int s = lane; s < S; s += 32) {
    const float ms = pml[static_cast<size_t>(s) * rows_cap * 2];
    if (ms != -INFINITY) L += ex2(ms - M) * pml[static_cast<size_t>(s) * rows_cap * 2 + 1];
  }
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) L += __shfl_xor_sync(0xffffffffu, L, x);
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  const float* po = o.part_o + (static_cast<size_t>(unit) * S * rows_cap + r) * D + lane * PER;
#pragma unroll 4
  for (int s = 0; s < S; ++s) {
    const float ms = pml[static_cast<size_t>(s) * rows_cap * 2];
    const float w = ms == -INFINITY ? 0.f : ex2(ms - M);
    const float* src = po + static_cast<size_t>(s) * rows_cap * D;
    if constexpr (PER == 4) {
      const float4 v = *reinterpret_cast<const float4*>(src);
      acc[0] += w * v.x, acc[1] += w * v.y, acc[2] += w * v.z, acc[3] += w * v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(src);
      acc[0] += w * v.x, acc[1] += w * v.y;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  float* dst = o.out + out_off + lane * PER;
  if constexpr (PER == 4) {
    *reinterpret_cast<float4*>(dst) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  } else {
    *reinterpret_cast<float2*>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
  }
  if (o.lse && lane == 0) o.lse[lse_off] = lse_from(M, L);
}

// Cross-chunk merge for many chunks and few rows (the token-dropped draft:
// g rows per unit, tens of chunks): one 256-thread block per output row.
// The chunks' (m, l) are reduced by all threads at once; each of 8 warps
// then sums every 8th chunk's o (lane l owns channels D/32 l ..), so a
// thread keeps ~S/8 independent loads in flight instead of S, and the 8
// warp sums meet in shared memory.  S <= kWideMaxS.
constexpr int kWideMaxS = 2048;

template <int D, typename Map>
__global__ void __launch_bounds__(256) splitk_combine_wide_kernel(SplitKOut o, int S, int rows_cap, int64_t n_rows,
                                                                  Map map) {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  constexpr int PER = D / 32;
  __shared__ float wts[kWideMaxS];
  __shared__ float red[8][D];
  __shared__ float ml[2][8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t fr = blockIdx.x;
  int unit, r;
  size_t out_off, lse_off;
  if (fr >= n_rows || !map.locate(fr, unit, r, out_off, lse_off)) return;  // block-uniform
  const size_t stride_ml = static_cast<size_t>(rows_cap) * 2;
  const float* pml = o.part_ml + static_cast<size_t>(unit) * S * stride_ml + 2 * r;
  float m = -INFINITY;
  for (int s = tid; s < S; s += 256) m = fmaxf(m, __ldcg(pml + s * stride_ml));
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, x));
  if (lane == 0) ml[0][warp] = m;
  __syncthreads();
  float M = ml[0][0];
#pragma unroll
  for (int w = 1; w < 8; ++w) M = fmaxf(M, ml[0][w]);
  float l = 0.f;
  for (int s = tid; s < S; s += 256) {
    const float ms = __ldcg(pml + s * stride_ml);
    const float w = (ms == -INFINITY || M == -INFINITY) ? 0.f : ex2(ms - M);
    wts[s] = w;
    if (w > 0.f) l += w * __ldcg(pml + s * stride_ml + 1);
  }
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) l += __shfl_xor_sync(0xffffffffu, l, x);
  if (lane == 0) ml[1][warp] = l;
  __syncthreads();
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) L += ml[1][w];
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  const float* po = o.part_o + (static_cast<size_t>(unit) * S * rows_cap + r) * D + lane * PER;
#pragma unroll 8
  for (int s = warp; s < S; s += 8) {
    const float w = wts[s];
    const float* src = po + static_cast<size_t>(s) * rows_cap * D;
    if constexpr (PER == 4) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
      acc[0] += w * v.x, acc[1] += w * v.y, acc[2] += w * v.z, acc[3] += w * v.w;
    } else {
      const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
      acc[0] += w * v.x, acc[1] += w * v.y;
    }
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) red[warp][lane * PER + i] = acc[i];
  __syncthreads();
  if (tid < D) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sum += red[w][tid];
    o.out[out_off + tid] = L > 0.f ? sum / L : 0.f;
  }
  if (o.lse && tid == 0) o.lse[lse_off] = lse_from(M, L);
}

// Host: launches splitk_combine_kernel<D> as a programmatic dependent of the
// kernel just enqueued on s.
template <int D, typename Map>
inline void launch_splitk_combine(const SplitKOut& o, int S, int rows_cap, int64_t n_rows, const Map& map,
                                  cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((n_rows + 3) / 4));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, splitk_combine_kernel<D, Map>, o, S, rows_cap, n_rows, map);
}

// Host: the wide merge (one block per row) as a programmatic dependent.
template <int D, typename Map>
inline void launch_splitk_combine_wide(const SplitKOut& o, int S, int rows_cap, int64_t n_rows, const Map& map,
                                       cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n_rows));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, splitk_combine_wide_kernel<D, Map>, o, S, rows_cap, n_rows, map);
}

}  // namespace vc
