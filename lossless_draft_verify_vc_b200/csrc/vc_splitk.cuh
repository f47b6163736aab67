// vc_splitk.cuh -- split-K bookkeeping shared by the attention kernels: the
// in-block merge of per-warp online-softmax states and the cross-block merge
// of per-chunk partials (the last block of a unit, found with an atomic
// ticket, merges; nobody waits).
//
// A partial of one (unit, chunk) holds, per query row r < rows:
//   o[r][0..D)  unnormalised sum_j 2^(s_j - m) v_j
//   ml[r]       (m, l) with l = sum_j 2^(s_j - m); m = -inf for "no keys"
// where s_j are scores already multiplied by sm_scale * log2(e).
#pragma once

#include "vc_common.cuh"

namespace vc {

// Merges the per-warp states staged in shared memory into one partial.
//   wst_o  per warp [rows][D] (strided)   wst_ml [nw][rows][2]
// Writes either the final normalised output (S == 1) or the chunk partial;
// with S > 1 the last block of the unit then merges all S partials.
struct SplitKOut {
  float* out;          // final output rows, row r at out + out_row_off(r)
  float* lse;          // optional natural-log lse per row (nullptr if unused)
  float* part_o;       // [units][S][rows][D]
  float* part_ml;      // [units][S][rows][2]
  uint32_t* tickets;   // [units]
};

__device__ __forceinline__ float lse_from(float m, float l) {
  // m, l in base 2 -> natural log of sum exp(s_nat)
  return (m + log2f(l)) * 0.6931471805599453f;
}

// Block-wide: every thread of the block must call it.  `row_out(r)` gives the
// element offset of row r in `out` (and `row_lse(r)` in lse).
// wst_o: warp w's rows start at wst_o + w * o_wstride (floats), row r at +r*D.
// rows_cap: rows reserved per (unit, chunk) in the partial arrays (>= rows).
template <int D, typename RowOff, typename RowLse>
__device__ void splitk_finish(const float* wst_o, int o_wstride, const float* wst_ml, int nw, int rows,
                              int rows_cap, int S, int chunk, int unit, const SplitKOut& o, RowOff row_out,
                              RowLse row_lse, float* smem_w) {
  const int tid = threadIdx.x;
  const int nthr = blockDim.x;
  // per-row block max and weights of each warp
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
  __threadfence();
  __syncthreads();
  __shared__ uint32_t ticket;
  if (tid == 0) ticket = atomicAdd(&o.tickets[unit], 1u);
  __syncthreads();
  if (ticket != static_cast<uint32_t>(S - 1)) return;
  __threadfence();
  // last block of this unit: merge the S partials
  const float* uo = o.part_o + static_cast<size_t>(unit) * S * rows_cap * D;
  const float* uml = o.part_ml + static_cast<size_t>(unit) * S * rows_cap * 2;
  for (int r = tid; r < rows; r += nthr) {
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, __ldcg(uml + (s * rows_cap + r) * 2));
    float L = 0.f;
    for (int s = 0; s < S; ++s) {
      const float ms = __ldcg(uml + (s * rows_cap + r) * 2);
      if (ms != -INFINITY) L += ex2(ms - M) * __ldcg(uml + (s * rows_cap + r) * 2 + 1);
    }
    smem_w[2 * r] = M;
    smem_w[2 * r + 1] = L;
  }
  __syncthreads();
  for (int e = tid; e < total; e += nthr) {
    const int r = e / D, d = e - r * D;
    const float M = smem_w[2 * r];
    float acc = 0.f;
    for (int s = 0; s < S; ++s) {
      const float ms = __ldcg(uml + (s * rows_cap + r) * 2);
      if (ms != -INFINITY) acc += ex2(ms - M) * __ldcg(uo + (static_cast<size_t>(s) * rows_cap + r) * D + d);
    }
    const float L = smem_w[2 * r + 1];
    o.out[row_out(r) + d] = L > 0.f ? acc / L : 0.f;
  }
  if (o.lse)
    for (int r = tid; r < rows; r += nthr) o.lse[row_lse(r)] = lse_from(smem_w[2 * r], smem_w[2 * r + 1]);
  if (tid == 0) o.tickets[unit] = 0;
}

}  // namespace vc
