// vc_accept.cu -- greedy acceptance of one VeriCache round.
//
// The verifier's K + 1 logit rows give one greedy prediction per drafted
// position plus one after the last; drafted tokens are kept left to right up
// to the first disagreement, where the verifier's token is emitted as the
// correction (the bonus token when all K agree) -- devshah.ca page "VeriCache:
// making lossy KV compression exact", section "The Core Idea".
//
// Layout of the work: grid (S, B*(K+1)).  Block (c, row) scans chunk c of one
// logit row with 16-byte streaming loads and reduces (value, index) pairs
// under the rule "larger value wins, NaN beats every number, ties go to the
// lower index".  The last block of a row (atomic ticket, no waiting) merges
// the S partials into target[row]; the last row of a request computes the
// accepted length and the correction.  Tickets reset themselves, so the
// workspace stays ready for the next call.
#include <climits>

#include "vc_common.cuh"

namespace vc {
namespace {

constexpr int kAcceptThreads = 256;
constexpr int kAcceptChunk = 16384;  // vocabulary entries per block
constexpr int kAcceptMaxSplit = 16;

struct Best {
  float v;
  int i;
};

__device__ __forceinline__ bool beats(float x, int i, float y, int j) {
  const bool xn = x != x, yn = y != y;
  if (xn || yn) return xn && (!yn || i < j);
  if (x != y) return x > y;
  return i < j;
}

__device__ __forceinline__ void take(Best& b, float x, int i) {
  if (beats(x, i, b.v, b.i)) {
    b.v = x;
    b.i = i;
  }
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <typename T>
__device__ __forceinline__ void take_vec(Best& b, uint4 w, int base) {
  if constexpr (sizeof(T) == 4) {
    take(b, __uint_as_float(w.x), base + 0);
    take(b, __uint_as_float(w.y), base + 1);
    take(b, __uint_as_float(w.z), base + 2);
    take(b, __uint_as_float(w.w), base + 3);
  } else {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = unpack_bf2(ws[j]);
      take(b, f.x, base + 2 * j);
      take(b, f.y, base + 2 * j + 1);
    }
  }
}

__device__ __forceinline__ Best warp_best(Best b) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float v = __shfl_xor_sync(0xffffffffu, b.v, o);
    int i = __shfl_xor_sync(0xffffffffu, b.i, o);
    take(b, v, i);
  }
  return b;
}

template <typename T>
__global__ void __launch_bounds__(kAcceptThreads) accept_kernel(const T* __restrict__ logits, int K, int V,
                                                                 int S, int chunk,
                                                                 const int32_t* __restrict__ draft,
                                                                 int32_t* target, int32_t* accept_len,
                                                                 int32_t* correction, uint32_t* row_cnt,
                                                                 uint32_t* req_cnt, Best* part) {
  constexpr int VEC = 16 / sizeof(T);
  const int row = blockIdx.y;
  const int c = blockIdx.x;
  const T* p = logits + static_cast<size_t>(row) * V;
  const int v0 = c * chunk;
  const int v1 = min(V, v0 + chunk);

  Best b{-INFINITY, INT_MAX};
  // scalar head up to 16-byte alignment, vector body, scalar tail
  const uintptr_t addr0 = reinterpret_cast<uintptr_t>(p + v0);
  int head = static_cast<int>(((16 - (addr0 & 15)) & 15) / sizeof(T));
  if (v0 + head > v1) head = v1 - v0;
  const int a = v0 + head;
  const int nvec = (v1 - a) / VEC;
  if (threadIdx.x < head) take(b, to_f32(p[v0 + threadIdx.x]), v0 + threadIdx.x);
  // four independent 16-byte loads in flight per thread before they are used
  // (the comparison rule does not depend on the order values are taken in)
  int j = threadIdx.x;
  for (; j + 3 * kAcceptThreads < nvec; j += 4 * kAcceptThreads) {
    const int b0 = a + j * VEC;
    const auto x0 = ld_stream(p + b0);
    const auto x1 = ld_stream(p + b0 + kAcceptThreads * VEC);
    const auto x2 = ld_stream(p + b0 + 2 * kAcceptThreads * VEC);
    const auto x3 = ld_stream(p + b0 + 3 * kAcceptThreads * VEC);
    take_vec<T>(b, x0, b0);
    take_vec<T>(b, x1, b0 + kAcceptThreads * VEC);
    take_vec<T>(b, x2, b0 + 2 * kAcceptThreads * VEC);
    take_vec<T>(b, x3, b0 + 3 * kAcceptThreads * VEC);
  }
  for (; j < nvec; j += kAcceptThreads) {
    const int base = a + j * VEC;
    take_vec<T>(b, ld_stream(p + base), base);
  }
  for (int t = a + nvec * VEC + threadIdx.x; t < v1; t += kAcceptThreads) take(b, to_f32(p[t]), t);

  __shared__ Best red[kAcceptThreads / 32];
  b = warp_best(b);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = b;
  __syncthreads();
  if (threadIdx.x != 0) return;
  for (int w = 1; w < kAcceptThreads / 32; ++w) take(b, red[w].v, red[w].i);

  if (S > 1) {
    part[static_cast<size_t>(row) * S + c] = b;
    __threadfence();
    if (atomicAdd(&row_cnt[row], 1u) != static_cast<uint32_t>(S - 1)) return;
    __threadfence();
    b = Best{-INFINITY, INT_MAX};
    for (int s = 0; s < S; ++s) {
      const float* q = reinterpret_cast<const float*>(&part[static_cast<size_t>(row) * S + s]);
      take(b, __ldcg(q), __ldcg(reinterpret_cast<const int*>(q + 1)));
    }
    row_cnt[row] = 0;
  }
  target[row] = b.i;

  // request-level ticket: the last of the K + 1 rows computes the acceptance
  const int req = row / (K + 1);
  __threadfence();
  if (atomicAdd(&req_cnt[req], 1u) != static_cast<uint32_t>(K)) return;
  __threadfence();
  const int32_t* tg = target + static_cast<size_t>(req) * (K + 1);
  const int32_t* dr = draft + static_cast<size_t>(req) * K;
  int acc = K;
  for (int i = 0; i < K; ++i) {
    if (__ldg(dr + i) != __ldcg(tg + i)) {
      acc = i;
      break;
    }
  }
  accept_len[req] = acc;
  correction[req] = __ldcg(tg + acc);
  req_cnt[req] = 0;
}

struct AcceptPlan {
  int S, chunk;
  size_t off_row, off_req, off_part, total;
};

AcceptPlan plan_accept(int B, int K, int V) {
  AcceptPlan pl{};
  pl.S = (V + kAcceptChunk - 1) / kAcceptChunk;
  if (pl.S > kAcceptMaxSplit) pl.S = kAcceptMaxSplit;
  if (pl.S < 1) pl.S = 1;
  pl.chunk = (V + pl.S - 1) / pl.S;
  pl.chunk = (pl.chunk + 7) / 8 * 8;
  pl.S = (V + pl.chunk - 1) / pl.chunk;
  if (pl.S < 1) pl.S = 1;
  const size_t rows = static_cast<size_t>(B) * (K + 1);
  pl.off_row = sizeof(WsHeader);
  pl.off_req = align_up(pl.off_row + rows * 4, 16);
  pl.off_part = align_up(pl.off_req + static_cast<size_t>(B) * 4, 16);
  pl.total = align_up(pl.off_part + rows * pl.S * sizeof(Best), 256);
  return pl;
}

}  // namespace
}  // namespace vc

extern "C" {

size_t vc_accept_workspace_size(int B, int K, int V) {
  if (B < 1 || K < 0 || V < 1) return 0;
  return vc::plan_accept(B, K, V).total;
}

vc_status vc_accept(const void* logits, int dtype, int B, int K, int V, const int32_t* draft, int32_t* target,
                    int32_t* accept_len, int32_t* correction, void* ws, size_t ws_bytes, void* stream) {
  VC_REQUIRE(B >= 1 && K >= 0 && K <= 64 && V >= 1, "vc_accept: need B >= 1, 0 <= K <= 64, V >= 1 (got %d, %d, %d)",
             B, K, V);
  VC_REQUIRE(dtype == VC_F32 || dtype == VC_BF16, "vc_accept: logits dtype must be VC_F32 or VC_BF16");
  VC_REQUIRE(logits && target && accept_len && correction && ws && (K == 0 || draft),
             "vc_accept: null pointer argument");
  VC_REQUIRE(vc::aligned16(logits) && vc::aligned16(ws), "vc_accept: logits and workspace must be 16-byte aligned");
  VC_REQUIRE(static_cast<int64_t>(B) * (K + 1) <= 65535, "vc_accept: too many logit rows");
  const vc::AcceptPlan pl = vc::plan_accept(B, K, V);
  VC_REQUIRE(ws_bytes >= pl.total, "vc_accept: workspace too small (%zu < %zu)", ws_bytes, pl.total);
  char* w = static_cast<char*>(ws);
  dim3 grid(pl.S, B * (K + 1));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* row_cnt = reinterpret_cast<uint32_t*>(w + pl.off_row);
  auto* req_cnt = reinterpret_cast<uint32_t*>(w + pl.off_req);
  auto* part = reinterpret_cast<vc::Best*>(w + pl.off_part);
  if (dtype == VC_F32)
    vc::accept_kernel<float><<<grid, vc::kAcceptThreads, 0, s>>>(static_cast<const float*>(logits), K, V, pl.S,
                                                                 pl.chunk, draft, target, accept_len, correction,
                                                                 row_cnt, req_cnt, part);
  else
    vc::accept_kernel<__nv_bfloat16><<<grid, vc::kAcceptThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(logits), K, V, pl.S, pl.chunk, draft, target, accept_len, correction,
        row_cnt, req_cnt, part);
  return vc::launch_status("vc_accept");
}

}  // extern "C"
