// vc_accept.cu -- greedy acceptance of one VeriCache round.
//
// The verifier's K + 1 logit rows give one greedy prediction per drafted
// position plus one after the last; drafted tokens are kept left to right up
// to the first disagreement, where the verifier's token is emitted as the
// correction (the bonus token when all K agree) -- devshah.ca page "VeriCache:
// making lossy KV compression exact", section "The Core Idea".
//
// Layout of the work: grid (S, B*(K+1)), S chosen so the grid is about one
// wave of 512-thread blocks.  Block (c, row) scans chunk c of one logit row
// with 16-byte streaming loads, eight in flight per thread, and reduces
// (value, index) pairs under the rule "larger value wins, NaN beats every
// number, ties go to the lower index".  Inside a thread the indices only
// grow, so a later value replaces the kept one only if it is strictly larger
// or a NaN over a number; the index rule decides between threads and blocks.  The last block of a row (atomic ticket, no waiting) merges
// the S partials into target[row]; the last row of a request computes the
// accepted length and the correction.  Tickets reset themselves, so the
// workspace stays ready for the next call.
#include <climits>

#include "vc_common.cuh"

namespace vc {
namespace {

constexpr int kAcceptThreads = 512;
constexpr int kAcceptMaxSplit = 16;
constexpr int kAcceptInFlight = 8;  // 16-byte loads in flight per thread

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

// x at a larger index than every value taken so far by this thread
__device__ __forceinline__ void take_later(Best& b, float x, int i) {
  if (x > b.v || (x != x && b.v == b.v) || b.i == INT_MAX) {
    b.v = x;
    b.i = i;
  }
}

// Largest of a 16-byte vector of logits, NaN if any is NaN (max.NaN).
__device__ __forceinline__ float max_nan_f32(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}
__device__ __forceinline__ uint32_t max_nan_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <typename T>
__device__ __forceinline__ float vec_max(uint4 w) {
  if constexpr (sizeof(T) == 4) {
    return max_nan_f32(max_nan_f32(__uint_as_float(w.x), __uint_as_float(w.y)),
                       max_nan_f32(__uint_as_float(w.z), __uint_as_float(w.w)));
  } else {
    const uint32_t m = max_nan_bf16x2(max_nan_bf16x2(w.x, w.y), max_nan_bf16x2(w.z, w.w));
    return max_nan_f32(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));  // bf16 -> fp32 is a shift
  }
}

template <typename T>
__device__ __forceinline__ void take_vec(Best& b, uint4 w, int base) {
  if constexpr (sizeof(T) == 4) {
    take_later(b, __uint_as_float(w.x), base + 0);
    take_later(b, __uint_as_float(w.y), base + 1);
    take_later(b, __uint_as_float(w.z), base + 2);
    take_later(b, __uint_as_float(w.w), base + 3);
  } else {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      take_later(b, __uint_as_float(ws[j] << 16), base + 2 * j);             // bf16 -> fp32 is a shift
      take_later(b, __uint_as_float(ws[j] & 0xffff0000u), base + 2 * j + 1);
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
  // scalar head up to 16-byte alignment, vector body, scalar tail; each
  // thread sees its indices in increasing order (head, then vectors j,
  // j + threads, ..., then the tail), so take_later applies
  const uintptr_t addr0 = reinterpret_cast<uintptr_t>(p + v0);
  int head = static_cast<int>(((16 - (addr0 & 15)) & 15) / sizeof(T));
  if (v0 + head > v1) head = v1 - v0;
  const int a = v0 + head;
  const int nvec = (v1 - a) / VEC;
  if (threadIdx.x < head) take_later(b, to_f32(p[v0 + threadIdx.x]), v0 + threadIdx.x);
  // Vector body, two passes over the thread's own vectors: (1) the running
  // maximum of whole vectors (max.NaN, a few instructions per 16 bytes) and
  // the first vector that reached it -- a later vector replaces it only if
  // its maximum is strictly larger or a NaN over a number, so ties keep the
  // earlier vector; (2) that one vector is read again (from L2) and its
  // first element equal to the maximum (or its first NaN) is the thread's
  // candidate.  kAcceptInFlight independent loads per thread before any is
  // used.
  float vrun = -INFINITY;
  int vbest = -1;  // element index of the vector holding vrun first
  for (int j0 = threadIdx.x; j0 < nvec; j0 += kAcceptInFlight * kAcceptThreads) {
    uint4 x[kAcceptInFlight];
#pragma unroll
    for (int f = 0; f < kAcceptInFlight; ++f) {
      const int j = j0 + f * kAcceptThreads;
      x[f] = j < nvec ? ld_stream(p + a + j * VEC) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int f = 0; f < kAcceptInFlight; ++f) {
      const int j = j0 + f * kAcceptThreads;
      if (j < nvec) {
        const float m = vec_max<T>(x[f]);
        if (vbest < 0 || m > vrun || (m != m && vrun == vrun)) {
          vrun = m;
          vbest = a + j * VEC;
        }
      }
    }
  }
  if (vbest >= 0) {
    Best vb{-INFINITY, INT_MAX};
    take_vec<T>(vb, *reinterpret_cast<const uint4*>(p + vbest), vbest);
    take_later(b, vb.v, vb.i);
  }
  for (int t = a + nvec * VEC + threadIdx.x; t < v1; t += kAcceptThreads) take_later(b, to_f32(p[t]), t);

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

// Resident accept blocks per SM (cached per device).
int accept_occupancy() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, accept_kernel<__nv_bfloat16>, kAcceptThreads, 0) !=
            cudaSuccess ||
        n < 1)
      n = 1;
    cache[dev] = n;
  }
  return cache[dev];
}

AcceptPlan plan_accept(int B, int K, int V) {
  AcceptPlan pl{};
  // at most one wave of blocks: S chunks per row with rows * S <= SMs x
  // resident blocks (a partial second wave would double the time of its
  // blocks), no chunk shorter than 8 loads per thread
  const int64_t nrows = static_cast<int64_t>(B) * (K + 1);
  const int64_t wave = static_cast<int64_t>(accept_occupancy()) * sm_count();
  int64_t S = wave / nrows;
  const int64_t smax = (V + 8 * kAcceptThreads - 1) / (8 * kAcceptThreads);
  if (S > smax) S = smax;
  if (S > kAcceptMaxSplit) S = kAcceptMaxSplit;
  pl.S = S < 1 ? 1 : static_cast<int>(S);
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
