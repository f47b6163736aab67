// vc_layer.cu -- one decoder layer of the verifier over the verification
// block, on caller-given (random) weights.
//
// Verification is one pass of the same model over the drafted block with the
// full cache ("VeriCache: making lossy KV compression exact", devshah.ca,
// "The Core Idea"; drafter and verifier share the weights and differ only in
// KV fidelity, "VeriCache: Turning Lossy KV Cache into Lossless LLM
// Inference", menfem.com, "Methodology").  The pages give no layer
// arithmetic; this is a Llama-style pre-norm layer:
//   h   = RMSNorm(x) w1                       rmsnorm_kernel
//   qkv = h Wqkv^T                            cuBLAS bf16 GEMM, fp32 accumulate
//   q, k = rotary(q, k); cache rows T-nq..T-1 = k, v        rope_store_kernel
//   o   = causal verification attention       vc_verify_attn (tcgen05)
//   x  += bf16(o) Wo^T                        cf32_to_bf16_kernel + GEMM (beta 1)
//   h2  = RMSNorm(x) w2;  [g | u] = h2 Wgu^T
//   a   = silu(g) u                           silu_mul_kernel
//   x  += a Wd^T                              GEMM (beta 1)
// Activations are bf16 between the steps (each step rounds its result once);
// norms, the rotary rotation and the SwiGLU product are computed in fp32 /
// fp64 from the bf16 inputs.  The projections are plain dense GEMMs and go
// to cuBLAS; the steps around them are this file's kernels.
#include <cublas_v2.h>

#include <mutex>

#include "vc_common.cuh"

namespace vc {
namespace {

constexpr int kNormThreads = 256;
constexpr size_t kCublasWs = 4u << 20;

// x[row] -> bf16(x / sqrt(mean(x^2) + eps) * w); dm a multiple of 8
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const __nv_bfloat16* __restrict__ x,
                                                                const __nv_bfloat16* __restrict__ w,
                                                                __nv_bfloat16* __restrict__ out, int dm, float eps) {
  const size_t row = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * dm);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  uint4* orow = reinterpret_cast<uint4*>(out + row * dm);
  const int nv = dm / 8;
  float ss = 0.f;
  for (int i = threadIdx.x; i < nv; i += kNormThreads) {
    const uint4 v = xr[i];
    const uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack_bf2(a[j]);
      ss = fmaf(f.x, f.x, ss);
      ss = fmaf(f.y, f.y, ss);
    }
  }
  __shared__ float red[kNormThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int k = 0; k < kNormThreads / 32; ++k) tot += red[k];
  const float inv = 1.0f / sqrtf(tot / static_cast<float>(dm) + eps);
  for (int i = threadIdx.x; i < nv; i += kNormThreads) {
    const uint4 v = xr[i], wv = wr[i];
    const uint32_t a[4] = {v.x, v.y, v.z, v.w}, b[4] = {wv.x, wv.y, wv.z, wv.w};
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack_bf2(a[j]), g = unpack_bf2(b[j]);
      r[j] = pack_bf2(f.x * inv * g.x, f.y * inv * g.y);
    }
    orow[i] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

// Rotary embedding (rotate-half pairs j, j + D/2, angle = pos theta^(-2j/D))
// of the block's q and k, computed in fp64 from the bf16 inputs and rounded
// once; q goes to a contiguous [B][nq][Hq][D] buffer, k and v to rows
// T - nq + i of the full cache [B][Hkv][T][D].  One thread per (token, head,
// pair) over the Hq + 2 Hkv heads of the qkv row (v heads copy both halves).
__global__ void rope_store_kernel(const __nv_bfloat16* __restrict__ qkv, int B, int nq, int Hq, int Hkv, int D,
                                  int64_t T, double theta, __nv_bfloat16* __restrict__ q_out,
                                  __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc) {
  const int half = D / 2;
  const int H = Hq + 2 * Hkv;
  const int64_t total = static_cast<int64_t>(B) * nq * H * half;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(e % half);
    const int hh = static_cast<int>((e / half) % H);
    const int64_t tok = e / (static_cast<int64_t>(half) * H);  // b * nq + i
    const int b = static_cast<int>(tok / nq), i = static_cast<int>(tok % nq);
    const __nv_bfloat16* src = qkv + tok * static_cast<int64_t>(H) * D + static_cast<int64_t>(hh) * D;
    const int64_t pos = T - nq + i;
    if (hh >= Hq + Hkv) {  // v: no rotation
      const int hk = hh - Hq - Hkv;
      __nv_bfloat16* dst = vc + ((static_cast<int64_t>(b) * Hkv + hk) * T + pos) * D;
      dst[j] = src[j];
      dst[j + half] = src[j + half];
      continue;
    }
    const double ang = static_cast<double>(pos) * pow(theta, -2.0 * j / D);
    double s, c;
    sincos(ang, &s, &c);
    const double a = __bfloat162float(src[j]), bb = __bfloat162float(src[j + half]);
    const __nv_bfloat16 r0 = __double2bfloat16(a * c - bb * s);
    const __nv_bfloat16 r1 = __double2bfloat16(a * s + bb * c);
    __nv_bfloat16* dst;
    if (hh < Hq) {
      dst = q_out + (tok * Hq + hh) * D;
    } else {
      const int hk = hh - Hq;
      dst = kc + ((static_cast<int64_t>(b) * Hkv + hk) * T + pos) * D;
    }
    dst[j] = r0;
    dst[j + half] = r1;
  }
}

__global__ void cf32_to_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, int64_t n) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[e] = __float2bfloat16_rn(x[e]);
}

// a[t][f] = bf16(silu(g) u) with [g | u] = gu[t] (F columns each)
__global__ void silu_mul_kernel(const __nv_bfloat16* __restrict__ gu, __nv_bfloat16* __restrict__ a, int64_t n_tok,
                                int F) {
  const int64_t total = n_tok * F;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = e / F;
    const int f = static_cast<int>(e % F);
    const float g = __bfloat162float(gu[t * 2 * F + f]);
    const float u = __bfloat162float(gu[t * 2 * F + F + f]);
    a[e] = __float2bfloat16_rn(g / (1.0f + expf(-g)) * u);
  }
}

struct LayerPlan {
  size_t off_h, off_qkv, off_q, off_of, off_ob, off_h2, off_gu, off_a, off_vws, off_cub, vws, total;
};

LayerPlan plan_layer(const vc_layer_shape& L, int B, int nq, int64_t T) {
  LayerPlan p{};
  const size_t n = static_cast<size_t>(B) * nq;
  const size_t qd = static_cast<size_t>(L.Hq) * L.D;
  const size_t n1 = static_cast<size_t>(L.Hq + 2 * L.Hkv) * L.D;
  vc_attn_shape sh{B, L.Hq, L.Hkv, L.D, 0.f};
  p.vws = vc_verify_attn_workspace_size(&sh, T, nq);
  size_t o = align_up(sizeof(WsHeader), 256);
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  p.off_h = take(n * L.d_model * 2);
  p.off_qkv = take(n * n1 * 2);
  p.off_q = take(n * qd * 2);
  p.off_of = take(n * qd * 4);
  p.off_ob = take(n * qd * 2);
  p.off_h2 = take(n * L.d_model * 2);
  p.off_gu = take(n * 2 * static_cast<size_t>(L.d_ff) * 2);
  p.off_a = take(n * static_cast<size_t>(L.d_ff) * 2);
  p.off_vws = take(p.vws);
  p.off_cub = take(kCublasWs);
  p.total = o;
  return p;
}

// One cuBLAS handle per (host thread, device).
cublasHandle_t cublas_handle() {
  thread_local cublasHandle_t h[64] = {nullptr};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!h[dev] && cublasCreate(&h[dev]) != CUBLAS_STATUS_SUCCESS) h[dev] = nullptr;
  return h[dev];
}

// row-major C[n][m] = A[n][k] B[m][k]^T (+ C when beta == 1), bf16 in/out, fp32 accumulate
bool gemm_nt(cublasHandle_t hd, int n, int m, int k, const void* A, const void* Bw, void* C, float beta) {
  const float alpha = 1.f;
  return cublasGemmEx(hd, CUBLAS_OP_T, CUBLAS_OP_N, m, n, k, &alpha, Bw, CUDA_R_16BF, k, A, CUDA_R_16BF, k, &beta, C,
                      CUDA_R_16BF, m, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) == CUBLAS_STATUS_SUCCESS;
}

int grid_for(int64_t n, int threads) {
  const int64_t b = (n + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  return static_cast<int>(b < 1 ? 1 : (b > cap ? cap : b));
}

vc_status check_layer(const vc_layer_shape* L, const vc_layer_weights* W, int B, int nq, int64_t T, const char* who) {
  VC_REQUIRE(L && W, "%s: null shape or weights", who);
  VC_REQUIRE(L->D == 64 || L->D == 128, "%s: head dim must be 64 or 128", who);
  VC_REQUIRE(L->Hq >= 1 && L->Hkv >= 1 && L->Hq % L->Hkv == 0 && L->Hq / L->Hkv <= 8,
             "%s: need Hq a multiple of Hkv and Hq/Hkv <= 8", who);
  VC_REQUIRE(L->d_model >= 8 && L->d_model % 8 == 0 && L->d_ff >= 8 && L->d_ff % 8 == 0,
             "%s: d_model and d_ff must be positive multiples of 8", who);
  VC_REQUIRE(L->rms_eps > 0.f && L->rope_theta > 1.f, "%s: need rms_eps > 0 and rope_theta > 1", who);
  VC_REQUIRE(B >= 1 && nq >= 1 && nq <= 32 && T >= nq && T < (int64_t(1) << 31), "%s: need B >= 1, 1 <= nq <= 32, "
             "nq <= T < 2^31", who);
  VC_REQUIRE(W->w1 && W->wqkv && W->wo && W->w2 && W->wgu && W->wd, "%s: null weight", who);
  VC_REQUIRE(aligned16(W->w1) && aligned16(W->wqkv) && aligned16(W->wo) && aligned16(W->w2) && aligned16(W->wgu) &&
                 aligned16(W->wd),
             "%s: weights must be 16-byte aligned", who);
  return VC_OK;
}

}  // namespace
}  // namespace vc

extern "C" {

size_t vc_verify_layer_workspace_size(const vc_layer_shape* shape, int B, int nq, int64_t T) {
  vc_layer_weights dummy{reinterpret_cast<const void*>(16), reinterpret_cast<const void*>(16),
                         reinterpret_cast<const void*>(16), reinterpret_cast<const void*>(16),
                         reinterpret_cast<const void*>(16), reinterpret_cast<const void*>(16)};
  if (vc::check_layer(shape, &dummy, B, nq, T, "vc_verify_layer_workspace_size") != VC_OK) return 0;
  return vc::plan_layer(*shape, B, nq, T).total;
}

vc_status vc_verify_layer(const vc_layer_shape* shape, const vc_layer_weights* w, int B, int nq, int64_t T, void* x,
                          void* k_cache, void* v_cache, void* ws, size_t ws_bytes, void* stream) {
  vc_status st = vc::check_layer(shape, w, B, nq, T, "vc_verify_layer");
  if (st != VC_OK) return st;
  VC_REQUIRE(x && k_cache && v_cache && ws, "vc_verify_layer: null x, cache or workspace");
  VC_REQUIRE(vc::aligned16(x) && vc::aligned16(k_cache) && vc::aligned16(v_cache) && vc::aligned16(ws),
             "vc_verify_layer: x, caches and workspace must be 16-byte aligned");
  const vc_layer_shape& L = *shape;
  const vc::LayerPlan p = vc::plan_layer(L, B, nq, T);
  VC_REQUIRE(ws_bytes >= p.total, "vc_verify_layer: workspace too small (%zu < %zu)", ws_bytes, p.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cublasHandle_t hd = vc::cublas_handle();
  if (!hd) return vc::set_error(VC_ERR_CUDA, "vc_verify_layer: cuBLAS handle creation failed");
  char* base = static_cast<char*>(ws);
  if (cublasSetStream(hd, s) != CUBLAS_STATUS_SUCCESS ||
      cublasSetWorkspace(hd, base + p.off_cub, vc::kCublasWs) != CUBLAS_STATUS_SUCCESS)
    return vc::set_error(VC_ERR_CUDA, "vc_verify_layer: cuBLAS stream / workspace setup failed");
  const int n = B * nq;
  const int qd = L.Hq * L.D;
  const int n1 = (L.Hq + 2 * L.Hkv) * L.D;
  auto* h = reinterpret_cast<__nv_bfloat16*>(base + p.off_h);
  auto* qkv = reinterpret_cast<__nv_bfloat16*>(base + p.off_qkv);
  auto* q = reinterpret_cast<__nv_bfloat16*>(base + p.off_q);
  auto* of = reinterpret_cast<float*>(base + p.off_of);
  auto* ob = reinterpret_cast<__nv_bfloat16*>(base + p.off_ob);
  auto* h2 = reinterpret_cast<__nv_bfloat16*>(base + p.off_h2);
  auto* gu = reinterpret_cast<__nv_bfloat16*>(base + p.off_gu);
  auto* a = reinterpret_cast<__nv_bfloat16*>(base + p.off_a);
  auto* xb = static_cast<__nv_bfloat16*>(x);
  auto bad = [&](const char* what) { return vc::set_error(VC_ERR_CUDA, "vc_verify_layer: %s failed", what); };

  vc::rmsnorm_kernel<<<n, vc::kNormThreads, 0, s>>>(xb, static_cast<const __nv_bfloat16*>(w->w1), h, L.d_model,
                                                    L.rms_eps);
  if (!vc::gemm_nt(hd, n, n1, L.d_model, h, w->wqkv, qkv, 0.f)) return bad("QKV projection");
  const int64_t nrot = static_cast<int64_t>(n) * (L.Hq + 2 * L.Hkv) * (L.D / 2);
  vc::rope_store_kernel<<<vc::grid_for(nrot, 256), 256, 0, s>>>(qkv, B, nq, L.Hq, L.Hkv, L.D, T,
                                                                 static_cast<double>(L.rope_theta), q,
                                                                 static_cast<__nv_bfloat16*>(k_cache),
                                                                 static_cast<__nv_bfloat16*>(v_cache));
  vc_attn_shape sh{B, L.Hq, L.Hkv, L.D, 0.f};
  st = vc_verify_attn(&sh, q, k_cache, v_cache, T, nq, of, nullptr, base + p.off_vws, p.vws, stream);
  if (st != VC_OK) return st;
  const int64_t no = static_cast<int64_t>(n) * qd;
  vc::cf32_to_bf16_kernel<<<vc::grid_for(no, 256), 256, 0, s>>>(of, ob, no);
  if (!vc::gemm_nt(hd, n, L.d_model, qd, ob, w->wo, xb, 1.f)) return bad("output projection");
  vc::rmsnorm_kernel<<<n, vc::kNormThreads, 0, s>>>(xb, static_cast<const __nv_bfloat16*>(w->w2), h2, L.d_model,
                                                    L.rms_eps);
  if (!vc::gemm_nt(hd, n, 2 * L.d_ff, L.d_model, h2, w->wgu, gu, 0.f)) return bad("gate/up projection");
  const int64_t na = static_cast<int64_t>(n) * L.d_ff;
  vc::silu_mul_kernel<<<vc::grid_for(na, 256), 256, 0, s>>>(gu, a, n, L.d_ff);
  if (!vc::gemm_nt(hd, n, L.d_model, L.d_ff, a, w->wd, xb, 1.f)) return bad("down projection");
  return vc::launch_status("vc_verify_layer");
}

}  // extern "C"
