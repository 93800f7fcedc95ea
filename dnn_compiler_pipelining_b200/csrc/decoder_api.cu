// decoder_api.cu -- C ABI of the LLaMA3 single-decoder-layer proxy (declared
// in include/decoder_layer.h): argument checks, the workspace plan, the
// per-(device, stream) cuBLAS handles, and the launch sequence
//   RMSNorm -> QKV GEMM -> RoPE + head split -> attention (attn_fwd) ->
//   head merge -> O GEMM (+ residual) -> RMSNorm -> gate/up GEMM -> SwiGLU ->
//   down GEMM (+ residual),
// all on the caller's stream.
#include <cublas_v2.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "attn.h"
#include "decoder_layer.h"
#include "decoder_sm100.cuh"

namespace attn_b200 {
namespace decoder {
namespace {

size_t r256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Byte offsets of the workspace regions of one call.
struct Plan {
  size_t cs, n, big, q, k, v, o, lse, h, g, total;
};

Plan plan(int B, int S, int hidden, int Hq, int Hkv, int D, int inter) {
  const size_t T = static_cast<size_t>(B) * S;
  const size_t qkv_cols = static_cast<size_t>(Hq + 2 * Hkv) * D;
  const size_t big_cols = qkv_cols > 2 * static_cast<size_t>(inter) ? qkv_cols
                                                                    : 2 * static_cast<size_t>(inter);
  Plan p;
  size_t at = 0;
  auto take = [&at](size_t bytes) {
    const size_t off = at;
    at += r256(bytes);
    return off;
  };
  p.cs = take(static_cast<size_t>(S) * (D / 2) * sizeof(float2));  // rotary table
  p.n = take(T * hidden * 2);                                       // RMSNorm outputs
  p.big = take(T * big_cols * 2);                                   // QKV, then gate/up
  p.q = take(T * Hq * D * 2);                                       // Q, then merged O
  p.k = take(T * Hkv * D * 2);
  p.v = take(T * Hkv * D * 2);
  p.o = take(T * Hq * D * 2);
  p.lse = take(T * Hq * 4);
  p.h = take(T * hidden * 2);                                       // residual stream
  p.g = take(T * inter * 2);                                        // SwiGLU output
  p.total = at;
  return p;
}

attn_status check_sizes(int B, int S, int hidden, int Hq, int Hkv, int D, int inter) {
  if (B < 1 || S < 1 || hidden < 8 || Hq < 1 || Hkv < 1 || inter < 8) return ATTN_ERR_SHAPE;
  if (Hq % Hkv != 0 || hidden % 8 != 0 || inter % 8 != 0) return ATTN_ERR_SHAPE;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  // GEMM sizes and leading dimensions are 32-bit in the library interface;
  // the attention keeps its own row limits
  const int64_t T = static_cast<int64_t>(B) * S;
  const int64_t lim = (int64_t(1) << 31) - 1;
  if (T > lim || static_cast<int64_t>(Hq + 2 * Hkv) * D > lim || 2 * int64_t(inter) > lim)
    return ATTN_ERR_SHAPE;
  // the element kernels run one thread per 8 outputs in 256-thread blocks
  int64_t per_token = static_cast<int64_t>(Hq + 2 * Hkv) * (D / 16);
  if (static_cast<int64_t>(Hq) * (D / 8) > per_token) per_token = static_cast<int64_t>(Hq) * (D / 8);
  if (inter / 8 > per_token) per_token = inter / 8;
  if (T * per_token / 256 >= lim) return ATTN_ERR_SHAPE;
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

std::map<std::pair<int, cudaStream_t>, cublasHandle_t> g_handles;
std::mutex g_handles_mutex;

// The cuBLAS handle bound to (current device, stream), created on first use.
cublasHandle_t handle_for(cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(g_handles_mutex);
  auto key = std::make_pair(dev, stream);
  auto it = g_handles.find(key);
  if (it != g_handles.end()) return it->second;
  cublasHandle_t h = nullptr;
  if (cublasCreate(&h) != CUBLAS_STATUS_SUCCESS) return nullptr;
  // split-K partial sums stay in fp32 (the default may reduce in the fp16
  // output type), so every GEMM output is rounded once
  if (cublasSetStream(h, stream) != CUBLAS_STATUS_SUCCESS ||
      cublasSetMathMode(h, static_cast<cublasMath_t>(
                               CUBLAS_DEFAULT_MATH |
                               CUBLAS_MATH_DISALLOW_REDUCED_PRECISION_REDUCTION)) !=
          CUBLAS_STATUS_SUCCESS) {
    cublasDestroy(h);
    return nullptr;
  }
  g_handles[key] = h;
  return h;
}

// Row-major Y[T, N] = X[T, K] * W[N, K]^T + beta * Y, fp16 operands, fp32
// accumulation, one rounding.  (Column-major view: Y^T = W * X^T.)
bool gemm_rows(cublasHandle_t h, const __half* X, const __half* W, __half* Y, int T, int N, int K,
               float beta) {
  const float alpha = 1.0f;
  return cublasGemmEx(h, CUBLAS_OP_T, CUBLAS_OP_N, N, T, K, &alpha, W, CUDA_R_16F, K, X,
                      CUDA_R_16F, K, &beta, Y, CUDA_R_16F, N, CUBLAS_COMPUTE_32F,
                      CUBLAS_GEMM_DEFAULT) == CUBLAS_STATUS_SUCCESS;
}

unsigned int blocks_for(int64_t n, int per_block) {
  return static_cast<unsigned int>((n + per_block - 1) / per_block);
}

}  // namespace
}  // namespace decoder
}  // namespace attn_b200

using namespace attn_b200::decoder;

extern "C" {

size_t attn_decoder_layer_workspace_bytes(int B, int S, int hidden, int Hq, int Hkv, int D,
                                          int inter) {
  if (check_sizes(B, S, hidden, Hq, Hkv, D, inter) != ATTN_OK) return 0;
  return plan(B, S, hidden, Hq, Hkv, D, inter).total;
}

attn_status attn_decoder_layer_fwd(const void* x, const void* w_attn_norm, const void* w_qkv,
                                   const void* w_o, const void* w_mlp_norm, const void* w_gate_up,
                                   const void* w_down, void* y, int B, int S, int hidden, int Hq,
                                   int Hkv, int D, int inter, float eps, float rope_theta,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !w_attn_norm || !w_qkv || !w_o || !w_mlp_norm || !w_gate_up || !w_down || !y ||
      !workspace)
    return ATTN_ERR_NULL;
  attn_status st = check_sizes(B, S, hidden, Hq, Hkv, D, inter);
  if (st != ATTN_OK) return st;
  if (!(eps >= 0.0f) || !std::isfinite(eps) || !(rope_theta > 1.0f) || !std::isfinite(rope_theta))
    return ATTN_ERR_SHAPE;
  const void* ptrs[] = {x, w_attn_norm, w_qkv, w_o, w_mlp_norm, w_gate_up, w_down, y};
  for (const void* p : ptrs)
    if (!aligned16(p)) return ATTN_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_ALIGN;
  const Plan pl = plan(B, S, hidden, Hq, Hkv, D, inter);
  if (workspace_bytes < pl.total) return ATTN_ERR_WORKSPACE;
  // y may be x itself: x is last read (residual copy) before y is first written

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cublasHandle_t hb = handle_for(cs);
  if (!hb) return ATTN_ERR_CUDA;

  char* ws = static_cast<char*>(workspace);
  float2* cs_tab = reinterpret_cast<float2*>(ws + pl.cs);
  __half* n = reinterpret_cast<__half*>(ws + pl.n);
  __half* big = reinterpret_cast<__half*>(ws + pl.big);
  __half* q = reinterpret_cast<__half*>(ws + pl.q);
  __half* k = reinterpret_cast<__half*>(ws + pl.k);
  __half* v = reinterpret_cast<__half*>(ws + pl.v);
  __half* o = reinterpret_cast<__half*>(ws + pl.o);
  float* lse = reinterpret_cast<float*>(ws + pl.lse);
  __half* h = reinterpret_cast<__half*>(ws + pl.h);
  __half* g = reinterpret_cast<__half*>(ws + pl.g);
  const __half* xin = static_cast<const __half*>(x);
  __half* out = static_cast<__half*>(y);
  const int T = B * S;
  const int qkv_cols = (Hq + 2 * Hkv) * D;
  const size_t row_bytes = static_cast<size_t>(T) * hidden * 2;

  // attention block: h = x + merge(attn(rope(split(rmsnorm(x) Wqkv^T)))) Wo^T
  rope_table_kernel<<<blocks_for(static_cast<int64_t>(S) * (D / 2), 256), 256, 0, cs>>>(
      cs_tab, S, D, std::log2(static_cast<double>(rope_theta)));
  rmsnorm_kernel<<<T, kRowThreads, 0, cs>>>(xin, static_cast<const __half*>(w_attn_norm), n,
                                            hidden, eps);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (!gemm_rows(hb, n, static_cast<const __half*>(w_qkv), big, T, qkv_cols, hidden, 0.0f))
    return ATTN_ERR_CUDA;
  rope_split_kernel<<<blocks_for(static_cast<int64_t>(T) * (Hq + 2 * Hkv) * (D / 16), 256), 256,
                      0, cs>>>(big, cs_tab, q, k, v, B, S, Hq, Hkv, D);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  st = attn_fwd(q, k, v, o, lse, B, Hq, Hkv, S, D, 1, stream);
  if (st != ATTN_OK) return st;
  merge_heads_kernel<<<blocks_for(static_cast<int64_t>(T) * Hq * (D / 8), 256), 256, 0, cs>>>(
      o, q, B, S, Hq, D);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyAsync(h, xin, row_bytes, cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (!gemm_rows(hb, q, static_cast<const __half*>(w_o), h, T, hidden, Hq * D, 1.0f))
    return ATTN_ERR_CUDA;

  // MLP block: y = h + (silu(n2 Wg^T) * (n2 Wu^T)) Wd^T, n2 = rmsnorm(h)
  rmsnorm_kernel<<<T, kRowThreads, 0, cs>>>(h, static_cast<const __half*>(w_mlp_norm), n, hidden,
                                            eps);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (!gemm_rows(hb, n, static_cast<const __half*>(w_gate_up), big, T, 2 * inter, hidden, 0.0f))
    return ATTN_ERR_CUDA;
  swiglu_kernel<<<blocks_for(static_cast<int64_t>(T) * (inter / 8), 256), 256, 0, cs>>>(big, g, T,
                                                                                       inter);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyAsync(out, h, row_bytes, cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (!gemm_rows(hb, g, static_cast<const __half*>(w_down), out, T, hidden, inter, 1.0f))
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

}  // extern "C"
