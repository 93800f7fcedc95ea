// decoder_api.cu -- C ABI of the LLaMA3 single-decoder-layer proxy (declared
// in include/decoder_layer.h): argument checks, the workspace plan, and the
// launch sequence
//   RMSNorm -> QKV GEMM with RoPE + head split in its epilogue -> attention
//   (attn_fwd) -> O GEMM reading the attention output head-major, + residual
//   -> RMSNorm -> gate/up GEMM with SwiGLU in its epilogue -> down GEMM +
//   residual,
// all on the caller's stream, every GEMM this library's tcgen05 kernel.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "decoder_layer.h"
#include "decoder_sm100.cuh"
#include "gemm_sm100.cuh"

namespace attn_b200 {
unsigned int* stream_status_block(cudaStream_t stream);  // attn_api.cu
namespace decoder {
namespace {

size_t r256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Byte offsets of the workspace regions of one call.
struct Plan {
  size_t cs, n, q, k, v, o, lse, h, g, total;
};

Plan plan(int B, int S, int hidden, int Hq, int Hkv, int D, int inter) {
  const size_t T = static_cast<size_t>(B) * S;
  Plan p;
  size_t at = 0;
  auto take = [&at](size_t bytes) {
    const size_t off = at;
    at += r256(bytes);
    return off;
  };
  p.cs = take(static_cast<size_t>(S) * (D / 2) * sizeof(float2));  // rotary table
  p.n = take(T * hidden * 2);                                       // RMSNorm outputs
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

std::atomic<uint64_t> g_gemm_timeout_ns{2000000000ull};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D fp16 view [rows, cols] (row-major, cols contiguous), 64 x 128 boxes
// with the 128-byte swizzle.
bool encode_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int g_sms = 0;
std::once_flag g_gemm_once;
bool g_gemm_ready = false;

using GemmKernel = void (*)(const CUtensorMap, const CUtensorMap, const gemm::GemmParams);
GemmKernel gemm_kernel_for(int epi) {
  switch (epi) {
    case gemm::kEpiStore: return gemm::gemm_kernel<gemm::kEpiStore>;
    case gemm::kEpiResidual: return gemm::gemm_kernel<gemm::kEpiResidual>;
    case gemm::kEpiRope: return gemm::gemm_kernel<gemm::kEpiRope>;
    default: return gemm::gemm_kernel<gemm::kEpiSwiGLU>;
  }
}

bool gemm_setup() {
  std::call_once(g_gemm_once, [] {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return;
    for (int e = 0; e < 4; ++e)
      if (cudaFuncSetAttribute(gemm_kernel_for(e), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(sizeof(gemm::SharedGemm))) != cudaSuccess)
        return;
    g_gemm_ready = true;
  });
  return g_gemm_ready;
}

// Y [T, N] = A [T, K] * W [N or 2N, K]^T with epilogue `epi`, on `stream`.
// `a` is row-major [T, K], or (p.a_head_major) the attention output
// [B, Hq, S, D], mapped as [B * Hq * S, D].
bool run_gemm(int epi, const __half* a, const __half* w, gemm::GemmParams p, cudaStream_t stream) {
  if (!gemm_setup()) return false;
  CUtensorMap ta, tw;
  const uint64_t a_rows = p.a_head_major ? static_cast<uint64_t>(p.T) * p.Hq
                                         : static_cast<uint64_t>(p.T);
  const uint64_t a_cols = p.a_head_major ? static_cast<uint64_t>(p.D) : static_cast<uint64_t>(p.K);
  const uint64_t w_rows = epi == gemm::kEpiSwiGLU ? 2 * static_cast<uint64_t>(p.N)
                                                  : static_cast<uint64_t>(p.N);
  if (!encode_map(&ta, a, a_rows, a_cols) || !encode_map(&tw, w, w_rows, p.K)) return false;
  p.n_tiles_m = (p.T + gemm::kTileM - 1) / gemm::kTileM;
  p.n_tiles_n = epi == gemm::kEpiSwiGLU ? (p.N + 127) / 128 : (p.N + gemm::kTileN - 1) / gemm::kTileN;
  p.n_tiles = p.n_tiles_m * p.n_tiles_n;
  p.timeout_ns = g_gemm_timeout_ns.load();
  const int pairs = p.n_tiles < g_sms / 2 ? p.n_tiles : g_sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(gemm::kThreads);
  cfg.dynamicSmemBytes = sizeof(gemm::SharedGemm);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_kernel_for(epi), ta, tw, p) == cudaSuccess;
}

unsigned int blocks_for(int64_t n, int per_block) {
  return static_cast<unsigned int>((n + per_block - 1) / per_block);
}

}  // namespace
}  // namespace decoder
}  // namespace attn_b200

using namespace attn_b200;
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

  char* ws = static_cast<char*>(workspace);
  float2* cs_tab = reinterpret_cast<float2*>(ws + pl.cs);
  __half* n = reinterpret_cast<__half*>(ws + pl.n);
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
  // the GEMMs report timeouts in the stream's status block, like attn_fwd
  unsigned int* gstat = stream_status_block(cs);
  if (!gstat) return ATTN_ERR_CUDA;

  gemm::GemmParams gp = {};
  gp.T = T;
  gp.S = S;
  gp.Hq = Hq;
  gp.Hkv = Hkv;
  gp.D = D;
  gp.status = gstat;

  // attention block: h = x + merge(attn(rope(split(rmsnorm(x) Wqkv^T)))) Wo^T
  rope_table_kernel<<<blocks_for(static_cast<int64_t>(S) * (D / 2), 256), 256, 0, cs>>>(
      cs_tab, S, D, std::log2(static_cast<double>(rope_theta)));
  rmsnorm_kernel<<<T, kRowThreads, 0, cs>>>(xin, static_cast<const __half*>(w_attn_norm), n,
                                            hidden, eps);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  {
    gemm::GemmParams p = gp;
    p.N = qkv_cols;
    p.K = hidden;
    p.q = q;
    p.k = k;
    p.v = v;
    p.cs = cs_tab;
    if (!run_gemm(gemm::kEpiRope, n, static_cast<const __half*>(w_qkv), p, cs)) return ATTN_ERR_CUDA;
  }
  st = attn_fwd(q, k, v, o, lse, B, Hq, Hkv, S, D, 1, stream);
  if (st != ATTN_OK) return st;
  {
    // the output projection reads O head-major when no 128-row block of
    // tokens straddles two sequences; otherwise O is merged token-major first
    gemm::GemmParams p = gp;
    p.N = hidden;
    p.K = Hq * D;
    p.r = xin;
    p.y = h;
    const __half* a = o;
    if (S % 128 == 0) {
      p.a_head_major = 1;
    } else {
      merge_heads_kernel<<<blocks_for(static_cast<int64_t>(T) * Hq * (D / 8), 256), 256, 0,
                           cs>>>(o, q, B, S, Hq, D);
      if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
      a = q;
    }
    if (!run_gemm(gemm::kEpiResidual, a, static_cast<const __half*>(w_o), p, cs)) return ATTN_ERR_CUDA;
  }

  // MLP block: y = h + (silu(n2 Wg^T) * (n2 Wu^T)) Wd^T, n2 = rmsnorm(h)
  rmsnorm_kernel<<<T, kRowThreads, 0, cs>>>(h, static_cast<const __half*>(w_mlp_norm), n, hidden,
                                            eps);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  {
    gemm::GemmParams p = gp;
    p.N = inter;
    p.K = hidden;
    p.y = g;
    if (!run_gemm(gemm::kEpiSwiGLU, n, static_cast<const __half*>(w_gate_up), p, cs))
      return ATTN_ERR_CUDA;
  }
  {
    gemm::GemmParams p = gp;
    p.N = hidden;
    p.K = inter;
    p.r = h;
    p.y = out;
    if (!run_gemm(gemm::kEpiResidual, g, static_cast<const __half*>(w_down), p, cs))
      return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // extern "C"
