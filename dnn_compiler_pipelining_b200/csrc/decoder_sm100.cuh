// decoder_sm100.cuh -- the elementwise and row kernels of the LLaMA3 decoder
// layer proxy around the attention forward (the PipeThreader pages' second
// workload: an FP16 single decoder layer of LLaMA3-8B / 70B, section 实验与结果,
// paper Sec. 6.3 / Fig. 13).  The GEMMs are library calls; the attention is
// this library's fused kernel.  Every kernel here is bound by HBM traffic: each
// element crosses HBM once in each direction, with 16-byte vector accesses.
// Rows are multiples of 8 fp16 elements and 16-byte aligned, which the entry
// point checks; RMSNorm's second read of a row hits L1/L2.  Each computes in
// fp32 with one rounding to fp16 per output.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace attn_b200 {
namespace decoder {

constexpr int kRowThreads = 256;  // threads per row in the row kernels

// 8 fp16 <-> fp32
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 v;
  __half2* h = reinterpret_cast<__half2*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  return v;
}

// Sum over the block (kRowThreads threads); every thread gets the total.
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kRowThreads / 32; ++w) t += red[w];
  return t;
}

// RMSNorm of one token row per block: y = x / sqrt(mean(x^2) + eps) * w,
// x, y [T, H] fp16, w [H] fp16; H % 8 == 0.  The sum of squares and the
// product are fp32; y is rounded once.
__global__ void __launch_bounds__(kRowThreads)
    rmsnorm_kernel(const __half* __restrict__ x, const __half* __restrict__ w,
                   __half* __restrict__ y, int H, float eps) {
  __shared__ float red[kRowThreads / 32];
  const int64_t row = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * H);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  uint4* yr = reinterpret_cast<uint4*>(y + row * H);
  const int n8 = H / 8;
  float ss = 0.f;
  for (int c = threadIdx.x; c < n8; c += kRowThreads) {
    float f[8];
    unpack8(xr[c], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
  }
  const float rstd = rsqrtf(block_sum(ss, red) / static_cast<float>(H) + eps);
  for (int c = threadIdx.x; c < n8; c += kRowThreads) {
    float f[8], g[8];
    unpack8(xr[c], f);
    unpack8(wr[c], g);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = f[i] * rstd * g[i];
    yr[c] = pack8(f);
  }
}

// Rotary table: cs[s * (D/2) + i] = (cos, sin) of s * theta^(-2i/D), angles
// and their cosines / sines in fp64, stored as fp32.
__global__ void rope_table_kernel(float2* __restrict__ cs, int S, int D, double log2_theta) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int half = D / 2;
  if (idx >= static_cast<int64_t>(S) * half) return;
  const int s = static_cast<int>(idx / half), i = static_cast<int>(idx % half);
  const double inv_freq = exp2(-(2.0 * i / D) * log2_theta);
  double sn, cn;
  sincos(static_cast<double>(s) * inv_freq, &sn, &cn);
  cs[idx] = make_float2(static_cast<float>(cn), static_cast<float>(sn));
}

// Splits the fused projection qkv [B*S, (Hq + 2*Hkv) * D] (per token: the Hq
// query heads, then the Hkv key heads, then the Hkv value heads, D columns
// each) into head-major Q [B, Hq, S, D], K, V [B, Hkv, S, D], rotating Q and
// K: for i < D/2 the pair (i, i + D/2) at position s turns by angle
// s * theta^(-2i/D).  One thread per (token, head, 8 consecutive i).
__global__ void rope_split_kernel(const __half* __restrict__ qkv, const float2* __restrict__ cs,
                                  __half* __restrict__ q, __half* __restrict__ k,
                                  __half* __restrict__ v, int B, int S, int Hq, int Hkv, int D) {
  const int heads = Hq + 2 * Hkv;
  const int chunks = D / 16;  // 8-wide chunks of the first half
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(B) * S * heads * chunks;
  if (idx >= total) return;
  const int c = static_cast<int>(idx % chunks);
  const int hs = static_cast<int>((idx / chunks) % heads);
  const int64_t t = idx / (static_cast<int64_t>(chunks) * heads);  // token b * S + s
  const int s = static_cast<int>(t % S);
  const int64_t b = t / S;
  const int half = D / 2;
  const int i0 = c * 8;
  const __half* src = qkv + (t * heads + hs) * D;
  const uint4 lo = *reinterpret_cast<const uint4*>(src + i0);
  const uint4 hi = *reinterpret_cast<const uint4*>(src + half + i0);
  __half* dst;
  if (hs < Hq) {
    dst = q + ((b * Hq + hs) * S + s) * D;
  } else if (hs < Hq + Hkv) {
    dst = k + ((b * Hkv + (hs - Hq)) * S + s) * D;
  } else {
    dst = v + ((b * Hkv + (hs - Hq - Hkv)) * S + s) * D;
    *reinterpret_cast<uint4*>(dst + i0) = lo;
    *reinterpret_cast<uint4*>(dst + half + i0) = hi;
    return;
  }
  float a[8], e[8], ra[8], re[8];
  unpack8(lo, a);
  unpack8(hi, e);
  const float2* row = cs + static_cast<int64_t>(s) * half + i0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 r = row[j];
    ra[j] = a[j] * r.x - e[j] * r.y;
    re[j] = e[j] * r.x + a[j] * r.y;
  }
  *reinterpret_cast<uint4*>(dst + i0) = pack8(ra);
  *reinterpret_cast<uint4*>(dst + half + i0) = pack8(re);
}

// Head-major O [B, Hq, S, D] -> token-major [B*S, Hq*D] for the output
// projection.  One thread per 8 consecutive d.
__global__ void merge_heads_kernel(const __half* __restrict__ o, __half* __restrict__ out, int B,
                                   int S, int Hq, int D) {
  const int chunks = D / 8;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(B) * Hq * S * chunks;
  if (idx >= total) return;
  // idx walks the destination in order: token, head, chunk
  const int c = static_cast<int>(idx % chunks);
  const int h = static_cast<int>((idx / chunks) % Hq);
  const int64_t t = idx / (static_cast<int64_t>(chunks) * Hq);
  const int s = static_cast<int>(t % S);
  const int64_t b = t / S;
  const uint4 val = *reinterpret_cast<const uint4*>(o + ((b * Hq + h) * S + s) * D + c * 8);
  *reinterpret_cast<uint4*>(out + idx * 8) = val;
}

// SwiGLU: g[t, j] = silu(gu[t, j]) * gu[t, I + j], gu [T, 2I] (gate columns,
// then up columns), g [T, I]; silu(a) = a / (1 + e^-a).  I % 8 == 0.
__global__ void swiglu_kernel(const __half* __restrict__ gu, __half* __restrict__ g, int64_t T,
                              int I) {
  const int chunks = I / 8;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= T * chunks) return;
  const int64_t t = idx / chunks;
  const int c = static_cast<int>(idx % chunks);
  const __half* row = gu + t * 2 * static_cast<int64_t>(I);
  float a[8], u[8];
  unpack8(*reinterpret_cast<const uint4*>(row + c * 8), a);
  unpack8(*reinterpret_cast<const uint4*>(row + I + c * 8), u);
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = a[j] / (1.0f + expf(-a[j])) * u[j];
  *reinterpret_cast<uint4*>(g + idx * 8) = pack8(a);
}

}  // namespace decoder
}  // namespace attn_b200
