// gemm_sm100.cuh -- the projection GEMMs of the LLaMA3 single-decoder-layer
// proxy (the PipeThreader pages' second workload, papers.lqhl.me
// "PipeThreader-OSDI25", section 实验与结果, paper Sec. 6.3 / Fig. 13), on
// tcgen05 tensor cores, with the layer's element steps fused into the
// epilogue:
//
//   Y[T, N] = A[T, K] * W[N, K]^T,  fp16 operands, fp32 accumulation,
//
// and per epilogue kind
//   kEpiStore    Y rounded to fp16,
//   kEpiResidual Y = round(R + A W^T) (R may be Y itself: read, then written
//                by the same thread),
//   kEpiRope     the fused Q/K/V projection: the accumulator is rounded to
//                fp16 (the value an unfused layer would store), Q and K heads
//                are rotated by RoPE in fp32 and rounded again, and every
//                head is written head-major into Q [B, Hq, S, D], K, V
//                [B, Hkv, S, D],
//   kEpiSwiGLU   the gate/up projection: a pair tile's 256 columns are 128
//                gate columns (W rows n0..) and the 128 matching up columns
//                (W rows I + n0..); both are rounded to fp16, then
//                G = round(silu(gate) * up) is written to G [T, I].
// The arithmetic after each rounding is the one the standalone element
// kernels use, so fused and unfused layers store the same tensors.
//
// Pairs of CTAs (2-CTA clusters) compute 256 x 256 tiles with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): CTA r holds rows
// [128 r, 128 r + 128) of the tile's A and W rows [128 r, 128 r + 128) of
// its B (no multicast: each CTA loads only its own halves), and its 128
// accumulator rows x 256 columns in its own TMEM, double-buffered (512
// columns) so that the epilogue of one tile overlaps the next tile's
// main loop.  K advances in 64-column stages (one 128-byte swizzle panel),
// 6 stages of 32 KiB per CTA.  The even CTA issues the MMAs; both CTAs' TMA
// loads complete on the even CTA's barriers.
//
// The A operand is either a row-major [T, K] matrix or, for the output
// projection, the attention output O [B, Hq, S, D] read head-major: K
// column k of token t = b S + s is O[b, k / D, s, k % D] (requires S % 128
// == 0, so a CTA's 128 rows never straddle two sequences).
#pragma once

#include <cuda_fp16.h>

#include "ptx_sm100.cuh"

namespace attn_b200 {
namespace gemm {

constexpr int kTileM = 256;   // per pair
constexpr int kTileN = 256;
constexpr int kTileK = 64;
constexpr int kStages = 6;
constexpr int kThreads = 256;  // warp 0 producer, warp 1 MMA, warps 4-7 epilogue
constexpr uint32_t kHalfBytes = 128u * kTileK * 2;  // 16 KiB: 128 rows x 64 fp16
constexpr uint32_t kAccCols = 256;

enum Epi : int { kEpiStore = 0, kEpiResidual = 1, kEpiRope = 2, kEpiSwiGLU = 3 };

struct GemmParams {
  int T, N, K;              // Y [T, N]; for kEpiSwiGLU N = I (W has 2 I rows)
  __half* y;                // kEpiStore / kEpiResidual / kEpiSwiGLU output
  const __half* r;          // kEpiResidual addend [T, N]
  // kEpiRope
  __half *q, *k, *v;
  const float2* cs;         // rotary table [S, D/2] (cos, sin)
  int S, Hq, Hkv, D;
  int a_head_major;         // A is O [B, Hq, S, D] read head-major (S % 128 == 0)
  int n_tiles_m, n_tiles_n, n_tiles;
  unsigned int* status;
  unsigned long long timeout_ns;
};

enum GemmSite : uint32_t {
  kSiteGemmProducer = 0x2101,
  kSiteGemmMmaFull = 0x2201,
  kSiteGemmMmaAcc = 0x2202,
  kSiteGemmEpilogue = 0x2401,
};

struct SharedGemm {
  uint8_t a[kStages][kHalfBytes];
  uint8_t b[kStages][kHalfBytes];
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(SharedGemm) <= 232448, "shared memory exceeds the 227 KiB per-block limit");

// ---- cluster (CTA pair) forms ------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Pair MMA (whole warp; one elected lane issues), descriptor offsets in
// 16-byte units.
template <uint32_t kOff>
__device__ __forceinline__ void mma2(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                     uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b64 da, db;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "add.s64 da, %1, %5;\n\t"
      "add.s64 db, %2, %5;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], da, db, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "n"(kOff)
      : "memory");
}
// Arrives once on the barrier at offset `bar` of both CTAs when every pair
// MMA the elected lane issued before it has completed.
__device__ __forceinline__ void commit2(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;\n\t}" ::"r"(bar),
      "h"(static_cast<uint16_t>(0x3))
      : "memory");
}
// Tile load into this CTA's shared memory whose bytes complete on `bar`,
// which may be the even CTA's barrier (a shared::cluster address).
__device__ __forceinline__ void tma_load2(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                          int32_t x, int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr)
               : "memory");
}

// Tile t of the static schedule: N-major, so that consecutive clusters share
// a block of W.
__device__ __forceinline__ void tile_coords(const GemmParams& p, int t, int& tm, int& tn) {
  tn = t / p.n_tiles_m;
  tm = t - tn * p.n_tiles_m;
}

// A's coordinates (x = column, y = row of the TMA view) of K stage kb for
// the CTA's 128 rows starting at token row0.
__device__ __forceinline__ void a_coords(const GemmParams& p, int row0, int kb, int& x, int& y) {
  if (!p.a_head_major) {
    x = kb * kTileK;
    y = row0;
    return;
  }
  const int col = kb * kTileK;
  const int h = col / p.D;
  const int b = row0 / p.S;
  const int s = row0 - b * p.S;
  x = col - h * p.D;
  y = (b * p.Hq + h) * p.S + s;
}

// W rows of this CTA's half of tile column tn.
__device__ __forceinline__ int w_row(const GemmParams& p, int tn, uint32_t rank, int epi) {
  if (epi == kEpiSwiGLU) return static_cast<int>(rank) * p.N + tn * 128;  // gate, then up
  return tn * kTileN + static_cast<int>(rank) * 128;
}

__device__ __forceinline__ float round_h(float x) { return __half2float(__float2half_rn(x)); }

// ---- epilogues (thread = one accumulator row = TMEM lane) --------------------
template <int kEpi>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, uint32_t acc, int row, int tn) {
  const bool valid = row < p.T;
  if constexpr (kEpi == kEpiStore || kEpi == kEpiResidual) {
#pragma unroll 1
    for (int c = 0; c < kTileN; c += 32) {
      uint32_t w[32];
      tmem_ld32(acc + c, w);
      tmem_wait_ld();
      reg_dep32(w);
      const int col = tn * kTileN + c;
      if (!valid || col >= p.N) continue;
      const size_t off = static_cast<size_t>(row) * p.N + col;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (col + 8 * g >= p.N) break;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(w[8 * g + e]);
        if constexpr (kEpi == kEpiResidual) {
          const uint4 rv = *reinterpret_cast<const uint4*>(p.r + off + 8 * g);
          const __half2* rh = reinterpret_cast<const __half2*>(&rv);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 t = __half22float2(rh[e]);
            f[2 * e] += t.x;
            f[2 * e + 1] += t.y;
          }
        }
        uint4 o;
        o.x = pack_half2(f[0], f[1]);
        o.y = pack_half2(f[2], f[3]);
        o.z = pack_half2(f[4], f[5]);
        o.w = pack_half2(f[6], f[7]);
        *reinterpret_cast<uint4*>(p.y + off + 8 * g) = o;
      }
    }
  } else if constexpr (kEpi == kEpiSwiGLU) {
#pragma unroll 1
    for (int c = 0; c < 128; c += 32) {
      uint32_t wg[32], wu[32];
      tmem_ld32(acc + c, wg);
      tmem_ld32(acc + 128 + c, wu);
      tmem_wait_ld();
      reg_dep32(wg);
      reg_dep32(wu);
      const int col = tn * 128 + c;
      if (!valid || col >= p.N) continue;
      const size_t off = static_cast<size_t>(row) * p.N + col;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (col + 8 * g >= p.N) break;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float a = round_h(__uint_as_float(wg[8 * g + e]));
          const float u = round_h(__uint_as_float(wu[8 * g + e]));
          f[e] = a / (1.0f + expf(-a)) * u;
        }
        uint4 o;
        o.x = pack_half2(f[0], f[1]);
        o.y = pack_half2(f[2], f[3]);
        o.z = pack_half2(f[4], f[5]);
        o.w = pack_half2(f[6], f[7]);
        *reinterpret_cast<uint4*>(p.y + off + 8 * g) = o;
      }
    }
  } else {  // kEpiRope
    const int D = p.D, half = D / 2;
    const int b = row / p.S, s = row - (row / p.S) * p.S;
#pragma unroll 1
    for (int hd = 0; hd < kTileN; hd += D) {
      const int col0 = tn * kTileN + hd;       // first column of the head
      const int hs = col0 / D;                 // head index over Q, K, V heads
      const bool in_range = valid && col0 < p.N;
      __half* dst;
      bool rotate = true;
      if (hs < p.Hq) {
        dst = p.q + ((static_cast<size_t>(b) * p.Hq + hs) * p.S + s) * D;
      } else if (hs < p.Hq + p.Hkv) {
        dst = p.k + ((static_cast<size_t>(b) * p.Hkv + (hs - p.Hq)) * p.S + s) * D;
      } else {
        dst = p.v + ((static_cast<size_t>(b) * p.Hkv + (hs - p.Hq - p.Hkv)) * p.S + s) * D;
        rotate = false;
      }
#pragma unroll 1
      for (int i0 = 0; i0 < half; i0 += 32) {
        uint32_t wl[32], wh[32];
        tmem_ld32(acc + hd + i0, wl);
        tmem_ld32(acc + hd + half + i0, wh);
        tmem_wait_ld();
        reg_dep32(wl);
        reg_dep32(wh);
        if (!in_range) continue;
        const float2* csr = p.cs + static_cast<size_t>(s) * half + i0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float lo[8], hi[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a = round_h(__uint_as_float(wl[8 * g + e]));
            const float h2 = round_h(__uint_as_float(wh[8 * g + e]));
            if (rotate) {
              const float2 r = csr[8 * g + e];
              lo[e] = a * r.x - h2 * r.y;
              hi[e] = h2 * r.x + a * r.y;
            } else {
              lo[e] = a;
              hi[e] = h2;
            }
          }
          uint4 ol, oh;
          ol.x = pack_half2(lo[0], lo[1]);
          ol.y = pack_half2(lo[2], lo[3]);
          ol.z = pack_half2(lo[4], lo[5]);
          ol.w = pack_half2(lo[6], lo[7]);
          oh.x = pack_half2(hi[0], hi[1]);
          oh.y = pack_half2(hi[2], hi[3]);
          oh.z = pack_half2(hi[4], hi[5]);
          oh.w = pack_half2(hi[6], hi[7]);
          *reinterpret_cast<uint4*>(dst + i0 + 8 * g) = ol;
          *reinterpret_cast<uint4*>(dst + half + i0 + 8 * g) = oh;
        }
      }
    }
  }
}

// Grid: 2 * (number of pairs); cluster dims (2, 1, 1).
template <int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  SharedGemm* sm = reinterpret_cast<SharedGemm*>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const uint64_t to = p.timeout_ns;
  // both CTAs of a pair take the same branch: the alignment of the dynamic
  // shared memory base is the same in every CTA of the launch
  if (smem_addr(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(&p.status[0], kStatusSmemAlign);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&sm->full[s]), 1);
      mbar_init(smem_addr(&sm->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_addr(&sm->acc_full[b]), 1);
      mbar_init(smem_addr(&sm->acc_empty[b]), 8);  // 4 epilogue warps in each CTA
    }
    mbar_init(smem_addr(&sm->drain), 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc2(smem_addr(&sm->tmem_base), 2 * kAccCols);
    tmem_relinquish2();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_w);
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;
  const int n_k = (p.K + kTileK - 1) / kTileK;
  int loads = 0;  // stages loaded by this CTA

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol_a = l2_policy_evict_first();
      const uint64_t pol_w = l2_policy_evict_last();
      bool ok = true;
      for (int t = pair; ok && t < p.n_tiles; t += n_pairs) {
        int tm, tn;
        tile_coords(p, t, tm, tn);
        const int row0 = tm * kTileM + static_cast<int>(rank) * 128;
        const int wr = w_row(p, tn, rank, kEpi);
        for (int kb = 0; kb < n_k; ++kb, ++loads) {
          const int st = loads % kStages;
          if (loads >= kStages &&
              !mbar_wait(smem_addr(&sm->empty[st]), ((loads / kStages) & 1) ^ 1, abort, to,
                         p.status, kSiteGemmProducer)) {
            ok = false;
            break;
          }
          const uint32_t full = map_rank(smem_addr(&sm->full[st]), 0);
          if (rank == 0) mbar_arrive_expect_tx(smem_addr(&sm->full[st]), 4 * kHalfBytes);
          int ax, ay;
          a_coords(p, row0, kb, ax, ay);
          tma_load2(smem_addr(sm->a[st]), &tm_a, full, ax, ay, pol_a);
          tma_load2(smem_addr(sm->b[st]), &tm_w, full, kb * kTileK, wr, pol_w);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA (even CTA)
    if (rank == 0) {
      const uint32_t idesc = idesc_f16_f32(kTileM, kTileN, false, false);
      int used = 0, tiles = 0;
      bool ok = true;
      for (int t = pair; ok && t < p.n_tiles; t += n_pairs, ++tiles) {
        const int b = tiles & 1;
        if (tiles >= 2)
          ok = mbar_wait<true>(smem_addr(&sm->acc_empty[b]), ((tiles >> 1) - 1) & 1, abort, to,
                               p.status, kSiteGemmMmaAcc);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + b * kAccCols;
        for (int kb = 0; kb < n_k; ++kb, ++used) {
          const int st = used % kStages;
          ok = mbar_wait<true>(smem_addr(&sm->full[st]), (used / kStages) & 1, abort, to,
                               p.status, kSiteGemmMmaFull);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const uint64_t ad = smem_desc_sw128(smem_addr(sm->a[st]), 16, 1024);
          const uint64_t bd = smem_desc_sw128(smem_addr(sm->b[st]), 16, 1024);
          mma2<0>(d, ad, bd, idesc, kb > 0 ? 1u : 0u);
          mma2<2>(d, ad, bd, idesc, 1u);
          mma2<4>(d, ad, bd, idesc, 1u);
          mma2<6>(d, ad, bd, idesc, 1u);
          commit2(smem_addr(&sm->empty[st]));  // both CTAs' stage st is free
        }
        if (ok) commit2(smem_addr(&sm->acc_full[b]));
      }
      // the pair form, like the MMAs it tracks (it also arrives, unused, on
      // the odd CTA's drain barrier)
      commit2(smem_addr(&sm->drain));
      drain_wait(smem_addr(&sm->drain), 0, to, p.status);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue
    const int r = (warp - 4) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t acc_empty0 = map_rank(smem_addr(&sm->acc_empty[0]), 0);
    int tiles = 0;
    bool ok = true;
    for (int t = pair; ok && t < p.n_tiles; t += n_pairs, ++tiles) {
      const int b = tiles & 1;
      ok = mbar_wait(smem_addr(&sm->acc_full[b]), (tiles >> 1) & 1, abort, to, p.status,
                     kSiteGemmEpilogue);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      int tm, tn;
      tile_coords(p, t, tm, tn);
      const int row = tm * kTileM + static_cast<int>(rank) * 128 + r;
      epilogue_tile<kEpi>(p, lane_base + b * kAccCols, row, tn);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty0 + b * 8);
    }
  }

  // After a wait gave up, loads may still be in flight.  The odd CTA's
  // loads complete on the even CTA's barriers, which cannot see how far
  // the odd CTA got, so both producers give every copy in flight a fixed
  // 50 us to land (the normal path needs none: every load was consumed).
  if (warp == 0 && lane == 0 && *abort) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 50000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, 2 * kAccCols);
  }
}

}  // namespace gemm
}  // namespace attn_b200
