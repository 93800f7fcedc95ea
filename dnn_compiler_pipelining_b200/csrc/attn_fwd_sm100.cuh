// attn_fwd_sm100.cuh -- fused attention forward for sm_100a (B200).
//
// One pass computes O = softmax(Q K^T / sqrt(D) [+ causal mask]) V and the
// row log-sum-exp, for grouped-query heads, without writing the score matrix
// to memory.  This is the FlashAttention forward that the PipeThreader pages
// evaluate (papers.lqhl.me "PipeThreader-OSDI25", section 实验与结果, paper
// Sec. 6.2 / Fig. 12).  Their pipeline (section 核心方法, "sTask / sEU") splits
// the operator into load, mma and softmax tasks on TMA, TensorCore and CUDA
// cores and overlaps them inside an SM; here that split is fixed by hand as
// warp roles:
//
//   warp 4       TMA producer: Q tile once, then K_j / V_j tiles into a ring
//                of kStages shared-memory stages.
//   warp 5       MMA issuer (one thread): S_j = Q K_j^T into TMEM, then
//                O += P_j V_j with P read from TMEM; tcgen05.commit signals
//                mbarriers when they finish.
//   warps 0..3   softmax, one query row per thread (TMEM lane = row): load
//                S_j, apply the causal mask on the diagonal tile, update the
//                running max, exponentiate, write P_j (fp16) over S_j in
//                TMEM; rescale O when the running max grew by more than
//                kRescaleLog2 (lazy rescaling is exact: O and the row sum l
//                always share the same reference max); finally O / l and
//                LSE.
//
// TMEM (512 columns): S/P buffer 0 at [0,128), buffer 1 at [128,256),
// O at [256,384).  Two S buffers let the tensor core compute S_{j+1} while
// the softmax works on S_j.
//
// Shared memory tiles are 128 rows x 128 fp16 stored as two 64-column panels
// of 16 KiB in the TMA 128-byte swizzle, which is also the tcgen05 "SW128"
// canonical layout: Q and K are K-major operands, V is an MN-major operand.
#pragma once

#include <cuda_fp16.h>

#include "ptx_sm100.cuh"

namespace attn_b200 {

constexpr int kBlockM = 128;   // query rows per tile
constexpr int kBlockN = 128;   // keys per tile
constexpr int kHeadDim = 128;  // D
constexpr uint32_t kTileBytes = kBlockM * kHeadDim * 2;  // 32 KiB fp16 tile
constexpr uint32_t kPanelBytes = kTileBytes / 2;         // 64-column swizzle panel
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8
constexpr float kLn2 = 0.69314718055994531f;

struct FwdParams {
  __half* o;
  float* lse;
  int B, Hq, Hkv, S;
  int causal;
  float scale_log2;  // log2(e) / sqrt(D)
  unsigned long long timeout_ns;
};

// wait sites recorded in the status word when a bounded wait runs out
enum WaitSite : uint32_t {
  kSiteProducerEmpty = 0x101,
  kSiteMmaQ = 0x201,
  kSiteMmaK = 0x202,
  kSiteMmaP = 0x203,
  kSiteMmaV = 0x204,
  kSiteSoftmaxS = 0x301,
  kSiteSoftmaxO = 0x302,
  kSiteEpilogueO = 0x303,
};

template <int kStages>
struct alignas(1024) SharedV1 {
  uint8_t q[kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full;
  uint64_t k_full[kStages];
  uint64_t v_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;

// Waits that must finish even after another role gave up (in-flight copies
// and MMAs complete on their own); bounded all the same.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  int never = 0;
  mbar_wait(bar, parity, &never, timeout_ns, 0x401);
}

template <int kStages>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_v1_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Smem = SharedV1<kStages>;
  extern __shared__ uint8_t smem_raw[];
  Smem* sm = reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int n_qb = p.S / kBlockM;
  const int qb = n_qb - 1 - static_cast<int>(blockIdx.x);  // heaviest causal tiles first
  const int hq = blockIdx.y;
  const int b = blockIdx.z;
  const int g = hq / (p.Hq / p.Hkv);
  const int n_kv = p.causal ? qb + 1 : n_qb;
  const int q_row0 = (b * p.Hq + hq) * p.S + qb * kBlockM;
  const int kv_row0 = (b * p.Hkv + g) * p.S;
  const uint64_t to = p.timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&sm->q_full), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&sm->k_full[s]), 1);
      mbar_init(smem_addr(&sm->v_full[s]), 1);
      mbar_init(smem_addr(&sm->kv_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_addr(&sm->s_full[s]), 1);
      mbar_init(smem_addr(&sm->p_full[s]), kBlockM);
      mbar_init(smem_addr(&sm->pv_done[s]), 1);
    }
    mbar_init(smem_addr(&sm->drain), 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(&sm->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint32_t q_s = smem_addr(sm->q);
      mbar_arrive_expect_tx(smem_addr(&sm->q_full), kTileBytes);
      tma_load_2d(q_s, &tm_q, smem_addr(&sm->q_full), 0, q_row0);
      tma_load_2d(q_s + kPanelBytes, &tm_q, smem_addr(&sm->q_full), 64, q_row0);
      int j = 0;
      for (; j < n_kv; ++j) {
        const int st = j % kStages;
        const int rnd = j / kStages;
        if (rnd > 0 &&
            !mbar_wait(smem_addr(&sm->kv_empty[st]), (rnd - 1) & 1, abort, to, kSiteProducerEmpty))
          break;
        const int row = kv_row0 + j * kBlockN;
        const uint32_t kf = smem_addr(&sm->k_full[st]);
        const uint32_t vf = smem_addr(&sm->v_full[st]);
        const uint32_t k_s = smem_addr(sm->k[st]);
        const uint32_t v_s = smem_addr(sm->v[st]);
        mbar_arrive_expect_tx(kf, kTileBytes);
        tma_load_2d(k_s, &tm_k, kf, 0, row);
        tma_load_2d(k_s + kPanelBytes, &tm_k, kf, 64, row);
        mbar_arrive_expect_tx(vf, kTileBytes);
        tma_load_2d(v_s, &tm_v, vf, 0, row);
        tma_load_2d(v_s + kPanelBytes, &tm_v, vf, 64, row);
      }
      if (*abort) {
        // let every copy still in flight land before the CTA exits
        drain_wait(smem_addr(&sm->q_full), 0, to);
        for (int t = (j > kStages ? j - kStages : 0); t < j; ++t) {
          drain_wait(smem_addr(&sm->k_full[t % kStages]), (t / kStages) & 1, to);
          drain_wait(smem_addr(&sm->v_full[t % kStages]), (t / kStages) & 1, to);
        }
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16_f32(kBlockM, kBlockN, false, false);
      constexpr uint32_t idesc_pv = idesc_f16_f32(kBlockM, kHeadDim, false, true);
      const uint32_t q_s = smem_addr(sm->q);
      // O += P_t V_t; returns false if a wait ran out
      auto issue_pv = [&](int t) -> bool {
        const int pb = t & 1;
        const int st = t % kStages;
        if (!mbar_wait(smem_addr(&sm->p_full[pb]), (t >> 1) & 1, abort, to, kSiteMmaP)) return false;
        if (!mbar_wait(smem_addr(&sm->v_full[st]), (t / kStages) & 1, abort, to, kSiteMmaV))
          return false;
        tc_fence_after();
        const uint32_t v_s = smem_addr(sm->v[st]);
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk) {
          // V is MN-major: 16 keys = two 8-row groups of 1 KiB; the two
          // 64-column panels of D are kPanelBytes apart.
          const uint64_t bdesc = smem_desc_sw128(v_s + kk * 2048, kPanelBytes, 1024);
          mma_f16_ts(tmem + kTmemO, tmem + pb * 128 + kk * 8, bdesc, idesc_pv,
                     (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(smem_addr(&sm->kv_empty[st]));
        tc_commit(smem_addr(&sm->pv_done[pb]));
        return true;
      };
      bool ok = mbar_wait(smem_addr(&sm->q_full), 0, abort, to, kSiteMmaQ);
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j % kStages;
        if (!mbar_wait(smem_addr(&sm->k_full[st]), (j / kStages) & 1, abort, to, kSiteMmaK)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_s = smem_addr(sm->k[st]);
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          // K-major: 16 columns = 32 bytes inside a 128-byte swizzled row;
          // columns 64..127 live in the second panel.
          const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
          mma_f16_ss(tmem + (j & 1) * 128, smem_desc_sw128(q_s + off, 16, 1024),
                     smem_desc_sw128(k_s + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(smem_addr(&sm->s_full[j & 1]));
        if (j > 0 && !issue_pv(j - 1)) ok = false;
      }
      if (ok) issue_pv(n_kv - 1);
      // every MMA issued must complete before TMEM is released
      tc_commit(smem_addr(&sm->drain));
      drain_wait(smem_addr(&sm->drain), 0, to);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax
    const int r = threadIdx.x;  // query row inside the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sc = p.scale_log2;
    float m_use = -INFINITY;  // reference max (log2 units) shared by O and l
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      // tcgen05.ld/st are warp-collective: every wait outcome is made
      // warp-uniform before the warp touches TMEM.
      ok = mbar_wait(smem_addr(&sm->s_full[sb]), (j >> 1) & 1, abort, to, kSiteSoftmaxS);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_t = lane_base + sb * 128;
      uint32_t u[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_t + c * 32, u[c]);
      tmem_wait_ld();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(u[c][i]);
      if (p.causal && j == qb) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > r) sv[c] = -INFINITY;
      }
      float mx = sv[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, sv[c]);
      const float cand = mx * sc;
      if (j == 0) {
        m_use = cand;
      } else {
        const bool grow = cand > m_use + kRescaleLog2;
        if (__any_sync(0xffffffffu, grow)) {
          const float alpha = grow ? ex2_approx(m_use - cand) : 1.0f;
          // O must already hold P_{j-1} V_{j-1} before it is rescaled
          ok = mbar_wait(smem_addr(&sm->pv_done[(j - 1) & 1]), ((j - 1) >> 1) & 1, abort, to,
                         kSiteSoftmaxO);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[32];
            tmem_ld32(lane_base + kTmemO + c * 32, w);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * alpha);
            tmem_st32(lane_base + kTmemO + c * 32, w);
          }
          if (grow) {
            l *= alpha;
            m_use = cand;
          }
        }
      }
      const float neg_m = -m_use;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t ph[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = ex2_approx(fmaf(sv[c * 64 + 2 * i], sc, neg_m));
          const float p1 = ex2_approx(fmaf(sv[c * 64 + 2 * i + 1], sc, neg_m));
          l += p0 + p1;
          ph[i] = pack_half2(p0, p1);
        }
        tmem_st32(s_t + c * 32, ph);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_addr(&sm->p_full[sb]));
    }
    if (ok) {
      const int t = n_kv - 1;
      ok = mbar_wait(smem_addr(&sm->pv_done[t & 1]), (t >> 1) & 1, abort, to, kSiteEpilogueO);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const float inv_l = 1.0f / l;
        uint4* orow = reinterpret_cast<uint4*>(p.o + static_cast<size_t>(q_row0 + r) * kHeadDim);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t w[32];
          tmem_ld32(lane_base + kTmemO + c * 32, w);
          tmem_wait_ld();
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 pk;
            pk.x = pack_half2(__uint_as_float(w[v4 * 8 + 0]) * inv_l,
                              __uint_as_float(w[v4 * 8 + 1]) * inv_l);
            pk.y = pack_half2(__uint_as_float(w[v4 * 8 + 2]) * inv_l,
                              __uint_as_float(w[v4 * 8 + 3]) * inv_l);
            pk.z = pack_half2(__uint_as_float(w[v4 * 8 + 4]) * inv_l,
                              __uint_as_float(w[v4 * 8 + 5]) * inv_l);
            pk.w = pack_half2(__uint_as_float(w[v4 * 8 + 6]) * inv_l,
                              __uint_as_float(w[v4 * 8 + 7]) * inv_l);
            orow[c * 4 + v4] = pk;
          }
        }
        p.lse[q_row0 + r] = (m_use + log2f(l)) * kLn2;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn_b200
