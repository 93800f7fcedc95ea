// attn_fwd_db_sm100.cuh -- the fused attention forward with S double-buffered
// in TMEM, one 128-row tile per work item, on sm_100a (B200).
//
// Same operation, numerics, roles and work walk as attn_fwd_sm100.cuh (the
// FlashAttention forward the PipeThreader pages evaluate, papers.lqhl.me
// "PipeThreader-OSDI25", section 实验与结果, paper Sec. 6.2 / Fig. 12), with
// a different pipeline: the pages' point that the schedule of the load, mma
// and softmax tasks matters as much as the tiling (section 关键观察, 观察 2)
// is kept by building both and choosing per shape class from measurements.
//
//   * A work item is one 128-row tile of queries.
//   * S is double-buffered in TMEM: S[0] [0, kBN), S[1] [kBN, 2 kBN), O at
//     [256, 256 + kD).  The issuer computes S(g+2) right after PV(g) (g
//     counts this CTA's key blocks across items, so the buffers alternate
//     without a break at item boundaries).  The softmax of block g+1 then
//     runs while the tensor core works on PV(g) and S(g+2): the softmax is
//     not on the chain between two MMAs of the same tile, as it is in the
//     two-tile ping-pong kernel.
//   * kSplit = 2 runs two softmax warps on each TMEM lane quadrant (so two
//     instruction streams feed each SM sub-partition's MUFU unit); each
//     takes half of a block's keys, and the two exchange their partial row
//     maxima through shared memory.
//   * Head dimension 256 (the pages name large head dimensions as the case
//     where shared memory runs short, section 设计取舍, "边界条件": RetNet)
//     uses 64-key blocks: Q (64 KiB) plus a 3-stage K ring and a 2-stage V
//     ring of 32 KiB tiles fill 224 KiB.
//
// Because O may still lack PV(g-1) while the softmax of block g runs, a
// lazy rescale (the row max grew by more than 2^8) first waits for PV(g-1)
// to complete (pv_done, one phase per block, never more than one phase
// ahead of the softmax).
//
// Warp roles (512 threads): warps 0-3 (and 4-7 when kSplit = 2) softmax,
// warps 8-11 epilogue, warp 12 Q/K producer, warp 13 MMA issuer, warp 14 V
// producer.
#pragma once

#include <cuda_fp16.h>

#include <utility>

#include "attn_fwd_sm100.cuh"

namespace attn_b200 {
namespace db {

template <int kD>
struct Cfg {
  static constexpr int kBN = kD == 256 ? 64 : 128;               // keys per K/V tile
  static constexpr int kStagesK = 3;
  static constexpr int kStagesV = 2;
  static constexpr uint32_t kQPanel = 128u * 128u;               // 128 rows x 64 fp16
  static constexpr uint32_t kKvPanel = static_cast<uint32_t>(kBN) * 128u;
  static constexpr uint32_t kQBytes = kQPanel * (kD / 64);
  static constexpr uint32_t kKvBytes = kKvPanel * (kD / 64);
  static constexpr uint32_t kTmemO = 256u;
};

template <int kD, int kSplit = 1>
struct SharedDb {
  using C = Cfg<kD>;
  uint8_t q[C::kQBytes];
  uint8_t k[C::kStagesK][C::kKvBytes];
  uint8_t v[C::kStagesV][C::kKvBytes];
  float stat_m[kBlockM];
  float stat_l[kSplit][kBlockM];        // [column half][row]
  float red_max[kSplit][2][kBlockM];    // [block parity][column half][row] (kSplit = 2)
  uint64_t xmax[kSplit][4];             // [block parity][lane quadrant]: both halves posted
  uint32_t redo_bits[kRedoWords];
  uint64_t q_full, q_empty;
  uint64_t k_full[C::kStagesK], k_empty[C::kStagesK], v_full[C::kStagesV], v_empty[C::kStagesV];
  uint64_t s_full[2], p_full[2];  // [S buffer]
  uint64_t pv_done;               // one phase per PV (per key block)
  uint64_t o_done, o_free, stats_ready, stats_free;
  uint64_t redo_ready;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(SharedDb<256, 1>) <= 232448, "shared memory exceeds the 227 KiB per-block limit");
static_assert(sizeof(SharedDb<128, 2>) <= 232448, "shared memory exceeds the 227 KiB per-block limit");

__device__ __forceinline__ uint32_t tmem_s(int b, int bn) {
  return static_cast<uint32_t>(b) * static_cast<uint32_t>(bn);
}

// Key blocks of the item's tile (items are one 128-row tile).
template <int kBN>
__device__ __forceinline__ int n_blocks(const FwdParams& p, const Item& it) {
  if (it.n_kv[0] == 0) return 0;
  const int nk = (p.Sk + kBN - 1) / kBN;
  if (!p.causal) return nk;
  const int last_row = min(it.qb0 * kBlockM + kBlockM - 1, p.S - 1);
  return min(nk, (last_row + p.off) / kBN + 1);
}

// S(g) = Q K^T: kD / 16 MMAs of M = 128, N = kBN, K = 16.
template <int kD, int kk>
__device__ __forceinline__ void qk_step(uint32_t d, uint64_t qd, uint64_t kd, uint32_t idesc) {
  using C = Cfg<kD>;
  constexpr uint32_t a_off = ((kk >> 2) * C::kQPanel + (kk & 3) * 32) >> 4;
  constexpr uint32_t b_off = ((kk >> 2) * C::kKvPanel + (kk & 3) * 32) >> 4;
  mma_ss<a_off, b_off>(d, qd, kd, idesc, kk > 0 ? 1u : 0u);
}
template <int kD, int... kK>
__device__ __forceinline__ void qk_steps(uint32_t d, uint64_t qd, uint64_t kd, uint32_t idesc,
                                         std::integer_sequence<int, kK...>) {
  (qk_step<kD, kK>(d, qd, kd, idesc), ...);
}
template <int kD>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_s, uint32_t k_s) {
  const uint32_t idesc = idesc_f16_f32(kBlockM, Cfg<kD>::kBN, false, false);
  qk_steps<kD>(d_tmem, smem_desc_sw128(q_s, 16, 1024), smem_desc_sw128(k_s, 16, 1024), idesc,
               std::make_integer_sequence<int, kD / 16>{});
}

// O (+)= P V: kBN / 16 MMAs of M = 128, N = kD, K = 16 keys; A = P from TMEM
// (8 columns per MMA), B = V MN-major: 64-column groups of D one panel apart
// (LBO), 8-key groups 1 KiB apart (SBO), 16 keys = 2 KiB per step.
template <int kk>
__device__ __forceinline__ void pv_step(uint32_t o, uint32_t pt, uint64_t vd, uint32_t idesc,
                                        uint32_t acc) {
  mma_ts<kk * 8, (kk * 2048) / 16>(o, pt, vd, idesc, (acc || kk > 0) ? 1u : 0u);
}
template <int... kK>
__device__ __forceinline__ void pv_steps(uint32_t o, uint32_t pt, uint64_t vd, uint32_t idesc,
                                         uint32_t acc, std::integer_sequence<int, kK...>) {
  (pv_step<kK>(o, pt, vd, idesc, acc), ...);
}
template <int kD>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_s,
                                         bool accumulate) {
  using C = Cfg<kD>;
  const uint32_t idesc = idesc_f16_f32(kBlockM, kD, false, true);
  const uint64_t vd = smem_desc_sw128(v_s, C::kKvPanel, 1024);
  pv_steps(o_tmem, p_tmem, vd, idesc, accumulate ? 1u : 0u,
           std::make_integer_sequence<int, C::kBN / 16>{});
}

template <class Sm, bool kSpin = false>
__device__ __forceinline__ int walk(ItemWalk& w, const FwdParams& p, Sm* sm,
                                    volatile int* abort, bool& ok, uint32_t site) {
  if (!w.exact) {
    const int id = seq_item(p, w.k);
    if (id >= 0) {
      ++w.k;
      return id;
    }
    w.n_fast = w.k;
    w.exact = true;
    w.k = 0;
    if (!mbar_wait<kSpin>(smem_addr(&sm->redo_ready), 0, abort, p.timeout_ns, p.status, site)) {
      ok = false;
      return -1;
    }
  }
  while (w.k < w.n_fast && !((sm->redo_bits[w.k >> 5] >> (w.k & 31)) & 1u)) ++w.k;
  if (w.k >= w.n_fast) return -1;
  return seq_item(p, w.k++);
}

template <int kD, class Sm>
__device__ __forceinline__ void producer(Sm* sm, const FwdParams& p,
                                         const CUtensorMap* tm_q, const CUtensorMap* tm_kv,
                                         bool is_v, volatile int* abort) {
  using C = Cfg<kD>;
  constexpr int kPanels = kD / 64;
  const uint64_t to = p.timeout_ns;
  const uint64_t keep = l2_policy_evict_last();
  const uint64_t once = l2_policy_evict_first();
  const int depth = is_v ? C::kStagesV : C::kStagesK;
  int rc = 0, qcnt = 0;
  bool ok = true;
  ItemWalk w;
  int item;
  while (ok && (item = walk(w, p, sm, abort, ok, kSiteProducerRedo)) >= 0) {
    const Item it = decode_item(p, item);
    const int n = n_blocks<C::kBN>(p, it);
    if (!is_v) {
      if (qcnt > 0 && !mbar_wait(smem_addr(&sm->q_empty), (qcnt - 1) & 1, abort, to, p.status,
                                 kSiteProducerQ)) {
        ok = false;
        break;
      }
      const int q_row = (it.b * p.Hq + it.hq) * p.S + it.qb0 * kBlockM;
      mbar_arrive_expect_tx(smem_addr(&sm->q_full), C::kQBytes);
#pragma unroll
      for (int pn = 0; pn < kPanels; ++pn)
        tma_load_2d(smem_addr(sm->q) + pn * C::kQPanel, tm_q, smem_addr(&sm->q_full), 64 * pn,
                    q_row, once);
      ++qcnt;
    }
    const int kv_row = (it.b * p.Hkv + it.g) * p.Sk;
    for (int j = 0; j < n; ++j, ++rc) {
      const int st = rc % depth;
      const uint32_t empty = smem_addr(is_v ? &sm->v_empty[st] : &sm->k_empty[st]);
      if (rc >= depth && !mbar_wait(empty, ((rc / depth) & 1) ^ 1, abort, to, p.status,
                                    is_v ? kSiteProducerV : kSiteProducerK)) {
        ok = false;
        break;
      }
      const uint32_t full = smem_addr(is_v ? &sm->v_full[st] : &sm->k_full[st]);
      const uint32_t dst = smem_addr(is_v ? sm->v[st] : sm->k[st]);
      mbar_arrive_expect_tx(full, C::kKvBytes);
#pragma unroll
      for (int pn = 0; pn < kPanels; ++pn)
        tma_load_2d(dst + pn * C::kKvPanel, tm_kv, full, 64 * pn, kv_row + j * C::kBN, keep);
    }
  }
  if (!is_v && ok && w.exact) {
    int c = 0;
    for (int i = 0; i < kRedoWords; ++i) c += __popc(sm->redo_bits[i]);
    if (c) atomicAdd(&p.status[2], static_cast<unsigned int>(c));
  }
  if (*abort) {
    if (!is_v && qcnt > 0) drain_wait(smem_addr(&sm->q_full), (qcnt - 1) & 1, to, p.status);
    for (int t = (rc > depth ? rc - depth : 0); t < rc; ++t)
      drain_wait(smem_addr(is_v ? &sm->v_full[t % depth] : &sm->k_full[t % depth]),
                 (t / depth) & 1, to, p.status);
  }
}

// MMA issuer (whole warp).  Per item of n blocks, step t = 0..n+1 issues
// PV(t-2) (t >= 2) and then S(t) (t < n); g0 + t is the CTA-wide block
// index that picks the S buffer.  One thread issues every MMA: S(t)
// overwrites the columns PV(t-2) reads and every PV accumulates into O, and
// only MMAs of one thread are ordered by the pipe.
template <int kD, class Sm>
__device__ __forceinline__ void mma(Sm* sm, const FwdParams& p, uint32_t tmem,
                                    volatile int* abort) {
  using C = Cfg<kD>;
  const uint64_t to = p.timeout_ns;
  int g0 = 0;     // key blocks of earlier items
  int qcnt = 0;   // items so far
  bool ok = true;
  ItemWalk w;
  int item;
  while (ok && (item = walk(w, p, sm, abort, ok, kSiteMmaRedo)) >= 0) {
    const bool hilo = w.exact;
    const Item it = decode_item(p, item);
    const int n = n_blocks<C::kBN>(p, it);
    for (int t = 0; ok && t < n + 2; ++t) {
      if (t >= 2) {
        const int j = t - 2, g = g0 + j, b = g & 1;
        ok = mbar_wait(smem_addr(&sm->v_full[g % C::kStagesV]), (g / C::kStagesV) & 1, abort, to,
                       p.status, kSiteMmaV);
        if (ok && j == 0 && qcnt > 0)
          ok = mbar_wait(smem_addr(&sm->o_free), (qcnt - 1) & 1, abort, to, p.status, kSiteMmaO);
        ok = ok && mbar_wait(smem_addr(&sm->p_full[b]), (g >> 1) & 1, abort, to, p.status,
                             kSiteMmaP);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t v_s = smem_addr(sm->v[g % C::kStagesV]);
        const uint32_t p_t = tmem + tmem_s(b, C::kBN);
        issue_pv<kD>(tmem + C::kTmemO, p_t, v_s, j > 0);
        if (hilo) issue_pv<kD>(tmem + C::kTmemO, p_t + C::kBN / 2, v_s, true);
        tc_commit(smem_addr(&sm->pv_done));
        tc_commit(smem_addr(&sm->v_empty[g % C::kStagesV]));
        if (j == n - 1) tc_commit(smem_addr(&sm->o_done));
      }
      if (t < n) {
        const int g = g0 + t, b = g & 1;
        ok = mbar_wait(smem_addr(&sm->k_full[g % C::kStagesK]), (g / C::kStagesK) & 1, abort, to,
                       p.status, kSiteMmaK);
        if (ok && t == 0)
          ok = mbar_wait(smem_addr(&sm->q_full), qcnt & 1, abort, to, p.status, kSiteMmaQ);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        issue_qk<kD>(tmem + tmem_s(b, C::kBN), smem_addr(sm->q), smem_addr(sm->k[g % C::kStagesK]));
        tc_commit(smem_addr(&sm->s_full[b]));
        tc_commit(smem_addr(&sm->k_empty[g % C::kStagesK]));
        if (t == n - 1) tc_commit(smem_addr(&sm->q_empty));
      }
    }
    g0 += n;
    ++qcnt;
  }
  tc_commit(smem_addr(&sm->drain));
  drain_wait(smem_addr(&sm->drain), 0, to, p.status);
}

// The key blocks of one item for one softmax warp: TMEM lane quadrant
// `quad` (rows 32 quad ..), column half h of each key block (kSplit = 2) or
// all of it (kSplit = 1).  kHilo: the exact pass.  Returns false if a wait
// gave up; m_use and l hold the row's statistics (l: this half's) on return.
template <int kD, int kSplit, int kEmu, bool kHilo>
__device__ __forceinline__ bool softmax_item(SharedDb<kD, kSplit>* sm, const FwdParams& p,
                                             uint32_t lane_base, int quad, int h, int r, int lane,
                                             int n, int key_lim, int j_mask, int& g, float& m_use,
                                             float& l, volatile int* abort) {
  using C = Cfg<kD>;
  constexpr int kCols = C::kBN / kSplit;  // keys of a block this warp handles
  const uint64_t to = p.timeout_ns;
  const uint32_t o_t = lane_base + C::kTmemO + h * (kD / kSplit);
  const float sc = p.scale_log2;
  m_use = -INFINITY;
  l = 0.f;
  for (int j = 0; j < n; ++j, ++g) {
    const int b = g & 1;
    const uint32_t s_t = lane_base + tmem_s(b, C::kBN);
    bool ok = mbar_wait(smem_addr(&sm->s_full[b]), (g >> 1) & 1, abort, to, p.status,
                        kSiteSoftmaxS);
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
    uint32_t u[kCols];
#pragma unroll
    for (int c = 0; c < kCols; c += 32) tmem_ld32(s_t + h * kCols + c, &u[c]);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < kCols; c += 32) reg_dep32(&u[c]);
    if (j >= j_mask) {
      const int lim = key_lim - j * C::kBN - h * kCols;
#pragma unroll
      for (int c = 0; c < kCols; ++c)
        if (c > lim) u[c] = 0xff800000u;  // -inf
    }
    float mx8[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) mx8[t] = fmaxf(__uint_as_float(u[t]), __uint_as_float(u[8 + t]));
#pragma unroll
    for (int c = 16; c + 16 <= kCols; c += 16)
#pragma unroll
      for (int t = 0; t < 8; ++t)
        mx8[t] = fmax3(mx8[t], __uint_as_float(u[c + t]), __uint_as_float(u[c + 8 + t]));
    float cand = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                       fmaxf(mx8[6], mx8[7]));
    if constexpr (kSplit == 2) {
      // the partner warp (same rows, other half of the keys) posts its
      // partial maximum too; xmax[block parity][quad] completes when both
      // have.  A slot is written again two blocks later, after the partner
      // passed the next block's exchange and so read this one.
      sm->red_max[g & 1][h][r] = cand;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&sm->xmax[g & 1][quad]));
      ok = mbar_wait<true>(smem_addr(&sm->xmax[g & 1][quad]), (g >> 1) & 1, abort, to, p.status,
                           kSiteSoftmaxStats);
      if (!__all_sync(0xffffffffu, ok)) return false;
      cand = fmaxf(cand, sm->red_max[g & 1][h ^ 1][r]);
    }
    cand *= sc;
    if (j == 0) {
      m_use = cand;
    } else {
      const bool grow = cand > m_use + kRescaleLog2;
      if (__any_sync(0xffffffffu, grow)) {
        // O must hold PV(g-1) before it is rescaled
        ok = mbar_wait(smem_addr(&sm->pv_done), (g - 1) & 1, abort, to, p.status, kSiteSoftmaxS);
        if (!__all_sync(0xffffffffu, ok)) return false;
        tc_fence_after();
        const float alpha = grow ? ex2_approx(m_use - cand) : 1.0f;
#pragma unroll 1
        for (int c = 0; c < kD / kSplit; c += 32) {
          uint32_t wv[32];
          tmem_ld32(o_t + c, wv);
          tmem_wait_ld();
          reg_dep32(wv);
#pragma unroll
          for (int i = 0; i < 32; ++i) wv[i] = __float_as_uint(__uint_as_float(wv[i]) * alpha);
          tmem_st32(o_t + c, wv);
        }
        if (grow) {
          l *= alpha;
          m_use = cand;
        }
      }
    }
    const float neg_m = -m_use;
    float lp[4] = {0.f, 0.f, 0.f, 0.f};
    // this warp's keys go to P columns [h kCols / 2, (h + 1) kCols / 2)
    const uint32_t p_t = s_t + h * (kCols / 2);
    if constexpr (!kHilo) {
      const float2 sc2 = make_float2(sc, sc);
      const float2 nm2 = make_float2(neg_m, neg_m);
#pragma unroll
      for (int c = 0; c < kCols / 16; ++c) {
        uint32_t ph[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 s2 = make_float2(__uint_as_float(u[c * 16 + 2 * i]),
                                        __uint_as_float(u[c * 16 + 2 * i + 1]));
          const float2 x2 = __ffma2_rn(s2, sc2, nm2);
          float2 p2;
          if (i < kEmu) {
            p2 = exp2_poly2(x2);
          } else {
            p2.x = ex2_approx(x2.x);
            p2.y = ex2_approx(x2.y);
          }
          ph[i] = pack_half2(p2.x, p2.y);
          lp[i & 3] = add_half2_f32(ph[i], lp[i & 3]);
        }
        tmem_st8(p_t + c * 8, ph);
      }
    } else {
      // P = hi + lo: hi over P's columns, lo kBN / 2 columns further
#pragma unroll
      for (int c = 0; c < kCols / 16; ++c) {
        uint32_t ph[8], pl[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(u[c * 16 + 2 * i]), sc, neg_m));
          const float p1 = ex2_approx(fmaf(__uint_as_float(u[c * 16 + 2 * i + 1]), sc, neg_m));
          ph[i] = pack_half2(p0, p1);
          const float2 hh = __half22float2(*reinterpret_cast<const __half2*>(&ph[i]));
          pl[i] = pack_half2(p0 - hh.x, p1 - hh.y);
          lp[i & 3] += p0 + p1;
        }
        tmem_st8(p_t + c * 8, ph);
        tmem_st8(p_t + C::kBN / 2 + c * 8, pl);
      }
    }
    l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sm->p_full[b]));
  }
  return true;
}

template <int kD, int kSplit, int kEmu>
__device__ __forceinline__ void softmax(SharedDb<kD, kSplit>* sm, const FwdParams& p,
                                        uint32_t tmem, int warp, int lane, volatile int* abort) {
  using C = Cfg<kD>;
  const int quad = warp & 3;
  const int h = kSplit == 2 ? (warp >> 2) : 0;
  const int r = quad * 32 + lane;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  int g = 0;      // key blocks so far (all items)
  int acnt = 0;   // items so far
  bool ok = true;
  ItemWalk w;
  int item;
  while (ok && (item = walk(w, p, sm, abort, ok, kSiteSoftmaxRedo)) >= 0) {
    const Item it = decode_item(p, item);
    const int n = n_blocks<C::kBN>(p, it);
    const int i_row = it.qb0 * kBlockM + r;
    const int key_lim = p.causal ? min(i_row + p.off, p.Sk - 1) : p.Sk - 1;
    // the first block in which some lane of the warp has keys to mask
    const int j_mask = (__shfl_sync(0xffffffffu, key_lim, 0) + 1) / C::kBN;
    float m_use, l;
    ok = w.exact ? softmax_item<kD, kSplit, kEmu, true>(sm, p, lane_base, quad, h, r, lane, n,
                                                         key_lim, j_mask, g, m_use, l, abort)
                 : softmax_item<kD, kSplit, kEmu, false>(sm, p, lane_base, quad, h, r, lane, n,
                                                          key_lim, j_mask, g, m_use, l, abort);
    if (!ok) break;
    ok = acnt == 0 ||
         mbar_wait(smem_addr(&sm->stats_free), (acnt - 1) & 1, abort, p.timeout_ns, p.status,
                   kSiteSoftmaxStats);
    if (!__all_sync(0xffffffffu, ok)) {
      ok = false;
      break;
    }
    if (h == 0) sm->stat_m[r] = m_use;
    sm->stat_l[kSplit == 2 ? h : 0][r] = l;
    ++acnt;
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sm->stats_ready));
  }
}

// One item's O / l -> fp16 and LSE; `flag` as in the two-tile kernel.
template <int kD, int kSplit>
__device__ __forceinline__ bool epilogue_item(SharedDb<kD, kSplit>* sm, const FwdParams& p,
                                              uint32_t lane_base, int r, int lane, const Item& it,
                                              int& ecnt, bool& flag, volatile int* abort) {
  using C = Cfg<kD>;
  const uint64_t to = p.timeout_ns;
  const int a = ecnt++;
  bool ok = mbar_wait(smem_addr(&sm->o_done), a & 1, abort, to, p.status, kSiteEpilogueO) &&
            mbar_wait(smem_addr(&sm->stats_ready), a & 1, abort, to, p.status, kSiteEpilogueStats);
  if (!__all_sync(0xffffffffu, ok)) return false;
  tc_fence_after();
  const float m_use = sm->stat_m[r];
  float l = sm->stat_l[0][r];
  if constexpr (kSplit == 2) l += sm->stat_l[kSplit - 1][r];
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_addr(&sm->stats_free));
  const float inv_l = 1.0f / l;
  const int i_row = it.qb0 * kBlockM + r;
  const bool valid = i_row < p.S;
  const int row = (it.b * p.Hq + it.hq) * p.S + i_row;
  __half* orow = p.o + static_cast<size_t>(row) * kD;
  // full-sector stores when O is 32-byte aligned (rows are kD * 2 bytes apart)
  const bool sector_aligned = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
  float omax = 0.f;
#pragma unroll 4
  for (int c = 0; c < kD / 16; ++c) {
    uint32_t wv[16];
    tmem_ld16(lane_base + C::kTmemO + c * 16, wv);
    tmem_wait_ld();
    reg_dep16(wv);
    uint32_t pk[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float f0 = __uint_as_float(wv[2 * e]) * inv_l;
      const float f1 = __uint_as_float(wv[2 * e + 1]) * inv_l;
      omax = fmax3(omax, fabsf(f0), fabsf(f1));
      pk[e] = pack_half2(f0, f1);
    }
    if (valid) {
      if (sector_aligned) {
        st_global_v8(orow + c * 16, pk);
      } else {
        uint4* o16 = reinterpret_cast<uint4*>(orow + c * 16);
        o16[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        o16[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_addr(&sm->o_free));
  if (valid) p.lse[row] = (m_use + log2f(l)) * kLn2;
  flag |= valid && omax >= kRedoThreshold;
  return true;
}

template <int kD, int kSplit>
__device__ __forceinline__ void epilogue(SharedDb<kD, kSplit>* sm, const FwdParams& p, uint32_t tmem,
                                         int warp, int lane, volatile int* abort) {
  const int r = (warp - kEpilogueWarp0) * 32 + lane;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  int ecnt = 0;
  bool ok = true;
  int k = 0;
  for (int item; ok && (item = seq_item(p, k)) >= 0; ++k) {
    bool flag = false;
    ok = epilogue_item<kD, kSplit>(sm, p, lane_base, r, lane, decode_item(p, item), ecnt, flag,
                                   abort);
    if (ok && __any_sync(0xffffffffu, flag) && lane == 0)
      atomicOr(&sm->redo_bits[k >> 5], 1u << (k & 31));
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_addr(&sm->redo_ready));
  if (!ok) return;
  ok = mbar_wait(smem_addr(&sm->redo_ready), 0, abort, p.timeout_ns, p.status, kSiteEpilogueRedo);
  if (!__all_sync(0xffffffffu, ok)) return;
  for (int kk = 0; ok && kk < k; ++kk) {
    if (!((sm->redo_bits[kk >> 5] >> (kk & 31)) & 1u)) continue;
    bool flag = false;
    ok = epilogue_item<kD, kSplit>(sm, p, lane_base, r, lane, decode_item(p, seq_item(p, kk)),
                                   ecnt, flag, abort);
  }
}

// Items are one 128-row tile (the host sets item_tiles = 1); the K and V
// maps use boxes of Cfg<kD>::kBN rows.
template <int kD, int kSplit = 1, int kEmu = 0>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_db_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = Cfg<kD>;
  static_assert(kSplit == 1 || kSplit == 2, "one or two softmax warps per lane quadrant");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  SharedDb<kD, kSplit>* sm = reinterpret_cast<SharedDb<kD, kSplit>*>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (smem_addr(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(&p.status[0], kStatusSmemAlign);
    return;
  }
  if (seq_item(p, 0) < 0) return;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&sm->q_full), 1);
    mbar_init(smem_addr(&sm->q_empty), 1);
    for (int s = 0; s < C::kStagesK; ++s) {
      mbar_init(smem_addr(&sm->k_full[s]), 1);
      mbar_init(smem_addr(&sm->k_empty[s]), 1);
    }
    for (int s = 0; s < C::kStagesV; ++s) {
      mbar_init(smem_addr(&sm->v_full[s]), 1);
      mbar_init(smem_addr(&sm->v_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_addr(&sm->s_full[b]), 1);
      mbar_init(smem_addr(&sm->p_full[b]), 4 * kSplit);
    }
    for (int x = 0; x < kSplit; ++x)
      for (int q = 0; q < 4; ++q) mbar_init(smem_addr(&sm->xmax[x][q]), 2);
    mbar_init(smem_addr(&sm->pv_done), 1);
    mbar_init(smem_addr(&sm->o_done), 1);
    mbar_init(smem_addr(&sm->o_free), 4);
    mbar_init(smem_addr(&sm->stats_ready), 4 * kSplit);
    mbar_init(smem_addr(&sm->stats_free), 4);
    mbar_init(smem_addr(&sm->redo_ready), 4);
    mbar_init(smem_addr(&sm->drain), 1);
    for (int i = 0; i < kRedoWords; ++i) sm->redo_bits[i] = 0;
    sm->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(&sm->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;

  if (warp >= kProducerWarp) {
    regs_dec<kRegsOther>();
    if (warp == kProducerWarp || warp == kProducerVWarp) {
      if (lane == 0)
        producer<kD>(sm, p, &tm_q, warp == kProducerVWarp ? &tm_v : &tm_k, warp == kProducerVWarp,
                     abort);
    } else if (warp == kMmaWarp) {
      mma<kD>(sm, p, tmem, abort);
    }
    __syncwarp();
  } else if (warp >= kEpilogueWarp0) {
    regs_dec<kRegsEpilogue>();
    epilogue<kD, kSplit>(sm, p, tmem, warp, lane, abort);
  } else {
    regs_inc<kRegsSoftmax>();
    if (warp < 4 * kSplit) softmax<kD, kSplit, kEmu>(sm, p, tmem, warp, lane, abort);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace db
}  // namespace attn_b200
