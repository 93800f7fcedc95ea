// attn_fwd_pair_sm100.cuh -- the fused attention forward pass on CTA pairs.
//
// Same computation as attn_fwd_sm100.cuh (O = softmax(Q K^T / sqrt(D)
// [+ causal mask]) V and the row log-sum-exp; the FlashAttention forward that
// the PipeThreader pages evaluate, papers.lqhl.me "PipeThreader-OSDI25",
// section 实验与结果, paper Sec. 6.2 / Fig. 12), with its load / mma /
// softmax tasks mapped onto two SMs at once:
//
// A 2-CTA cluster takes one work item, 256 query rows of one (batch, query
// head); CTA r of the pair owns rows [128 r, 128 r + 128) of the item.  The
// even CTA issues every MMA as tcgen05.mma.cta_group::2 with M = 256: each
// CTA holds its own 128 rows of Q (and of S, P, O in its own TMEM) but only
// half of each key block's operand -- 64 of the 128 keys of K_j, and 64 of
// the 128 head-dimension columns of V_j -- so every K/V byte crosses from L2
// into shared memory once per pair, not once per SM.
//
// Each CTA's TMEM (512 columns) holds three S buffers and the O accumulator:
//   S[0] [0,128)  S[1] [128,256)  S[2] [256,384)   (key block g of the
//   pair's block sequence goes to S[g % 3]; P_g, fp16, is written over its
//   first 64 columns)
//   O    [384,512)
// The MMA warp issues S(g+3) right after PV(g), so the S of the next two
// blocks is always ready when a softmax warpgroup turns to it.
//
// The softmax runs in two warpgroups that take alternate key blocks (WG0
// the even blocks g, WG1 the odd ones).  The running row max is handed from
// block to block through shared memory (m_ready / m_pub); each warpgroup
// keeps its own partial row sum l relative to the last max it used, and the
// epilogue combines the two.  While one warpgroup computes the max of its
// block, the other's exponentials keep the MUFU unit busy.
//
// Warp roles (512 threads per CTA):
//   warps 0-3   softmax warpgroup 0 (one query row per thread = TMEM lane)
//   warps 4-7   softmax warpgroup 1
//   warps 8-11  epilogue: O / l -> fp16, LSE
//   warp 12     TMA producer of Q (per item) and this CTA's half of K_j
//   warp 13     S = Q K^T issuer (even CTA, one thread); TMEM allocation (both)
//   warp 14     TMA producer of this CTA's half of V_j
//   warp 15     O += P V issuer (even CTA, one thread)
// Two issuing threads keep the tensor core fed: a single thread waiting on
// K, V and P and issuing 16 MMAs and their commits per block measured about
// 2.6x the 1024 cycles the MMAs themselves take.  S(g + 3) overwrites the S
// buffer of block g, so the S issuer waits for PV(g) to complete (s_free).
//
// Signals between the two CTAs: the odd CTA's loads complete their bytes
// on the even CTA's "full" barriers; the even CTA's commits arrive on the
// barrier of the same offset in both CTAs (multicast); the odd CTA's
// softmax and epilogue warps arrive on the even CTA's p_full / o_free.
#pragma once

#include <cuda_fp16.h>

#include "attn_fwd_sm100.cuh"
#include "ptx_sm100.cuh"

namespace attn_b200 {
namespace pair {

constexpr int kStagesK = 4;                            // K ring (this CTA's 64 keys of a block)
constexpr int kStagesV = 4;                            // V ring (this CTA's 64 columns of a block)
constexpr uint32_t kHalfBytes = kTileBytes / 2;        // 16 KiB
constexpr uint32_t kKPanelBytes = kHalfBytes / 2;      // 64 keys x 64 columns
constexpr int kThreads = 512;
constexpr int kEpilogueWarp0 = 8;
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kProducerVWarp = 14;
constexpr int kMmaPvWarp = 15;
constexpr int kRegsSoftmax = 184;
constexpr int kRegsEpilogue = 80;
constexpr int kRegsOther = 64;
static_assert(256 * kRegsSoftmax + 128 * kRegsEpilogue + 128 * kRegsOther <= 65536,
              "register split exceeds the register file");
constexpr uint16_t kBothCtas = 0x3;
constexpr int kSBufs = 3;
// Of every 8 column pairs, how many take 2^x from the FMA-pipe polynomial
// (exp2_poly2) instead of the MUFU unit.
constexpr int kPairEmuPairs = 0;

__device__ __forceinline__ uint32_t tmem_s(int b) { return static_cast<uint32_t>(b) * 128u; }
constexpr uint32_t kTmemO = 384u;

enum PairWaitSite : uint32_t {
  kSitePairProducerQ = 0x1101,
  kSitePairProducerK = 0x1102,
  kSitePairProducerV = 0x1103,
  kSitePairMmaQ = 0x1201,
  kSitePairMmaK = 0x1202,
  kSitePairMmaV = 0x1203,
  kSitePairMmaP = 0x1204,
  kSitePairMmaO = 0x1205,
  kSitePairMmaS = 0x1206,
  kSitePairSoftmaxS = 0x1301,
  kSitePairSoftmaxStats = 0x1302,
  kSitePairSoftmaxPV = 0x1303,
  kSitePairEpilogueO = 0x1401,
  kSitePairEpilogueStats = 0x1402,
  kSitePairDrain = 0x1501,
};

// Identical layout in both CTAs: the pair MMAs address the odd CTA's
// operands and barriers at the even CTA's offsets.
struct SharedPair {
  uint8_t q[2][kTileBytes];         // [item parity] this CTA's 128 rows, two 64-column panels
  uint8_t k[kStagesK][kHalfBytes];  // 64 keys x 128 columns, two panels of 8 KiB
  uint8_t v[kStagesV][kHalfBytes];  // 128 keys x 64 columns (one panel)
  float stat_m[2][2][kBlockM];      // [item parity][softmax warpgroup][row]
  float stat_l[2][2][kBlockM];
  float m_pub[2][kBlockM];          // [block parity][row]: row max after that block
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kStagesK], k_empty[kStagesK], v_full[kStagesV], v_empty[kStagesV];
  uint64_t s_full[kSBufs], p_full[kSBufs], s_free[kSBufs];  // [S buffer]
  uint64_t pv_done[2], m_ready[2];             // [block parity]
  uint64_t o_done, o_free;
  uint64_t stats_ready[2], stats_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int item_flag[2];
  int item_warps[2];
};
static_assert(sizeof(SharedPair) <= 232448, "shared memory exceeds the 227 KiB per-block limit");

// Work item of a pair: the same ids as the single-CTA pass (kv-head major,
// 256-row blocks from last to first), so the redo list is shared.
struct PairItem {
  int b, hq, g, qb2;
  bool half1;    // the odd CTA's 128 rows exist (S / 128 may be odd)
  int n_blocks;  // key blocks the pair computes
};

__device__ __forceinline__ PairItem decode_pair_item(const FwdParams& p, int id) {
  const int per_kv = p.group * p.n_qb2;
  const int kvh = id / per_kv;
  const int rem = id - kvh * per_kv;
  PairItem it;
  it.b = kvh / p.Hkv;
  it.g = kvh - it.b * p.Hkv;
  it.qb2 = p.n_qb2 - 1 - rem / p.group;
  it.hq = it.g * p.group + rem % p.group;
  it.half1 = 2 * it.qb2 + 1 < p.n_qb;
  if (p.causal)
    it.n_blocks = it.half1 ? 2 * it.qb2 + 2 : 2 * it.qb2 + 1;
  else
    it.n_blocks = p.n_qb;
  return it;
}

// S(g) = Q K_j^T over the pair: 8 MMAs of K = 16.  Q panels are 16 KiB
// apart, this CTA's K panels (64 rows) 8 KiB apart.
template <int kk>
__device__ __forceinline__ void qk_step_pair(uint32_t d_tmem, uint64_t qd, uint64_t kd,
                                             uint32_t idesc) {
  constexpr uint32_t a_off = ((kk >> 2) * kPanelBytes + (kk & 3) * 32) >> 4;
  constexpr uint32_t b_off = ((kk >> 2) * kKPanelBytes + (kk & 3) * 32) >> 4;
  mma_pair_ss_off<a_off, b_off>(d_tmem, qd, kd, idesc, kk > 0 ? 1u : 0u);
}
__device__ __forceinline__ void issue_qk_pair(uint32_t d_tmem, uint32_t q_s, uint32_t k_s) {
  const uint32_t idesc = idesc_f16_f32(2 * kBlockM, kBlockN, false, false);
  const uint64_t qd = smem_desc_sw128(q_s, 16, 1024);
  const uint64_t kd = smem_desc_sw128(k_s, 16, 1024);
  qk_step_pair<0>(d_tmem, qd, kd, idesc);
  qk_step_pair<1>(d_tmem, qd, kd, idesc);
  qk_step_pair<2>(d_tmem, qd, kd, idesc);
  qk_step_pair<3>(d_tmem, qd, kd, idesc);
  qk_step_pair<4>(d_tmem, qd, kd, idesc);
  qk_step_pair<5>(d_tmem, qd, kd, idesc);
  qk_step_pair<6>(d_tmem, qd, kd, idesc);
  qk_step_pair<7>(d_tmem, qd, kd, idesc);
}

// O (+)= P V over the pair: A = P from each CTA's TMEM (8 columns = 16 keys
// per MMA), B = V, MN-major; each CTA holds one 64-column panel of V_j.
template <int kk>
__device__ __forceinline__ void pv_step_pair(uint32_t o_tmem, uint32_t p_tmem, uint64_t vd,
                                             uint32_t idesc, uint32_t acc) {
  constexpr uint32_t a_off = kk * 8;
  constexpr uint32_t b_off = (kk * 2048) / 16;
  mma_pair_ts_off<a_off, b_off>(o_tmem, p_tmem, vd, idesc, (acc || kk > 0) ? 1u : 0u);
}
__device__ __forceinline__ void issue_pv_pair(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_s,
                                              bool accumulate) {
  const uint32_t idesc = idesc_f16_f32(2 * kBlockM, kHeadDim, false, true);
  const uint64_t vd = smem_desc_sw128(v_s, kPanelBytes, 1024);
  const uint32_t acc = accumulate ? 1u : 0u;
  pv_step_pair<0>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step_pair<1>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step_pair<2>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step_pair<3>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step_pair<4>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step_pair<5>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step_pair<6>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step_pair<7>(o_tmem, p_tmem, vd, idesc, acc);
}

__device__ __forceinline__ void pair_sleep_ns(uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (global_timer_ns() - t0 < ns) __nanosleep(1000);
}

// Cursor over the key blocks of a pair's items, in issue order: item k,
// block j of n, global block index g.
struct BlockCursor {
  int k, j, n, g, item;
  PairItem it;
};

__device__ __forceinline__ bool cursor_start(BlockCursor& c, const FwdParams& p, int pair_id,
                                             int n_pairs) {
  c.k = 0;
  c.j = 0;
  c.g = 0;
  c.item = pair_id;
  if (c.item >= p.n_items) return false;
  c.it = decode_pair_item(p, c.item);
  c.n = c.it.n_blocks;
  return true;
}

__device__ __forceinline__ bool cursor_next(BlockCursor& c, const FwdParams& p, int n_pairs) {
  ++c.g;
  if (++c.j < c.n) return true;
  c.j = 0;
  ++c.k;
  c.item += n_pairs;
  if (c.item >= p.n_items) return false;
  c.it = decode_pair_item(p, c.item);
  c.n = c.it.n_blocks;
  return true;
}

// The fused pass on CTA pairs (records items for the redo pass exactly as
// attn_fwd_kernel<0> does).  Launched with 2-CTA clusters; the grid is an
// even number of CTAs, pair c taking items c, c + pairs, ...
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  SharedPair* sm = reinterpret_cast<SharedPair*>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t to = p.timeout_ns;
  // both CTAs of a pair take the same branch here (same kernel, same layout)
  if (cluster_nctarank() != 2 || (smem_addr(smem_raw) & 1023u)) {
    if (threadIdx.x == 0) atomicOr(&g_attn_status[0], kStatusSmemAlign);
    return;
  }
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair_id = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_addr(&sm->q_full[b]), 1);
      mbar_init(smem_addr(&sm->q_empty[b]), 1);
      mbar_init(smem_addr(&sm->pv_done[b]), 1);
      mbar_init(smem_addr(&sm->m_ready[b]), kBlockM);
      mbar_init(smem_addr(&sm->stats_ready[b]), 2 * kBlockM);
      mbar_init(smem_addr(&sm->stats_free[b]), kBlockM);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(smem_addr(&sm->s_full[b]), 1);
      // P of the block in S[b]: 4 softmax warps x 2 CTAs.  Indexed by buffer,
      // not by warpgroup: a warpgroup may finish two of its blocks before
      // the MMA thread takes the first (at an item boundary), but block
      // g + 3 (same buffer) waits for PV(g), so this barrier never runs two
      // phases ahead of its waiter.
      mbar_init(smem_addr(&sm->p_full[b]), 8);
      mbar_init(smem_addr(&sm->s_free[b]), 1);
    }
    mbar_init(smem_addr(&sm->o_done), 1);
    mbar_init(smem_addr(&sm->o_free), 8);         // 4 epilogue warps x 2 CTAs
    for (int st = 0; st < kStagesK; ++st) {
      mbar_init(smem_addr(&sm->k_full[st]), 1);
      mbar_init(smem_addr(&sm->k_empty[st]), 1);
    }
    for (int st = 0; st < kStagesV; ++st) {
      mbar_init(smem_addr(&sm->v_full[st]), 1);
      mbar_init(smem_addr(&sm->v_empty[st]), 1);
    }
    mbar_init(smem_addr(&sm->drain), 2);  // one commit per issuing thread
    sm->abort = 0;
    sm->item_flag[0] = sm->item_flag[1] = 0;
    sm->item_warps[0] = sm->item_warps[1] = 0;
    fence_mbar_init();
  }
  // the other CTA's barriers exist before anything signals them
  cluster_sync();
  if (pair_id >= p.n_items) return;  // same for both CTAs of the pair

  if (warp == kMmaWarp) {
    tmem_alloc_pair(smem_addr(&sm->tmem_base), kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  // both CTAs' TMEM is allocated before the first pair MMA
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;
  const uint32_t peer_abort = smem_map_rank(smem_addr(&sm->abort), rank ^ 1u);

  if (warp >= kProducerWarp) {
    regs_dec<kRegsOther>();
    if ((warp == kProducerWarp || warp == kProducerVWarp) && lane == 0) {
      // ------------------------------------------------------------ producers
      const bool is_v = warp == kProducerVWarp;
      const uint64_t keep = l2_policy_evict_last();
      const uint64_t once = l2_policy_evict_first();
      const int depth = is_v ? kStagesV : kStagesK;
      int gb = 0;  // key blocks loaded so far (all items)
      int k = 0;
      bool ok = true;
      for (int item; ok && (item = pair_id + k * n_pairs) < p.n_items; ++k) {
        const PairItem it = decode_pair_item(p, item);
        if (!is_v) {
          const int qb = k & 1;
          if (k >= 2 && !mbar_wait_pair(smem_addr(&sm->q_empty[qb]), ((k >> 1) - 1) & 1, abort,
                                        peer_abort, to, kSitePairProducerQ)) {
            ok = false;
            break;
          }
          const uint32_t qf = smem_addr(&sm->q_full[qb]);
          if (leader) mbar_arrive_expect_tx(qf, 2 * kTileBytes);
          const uint32_t qf0 = smem_map_rank(qf, 0);
          const int q_row = (it.b * p.Hq + it.hq) * p.S + it.qb2 * kItemRows + rank * kBlockM;
          const uint32_t q_s = smem_addr(sm->q[qb]);
          tma_load_2d_pair(q_s, &tm_q, qf0, 0, q_row, once);
          tma_load_2d_pair(q_s + kPanelBytes, &tm_q, qf0, 64, q_row, once);
        }
        const int kv_row = (it.b * p.Hkv + it.g) * p.S;
        for (int j = 0; j < it.n_blocks; ++j, ++gb) {
          const int st = gb % depth;
          const uint32_t empty = smem_addr(is_v ? &sm->v_empty[st] : &sm->k_empty[st]);
          if (gb >= depth &&
              !mbar_wait_pair(empty, ((gb / depth) & 1) ^ 1, abort, peer_abort, to,
                              is_v ? kSitePairProducerV : kSitePairProducerK)) {
            ok = false;
            break;
          }
          const uint32_t full = smem_addr(is_v ? &sm->v_full[st] : &sm->k_full[st]);
          if (leader) mbar_arrive_expect_tx(full, 2 * kHalfBytes);
          const uint32_t full0 = smem_map_rank(full, 0);
          if (is_v) {
            // all 128 keys, head-dimension columns [64 rank, 64 rank + 64)
            tma_load_2d_pair(smem_addr(sm->v[st]), &tm_v, full0, 64 * rank, kv_row + j * kBlockN,
                             keep);
          } else {
            // keys [64 rank, 64 rank + 64) of the block, both column panels
            const int key_row = kv_row + j * kBlockN + 64 * rank;
            tma_load_2d_pair(smem_addr(sm->k[st]), &tm_k, full0, 0, key_row, keep);
            tma_load_2d_pair(smem_addr(sm->k[st]) + kKPanelBytes, &tm_k, full0, 64, key_row, keep);
          }
        }
      }
      if (*abort) {
        // copies still in flight land within microseconds; the even CTA's
        // full barriers count both CTAs' bytes, so it also waits on those
        if (leader) {
          if (!is_v && k > 0) drain_wait(smem_addr(&sm->q_full[(k - 1) & 1]), ((k - 1) >> 1) & 1, to);
          for (int t = (gb > depth ? gb - depth : 0); t < gb; ++t)
            drain_wait(smem_addr(is_v ? &sm->v_full[t % depth] : &sm->k_full[t % depth]),
                       (t / depth) & 1, to);
        } else {
          pair_sleep_ns(200000);
        }
      }
    } else if (warp == kMmaWarp && lane == 0 && leader) {
      // ---------------------------------------------------------- S issuer
      BlockCursor cs;
      bool more = cursor_start(cs, p, pair_id, n_pairs);
      while (more) {
        const int qb = cs.k & 1;
        const int sb = cs.g % kSBufs;
        const int st_k = cs.g % kStagesK;
        // Q of a new item; the S buffer (PV of block g - 3 has read its P); K_j
        const bool ok =
            (cs.j != 0 || mbar_wait_pair(smem_addr(&sm->q_full[qb]), (cs.k >> 1) & 1, abort,
                                         peer_abort, to, kSitePairMmaQ)) &&
            (cs.g < kSBufs || mbar_wait_pair(smem_addr(&sm->s_free[sb]), ((cs.g / kSBufs) - 1) & 1,
                                             abort, peer_abort, to, kSitePairMmaS)) &&
            mbar_wait_pair(smem_addr(&sm->k_full[st_k]), (cs.g / kStagesK) & 1, abort, peer_abort,
                           to, kSitePairMmaK);
        if (!ok) break;
        tc_fence_after();
        issue_qk_pair(tmem + tmem_s(sb), smem_addr(sm->q[qb]), smem_addr(sm->k[st_k]));
        tc_commit_pair(smem_addr(&sm->s_full[sb]), kBothCtas);
        tc_commit_pair(smem_addr(&sm->k_empty[st_k]), kBothCtas);
        if (cs.j == cs.n - 1) tc_commit_pair(smem_addr(&sm->q_empty[qb]), kBothCtas);
        more = cursor_next(cs, p, n_pairs);
      }
      // every MMA issued must complete before either CTA releases its TMEM
      tc_commit_pair(smem_addr(&sm->drain), kBothCtas);
    } else if (warp == kMmaPvWarp && lane == 0 && leader) {
      // --------------------------------------------------------- PV issuer
      BlockCursor cp;
      bool more = cursor_start(cp, p, pair_id, n_pairs);
      while (more) {
        const int st_v = cp.g % kStagesV;
        const int sb = cp.g % kSBufs;
        // the epilogue has read O of the previous item; V_j; P of this block
        const bool ok =
            (cp.j != 0 || cp.k == 0 ||
             mbar_wait_pair(smem_addr(&sm->o_free), (cp.k - 1) & 1, abort, peer_abort, to,
                            kSitePairMmaO)) &&
            mbar_wait_pair(smem_addr(&sm->v_full[st_v]), (cp.g / kStagesV) & 1, abort, peer_abort,
                           to, kSitePairMmaV) &&
            mbar_wait_pair(smem_addr(&sm->p_full[sb]), (cp.g / kSBufs) & 1, abort, peer_abort, to,
                           kSitePairMmaP);
        if (!ok) break;
        tc_fence_after();
        issue_pv_pair(tmem + kTmemO, tmem + tmem_s(sb), smem_addr(sm->v[st_v]), cp.j > 0);
        tc_commit_pair(smem_addr(&sm->pv_done[cp.g & 1]), kBothCtas);
        tc_commit_pair(smem_addr(&sm->v_empty[st_v]), kBothCtas);
        tc_commit_pair(smem_addr(&sm->s_free[sb]), 0x1);
        if (cp.j == cp.n - 1) tc_commit_pair(smem_addr(&sm->o_done), kBothCtas);
        more = cursor_next(cp, p, n_pairs);
      }
      tc_commit_pair(smem_addr(&sm->drain), kBothCtas);
    }
    __syncwarp();
    if (warp == kMmaWarp) {
      // both CTAs: the drain commit has landed (or the wait gave up)
      if (lane == 0) drain_wait(smem_addr(&sm->drain), 0, to);
      __syncwarp();
    }
  } else if (warp >= kEpilogueWarp0) {
    // -------------------------------------------------------------- epilogue
    regs_dec<kRegsEpilogue>();
    const int r = (warp - kEpilogueWarp0) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t o_free0 = smem_map_rank(smem_addr(&sm->o_free), 0);
    const uint32_t item_flag0[2] = {smem_map_rank(smem_addr(&sm->item_flag[0]), 0),
                                    smem_map_rank(smem_addr(&sm->item_flag[1]), 0)};
    const uint32_t item_warps0[2] = {smem_map_rank(smem_addr(&sm->item_warps[0]), 0),
                                     smem_map_rank(smem_addr(&sm->item_warps[1]), 0)};
    int k = 0;
    for (int item; (item = pair_id + k * n_pairs) < p.n_items; ++k) {
      const PairItem it = decode_pair_item(p, item);
      const int ib = k & 1;
      bool ok = mbar_wait_pair(smem_addr(&sm->o_done), k & 1, abort, peer_abort, to,
                               kSitePairEpilogueO) &&
                mbar_wait_pair(smem_addr(&sm->stats_ready[ib]), (k >> 1) & 1, abort, peer_abort, to,
                               kSitePairEpilogueStats);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      // the two warpgroups' partial sums, each relative to the last max it used
      const float m0 = sm->stat_m[ib][0][r], l0 = sm->stat_l[ib][0][r];
      const float m1 = sm->stat_m[ib][1][r], l1 = sm->stat_l[ib][1][r];
      mbar_arrive(smem_addr(&sm->stats_free[ib]));
      bool flag = false;
      if (rank == 0 || it.half1) {
        const float m_use = fmaxf(m0, m1);
        const float l = (l0 > 0.f ? l0 * ex2_approx(m0 - m_use) : 0.f) +
                        (l1 > 0.f ? l1 * ex2_approx(m1 - m_use) : 0.f);
        const float inv_l = 1.0f / l;
        const int row = (it.b * p.Hq + it.hq) * p.S + it.qb2 * kItemRows + rank * kBlockM + r;
        uint4* orow = reinterpret_cast<uint4*>(p.o + static_cast<size_t>(row) * kHeadDim);
        float omax = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w[16];
          tmem_ld16(lane_base + kTmemO + c * 16, w);
          tmem_wait_ld();
          reg_dep16(w);
#pragma unroll
          for (int v4 = 0; v4 < 2; ++v4) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              f[e] = __uint_as_float(w[v4 * 8 + e]) * inv_l;
              omax = fmaxf(omax, fabsf(f[e]));
            }
            uint4 pk;
            pk.x = pack_half2(f[0], f[1]);
            pk.y = pack_half2(f[2], f[3]);
            pk.z = pack_half2(f[4], f[5]);
            pk.w = pack_half2(f[6], f[7]);
            orow[c * 2 + v4] = pk;
          }
        }
        p.lse[row] = (m_use + log2f(l)) * kLn2;
        flag = omax >= kRedoThreshold;
      }
      // One redo-list entry per item if any row of either CTA needs it: the
      // 8 epilogue warps of the pair count in on the even CTA's words, and
      // the last one appends.  This comes before the o_free arrive, so no
      // warp reaches item k + 2 (whose first PV waits for o_free of item
      // k + 1) before all 8 have left the parity slot of item k.
      const bool any = __any_sync(0xffffffffu, flag);
      if (lane == 0) {
        if (any) atom_or_cluster(item_flag0[ib], 1u);
        if (atom_add_cluster(item_warps0[ib], 1u) == 7u) {
          atom_exch_cluster(item_warps0[ib], 0u);
          if (atom_exch_cluster(item_flag0[ib], 0u)) {
            const unsigned int slot = atomicAdd(p.redo, 1u);
            if (slot < p.redo_capacity)
              p.redo[kRedoHeaderWords + slot] = static_cast<unsigned int>(item);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(o_free0);
    }
  } else {
    // -------------------------------------------------------------- softmax
    regs_inc<kRegsSoftmax>();
    const int wg = warp >> 2;  // this warpgroup takes the blocks g with g % 2 == wg
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t o_t = lane_base + kTmemO;
    const uint32_t p_full0[kSBufs] = {smem_map_rank(smem_addr(&sm->p_full[0]), 0),
                                      smem_map_rank(smem_addr(&sm->p_full[1]), 0),
                                      smem_map_rank(smem_addr(&sm->p_full[2]), 0)};
    const float sc = p.scale_log2;
    const float2 sc2 = make_float2(sc, sc);
    int g = 0;  // global block index (all items of the pair)
    int k = 0;
    bool ok = true;
    for (int item; ok && (item = pair_id + k * n_pairs) < p.n_items; ++k) {
      const PairItem it = decode_pair_item(p, item);
      const bool active = rank == 0 || it.half1;
      // this CTA's diagonal key block (causal): rows start at 128 (2 qb2 + rank)
      const int diag = p.causal ? 2 * it.qb2 + static_cast<int>(rank) : (1 << 30);
      float m_ref = -INFINITY;  // the max this warpgroup's l is relative to
      float l = 0.f;
      for (int j = 0; j < it.n_blocks; ++j, ++g) {
        if ((g & 1) != wg) continue;
        ok = mbar_wait_pair(smem_addr(&sm->s_full[g % kSBufs]), (g / kSBufs) & 1, abort, peer_abort,
                            to, kSitePairSoftmaxS);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t s_t = lane_base + tmem_s(g % kSBufs);
        uint32_t u[128];
        float cand = -INFINITY;
        if (active) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld32(s_t + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c * 32]));
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) reg_dep32(&u[c * 32]);
          if (j >= diag) {
            // the diagonal block keeps keys <= row; blocks past it keep none
            const int lim = j == diag ? r : -1;
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c > lim) u[c] = 0xff800000u;  // -inf
          }
          // row max: 8 independent chains (chain t takes columns t, t + 8,
          // ..., t + 120) of 3-input max, then a tree
          float mx8[8];
#pragma unroll
          for (int t = 0; t < 8; ++t)
            mx8[t] = fmax3(__uint_as_float(u[t]), __uint_as_float(u[8 + t]),
                           __uint_as_float(u[16 + t]));
#pragma unroll
          for (int c = 24; c < 120; c += 16)
#pragma unroll
            for (int t = 0; t < 8; ++t)
              mx8[t] = fmax3(mx8[t], __uint_as_float(u[c + t]), __uint_as_float(u[c + 8 + t]));
#pragma unroll
          for (int t = 0; t < 8; ++t) mx8[t] = fmaxf(mx8[t], __uint_as_float(u[120 + t]));
          cand = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                       fmaxf(mx8[6], mx8[7])) * sc;
        }
        // the row max after block g - 1 (the other warpgroup's block; for
        // the first block of an item it belongs to the previous item and
        // is not used, but every phase is waited on)
        float m_prev = -INFINITY;
        if (g > 0) {
          ok = mbar_wait_pair(smem_addr(&sm->m_ready[(g - 1) & 1]), ((g - 1) >> 1) & 1, abort,
                              peer_abort, to, kSitePairSoftmaxS);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          if (j > 0) m_prev = sm->m_pub[(g - 1) & 1][r];
        }
        // lazy rescaling: the reference max moves only when the row max
        // grows by more than 2^kRescaleLog2 (the first block sets it)
        const bool grow = j == 0 || cand > m_prev + kRescaleLog2;
        const float m_use = grow ? cand : m_prev;
        sm->m_pub[g & 1][r] = m_use;
        mbar_arrive(smem_addr(&sm->m_ready[g & 1]));
        if (active) {
          if (j > 0 && __any_sync(0xffffffffu, grow)) {
            // O must hold every PV of this item so far: PV(g - 1) may still
            // be in flight
            ok = mbar_wait_pair(smem_addr(&sm->pv_done[(g - 1) & 1]), ((g - 1) >> 1) & 1, abort,
                                peer_abort, to, kSitePairSoftmaxPV);
            if (!__all_sync(0xffffffffu, ok)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float alpha = grow ? ex2_approx(m_prev - cand) : 1.0f;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t w[32];
              tmem_ld32(o_t + c * 32, w);
              tmem_wait_ld();
              reg_dep32(w);
#pragma unroll
              for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * alpha);
              tmem_st32(o_t + c * 32, w);
            }
          }
          // this warpgroup's partial sum follows the reference max
          if (m_use != m_ref) {
            l = (l > 0.f) ? l * ex2_approx(m_ref - m_use) : 0.f;
            m_ref = m_use;
          }
          // P rounded to fp16 over the first 64 columns of S; l sums exactly
          // the rounded values
          const float2 nm2 = make_float2(-m_use, -m_use);
          float lp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t ph[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 s2 = make_float2(__uint_as_float(u[c * 16 + 2 * i]),
                                            __uint_as_float(u[c * 16 + 2 * i + 1]));
              const float2 x2 = __ffma2_rn(s2, sc2, nm2);
              if (i < kPairEmuPairs) {
                const float2 e2 = exp2_poly2(x2);
                ph[i] = pack_half2(e2.x, e2.y);
              } else {
                ph[i] = pack_half2(ex2_approx(x2.x), ex2_approx(x2.y));
              }
              lp[i & 3] = add_half2_f32(ph[i], lp[i & 3]);
            }
            tmem_st8(s_t + c * 8, ph);
          }
          l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(p_full0[g % kSBufs]);
      }
      if (!ok) break;
      // the epilogue has read the statistics of item k - 2
      ok = k < 2 || mbar_wait_pair(smem_addr(&sm->stats_free[k & 1]), ((k >> 1) - 1) & 1, abort,
                                   peer_abort, to, kSitePairSoftmaxStats);
      if (!__all_sync(0xffffffffu, ok)) break;
      sm->stat_m[k & 1][wg][r] = m_ref;
      sm->stat_l[k & 1][wg][r] = l;
      mbar_arrive(smem_addr(&sm->stats_ready[k & 1]));
    }
  }

  tc_fence_before();
  // every role of both CTAs is done, and the MMAs have drained
  cluster_sync();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace pair
}  // namespace attn_b200
