// attn_fwd_sm100.cuh -- fused attention forward for sm_100a (B200).
//
// One pass computes O = softmax(Q K^T / sqrt(D) [+ causal mask]) V and the
// row log-sum-exp for grouped-query heads, without writing the score matrix
// to memory: the FlashAttention forward that the PipeThreader pages evaluate
// (papers.lqhl.me "PipeThreader-OSDI25", section 实验与结果, paper Sec. 6.2 /
// Fig. 12).  The pages build it from load, mma and softmax tasks on TMA,
// TensorCore and CUDA-core units overlapped inside an SM (section 核心方法,
// "sTask / sEU"; dependences kept by barrier-sTasks, "sTask-graph ->
// sProgram").  Here that split is fixed by hand for B200:
//
// Persistent kernel, one CTA per SM.  A work item is 256 query rows of one
// (batch, query head): two 128-row tiles, A and B, that share every K/V tile
// and take turns on the tensor core, so one tile's softmax runs while the
// other tile's MMAs do.  Items are ordered kv-head by kv-head (the query
// heads of a group and all their row blocks close together, so K/V stay in
// L2) and handed out round-robin to the CTAs.
//
// Warp roles (512 threads, registers re-split with setmaxnreg):
//   warps 0-3   softmax of tile A   (one query row per thread = TMEM lane)
//   warps 4-7   softmax of tile B
//   warps 8-11  epilogue: O / l -> fp16, LSE, for both tiles
//   warp 12     TMA producer of Q_A, Q_B (per item) and K_j (a ring)
//   warp 13     MMA issuer (one thread): S_X = Q_X K_j^T, O_X += P_X V_j
//   warp 14     TMA producer of V_j (its own ring)
//   warp 15     idle
//
// K_j and V_j have separate rings and are released separately, each as soon
// as the last MMA reading it completes (K after both S(j), V after both
// PV(j)); a K load is then never held back by the later V release.
//
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384),
// O_B [384,512).  P_X (fp16) is written over the first 64 columns of S_X
// (and, in the redo pass, its low half over the next 64).
//
// Per tile X and key block j the MMA thread issues PV_X(j-1) and then
// S_X(j); tcgen05 operations complete in order, so when S_X(j) signals
// s_full, O_X already holds P_X(j-1) V_{j-1} and the softmax may rescale it.
//
// Numerics: P is rounded to fp16 and the row sum l accumulates exactly those
// rounded values, so O / l uses one consistent set of weights.  Lazy
// rescaling keeps a reference max per row and rescales O only when the row
// max grows by more than 2^kRescaleLog2 (exact: O and l share the
// reference).  The output is rounded to fp16, whose half-ulp for |O| >= 4 is
// 1.95e-3, so rows there need more than fp16 weights can give.  The fast
// pass (mode 0) therefore records each item with a row max|O| >=
// kRedoThreshold, and a second launch (mode 1) recomputes just those items
// with P split as hi + lo fp16 (about 22-bit weights, one extra PV MMA).
#pragma once

#include <cuda_fp16.h>

#include "ptx_sm100.cuh"

namespace attn_b200 {

constexpr int kBlockM = 128;   // query rows per tile
constexpr int kBlockN = 128;   // keys per K/V tile
constexpr int kHeadDim = 128;  // D
constexpr int kItemRows = 2 * kBlockM;
constexpr int kStagesK = 3;    // K ring depth
constexpr int kStagesV = 2;    // V ring depth (V_j is needed one softmax later than K_j)
constexpr int kThreads = 512;
constexpr uint32_t kTileBytes = kBlockM * kHeadDim * 2;  // 32 KiB fp16 tile
constexpr uint32_t kPanelBytes = kTileBytes / 2;         // one 64-column swizzle panel
constexpr float kRescaleLog2 = 8.0f;
// Of every 8 column pairs, how many take 2^x from the FMA-pipe polynomial
// instead of the MUFU unit: the kernel's kEmu template argument, one of
// kEmuChoices.  Which one runs for a call is a per-shape-class table measured
// on B200.  There no class gained from the polynomial: at D = 128, S = 8192
// causal, 0..4 pairs gave 1008, 971, 946, 911, 884 TFLOP/s, and at D = 64
// (half the tensor work per exponential) 1 pair tied with 0 and more lost, so
// the softmax is bound by its latency chain, not by MUFU throughput.
constexpr int kEmuChoices[] = {0, 1, 2, 3, 4};
constexpr int kNumVariants = sizeof(kEmuChoices) / sizeof(kEmuChoices[0]);
constexpr float kRedoThreshold = 3.98f;
constexpr float kLn2 = 0.69314718055994531f;

constexpr int kEpilogueWarp0 = 8;
constexpr int kProducerWarp = 12;   // Q and K
constexpr int kMmaWarp = 13;
constexpr int kProducerVWarp = 14;  // V
constexpr int kRegsSoftmax = 192;
constexpr int kRegsEpilogue = 80;
constexpr int kRegsOther = 48;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsEpilogue + 128 * kRegsOther <= kThreads * 128,
              "register split exceeds the launch allocation");

constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t tmem_s_col(int x) { return x * 128u; }
__device__ __forceinline__ uint32_t tmem_o_col(int x) { return 256u + x * 128u; }

// redo list (device scratch): header {count, done, -, -} then item ids
constexpr int kRedoHeaderWords = 4;

struct FwdParams {
  __half* o;
  float* lse;
  int B, Hq, Hkv, S;  // S: query rows per head (Sq)
  int Sk;             // keys per kv head
  int causal;
  int off;            // causal window offset Sk - Sq: query i sees keys j <= i + off
  int n_items;        // B * Hq * n_qb2
  int n_qb;           // ceil(S / 128) row blocks
  int n_kb;           // ceil(Sk / 128) key blocks
  int s_tail;         // rows in the last row block, 1..128
  int n_qb2;         // ceil(n_qb / 2) items per (batch, head)
  int group;         // Hq / Hkv
  float scale_log2;  // log2(e) / sqrt(D)
  unsigned long long timeout_ns;
  unsigned int* redo;  // redo list
  unsigned int redo_capacity;
};

enum WaitSite : uint32_t {
  kSiteProducerQ = 0x101,
  kSiteProducerK = 0x102,
  kSiteProducerV = 0x103,
  kSiteMmaQ = 0x201,
  kSiteMmaK = 0x202,
  kSiteMmaV = 0x203,
  kSiteMmaP = 0x204,
  kSiteMmaO = 0x205,
  kSiteSoftmaxS = 0x301,
  kSiteSoftmaxStats = 0x302,
  kSiteEpilogueO = 0x401,
  kSiteEpilogueStats = 0x402,
  kSiteDrain = 0x501,
};

// Bytes of one 128-row fp16 tile of head dimension kD (kD / 64 panels of 64
// columns, 128 bytes per row of a panel).
template <int kD>
__host__ __device__ constexpr uint32_t tile_bytes() {
  return static_cast<uint32_t>(kBlockM) * kD * 2;
}

// Shared memory: the tiles first (224 KiB at kD = 128; each 1 KiB aligned,
// as the 128-byte swizzle needs), then the row statistics and the barriers.
// The dynamic shared memory base is checked to be 1 KiB aligned at launch.
template <int kD>
struct SharedFwdT {
  uint8_t q[2][tile_bytes<kD>()];
  uint8_t k[kStagesK][tile_bytes<kD>()];
  uint8_t v[kStagesV][tile_bytes<kD>()];
  float stat_m[2][kBlockM];  // [tile][row], handed from softmax to epilogue
  float stat_l[2][kBlockM];
  uint64_t q_full, q_empty;
  uint64_t k_full[kStagesK], k_empty[kStagesK], v_full[kStagesV], v_empty[kStagesV];
  uint64_t s_full[2], p_full[2], o_done[2], o_free[2], stats_ready[2], stats_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int item_flag[2];   // [item parity]: a row of the item needs the redo pass
  int item_warps[2];  // [item parity]: epilogue warps done with the item
  unsigned int n_listed;
};

static_assert(sizeof(SharedFwdT<128>) <= 232448, "shared memory exceeds the 227 KiB per-block limit");
using SharedFwd = SharedFwdT<128>;

struct Item {
  int b, hq, g, qb2;
  int n_kv[2];   // key blocks of tile A, tile B (0: tile B lies past the end)
  int n_blocks;  // max of the two
};

__device__ __forceinline__ Item decode_item(const FwdParams& p, int id) {
  // kv-head major; inside a kv head: row blocks from last to first, the
  // group's query heads adjacent
  const int per_kv = p.group * p.n_qb2;
  const int kvh = id / per_kv;
  const int rem = id - kvh * per_kv;
  Item it;
  it.b = kvh / p.Hkv;
  it.g = kvh - it.b * p.Hkv;
  it.qb2 = p.n_qb2 - 1 - rem / p.group;
  it.hq = it.g * p.group + rem % p.group;
  const bool b_active = 2 * it.qb2 + 1 < p.n_qb;
  if (p.causal) {
    // the tile's last row sees keys up to row + off; no further key block
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int last_row = min((2 * it.qb2 + x) * kBlockM + kBlockM - 1, p.S - 1);
      it.n_kv[x] = min(p.n_kb, (last_row + p.off) / kBlockN + 1);
    }
    if (!b_active) it.n_kv[1] = 0;
  } else {
    it.n_kv[0] = p.n_kb;
    it.n_kv[1] = b_active ? p.n_kb : 0;
  }
  it.n_blocks = it.n_kv[1] > it.n_kv[0] ? it.n_kv[1] : it.n_kv[0];
  return it;
}

// k-th work item of this CTA, or -1 when done.
template <int kMode>
__device__ __forceinline__ int work_item(const FwdParams& p, int k, unsigned int n_listed) {
  const long long idx = static_cast<long long>(blockIdx.x) + static_cast<long long>(k) * gridDim.x;
  if (kMode == 1 && n_listed <= p.redo_capacity) {
    if (idx >= n_listed) return -1;
    const unsigned int id = p.redo[kRedoHeaderWords + idx];
    // an id from another call's list (left by a launch that failed) is
    // replaced by item 0: recomputing a valid item is always harmless
    return id < static_cast<unsigned int>(p.n_items) ? static_cast<int>(id) : 0;
  }
  return idx < p.n_items ? static_cast<int>(idx) : -1;
}

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  int never = 0;
  mbar_wait(bar, parity, &never, timeout_ns, kSiteDrain);
}

template <int kDepth>
__device__ __forceinline__ uint32_t ring_parity(int rc) {
  return (rc / kDepth) & 1;
}

// S_X(j) = Q_X K^T: kD / 16 MMAs of K = 16 over the head dimension.  Both
// operands are K-major; 16 columns are 32 bytes inside a 128-byte swizzled
// row and columns 64..127 (kD = 128) live in the second panel.
// A descriptor's start address sits in its low bits (16-byte units), so a
// descriptor for base + off is the base descriptor plus off >> 4 (shared
// memory offsets stay below 256 KiB, so no carry leaves the field).
template <int kk>
__device__ __forceinline__ void qk_step(uint32_t d_tmem, uint64_t qd, uint64_t kd, uint32_t idesc) {
  constexpr uint32_t off = ((kk >> 2) * kPanelBytes + (kk & 3) * 32) >> 4;
  mma_f16_ss_off<off, off>(d_tmem, qd, kd, idesc, kk > 0 ? 1u : 0u);
}

template <int kD>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_s, uint32_t k_s) {
  static_assert(kD == 64 || kD == 128, "head dimension 64 or 128");
  const uint32_t idesc = idesc_f16_f32(kBlockM, kBlockN, false, false);
  const uint64_t qd = smem_desc_sw128(q_s, 16, 1024);
  const uint64_t kd = smem_desc_sw128(k_s, 16, 1024);
  qk_step<0>(d_tmem, qd, kd, idesc);
  qk_step<1>(d_tmem, qd, kd, idesc);
  qk_step<2>(d_tmem, qd, kd, idesc);
  qk_step<3>(d_tmem, qd, kd, idesc);
  if constexpr (kD == 128) {
    qk_step<4>(d_tmem, qd, kd, idesc);
    qk_step<5>(d_tmem, qd, kd, idesc);
    qk_step<6>(d_tmem, qd, kd, idesc);
    qk_step<7>(d_tmem, qd, kd, idesc);
  }
}

// O_X (+)= P V: A = P from TMEM (8 columns = 16 keys per MMA), B = V, an
// MN-major operand of N = kD (16 keys = two 8-row groups of 1 KiB; at kD = 128
// the two 64-column halves of D are a panel apart).
template <int kk>
__device__ __forceinline__ void pv_step(uint32_t o_tmem, uint32_t p_tmem, uint64_t vd,
                                        uint32_t idesc, uint32_t acc) {
  constexpr uint32_t a_off = kk * 8;            // TMEM columns
  constexpr uint32_t b_off = (kk * 2048) / 16;   // 16 keys of V, in 16-byte units
  mma_f16_ts_off<a_off, b_off>(o_tmem, p_tmem, vd, idesc, (acc || kk > 0) ? 1u : 0u);
}

template <int kD>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_s,
                                         bool accumulate) {
  const uint32_t idesc = idesc_f16_f32(kBlockM, kD, false, true);
  const uint64_t vd = smem_desc_sw128(v_s, kPanelBytes, 1024);
  const uint32_t acc = accumulate ? 1u : 0u;
  pv_step<0>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step<1>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step<2>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step<3>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step<4>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step<5>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step<6>(o_tmem, p_tmem, vd, idesc, acc);
  pv_step<7>(o_tmem, p_tmem, vd, idesc, acc);
}

// kMode 0: the fused pass over every item; kMode 1: the redo pass over the
// listed items with hi + lo probabilities.  kD: the head dimension, 64 or 128.
// kEmu: FMA-pipe exponentials per 8 column pairs in the fused pass (the redo
// pass takes every exponential from the MUFU unit and is built with 0).
template <int kMode, int kD = 128, int kEmu = 0>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  static_assert(kEmu >= 0 && kEmu <= 8 && (kMode == 0 || kEmu == 0), "kEmu: 0..8, fused pass");
  constexpr uint32_t kTile = tile_bytes<kD>();
  constexpr int kPanels = kD / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  SharedFwdT<kD>* sm = reinterpret_cast<SharedFwdT<kD>*>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t to = p.timeout_ns;
  if (smem_addr(smem_raw) & 1023u) {
    // the swizzled tiles need a 1 KiB aligned base; report instead of computing garbage
    if (threadIdx.x == 0) atomicOr(&g_attn_status[0], kStatusSmemAlign);
    return;
  }

  if (threadIdx.x == 0) {
    sm->n_listed = (kMode == 1) ? *reinterpret_cast<volatile unsigned int*>(p.redo) : 0u;
    mbar_init(smem_addr(&sm->q_full), 1);
    mbar_init(smem_addr(&sm->q_empty), 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(smem_addr(&sm->k_full[s]), 1);
      mbar_init(smem_addr(&sm->k_empty[s]), 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(smem_addr(&sm->v_full[s]), 1);
      mbar_init(smem_addr(&sm->v_empty[s]), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(smem_addr(&sm->s_full[x]), 1);
      mbar_init(smem_addr(&sm->p_full[x]), kBlockM);
      mbar_init(smem_addr(&sm->o_done[x]), 1);
      mbar_init(smem_addr(&sm->o_free[x]), kBlockM);
      mbar_init(smem_addr(&sm->stats_ready[x]), kBlockM);
      mbar_init(smem_addr(&sm->stats_free[x]), kBlockM);
    }
    mbar_init(smem_addr(&sm->drain), 1);
    sm->abort = 0;
    sm->item_flag[0] = sm->item_flag[1] = 0;
    sm->item_warps[0] = sm->item_warps[1] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const unsigned int n_listed = sm->n_listed;
  const bool has_work = work_item<kMode>(p, 0, n_listed) >= 0;

  if (has_work) {
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
      if ((warp == kProducerWarp || warp == kProducerVWarp) && lane == 0) {
        // ------------------------------------------------------------ producers
        // warp 12: Q_A, Q_B per item and K_j; warp 14: V_j
        const bool is_v = warp == kProducerVWarp;
        const uint64_t keep = l2_policy_evict_last();     // K/V: reused by many items
        const uint64_t once = l2_policy_evict_first();    // Q: read once
        int rc = 0;
        int k = 0;
        int item;
        bool ok = true;
        for (; ok && (item = work_item<kMode>(p, k, n_listed)) >= 0; ++k) {
          const Item it = decode_item(p, item);
          if (!is_v) {
            if (k > 0 &&
                !mbar_wait(smem_addr(&sm->q_empty), (k - 1) & 1, abort, to, kSiteProducerQ)) {
              ok = false;
              break;
            }
            const int q_row = (it.b * p.Hq + it.hq) * p.S + it.qb2 * kItemRows;
            const uint32_t qf = smem_addr(&sm->q_full);
            mbar_arrive_expect_tx(qf, 2 * kTile);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              const uint32_t q_s = smem_addr(sm->q[x]);
#pragma unroll
              for (int pn = 0; pn < kPanels; ++pn)
                tma_load_2d_hint(q_s + pn * kPanelBytes, &tm_q, qf, 64 * pn, q_row + x * kBlockM,
                                 once);
            }
          }
          const int kv_row = (it.b * p.Hkv + it.g) * p.Sk;
          for (int j = 0; j < it.n_blocks; ++j, ++rc) {
            const int depth = is_v ? kStagesV : kStagesK;
            const int st = rc % depth;
            const uint32_t empty = smem_addr(is_v ? &sm->v_empty[st] : &sm->k_empty[st]);
            if (rc >= depth && !mbar_wait(empty, ((rc / depth) & 1) ^ 1, abort, to,
                                          is_v ? kSiteProducerV : kSiteProducerK)) {
              ok = false;
              break;
            }
            const uint32_t full = smem_addr(is_v ? &sm->v_full[st] : &sm->k_full[st]);
            const uint32_t dst = smem_addr(is_v ? sm->v[st] : sm->k[st]);
            const CUtensorMap* map = is_v ? &tm_v : &tm_k;
            mbar_arrive_expect_tx(full, kTile);
#pragma unroll
            for (int pn = 0; pn < kPanels; ++pn)
              tma_load_2d_hint(dst + pn * kPanelBytes, map, full, 64 * pn, kv_row + j * kBlockN,
                               keep);
          }
        }
        if (*abort) {
          // every copy still in flight must land before the CTA exits: the
          // last Q load and the last load of each ring stage
          if (!is_v && k > 0) drain_wait(smem_addr(&sm->q_full), (k - 1) & 1, to);
          const int depth = is_v ? kStagesV : kStagesK;
          for (int t = (rc > depth ? rc - depth : 0); t < rc; ++t)
            drain_wait(smem_addr(is_v ? &sm->v_full[t % depth] : &sm->k_full[t % depth]),
                       ((t / depth) & 1), to);
        }
      } else if (warp == kMmaWarp && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr bool hilo = kMode == 1;
        int rc = 0;
        int pcnt[2] = {0, 0};
        int acnt[2] = {0, 0};  // items so far in which tile X was active
        bool ok = true;
        int item;
        for (int k = 0; ok && (item = work_item<kMode>(p, k, n_listed)) >= 0; ++k) {
          const Item it = decode_item(p, item);
          const int n_b = it.n_blocks;
          if (!mbar_wait(smem_addr(&sm->q_full), k & 1, abort, to, kSiteMmaQ)) {
            ok = false;
            break;
          }
          for (int j = 0; ok && j <= n_b; ++j) {
            // step j: PV_X(j-1) then S_X(j) for each tile; V_{j-1} and K_j are
            // awaited just before the first MMA that reads them
            const int st_k = (rc + j) % kStagesK;
            const int st_v = (rc + j + kStagesV - 1) % kStagesV;
            bool have_k = false, have_v = false;
            for (int x = 0; ok && x < 2; ++x) {
              const int n_x = it.n_kv[x];
              if (j >= 1 && j - 1 < n_x) {
                if (!have_v) {
                  ok = mbar_wait(smem_addr(&sm->v_full[st_v]), ring_parity<kStagesV>(rc + j - 1),
                                 abort, to, kSiteMmaV);
                  have_v = true;
                }
                // the epilogue must have read O_X of the tile's previous item
                ok = ok && (j != 1 || acnt[x] == 0 ||
                            mbar_wait(smem_addr(&sm->o_free[x]), (acnt[x] - 1) & 1, abort, to,
                                      kSiteMmaO));
                ok = ok && mbar_wait(smem_addr(&sm->p_full[x]), pcnt[x] & 1, abort, to, kSiteMmaP);
                if (!ok) break;
                ++pcnt[x];
                tc_fence_after();
                const uint32_t v_s = smem_addr(sm->v[st_v]);
                issue_pv<kD>(tmem + tmem_o_col(x), tmem + tmem_s_col(x), v_s, j - 1 > 0);
                if (hilo) issue_pv<kD>(tmem + tmem_o_col(x), tmem + tmem_s_col(x) + 64, v_s, true);
                if (j == n_x) tc_commit(smem_addr(&sm->o_done[x]));
              }
              if (j < n_x) {
                if (!have_k) {
                  ok = mbar_wait(smem_addr(&sm->k_full[st_k]), ring_parity<kStagesK>(rc + j), abort,
                                 to, kSiteMmaK);
                  have_k = true;
                  if (!ok) break;
                  tc_fence_after();
                }
                issue_qk<kD>(tmem + tmem_s_col(x), smem_addr(sm->q[x]), smem_addr(sm->k[st_k]));
                tc_commit(smem_addr(&sm->s_full[x]));
              }
            }
            if (ok && j < n_b) tc_commit(smem_addr(&sm->k_empty[st_k]));  // every S(j) issued
            if (ok && j == n_b - 1) tc_commit(smem_addr(&sm->q_empty));   // last S of the item
            if (ok && j >= 1) tc_commit(smem_addr(&sm->v_empty[st_v]));   // every PV(j-1) issued
          }
          rc += n_b;
          acnt[0] += it.n_kv[0] > 0;
          acnt[1] += it.n_kv[1] > 0;
        }
        // every MMA issued must complete before TMEM is released
        tc_commit(smem_addr(&sm->drain));
        drain_wait(smem_addr(&sm->drain), 0, to);
      }
      __syncwarp();
    } else if (warp >= kEpilogueWarp0) {
      // -------------------------------------------------------------- epilogue
      regs_dec<kRegsEpilogue>();
      const int r = (warp - kEpilogueWarp0) * 32 + lane;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      int acnt[2] = {0, 0};  // items so far in which tile X was active
      int item;
      for (int k = 0; (item = work_item<kMode>(p, k, n_listed)) >= 0; ++k) {
        const Item it = decode_item(p, item);
        bool flag = false;
        bool ok = true;
#pragma unroll 1
        for (int x = 0; x < 2; ++x) {
          if (it.n_kv[x] == 0) continue;
          const int a = acnt[x]++;
          ok = mbar_wait(smem_addr(&sm->o_done[x]), a & 1, abort, to, kSiteEpilogueO) &&
               mbar_wait(smem_addr(&sm->stats_ready[x]), a & 1, abort, to, kSiteEpilogueStats);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float m_use = sm->stat_m[x][r];
          const float l = sm->stat_l[x][r];
          mbar_arrive(smem_addr(&sm->stats_free[x]));  // the softmax may write the next item's
          const float inv_l = 1.0f / l;
          // rows past S (a ragged last block) are computed but not stored
          const int i_row = it.qb2 * kItemRows + x * kBlockM + r;
          const bool valid = i_row < p.S;
          const int row = (it.b * p.Hq + it.hq) * p.S + i_row;
          uint4* orow = reinterpret_cast<uint4*>(p.o + static_cast<size_t>(row) * kD);
          float omax = 0.f;
#pragma unroll
          for (int c = 0; c < kD / 16; ++c) {
            uint32_t w[16];
            tmem_ld16(lane_base + tmem_o_col(x) + c * 16, w);
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
              if (valid) orow[c * 2 + v4] = pk;
            }
          }
          tc_fence_before();
          mbar_arrive(smem_addr(&sm->o_free[x]));
          if (valid) p.lse[row] = (m_use + log2f(l)) * kLn2;
          flag |= valid && omax >= kRedoThreshold;
        }
        if (!ok) break;
        if (kMode == 0) {
          // One redo-list entry per item if any of its rows needs it.  The
          // last of the four epilogue warps to finish the item appends it (no
          // barrier, so a warp that gave up on a wait cannot block the
          // others).  Slots are per item parity: a warp reaches item k+2 only
          // after every warp has finished item k.
          const bool any = __any_sync(0xffffffffu, flag);
          if (lane == 0) {
            if (any) atomicOr(&sm->item_flag[k & 1], 1);
            __threadfence_block();
            if (atomicAdd(&sm->item_warps[k & 1], 1) == 3) {
              if (atomicExch(&sm->item_flag[k & 1], 0)) {
                const unsigned int slot = atomicAdd(p.redo, 1u);
                if (slot < p.redo_capacity)
                  p.redo[kRedoHeaderWords + slot] = static_cast<unsigned int>(item);
              }
              sm->item_warps[k & 1] = 0;
            }
          }
        }
      }
    } else {
      // -------------------------------------------------------------- softmax
      regs_inc<kRegsSoftmax>();
      const int x = warp >> 2;  // tile
      const int r = (warp & 3) * 32 + lane;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      const uint32_t s_t = lane_base + tmem_s_col(x);
      const uint32_t o_t = lane_base + tmem_o_col(x);
      const float sc = p.scale_log2;
      constexpr bool hilo = kMode == 1;
      int scnt = 0;
      int acnt = 0;  // items so far in which this tile was active
      int item;
      for (int k = 0; (item = work_item<kMode>(p, k, n_listed)) >= 0; ++k) {
        const Item it = decode_item(p, item);
        const int n_x = it.n_kv[x];
        if (n_x == 0) continue;
        // the last key this row sees: row + off (causal), and never past Sk
        // (a ragged last key block reads the next head's rows, or zero fill
        // past the tensor); rows past S are computed but not stored
        const int i_row = (2 * it.qb2 + x) * kBlockM + r;
        const int key_lim = p.causal ? min(i_row + p.off, p.Sk - 1) : p.Sk - 1;
        // key_lim grows with the lane, so from this block on (warp-uniform)
        // some lane of the warp has keys to mask
        const int j_mask = (__shfl_sync(0xffffffffu, key_lim, 0) + 1) / kBlockN;
        float m_use = -INFINITY;
        float l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_x; ++j, ++scnt) {
          ok = mbar_wait(smem_addr(&sm->s_full[x]), scnt & 1, abort, to, kSiteSoftmaxS);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // the row of S_X in 128 registers (fp32 bits)
          uint32_t u[128];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld32(s_t + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c * 32]));
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) reg_dep32(&u[c * 32]);
          // keys past the row's limit -> -inf (the causal diagonal, a
          // ragged last key block)
          if (j >= j_mask) {
            const int lim = key_lim - j * kBlockN;
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
          const float cand = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                   fmaxf(mx8[6], mx8[7])) * sc;
          if (j == 0) {
            m_use = cand;
          } else {
            const bool grow = cand > m_use + kRescaleLog2;
            if (__any_sync(0xffffffffu, grow)) {
              // O_X holds P(j-1) V_{j-1} already (it completed before S(j))
              const float alpha = grow ? ex2_approx(m_use - cand) : 1.0f;
#pragma unroll 1
              for (int c = 0; c < kD / 32; ++c) {
                uint32_t w[32];
                tmem_ld32(o_t + c * 32, w);
                tmem_wait_ld();
                reg_dep32(w);
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * alpha);
                tmem_st32(o_t + c * 32, w);
              }
              if (grow) {
                l *= alpha;
                m_use = cand;
              }
            }
          }
          const float neg_m = -m_use;
          float lp[4] = {0.f, 0.f, 0.f, 0.f};
          if constexpr (!hilo) {
            // P rounded to fp16; l sums exactly the rounded values.  In every
            // 16 columns, kEmu pairs take 2^x from the FMA-pipe polynomial
            // and the rest from the MUFU unit.
            const float2 sc2 = make_float2(sc, sc);
            const float2 nm2 = make_float2(neg_m, neg_m);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
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
              tmem_st8(s_t + c * 8, ph);
            }
          } else {
            // P = hi + lo, both fp16: hi over columns [0,64), lo over [64,128)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t ph[8], pl[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(u[c * 16 + 2 * i]), sc, neg_m));
                const float p1 = ex2_approx(fmaf(__uint_as_float(u[c * 16 + 2 * i + 1]), sc, neg_m));
                ph[i] = pack_half2(p0, p1);
                const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&ph[i]));
                pl[i] = pack_half2(p0 - h.x, p1 - h.y);
                lp[i & 3] += p0 + p1;
              }
              tmem_st8(s_t + c * 8, ph);
              tmem_st8(s_t + 64 + c * 8, pl);
            }
          }
          l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(smem_addr(&sm->p_full[x]));
        }
        if (!ok) break;
        // the epilogue must have read this tile's previous statistics
        ok = acnt == 0 ||
             mbar_wait(smem_addr(&sm->stats_free[x]), (acnt - 1) & 1, abort, to, kSiteSoftmaxStats);
        if (!__all_sync(0xffffffffu, ok)) break;
        sm->stat_m[x][r] = m_use;
        sm->stat_l[x][r] = l;
        ++acnt;
        mbar_arrive(smem_addr(&sm->stats_ready[x]));
      }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
  }

  if (kMode == 1) {
    // the last CTA out empties the redo list for the next call on this stream
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      const unsigned int prev = atomicAdd(p.redo + 1, 1u);
      if (prev == gridDim.x - 1) {
        p.redo[0] = 0;
        p.redo[1] = 0;
        __threadfence();
      }
    }
  }
}

}  // namespace attn_b200
