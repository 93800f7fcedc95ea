// attn_fwd_sm100.cuh -- fused attention forward for sm_100a (B200).
//
// One launch computes O = softmax(Q K^T / sqrt(D) [+ causal mask]) V and the
// row log-sum-exp for grouped-query heads, without writing the score matrix
// to memory: the FlashAttention forward that the PipeThreader pages evaluate
// (papers.lqhl.me "PipeThreader-OSDI25", section 实验与结果, paper Sec. 6.2 /
// Fig. 12).  The pages build it from load, mma and softmax tasks on TMA,
// TensorCore and CUDA-core units overlapped inside an SM (section 核心方法,
// "sTask / sEU"; dependences kept by barrier-sTasks, "sTask-graph ->
// sProgram").  Here that split is fixed by hand for B200:
//
// Persistent kernel, one CTA per SM, a static list of work items per CTA.
// A work item is 256 query rows of one (batch, query head) -- two 128-row
// tiles, A and B, that share every K/V tile and take turns on the tensor
// core, so one tile's softmax runs while the other tile's MMAs do -- or, for
// launches with fewer items than SMs, 128 rows (tile A only).  Items are
// numbered either kv-head by kv-head (the query heads of a group and all
// their row blocks close together, so K/V stay in L2; item k of a CTA is
// blockIdx + k * grid) or, when all of K and V fit in L2, longest first with
// the CTAs taking them in a snake order (forward on even rounds, backward on
// odd ones), which balances the causal triangle.
//
// Warp roles (512 threads, registers re-split with setmaxnreg):
//   warps 0-3   softmax of tile A   (one query row per thread = TMEM lane)
//   warps 4-7   softmax of tile B
//   warps 8-11  epilogue: O / l -> fp16, LSE, for both tiles
//   warp 12     TMA producer of Q_A, Q_B (per item) and K_j (a ring)
//   warp 13     MMA issuer: S_X = Q_X K_j^T, O_X += P_X V_j (both tiles)
//   warp 14     TMA producer of V_j (its own ring)
//   warp 15     idle
// The MMA warp runs whole: every lane takes the same branches and waits, and
// one elected lane issues each MMA and commit.  One thread issues every MMA:
// a second issuing warp, even one taking strict turns with the first so that
// the pipe sees the same order, measured 20% slower on B200.
//
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384),
// O_B [384,512).  P_X (fp16) is written over the first 64 columns of S_X
// (in the exact pass its low half over the next 64).
//
// Per tile X and key block j the issuer issues PV_X(j-1) and then S_X(j);
// tcgen05 operations of one thread complete in order, so when S_X(j)
// signals s_full, O_X already holds P_X(j-1) V_{j-1} and the softmax may
// rescale it, and P_X(j-1) has been read before S_X(j) overwrites it.
//
// Numerics: P is rounded to fp16 and the row sum l accumulates exactly those
// rounded values, so O / l uses one consistent set of weights.  Lazy
// rescaling keeps a reference max per row and rescales O only when the row
// max grows by more than 2^kRescaleLog2 (exact: O and l share the
// reference).  The output is rounded to fp16, whose half-ulp for |O| >= 4 is
// 1.95e-3, so rows there need more than fp16 weights can give: the epilogue
// marks every 128-row tile with a row max|O| >= kRedoThreshold in a
// shared-memory bit set, and after its last item the CTA recomputes the
// marked tiles (an item whose other tile is unmarked runs with that tile
// left out) with P split as hi + lo fp16 (about 22-bit weights, one extra
// PV MMA per block): the exact pass, in the same launch.
#pragma once

#include <cuda_fp16.h>

#include "ptx_sm100.cuh"

namespace attn_b200 {

constexpr int kBlockM = 128;   // query rows per tile
constexpr int kBlockN = 128;   // keys per K/V tile
constexpr int kStagesK = 3;    // K ring depth
constexpr int kStagesV = 2;    // V ring depth (V_j is needed one softmax later than K_j)
constexpr int kThreads = 512;
constexpr uint32_t kPanelBytes = 16384;  // 128 rows x 64 fp16: one 128-byte swizzle panel
constexpr float kRescaleLog2 = 8.0f;
constexpr float kRedoThreshold = 3.98f;
constexpr float kLn2 = 0.69314718055994531f;
constexpr float kLog2e = 1.44269504088896341f;
// Items of one CTA in one launch are at most 32 * kRedoWords (the exact-pass
// bit sets: one bit per item, or per tile in the two-tile kernel); the host
// splits larger calls.
constexpr int kRedoWords = 64;
constexpr int kMaxItemsPerCta = 32 * kRedoWords;

constexpr int kEpilogueWarp0 = 8;
constexpr int kProducerWarp = 12;   // Q and K
constexpr int kMmaWarp = 13;
constexpr int kProducerVWarp = 14;  // V
constexpr int kMmaWarpB = 15;       // tile B's issuer when there are two
constexpr int kRegsSoftmax = 192;
constexpr int kRegsEpilogue = 64;
constexpr int kRegsOther = 64;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsEpilogue + 128 * kRegsOther <= kThreads * 128,
              "register split exceeds the launch allocation");

constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t tmem_s_col(int x) { return x * 128u; }
__device__ __forceinline__ uint32_t tmem_o_col(int x) { return 256u + x * 128u; }

// Of every 8 column pairs, how many take 2^x from the FMA-pipe polynomial
// instead of the MUFU unit (the kernel's kEmu argument).
constexpr int kEmuMax = 4;

// Division by a divisor fixed for the launch, without the hardware integer
// divide: that goes through the reciprocal of the MUFU unit, which the
// softmax keeps busy with exponentials, and measured ~1800 cycles for the
// three divisions of an item decode.  q = (umulhi(n, m) + n) >> s, exact for
// 0 <= n < 2^31, with s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1:
// the round-up multiplier of Granlund and Montgomery ("Division by invariant
// integers using multiplication", PLDI 1994), 2^32 + m = floor(2^(32+s)/d)+1,
// split so that the product fits 32-bit operations (n < 2^31 keeps the sum
// below 2^32).
struct FastDiv {
  uint32_t d, m, s;
};

inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  const uint64_t m = ((1ull << 32) * ((1ull << s) - d)) / d + 1;
  return {d, static_cast<uint32_t>(m), s};
}

__host__ __device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv& f) {
#ifdef __CUDA_ARCH__
  const uint32_t hi = __umulhi(n, f.m);
#else
  const uint32_t hi = static_cast<uint32_t>((static_cast<uint64_t>(n) * f.m) >> 32);
#endif
  return (hi + n) >> f.s;
}

struct FwdParams {
  __half* o;
  float* lse;
  unsigned int* status;  // kStatusWords words of device memory for this call
  int B, Hq, Hkv, S;     // S: query rows per head (Sq)
  int Sk;                // keys per kv head
  int causal;
  int off;               // causal window offset Sk - Sq: query i sees keys j <= i + off
  int n_qb;              // ceil(S / 128) row blocks
  int n_kb;              // ceil(Sk / 128) key blocks
  int group;             // Hq / Hkv
  int item_tiles;        // 2: items of two 128-row tiles; 1: one tile
  int pair_heads;        // two-tile items: 1 = the same rows of two query heads of a kv
                         // group, 0 = two consecutive row blocks of one head
  int n_qi;              // items per (batch, head or head pair)
  int n_items;
  int order;             // 0: kv-head major, round robin; 1: longest first, snake
  FastDiv div_major;     // items per kv head (order 0) or per row block (order 1)
  FastDiv div_members;   // query heads (or head pairs) per kv group
  FastDiv div_hkv;       // Hkv
  float scale_log2;      // log2(e) / sqrt(D)
  unsigned long long timeout_ns;
};

enum WaitSite : uint32_t {
  kSiteProducerQ = 0x101,
  kSiteProducerK = 0x102,
  kSiteProducerV = 0x103,
  kSiteProducerRedo = 0x104,
  kSiteMmaQ = 0x201,
  kSiteMmaK = 0x202,
  kSiteMmaV = 0x203,
  kSiteMmaP = 0x204,
  kSiteMmaO = 0x205,
  kSiteMmaRedo = 0x206,
  kSiteSoftmaxS = 0x301,
  kSiteSoftmaxStats = 0x302,
  kSiteSoftmaxRedo = 0x303,
  kSiteEpilogueO = 0x401,
  kSiteEpilogueStats = 0x402,
  kSiteEpilogueRedo = 0x403,
  kSiteDrain = 0x501,
};

// Bytes of one 128-row fp16 tile of head dimension kD (kD / 64 panels of 64
// columns, 128 bytes per row of a panel).
template <int kD>
__host__ __device__ constexpr uint32_t tile_bytes() {
  return static_cast<uint32_t>(kBlockM) * kD * 2;
}

// Shared memory: the tiles first (224 KiB at kD = 128; each 1 KiB aligned,
// as the 128-byte swizzle needs), then the row statistics, the exact-pass
// bit set and the barriers.  The dynamic shared memory base is checked to be
// 1 KiB aligned at launch.
template <int kD>
struct SharedFwdT {
  uint8_t q[2][tile_bytes<kD>()];
  uint8_t k[kStagesK][tile_bytes<kD>()];
  uint8_t v[kStagesV][tile_bytes<kD>()];
  float stat_m[2][kBlockM];  // [tile][row], handed from softmax to epilogue
  float stat_l[2][kBlockM];
  uint32_t redo_bits[2 * kRedoWords];  // bit 2k + x: tile x of item k needs the exact pass
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kStagesK], k_empty[kStagesK], v_full[kStagesV], v_empty[kStagesV];
  uint64_t s_full[2], p_full[2], o_done[2], o_free[2], stats_ready[2], stats_free[2];
  uint64_t redo_ready;  // the epilogue has marked every item of the fast pass
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(SharedFwdT<128>) <= 232448, "shared memory exceeds the 227 KiB per-block limit");

// Tile x of an item is row block qb0 + x * dqb of query head hq + x * dhq.
struct Item {
  int b, hq, g;
  int qb0;       // row block of tile A
  int dqb, dhq;  // (1, 0): two row blocks of one head; (0, 1): two heads of one kv group
  int n_kv[2];   // key blocks of tile A, tile B (0: the tile is not part of the item)
  int n_blocks;  // max of the two
};

__device__ __forceinline__ Item decode_item(const FwdParams& p, int id) {
  // the query heads (or head pairs) of a kv group an item can start at
  const int members = static_cast<int>(p.div_members.d);
  const int major = static_cast<int>(p.div_major.d);
  int qi, kvh, member;
  if (p.order == 0) {
    // kv-head major; inside a kv head: row blocks from last to first, the
    // group's query heads adjacent
    kvh = static_cast<int>(fast_div(id, p.div_major));
    const int rem = id - kvh * major;
    const int t = static_cast<int>(fast_div(rem, p.div_members));
    qi = p.n_qi - 1 - t;
    member = rem - t * members;
  } else {
    // row blocks from last (longest) to first; inside one, kv-head major
    const int r = static_cast<int>(fast_div(id, p.div_major));
    const int rem = id - r * major;
    qi = p.n_qi - 1 - r;
    kvh = static_cast<int>(fast_div(rem, p.div_members));
    member = rem - kvh * members;
  }
  Item it;
  it.b = static_cast<int>(fast_div(kvh, p.div_hkv));
  it.g = kvh - it.b * p.Hkv;
  it.dhq = p.pair_heads;
  it.dqb = p.pair_heads ? 0 : 1;
  it.hq = it.g * p.group + member * (1 + p.pair_heads);
  it.qb0 = p.pair_heads ? qi : qi * p.item_tiles;
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int qb = it.qb0 + x * it.dqb;
    if (x >= p.item_tiles || qb >= p.n_qb) {
      it.n_kv[x] = 0;
    } else if (p.causal) {
      // the tile's last row sees keys up to row + off; no further key block
      const int last_row = min(qb * kBlockM + kBlockM - 1, p.S - 1);
      it.n_kv[x] = min(p.n_kb, (last_row + p.off) / kBlockN + 1);
    } else {
      it.n_kv[x] = p.n_kb;
    }
  }
  it.n_blocks = max(it.n_kv[0], it.n_kv[1]);
  return it;
}

// k-th item of this CTA's fast pass, or -1 when its list has ended.
__device__ __forceinline__ int seq_item(const FwdParams& p, int k) {
  const long long G = gridDim.x;
  const long long c = blockIdx.x;
  const long long kk = k;
  const long long id = p.order == 0 ? c + kk * G : kk * G + ((k & 1) ? G - 1 - c : c);
  return id < p.n_items ? static_cast<int>(id) : -1;
}

// Walks this CTA's items: the fast pass over its list, then -- once the
// epilogue has marked them -- the exact pass over the marked ones.  Every
// role walks the same sequence.
struct ItemWalk {
  int k;        // index in this CTA's list
  int n_fast;   // length of the list (known once the fast pass ended)
  bool exact;   // in the exact pass
  __device__ __forceinline__ ItemWalk() : k(0), n_fast(-1), exact(false) {}
};

// The tiles of item k (bit x: tile x) that the exact pass recomputes.
template <int kD>
__device__ __forceinline__ uint32_t redo_marked(const SharedFwdT<kD>* sm, int k) {
  return (sm->redo_bits[(2 * k) >> 5] >> ((2 * k) & 31)) & 3u;
}

// An item of the exact pass keeps only its marked tiles.
__device__ __forceinline__ Item exact_tiles(Item it, uint32_t tiles) {
#pragma unroll
  for (int x = 0; x < 2; ++x)
    if (!((tiles >> x) & 1u)) it.n_kv[x] = 0;
  it.n_blocks = max(it.n_kv[0], it.n_kv[1]);
  return it;
}

// decode_item, restricted in the exact pass to the marked tiles of the item
// the walk just returned.
template <int kD>
__device__ __forceinline__ Item walk_item(const FwdParams& p, const SharedFwdT<kD>* sm,
                                          const ItemWalk& w, int item) {
  const Item it = decode_item(p, item);
  return w.exact ? exact_tiles(it, redo_marked(sm, w.k - 1)) : it;
}

// Next item of the walk, or -1 at the end.  At the switch from the fast pass
// to the exact pass it waits (bounded) until the epilogue has marked every
// item; `ok` turns false if that wait gives up.
template <int kD, bool kSpin = false>
__device__ __forceinline__ int walk_next(ItemWalk& w, const FwdParams& p, SharedFwdT<kD>* sm,
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
  while (w.k < w.n_fast && !redo_marked(sm, w.k)) ++w.k;
  if (w.k >= w.n_fast) return -1;
  return seq_item(p, w.k++);
}

template <int kDepth>
__device__ __forceinline__ uint32_t ring_parity(int rc) {
  return (rc / kDepth) & 1;
}

// S_X(j) = Q_X K^T: kD / 16 MMAs of K = 16 over the head dimension.  Both
// operands are K-major; 16 columns are 32 bytes inside a 128-byte swizzled
// row and columns 64..127 (kD = 128) live in the second panel.
template <int kk>
__device__ __forceinline__ void qk_step(uint32_t d_tmem, uint64_t qd, uint64_t kd, uint32_t idesc) {
  constexpr uint32_t off = ((kk >> 2) * kPanelBytes + (kk & 3) * 32) >> 4;
  mma_ss<off, off>(d_tmem, qd, kd, idesc, kk > 0 ? 1u : 0u);
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
  constexpr uint32_t b_off = (kk * 2048) / 16;  // 16 keys of V, in 16-byte units
  mma_ts<a_off, b_off>(o_tmem, p_tmem, vd, idesc, (acc || kk > 0) ? 1u : 0u);
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

// ---------------------------------------------------------------------------
// roles
// ---------------------------------------------------------------------------

// TMA producer (one thread): Q_A, Q_B per item and K_j (is_v false), or V_j.
template <int kD>
__device__ __forceinline__ void producer_role(SharedFwdT<kD>* sm, const FwdParams& p,
                                              const CUtensorMap* tm_q, const CUtensorMap* tm_kv,
                                              bool is_v, volatile int* abort) {
  constexpr uint32_t kTile = tile_bytes<kD>();
  constexpr int kPanels = kD / 64;
  const uint64_t to = p.timeout_ns;
  const uint64_t keep = l2_policy_evict_last();   // K/V: reused by many items
  const uint64_t once = l2_policy_evict_first();  // Q: read once
  const int depth = is_v ? kStagesV : kStagesK;
  int rc = 0;
  int qcnt[2] = {0, 0};
  bool ok = true;
  ItemWalk w;
  int item;
  while (ok && (item = walk_next(w, p, sm, abort, ok, kSiteProducerRedo)) >= 0) {
    const Item it = walk_item(p, sm, w, item);
    if (!is_v) {
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (!ok || it.n_kv[x] == 0) continue;
        if (qcnt[x] > 0 && !mbar_wait(smem_addr(&sm->q_empty[x]), (qcnt[x] - 1) & 1, abort, to,
                                      p.status, kSiteProducerQ)) {
          ok = false;
          continue;
        }
        const int q_row =
            (it.b * p.Hq + it.hq + x * it.dhq) * p.S + (it.qb0 + x * it.dqb) * kBlockM;
        const uint32_t qf = smem_addr(&sm->q_full[x]);
        mbar_arrive_expect_tx(qf, kTile);
#pragma unroll
        for (int pn = 0; pn < kPanels; ++pn)
          tma_load_2d(smem_addr(sm->q[x]) + pn * kPanelBytes, tm_q, qf, 64 * pn, q_row, once);
        ++qcnt[x];
      }
      if (!ok) break;
    }
    const int kv_row = (it.b * p.Hkv + it.g) * p.Sk;
    for (int j = 0; j < it.n_blocks; ++j, ++rc) {
      const int st = rc % depth;
      const uint32_t empty = smem_addr(is_v ? &sm->v_empty[st] : &sm->k_empty[st]);
      if (rc >= depth && !mbar_wait(empty, ((rc / depth) & 1) ^ 1, abort, to, p.status,
                                    is_v ? kSiteProducerV : kSiteProducerK)) {
        ok = false;
        break;
      }
      const uint32_t full = smem_addr(is_v ? &sm->v_full[st] : &sm->k_full[st]);
      const uint32_t dst = smem_addr(is_v ? sm->v[st] : sm->k[st]);
      mbar_arrive_expect_tx(full, kTile);
#pragma unroll
      for (int pn = 0; pn < kPanels; ++pn)
        tma_load_2d(dst + pn * kPanelBytes, tm_kv, full, 64 * pn, kv_row + j * kBlockN, keep);
    }
  }
  if (!is_v && ok && w.exact) {
    // count this CTA's exact-pass items (any tile marked) for the status block
    int n = 0;
    for (int i = 0; i < 2 * kRedoWords; ++i)
      n += __popc((sm->redo_bits[i] | (sm->redo_bits[i] >> 1)) & 0x55555555u);
    if (n) atomicAdd(&p.status[2], static_cast<unsigned int>(n));
  }
  if (*abort) {
    // every copy still in flight must land before the CTA exits: the last Q
    // load of each tile and the last load of each ring stage
    if (!is_v)
#pragma unroll
      for (int x = 0; x < 2; ++x)
        if (qcnt[x] > 0) drain_wait(smem_addr(&sm->q_full[x]), (qcnt[x] - 1) & 1, to, p.status);
    for (int t = (rc > depth ? rc - depth : 0); t < rc; ++t)
      drain_wait(smem_addr(is_v ? &sm->v_full[t % depth] : &sm->k_full[t % depth]),
                 (t / depth) & 1, to, p.status);
  }
}

// Single MMA issuer (a whole warp; one elected lane issues).  Per item and
// key block j it waits for the step's V and K stages (and, at j = 0, the
// tiles' Q), then issues for tile A and tile B the group PV_X(j-1), S_X(j),
// each after its P (and, at j = 1, the epilogue's release of O).
template <int kD>
__device__ __forceinline__ void mma_role(SharedFwdT<kD>* sm, const FwdParams& p, uint32_t tmem,
                                         volatile int* abort) {
  constexpr int x_lo = 0, x_hi = 1;
  const uint64_t to = p.timeout_ns;
  int rc = 0;
  int pcnt[2] = {0, 0};  // P handoffs consumed
  int qcnt[2] = {0, 0};  // items in which the tile was active
  bool ok = true;
  ItemWalk w;
  int item;
  while (ok && (item = walk_next<kD, true>(w, p, sm, abort, ok, kSiteMmaRedo)) >= 0) {
    const Item it = walk_item(p, sm, w, item);
    const bool hilo = w.exact;
    const int n_b = it.n_blocks;
    for (int j = 0; ok && j <= n_b; ++j) {
      const int st_k = (rc + j) % kStagesK;
      const int st_v = (rc + j + kStagesV - 1) % kStagesV;
      // the stages this step reads are awaited before anything is issued
      const bool need_k = j < n_b;
      const bool need_v = j >= 1;
      if (need_v)
        ok = mbar_wait<true>(smem_addr(&sm->v_full[st_v]), ring_parity<kStagesV>(rc + j - 1),
                             abort, to, p.status, kSiteMmaV);
      if (ok && need_k)
        ok = mbar_wait<true>(smem_addr(&sm->k_full[st_k]), ring_parity<kStagesK>(rc + j), abort,
                             to, p.status, kSiteMmaK);
      if (ok && j == 0) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (x < x_lo || x > x_hi || it.n_kv[x] == 0 || !ok) continue;
          ok = mbar_wait<true>(smem_addr(&sm->q_full[x]), qcnt[x] & 1, abort, to, p.status,
                               kSiteMmaQ);
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (x < x_lo || x > x_hi || !ok) continue;
        const int n_x = it.n_kv[x];
        if (j >= 1 && j - 1 < n_x) {
          // the epilogue must have read O_X of the tile's previous item
          if (j == 1 && qcnt[x] > 0)
            ok = mbar_wait<true>(smem_addr(&sm->o_free[x]), (qcnt[x] - 1) & 1, abort, to,
                                 p.status, kSiteMmaO);
          ok = ok && mbar_wait<true>(smem_addr(&sm->p_full[x]), pcnt[x] & 1, abort, to, p.status,
                                     kSiteMmaP);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) continue;
          ++pcnt[x];
          tc_fence_after();
          const uint32_t v_s = smem_addr(sm->v[st_v]);
          issue_pv<kD>(tmem + tmem_o_col(x), tmem + tmem_s_col(x), v_s, j - 1 > 0);
          if (hilo) issue_pv<kD>(tmem + tmem_o_col(x), tmem + tmem_s_col(x) + 64, v_s, true);
          if (j == n_x) tc_commit(smem_addr(&sm->o_done[x]));
        }
        if (j < n_x) {
          issue_qk<kD>(tmem + tmem_s_col(x), smem_addr(sm->q[x]), smem_addr(sm->k[st_k]));
          tc_commit(smem_addr(&sm->s_full[x]));
          if (j == n_x - 1) tc_commit(smem_addr(&sm->q_empty[x]));  // last S of the item
        }
      }
      if (!ok) break;
      // ring releases: the K stage of block j once every S(j) completed,
      // the V stage of block j-1 once every PV(j-1) did
      if (j < n_b) tc_commit(smem_addr(&sm->k_empty[st_k]));
      if (j >= 1) tc_commit(smem_addr(&sm->v_empty[st_v]));
    }
    rc += n_b;
#pragma unroll
    for (int x = 0; x < 2; ++x) qcnt[x] += it.n_kv[x] > 0 ? 1 : 0;
  }
  // every MMA issued must complete before TMEM is released
  tc_commit(smem_addr(&sm->drain[0]));
  drain_wait(smem_addr(&sm->drain[0]), 0, to, p.status);
}

// Epilogue of one item (warps 8-11; thread r owns row r of both tiles):
// O / l -> fp16 and LSE.  Returns false if a wait gave up; bit x of `flag`
// is set when a stored row of tile x has max|O| >= kRedoThreshold.
template <int kD>
__device__ __forceinline__ bool epilogue_item(SharedFwdT<kD>* sm, const FwdParams& p,
                                              uint32_t lane_base, int r, int lane, const Item& it,
                                              int (&ecnt)[2], uint32_t& flag, volatile int* abort) {
  const uint64_t to = p.timeout_ns;
  bool ok = true;
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    if (it.n_kv[x] == 0 || !ok) continue;
    const int a = ecnt[x]++;
    ok = mbar_wait(smem_addr(&sm->o_done[x]), a & 1, abort, to, p.status, kSiteEpilogueO) &&
         mbar_wait(smem_addr(&sm->stats_ready[x]), a & 1, abort, to, p.status,
                   kSiteEpilogueStats);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) continue;
    tc_fence_after();
    const float m_use = sm->stat_m[x][r];
    const float l = sm->stat_l[x][r];
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sm->stats_free[x]));  // the softmax may write the next
    const float inv_l = 1.0f / l;
    // rows past S (a ragged last block) are computed but not stored
    const int i_row = (it.qb0 + x * it.dqb) * kBlockM + r;
    const bool valid = i_row < p.S;
    const int row = (it.b * p.Hq + it.hq + x * it.dhq) * p.S + i_row;
    __half* orow = p.o + static_cast<size_t>(row) * kD;
    // rows are kD * 2 bytes apart, so every 16-column chunk of O is 32-byte
    // aligned when the tensor is: then each chunk goes out as one full-sector
    // store, else as two 16-byte stores
    const bool sector_aligned = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
    float omax = 0.f;
#pragma unroll
    for (int c = 0; c < kD / 16; ++c) {
      uint32_t wv[16];
      tmem_ld16(lane_base + tmem_o_col(x) + c * 16, wv);
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
    if (lane == 0) mbar_arrive(smem_addr(&sm->o_free[x]));
    if (valid) p.lse[row] = (m_use + log2f(l)) * kLn2;
    if (valid && omax >= kRedoThreshold) flag |= 1u << x;
  }
  return ok;
}

// Epilogue role: the fast pass over the CTA's list, marking items for the
// exact pass; then it releases the other roles into the exact pass and
// stores the marked items again from their recomputed O.
template <int kD>
__device__ __forceinline__ void epilogue_role(SharedFwdT<kD>* sm, const FwdParams& p,
                                              uint32_t tmem, int warp, int lane,
                                              volatile int* abort) {
  const int r = (warp - kEpilogueWarp0) * 32 + lane;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  int ecnt[2] = {0, 0};  // items so far in which tile X was active
  bool ok = true;
  int k = 0;
  for (int item; ok && (item = seq_item(p, k)) >= 0; ++k) {
    uint32_t flag = 0;
    ok = epilogue_item(sm, p, lane_base, r, lane, decode_item(p, item), ecnt, flag, abort);
    const uint32_t tiles = __reduce_or_sync(0xffffffffu, flag);
    if (ok && tiles && lane == 0) atomicOr(&sm->redo_bits[(2 * k) >> 5], tiles << ((2 * k) & 31));
  }
  // every fast-pass item is marked or not: release the others (also when
  // this warp gave up, so that no role waits for the marks forever)
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_addr(&sm->redo_ready));
  if (!ok) return;
  ok = mbar_wait(smem_addr(&sm->redo_ready), 0, abort, p.timeout_ns, p.status,
                 kSiteEpilogueRedo);
  if (!__all_sync(0xffffffffu, ok)) return;
  for (int kk = 0; ok && kk < k; ++kk) {
    const uint32_t tiles = redo_marked(sm, kk);
    if (!tiles) continue;
    uint32_t flag = 0;
    ok = epilogue_item(sm, p, lane_base, r, lane, exact_tiles(decode_item(p, seq_item(p, kk)), tiles),
                       ecnt, flag, abort);
  }
}

// The key blocks of one item in the fast pass, for one tile's softmax warp
// (thread = query row = TMEM lane).  Returns false if a wait gave up; m_use
// and l hold the row's statistics on return.
template <int kD, int kEmu>
__device__ __forceinline__ bool softmax_item(SharedFwdT<kD>* sm, const FwdParams& p, int x,
                                             uint32_t s_t, uint32_t o_t, int n_x, int key_lim,
                                             int j_mask, int lane, int& scnt, float& m_use,
                                             float& l, volatile int* abort) {
  const uint64_t to = p.timeout_ns;
  const float sc = p.scale_log2;
  m_use = -INFINITY;
  l = 0.f;
  for (int j = 0; j < n_x; ++j, ++scnt) {
    bool ok = mbar_wait(smem_addr(&sm->s_full[x]), scnt & 1, abort, to, p.status, kSiteSoftmaxS);
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
    // the row of S_X in 128 registers (fp32 bits)
    uint32_t u[128];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(s_t + c * 32, &u[c * 32]);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 4; ++c) reg_dep32(&u[c * 32]);
    // keys past the row's limit -> -inf (the causal diagonal, a ragged last
    // key block)
    if (j >= j_mask) {
      const int lim = key_lim - j * kBlockN;
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (c > lim) u[c] = 0xff800000u;  // -inf
    }
    // row max: 8 independent chains (chain t takes columns t, t + 8, ...) of
    // 3-input max, then a tree
    float mx8[8];
#pragma unroll
    for (int t = 0; t < 8; ++t)
      mx8[t] = fmax3(__uint_as_float(u[t]), __uint_as_float(u[8 + t]), __uint_as_float(u[16 + t]));
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
          uint32_t wv[32];
          tmem_ld32(o_t + c * 32, wv);
          tmem_wait_ld();
          reg_dep32(wv);
#pragma unroll
          for (int i = 0; i < 32; ++i) wv[i] = __float_as_uint(__uint_as_float(wv[i]) * alpha);
          tmem_st32(o_t + c * 32, wv);
        }
        if (grow) {
          l *= alpha;
          m_use = cand;
        }
      }
    }
    const float neg_m = -m_use;
    float lp[4] = {0.f, 0.f, 0.f, 0.f};
    // P rounded to fp16; l sums exactly the rounded values.  In every 16
    // columns, kEmu pairs take 2^x from the FMA-pipe polynomial and the rest
    // from the MUFU unit.
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
    l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sm->p_full[x]));
  }
  return true;
}

// The key blocks of one item in the exact pass.  The fast pass has already
// stored the row's LSE = ln 2 * (m + log2 l) in log2 units m + log2 l, which
// bounds every scaled logit of the row from above: l sums the weights
// against m, the largest of them among them, even when a lazy rescale left m
// below the row max.  With m_ref = that bound - kRescaleLog2, the weights
// p = 2^(s * scale - m_ref) stay <= 2^kRescaleLog2 (the fast pass's range,
// well inside fp16 and away from its subnormals) with no running max and no
// rescale of O.  P goes to the PV MMAs as hi + lo fp16 (hi over columns
// [0, 64), lo over [64, 128)); l sums the fp32 p.  Returns false if a wait
// gave up.
template <int kD>
__device__ __forceinline__ bool softmax_item_exact(SharedFwdT<kD>* sm, const FwdParams& p, int x,
                                                   uint32_t s_t, int n_x, int key_lim,
                                                   int j_mask, int lane, int& scnt, float m_ref,
                                                   float& l, volatile int* abort) {
  const uint64_t to = p.timeout_ns;
  const float sc = p.scale_log2;
  const float neg_m = -m_ref;
  l = 0.f;
  for (int j = 0; j < n_x; ++j, ++scnt) {
    bool ok = mbar_wait(smem_addr(&sm->s_full[x]), scnt & 1, abort, to, p.status, kSiteSoftmaxS);
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
    // the whole row of S first: P's low parts go over columns [64, 128)
    uint32_t u[128];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(s_t + c * 32, &u[c * 32]);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 4; ++c) reg_dep32(&u[c * 32]);
    if (j >= j_mask) {
      const int lim = key_lim - j * kBlockN;
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (c > lim) u[c] = 0xff800000u;  // -inf
    }
    float lp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
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
      tmem_st8(s_t + c * 8, ph);
      tmem_st8(s_t + 64 + c * 8, pl);
    }
    l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sm->p_full[x]));
  }
  return true;
}

// Softmax of tile x (warps 4x..4x+3).
template <int kD, int kEmu>
__device__ __forceinline__ void softmax_role(SharedFwdT<kD>* sm, const FwdParams& p, uint32_t tmem,
                                             int warp, int lane, volatile int* abort) {
  const int x = warp >> 2;  // tile
  const int r = (warp & 3) * 32 + lane;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  const uint32_t s_t = lane_base + tmem_s_col(x);
  const uint32_t o_t = lane_base + tmem_o_col(x);
  int scnt = 0;
  int acnt = 0;  // items so far in which this tile was active
  bool ok = true;
  ItemWalk w;
  int item;
  while (ok && (item = walk_next(w, p, sm, abort, ok, kSiteSoftmaxRedo)) >= 0) {
    const Item it = walk_item(p, sm, w, item);
    const int n_x = x ? it.n_kv[1] : it.n_kv[0];
    if (n_x == 0) continue;
    // the last key this row sees: row + off (causal), and never past Sk (a
    // ragged last key block reads the next head's rows, or zero fill past
    // the tensor); rows past S are computed but not stored
    const int i_row = (it.qb0 + x * it.dqb) * kBlockM + r;
    const int key_lim = p.causal ? min(i_row + p.off, p.Sk - 1) : p.Sk - 1;
    // key_lim grows with the lane, so from this block on (warp-uniform) some
    // lane of the warp has keys to mask
    const int j_mask = (__shfl_sync(0xffffffffu, key_lim, 0) + 1) / kBlockN;
    float m_use, l;
    if (w.exact) {
      // the fast pass stored this row's LSE (rows past S: not stored, not
      // needed, any finite reference does)
      const int hq = it.hq + x * it.dhq;
      const float lse = i_row < p.S ? p.lse[(static_cast<size_t>(it.b) * p.Hq + hq) * p.S + i_row]
                                    : 0.f;
      m_use = lse * kLog2e - kRescaleLog2;
      ok = softmax_item_exact<kD>(sm, p, x, s_t, n_x, key_lim, j_mask, lane, scnt, m_use, l,
                                  abort);
    } else {
      ok = softmax_item<kD, kEmu>(sm, p, x, s_t, o_t, n_x, key_lim, j_mask, lane, scnt, m_use,
                                  l, abort);
    }
    if (!ok) break;
    // the epilogue must have read this tile's previous statistics
    ok = acnt == 0 || mbar_wait(smem_addr(&sm->stats_free[x]), (acnt - 1) & 1, abort,
                                p.timeout_ns, p.status, kSiteSoftmaxStats);
    if (!__all_sync(0xffffffffu, ok)) {
      ok = false;
      break;
    }
    sm->stat_m[x][r] = m_use;
    sm->stat_l[x][r] = l;
    ++acnt;
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sm->stats_ready[x]));
  }
}

// kD: the head dimension, 64 or 128.  kEmu: FMA-pipe exponentials per 8
// column pairs in the fast pass.
template <int kD = 128, int kEmu = 0>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  static_assert(kEmu >= 0 && kEmu <= kEmuMax, "kEmu: 0..4");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  SharedFwdT<kD>* sm = reinterpret_cast<SharedFwdT<kD>*>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (smem_addr(smem_raw) & 1023u) {
    // the swizzled tiles need a 1 KiB aligned base; report instead of computing garbage
    if (threadIdx.x == 0) atomicOr(&p.status[0], kStatusSmemAlign);
    return;
  }
  if (seq_item(p, 0) < 0) return;  // no item for this CTA (the grid never exceeds the items)

  if (threadIdx.x == 0) {
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      mbar_init(smem_addr(&sm->q_full[x]), 1);
      mbar_init(smem_addr(&sm->q_empty[x]), 1);
      mbar_init(smem_addr(&sm->s_full[x]), 1);
      mbar_init(smem_addr(&sm->p_full[x]), 4);  // one arrive per softmax warp
      mbar_init(smem_addr(&sm->o_done[x]), 1);
      mbar_init(smem_addr(&sm->o_free[x]), 4);  // one per epilogue warp
      mbar_init(smem_addr(&sm->stats_ready[x]), 4);
      mbar_init(smem_addr(&sm->stats_free[x]), 4);
      mbar_init(smem_addr(&sm->drain[x]), 1);
    }
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(smem_addr(&sm->k_full[s]), 1);
      mbar_init(smem_addr(&sm->k_empty[s]), 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(smem_addr(&sm->v_full[s]), 1);
      mbar_init(smem_addr(&sm->v_empty[s]), 1);
    }
    mbar_init(smem_addr(&sm->redo_ready), 4);
    for (int i = 0; i < 2 * kRedoWords; ++i) sm->redo_bits[i] = 0;
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
      if (lane == 0) producer_role<kD>(sm, p, &tm_q, warp == kProducerVWarp ? &tm_v : &tm_k,
                                       warp == kProducerVWarp, abort);
    } else if (warp == kMmaWarp) {
      mma_role<kD>(sm, p, tmem, abort);
    }
    __syncwarp();
  } else if (warp >= kEpilogueWarp0) {
    regs_dec<kRegsEpilogue>();
    epilogue_role<kD>(sm, p, tmem, warp, lane, abort);
  } else {
    regs_inc<kRegsSoftmax>();
    softmax_role<kD, kEmu>(sm, p, tmem, warp, lane, abort);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn_b200
