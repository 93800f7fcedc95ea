// attn_api.cu -- C ABI of libattn_b200.so (declared in include/attn.h):
// argument validation, TMA tensor-map encoding, kernel launch, the per-call
// status blocks, the host-buffer entry point and the self-tests.  The only
// device memory it allocates is one small status block per (device, stream)
// -- per (device, host thread) for cudaStreamPerThread -- once, on first use.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <array>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <map>
#include <mutex>
#include <thread>
#include <tuple>
#include <utility>

#include "attn.h"
#include "attn_fwd_db_sm100.cuh"
#include "attn_fwd_sm100.cuh"

namespace attn_b200 {
namespace {

constexpr int kMaxDevices = 64;

std::atomic<uint64_t> g_timeout_ns{2000000000ull};

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

// ---------------------------------------------------------------------------
// fused-kernel variants: a pipeline structure x kEmu FMA-pipe exponentials
// per 8 column pairs.  Structures: 0 two-tile ping-pong, the tiles two row
// blocks of one head; 1 the same kernel with the tiles the same rows of two
// query heads of one kv group (when the group has an even number of heads;
// else as 0); 2 one tile with S double-buffered in TMEM; 3 the same with two
// softmax warps per lane quadrant.  Head dimension 256 has only the double-buffered kernel with one
// softmax warp per quadrant (shared memory has no room for more): every
// structure maps to it there.
// ---------------------------------------------------------------------------
constexpr int kEmuChoices = kEmuMax + 1;  // 0..4
constexpr int kStructures = 4;
constexpr int kNumVariants = kStructures * kEmuChoices;
__host__ __device__ constexpr int variant_emu(int v) { return v % kEmuChoices; }
__host__ __device__ constexpr int variant_structure(int v) { return v / kEmuChoices; }

using FwdKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                           const FwdParams);
struct KernelChoice {
  FwdKernel fn;
  size_t smem;
  int one_tile;    // items are one 128-row tile
  int kv_box;      // rows of a K / V tile
  int pair_heads;  // two-tile items pair query heads
};

template <int kD, int kV>
KernelChoice kernel_choice_v() {
  constexpr int s = variant_structure(kV), e = variant_emu(kV);
  if constexpr (kD == 256) {
    return {&db::attn_fwd_db_kernel<256, 1, e>, sizeof(db::SharedDb<256, 1>), 1,
            db::Cfg<256>::kBN, 0};
  } else if constexpr (s == 0 || s == 1) {
    return {&attn_fwd_kernel<kD, e>, sizeof(SharedFwdT<kD>), 0, kBlockN, s == 1};
  } else {
    return {&db::attn_fwd_db_kernel<kD, s - 1, e>, sizeof(db::SharedDb<kD, s - 1>), 1,
            db::Cfg<kD>::kBN, 0};
  }
}
template <int kD, int... kV>
std::array<KernelChoice, sizeof...(kV)> kernel_table(std::integer_sequence<int, kV...>) {
  return {{kernel_choice_v<kD, kV>()...}};
}
template <int kD>
const KernelChoice& kernel_choice_d(int variant) {
  static const std::array<KernelChoice, kNumVariants> table =
      kernel_table<kD>(std::make_integer_sequence<int, kNumVariants>{});
  return table[variant];
}
const KernelChoice& kernel_choice(int D, int variant) {
  return D == 64 ? kernel_choice_d<64>(variant)
                 : D == 128 ? kernel_choice_d<128>(variant) : kernel_choice_d<256>(variant);
}

// Measured choice of variant per shape class: rules (D, causal, smallest Sk,
// largest Sk, variant), first match wins, no match -> variant 0.  The rows
// are written by the package's tuner from timings of every variant on B200.
struct VariantRule {
  int d, causal, sk_lo, sk_hi, variant;
};
constexpr VariantRule kVariantRules[] = {
#define VARIANT_RULE(d, causal, sk_lo, sk_hi, variant) {d, causal, sk_lo, sk_hi, variant},
#include "variant_table.inc"
#undef VARIANT_RULE
    {0, 0, 0, 0, 0}  // end (D is never 0)
};

int select_variant(int D, int causal, int Sk) {
  for (const VariantRule& r : kVariantRules)
    if (r.d == D && r.causal == (causal ? 1 : 0) && Sk >= r.sk_lo && Sk <= r.sk_hi &&
        r.variant >= 0 && r.variant < kNumVariants)
      return r.variant;
  return 0;
}

// every kernel checks 1 KiB alignment of its dynamic shared memory base
bool set_smem_attributes(int D) {
  for (int v = 0; v < kNumVariants; ++v) {
    const KernelChoice& k = kernel_choice(D, v);
    if (cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(k.smem)) != cudaSuccess)
      return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// per-device setup
// ---------------------------------------------------------------------------
// 0 = not done, 1 = ok, 2 = unsupported device.
std::atomic<int> g_dev_state[kMaxDevices];
int g_dev_sms[kMaxDevices];
int g_dev_l2[kMaxDevices];
std::mutex g_dev_mutex;

attn_status device_setup(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  *dev_out = dev;
  int st = g_dev_state[dev].load(std::memory_order_acquire);
  if (st == 1) return ATTN_OK;
  if (st == 2) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  st = g_dev_state[dev].load(std::memory_order_acquire);
  if (st == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (major != 10 || minor != 0) {
      g_dev_state[dev].store(2, std::memory_order_release);
      return ATTN_ERR_UNSUPPORTED;
    }
    if (cudaDeviceGetAttribute(&g_dev_sms[dev], cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&g_dev_l2[dev], cudaDevAttrL2CacheSize, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (!set_smem_attributes(128) || !set_smem_attributes(64) || !set_smem_attributes(256))
      return ATTN_ERR_CUDA;
    g_dev_state[dev].store(1, std::memory_order_release);
  }
  return g_dev_state[dev].load() == 1 ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// status blocks: kStatusWords words of device memory per (device, stream),
// zeroed on that stream when created.  The legacy default stream (0) is one
// stream shared by every host thread; cudaStreamPerThread names a different
// stream in each host thread, so it gets one block per (device, thread).
// ---------------------------------------------------------------------------
using StatusKey = std::tuple<int, cudaStream_t, std::thread::id>;
std::map<StatusKey, unsigned int*> g_status_blocks;
std::mutex g_status_mutex;

StatusKey status_key(int dev, cudaStream_t stream) {
  const bool per_thread = stream == cudaStreamPerThread;
  return StatusKey(dev, stream, per_thread ? std::this_thread::get_id() : std::thread::id());
}

unsigned int* status_block(int dev, cudaStream_t stream, bool create) {
  std::lock_guard<std::mutex> lock(g_status_mutex);
  const StatusKey key = status_key(dev, stream);
  auto it = g_status_blocks.find(key);
  if (it != g_status_blocks.end()) return it->second;
  if (!create) return nullptr;
  void* ptr = nullptr;
  const size_t bytes = kStatusWords * sizeof(unsigned int);
  if (cudaMalloc(&ptr, bytes) != cudaSuccess) return nullptr;
  if (cudaMemsetAsync(ptr, 0, bytes, stream) != cudaSuccess) {
    cudaFree(ptr);
    return nullptr;
  }
  g_status_blocks[key] = static_cast<unsigned int*>(ptr);
  return static_cast<unsigned int*>(ptr);
}

// ---------------------------------------------------------------------------
// launch
// ---------------------------------------------------------------------------
// 2-D view [rows, D] fp16 of a dense [.., S, D] tensor; boxes of 64 columns
// (one 128-byte swizzle panel) x box_rows rows.
bool encode_rows_map(CUtensorMap* map, const void* base, uint64_t rows, int D,
                     uint32_t box_rows = kBlockM) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

attn_status validate_sizes(int B, int Hq, int Hkv, int S, int D, int Sk = -1, int causal = 0) {
  if (Sk < 0) Sk = S;
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || Sk < 1 || D < 1) return ATTN_ERR_SHAPE;
  if (Hq % Hkv != 0) return ATTN_ERR_SHAPE;
  // a causal query with no visible key (Sq > Sk) has no softmax
  if (causal && S > Sk) return ATTN_ERR_SHAPE;
  if (static_cast<int64_t>(B) * Hkv * Sk >= (int64_t(1) << 31)) return ATTN_ERR_SHAPE;
  if (D != 64 && D != 128 && D != 256) return ATTN_ERR_UNSUPPORTED;
  // row indices are 32-bit signed in the kernel and in TMA coordinates
  const int64_t q_rows = static_cast<int64_t>(B) * Hq * S;
  if (q_rows >= (int64_t(1) << 31)) return ATTN_ERR_SHAPE;
  return ATTN_OK;
}

attn_status validate_pointers(const void* q, const void* k, const void* v, const void* o,
                              const float* lse) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return ATTN_ERR_ALIGN;
  return ATTN_OK;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Kernel parameters of one launch over B batch elements (Sq query rows over
// Sk keys) on a device with `sms` SMs and `l2` bytes of L2.
FwdParams make_params(void* o, float* lse, unsigned int* status, int B, int Hq, int Hkv, int Sq,
                      int Sk, int D, int causal, int sms, int l2, bool one_tile,
                      bool pair_heads) {
  FwdParams p;
  p.o = static_cast<__half*>(o);
  p.lse = lse;
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = Sq;
  p.Sk = Sk;
  p.causal = causal ? 1 : 0;
  p.off = causal ? Sk - Sq : 0;
  p.n_qb = (Sq + kBlockM - 1) / kBlockM;
  p.n_kb = (Sk + kBlockN - 1) / kBlockN;
  p.group = Hq / Hkv;
  // 256-row items (two tiles sharing each K/V tile) unless the kernel takes
  // one tile per item, or two-tile items would leave SMs idle
  const long long heads = static_cast<long long>(B) * Hq;
  p.item_tiles = (one_tile || heads * ((p.n_qb + 1) / 2) < sms) ? 1 : 2;
  p.pair_heads = (pair_heads && p.item_tiles == 2 && p.group % 2 == 0) ? 1 : 0;
  p.n_qi = p.pair_heads ? p.n_qb : (p.n_qb + p.item_tiles - 1) / p.item_tiles;
  p.n_items = static_cast<int>(heads / (1 + p.pair_heads) * p.n_qi);
  // Longest first (snake) balances a causal launch; it walks all kv heads at
  // once, so it is used only when all of K and V stay resident in L2.
  const double kv_bytes = 2.0 * B * Hkv * static_cast<double>(Sk) * D * 2;
  p.order = (causal && kv_bytes <= 0.5 * l2) ? 1 : 0;
  const int members = p.pair_heads ? p.group / 2 : p.group;
  p.div_members = make_fastdiv(static_cast<uint32_t>(members));
  p.div_major = make_fastdiv(static_cast<uint32_t>(
      p.order == 0 ? members * p.n_qi : static_cast<long long>(B) * Hkv * members));
  p.div_hkv = make_fastdiv(static_cast<uint32_t>(Hkv));
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  p.timeout_ns = g_timeout_ns.load();
  return p;
}

// One call: the batch is split into launches of at most kMaxItemsPerCta
// items per CTA (the exact pass's bit set), each with its own tensor maps.
attn_status launch_call(const void* q, const void* k, const void* v, void* o, float* lse,
                        unsigned int* status, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                        int causal, int variant, int dev, cudaStream_t cs) {
  const int sms = g_dev_sms[dev];
  const KernelChoice& kc = kernel_choice(D, variant);
  const FwdParams whole = make_params(o, lse, status, B, Hq, Hkv, Sq, Sk, D, causal, sms,
                                      g_dev_l2[dev], kc.one_tile != 0, kc.pair_heads != 0);
  const long long per_b = static_cast<long long>(whole.n_items) / B;
  const long long max_items = static_cast<long long>(sms) * kMaxItemsPerCta;
  const int chunk_b = static_cast<int>(per_b >= max_items ? 1 : max_items / per_b);
  if (per_b > max_items) return ATTN_ERR_SHAPE;  // one batch element would not fit
  const size_t q_b = static_cast<size_t>(Hq) * Sq * D;   // elements per batch element
  const size_t kv_b = static_cast<size_t>(Hkv) * Sk * D;
  const size_t l_b = static_cast<size_t>(Hq) * Sq;
  for (int b0 = 0; b0 < B; b0 += chunk_b) {
    const int nb = B - b0 < chunk_b ? B - b0 : chunk_b;
    const __half* qc = static_cast<const __half*>(q) + q_b * b0;
    const __half* kch = static_cast<const __half*>(k) + kv_b * b0;
    const __half* vc = static_cast<const __half*>(v) + kv_b * b0;
    __half* oc = static_cast<__half*>(o) + q_b * b0;
    float* lc = lse + l_b * b0;
    CUtensorMap tq, tk, tv;
    const uint32_t kv_box = static_cast<uint32_t>(kc.kv_box);
    if (!encode_rows_map(&tq, qc, static_cast<uint64_t>(nb) * Hq * Sq, D) ||
        !encode_rows_map(&tk, kch, static_cast<uint64_t>(nb) * Hkv * Sk, D, kv_box) ||
        !encode_rows_map(&tv, vc, static_cast<uint64_t>(nb) * Hkv * Sk, D, kv_box))
      return ATTN_ERR_CUDA;
    const FwdParams p = make_params(oc, lc, status, nb, Hq, Hkv, Sq, Sk, D, causal, sms,
                                    g_dev_l2[dev], kc.one_tile != 0, kc.pair_heads != 0);
    const int grid = p.n_items < sms ? p.n_items : sms;
    kc.fn<<<grid, kThreads, kc.smem, cs>>>(tq, tk, tv, p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// Streams of attn_fwd_host's copy / compute pipeline, created once per device
// (non-blocking, so they do not serialize with the legacy default stream).
constexpr int kHostChunks = 16;
// One call at a time uses a device's pipeline (`busy`): concurrent calls would
// share the compute stream's status block, and one could read and clear a
// timeout that the other's kernels raised.
struct HostPipe {
  cudaStream_t up, comp, down;
  std::mutex busy;
};
HostPipe* g_host_pipe[kMaxDevices];
std::mutex g_host_pipe_mutex;

HostPipe* host_pipe(int dev) {
  std::lock_guard<std::mutex> lock(g_host_pipe_mutex);
  if (!g_host_pipe[dev]) {
    HostPipe* hp = new HostPipe;
    if (cudaStreamCreateWithFlags(&hp->up, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp->comp, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp->down, cudaStreamNonBlocking) != cudaSuccess) {
      delete hp;
      return nullptr;
    }
    g_host_pipe[dev] = hp;
  }
  return g_host_pipe[dev];
}

// ---------------------------------------------------------------------------
// attn_fwd_noalloc's fixed scratch: the status block lives in this file-scope
// array instead of memory from cudaMalloc.  Every device that loads the
// library holds one copy until the process exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned int g_noalloc_status[kStatusWords];

// Device address of g_noalloc_status, looked up once per device with that
// device current (host code cannot use the symbol itself as an address).
unsigned int* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mutex;

unsigned int* noalloc_scratch(int dev) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_status) != cudaSuccess || !ptr) return nullptr;
    g_noalloc_ptr[dev] = static_cast<unsigned int*>(ptr);
  }
  return g_noalloc_ptr[dev];
}

// Reads (blocking) and clears one status block; ORs its flags into `words`.
bool drain_status_block(unsigned int* block, unsigned int (&words)[kStatusWords]) {
  unsigned int w[kStatusWords] = {0, 0, 0, 0};
  if (cudaMemcpy(w, block, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return false;
  if (w[0] | w[1] | w[2] | w[3]) {
    if (cudaMemset(block, 0, sizeof(w)) != cudaSuccess) return false;
  }
  words[0] |= w[0];
  if (words[1] == 0) words[1] = w[1];
  words[2] += w[2];
  return true;
}

attn_status status_of(const unsigned int (&words)[kStatusWords]) {
  if (words[0] & kStatusSmemAlign) return ATTN_ERR_CUDA;
  return (words[0] & kStatusTimeout) ? ATTN_ERR_DEVICE_TIMEOUT : ATTN_OK;
}

}  // namespace

// The status block of `stream` on the current device (created on first
// use), for the other kernels of this library (the decoder layer's GEMMs).
unsigned int* stream_status_block(cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  return status_block(dev, stream, true);
}

}  // namespace attn_b200

using namespace attn_b200;

extern "C" {

int attn_version(void) { return (2 << 16) | 0; }

const char* attn_status_string(attn_status s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_NULL: return "ATTN_ERR_NULL: a required pointer is NULL";
    case ATTN_ERR_SHAPE: return "ATTN_ERR_SHAPE: invalid or too large sizes";
    case ATTN_ERR_ALIGN: return "ATTN_ERR_ALIGN: a device pointer is not 16-byte aligned";
    case ATTN_ERR_UNSUPPORTED:
      return "ATTN_ERR_UNSUPPORTED: needs D == 64, 128 or 256 and an sm_100 device";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA: a CUDA call failed";
    case ATTN_ERR_DEVICE_TIMEOUT: return "ATTN_ERR_DEVICE_TIMEOUT: a kernel wait ran out";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE: device workspace too small";
    case ATTN_ERR_TOO_LARGE: return "ATTN_ERR_TOO_LARGE: more work than a fixed buffer holds";
  }
  return "ATTN_ERR_UNKNOWN";
}

uint64_t attn_set_wait_timeout_ns(uint64_t ns) {
  if (ns < 1000000ull) ns = 1000000ull;
  return g_timeout_ns.exchange(ns);
}

int attn_variant_count(void) { return kNumVariants; }

const char* attn_variant_name(int variant) {
  static char names[kNumVariants][64];
  static std::once_flag once;
  std::call_once(once, [] {
    static const char* kStructureNames[kStructures] = {
        "pingpong,row_pairs", "pingpong,head_pairs", "dbuf,softmax_split=1",
        "dbuf,softmax_split=2"};
    for (int v = 0; v < kNumVariants; ++v)
      std::snprintf(names[v], sizeof(names[v]), "%s,fma_exp2_pairs=%d/8",
                    kStructureNames[variant_structure(v)], variant_emu(v));
  });
  return (variant >= 0 && variant < kNumVariants) ? names[variant] : nullptr;
}

int attn_variant_select(int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal) {
  if (validate_sizes(B, Hq, Hkv, Sq, D, Sk, causal) != ATTN_OK) return -1;
  return select_variant(D, causal, Sk);
}

attn_status attn_fwd_variant(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal,
                             int variant, void* stream) {
  attn_status st = validate_pointers(q, k, v, o, lse);
  if (st != ATTN_OK) return st;
  st = validate_sizes(B, Hq, Hkv, Sq, D, Sk, causal);
  if (st != ATTN_OK) return st;
  if (variant < 0 || variant >= kNumVariants) return ATTN_ERR_UNSUPPORTED;
  int dev = 0;
  st = device_setup(&dev);
  if (st != ATTN_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  unsigned int* status = status_block(dev, cs, true);
  if (!status) return ATTN_ERR_CUDA;
  return launch_call(q, k, v, o, lse, status, B, Hq, Hkv, Sq, Sk, D, causal, variant, dev, cs);
}

attn_status attn_fwd_qk(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Sq, int Sk, int D, int causal, void* stream) {
  return attn_fwd_variant(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, D, causal,
                          select_variant(D, causal, Sk), stream);
}

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Hq, int Hkv, int S, int D, int causal, void* stream) {
  return attn_fwd_qk(q, k, v, o, lse, B, Hq, Hkv, S, S, D, causal, stream);
}

size_t attn_fwd_host_workspace_bytes(int B, int Hq, int Hkv, int S, int D) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || D < 1) return 0;
  const size_t q = static_cast<size_t>(B) * Hq * S * D * 2;
  const size_t kv = static_cast<size_t>(B) * Hkv * S * D * 2;
  const size_t l = static_cast<size_t>(B) * Hq * S * 4;
  return round256(q) * 2 + round256(kv) * 2 + round256(l);
}

attn_status attn_device_status_ex(void* stream, uint32_t* site, uint64_t* exact_items) {
  if (site) *site = 0;
  if (exact_items) *exact_items = 0;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return ATTN_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  unsigned int words[kStatusWords] = {0, 0, 0, 0};
  unsigned int* block = status_block(dev, cs, false);
  if (block && !drain_status_block(block, words)) return ATTN_ERR_CUDA;
  if (site) *site = words[1];
  if (exact_items) *exact_items = words[2];
  return status_of(words);
}

attn_status attn_device_status(void* stream, uint32_t* site) {
  return attn_device_status_ex(stream, site, nullptr);
}

attn_status attn_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* o_h,
                          float* lse_h, int B, int Hq, int Hkv, int S, int D, int causal,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!q_h || !k_h || !v_h || !o_h || !lse_h || !workspace) return ATTN_ERR_NULL;
  attn_status st = validate_sizes(B, Hq, Hkv, S, D);
  if (st != ATTN_OK) return st;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_ALIGN;
  const size_t need = attn_fwd_host_workspace_bytes(B, Hq, Hkv, S, D);
  if (workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  int dev = 0;
  st = device_setup(&dev);
  if (st != ATTN_OK) return st;
  // per batch element (BHSD: each b is one contiguous slice of every tensor)
  const size_t qb1 = static_cast<size_t>(Hq) * S * D * 2;
  const size_t kvb1 = static_cast<size_t>(Hkv) * S * D * 2;
  const size_t lb1 = static_cast<size_t>(Hq) * S * 4;
  char* w = static_cast<char*>(workspace);
  char* dq = w;
  char* dk = dq + round256(qb1 * B);
  char* dv = dk + round256(kvb1 * B);
  char* dout = dv + round256(kvb1 * B);
  char* dl = dout + round256(qb1 * B);
  const char* hq = static_cast<const char*>(q_h);
  const char* hk = static_cast<const char*>(k_h);
  const char* hv = static_cast<const char*>(v_h);
  char* ho = static_cast<char*>(o_h);
  char* hl = reinterpret_cast<char*>(lse_h);

  // Three-stage pipeline over chunks of the batch on this device's copy /
  // compute streams: uploads of chunk c+1 and downloads of chunk c-1 overlap
  // the kernels of chunk c (and each other: host links are full duplex).
  // Events order the stages per chunk and the whole call after the work
  // already on `stream`; `stream` waits for the last download.
  HostPipe* hp = host_pipe(dev);
  if (!hp) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> one_call(hp->busy);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int n_chunks = B < kHostChunks ? B : kHostChunks;
  cudaEvent_t ev[1 + 2 * kHostChunks + 1];
  int n_ev = 0;
  auto fail = [&](attn_status e) {
    cudaStreamSynchronize(hp->up);
    cudaStreamSynchronize(hp->comp);
    cudaStreamSynchronize(hp->down);
    for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);
    return e;
  };
  for (int i = 0; i < 2 + 2 * n_chunks; ++i) {
    if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess)
      return fail(ATTN_ERR_CUDA);
    ++n_ev;
  }
  cudaEvent_t ev_start = ev[0], ev_end = ev[1 + 2 * n_chunks];
  if (cudaEventRecord(ev_start, cs) != cudaSuccess ||
      cudaStreamWaitEvent(hp->up, ev_start, 0) != cudaSuccess)
    return fail(ATTN_ERR_CUDA);
  for (int c = 0; c < n_chunks; ++c) {
    const int b0 = static_cast<int>(static_cast<int64_t>(B) * c / n_chunks);
    const int b1 = static_cast<int>(static_cast<int64_t>(B) * (c + 1) / n_chunks);
    const int nb = b1 - b0;
    cudaEvent_t up_done = ev[1 + 2 * c], comp_done = ev[2 + 2 * c];
    if (cudaMemcpyAsync(dq + qb1 * b0, hq + qb1 * b0, qb1 * nb, cudaMemcpyHostToDevice,
                        hp->up) != cudaSuccess ||
        cudaMemcpyAsync(dk + kvb1 * b0, hk + kvb1 * b0, kvb1 * nb, cudaMemcpyHostToDevice,
                        hp->up) != cudaSuccess ||
        cudaMemcpyAsync(dv + kvb1 * b0, hv + kvb1 * b0, kvb1 * nb, cudaMemcpyHostToDevice,
                        hp->up) != cudaSuccess ||
        cudaEventRecord(up_done, hp->up) != cudaSuccess ||
        cudaStreamWaitEvent(hp->comp, up_done, 0) != cudaSuccess)
      return fail(ATTN_ERR_CUDA);
    st = attn_fwd(dq + qb1 * b0, dk + kvb1 * b0, dv + kvb1 * b0, dout + qb1 * b0,
                  reinterpret_cast<float*>(dl + lb1 * b0), nb, Hq, Hkv, S, D, causal, hp->comp);
    if (st != ATTN_OK) return fail(st);
    if (cudaEventRecord(comp_done, hp->comp) != cudaSuccess ||
        cudaStreamWaitEvent(hp->down, comp_done, 0) != cudaSuccess ||
        cudaMemcpyAsync(ho + qb1 * b0, dout + qb1 * b0, qb1 * nb, cudaMemcpyDeviceToHost,
                        hp->down) != cudaSuccess ||
        cudaMemcpyAsync(hl + lb1 * b0, dl + lb1 * b0, lb1 * nb, cudaMemcpyDeviceToHost,
                        hp->down) != cudaSuccess)
      return fail(ATTN_ERR_CUDA);
  }
  if (cudaEventRecord(ev_end, hp->down) != cudaSuccess ||
      cudaStreamWaitEvent(cs, ev_end, 0) != cudaSuccess)
    return fail(ATTN_ERR_CUDA);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return fail(ATTN_ERR_CUDA);
  // the kernels ran on the pipeline's compute stream: report its status
  st = attn_device_status(hp->comp, nullptr);
  for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);
  return st;
}

}  // extern "C"

namespace attn_b200 {
// One thread waits, with the kernels' bounded wait, on an mbarrier that no
// one arrives on, and records the timeout in `status`.
__global__ void selftest_wait_kernel(uint64_t timeout_ns, unsigned int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_addr(&bar), 0, &abort_flag, timeout_ns, status, 0x501);
}

// The fast pass's FMA-pipe exponential, evaluated elementwise (pairs).
__global__ void selftest_exp2_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], x[i])).x;
  }
}
}  // namespace attn_b200

extern "C" attn_status attn_selftest_exp2(const float* x, float* y, int n, void* stream) {
  if (!x || !y) return ATTN_ERR_NULL;
  if (n < 0) return ATTN_ERR_SHAPE;
  if (n == 0) return ATTN_OK;
  int dev = 0;
  attn_status st = device_setup(&dev);
  if (st != ATTN_OK) return st;
  const int pairs = (n + 1) / 2;
  selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

namespace attn_b200 {
__global__ void selftest_fastdiv_kernel(FastDiv f, const uint32_t* n, uint32_t* q, int count) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < count) q[i] = fast_div(n[i], f);
}
}  // namespace attn_b200

extern "C" attn_status attn_selftest_fastdiv(uint32_t d, const uint32_t* n, uint32_t* q,
                                             int count, int on_device, void* stream) {
  if (d == 0 || count < 0) return ATTN_ERR_SHAPE;
  if (count == 0) return ATTN_OK;
  if (!n || !q) return ATTN_ERR_NULL;
  const FastDiv f = make_fastdiv(d);
  if (!on_device) {
    for (int i = 0; i < count; ++i) q[i] = fast_div(n[i], f);
    return ATTN_OK;
  }
  int dev = 0;
  attn_status st = device_setup(&dev);
  if (st != ATTN_OK) return st;
  selftest_fastdiv_kernel<<<(count + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      f, n, q, count);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" attn_status attn_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
  int dev = 0;
  attn_status st = device_setup(&dev);
  if (st != ATTN_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  unsigned int* status = status_block(dev, cs, true);
  if (!status) return ATTN_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, cs>>>(timeout_ns, status);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return attn_device_status(stream, nullptr);
}

// ---------------------------------------------------------------------------
// attn_fwd_noalloc: the same launches as attn_fwd, with the call's status
// block in this file's fixed array instead of memory from cudaMalloc.
// ---------------------------------------------------------------------------
extern "C" attn_status attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                        float* lse, int B, int Hq, int Hkv, int S, int D,
                                        int causal, void* stream) {
  attn_status st = validate_pointers(q, k, v, o, lse);
  if (st != ATTN_OK) return st;
  st = validate_sizes(B, Hq, Hkv, S, D);
  if (st != ATTN_OK) return st;
  int dev = 0;
  st = device_setup(&dev);
  if (st != ATTN_OK) return st;
  unsigned int* scratch = noalloc_scratch(dev);
  if (!scratch) return ATTN_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return launch_call(q, k, v, o, lse, scratch, B, Hq, Hkv, S, S, D, causal,
                     select_variant(D, causal, S), dev, cs);
}

extern "C" attn_status attn_noalloc_status(void* stream, uint32_t* site, uint64_t* exact_items) {
  if (site) *site = 0;
  if (exact_items) *exact_items = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  unsigned int* scratch = noalloc_scratch(dev);
  if (!scratch) return ATTN_ERR_CUDA;
  unsigned int words[kStatusWords] = {0, 0, 0, 0};
  if (!drain_status_block(scratch, words)) return ATTN_ERR_CUDA;
  if (site) *site = words[1];
  if (exact_items) *exact_items = words[2];
  return status_of(words);
}
