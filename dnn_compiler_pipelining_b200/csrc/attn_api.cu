// attn_api.cu -- C ABI of libattn_b200.so (declared in include/attn.h):
// argument validation, TMA tensor-map encoding, kernel launch, the
// per-device status word, the host-buffer entry point and the bounded-wait
// self-test.  The only device memory it allocates is the redo list of each
// (device, stream) pair, once, on first use.
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
#include <utility>

#include "attn.h"
#include "attn_fwd_pair_sm100.cuh"
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

// Per-device one-time setup: architecture check and the kernel's shared
// memory opt-in.  0 = not done, 1 = ok, 2 = unsupported device.
std::atomic<int> g_dev_state[kMaxDevices];
int g_dev_sms[kMaxDevices];
int g_dev_pairs[kMaxDevices];  // 2-CTA clusters of the pair kernel resident at once
std::mutex g_dev_mutex;

// Redo lists (items the fast pass hands to the hi+lo pass), one per
// (device, stream): launches on one stream run in order, so a list is never
// shared by launches that could overlap.
constexpr unsigned int kRedoCapacity = 1u << 16;
std::map<std::pair<int, cudaStream_t>, unsigned int*> g_redo_lists;
std::mutex g_redo_mutex;

size_t redo_bytes() { return (kRedoHeaderWords + kRedoCapacity) * sizeof(unsigned int); }

// Returns the list for (dev, stream), allocating and zeroing it (on that
// stream) the first time.
unsigned int* redo_list(int dev, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_redo_mutex);
  auto key = std::make_pair(dev, stream);
  auto it = g_redo_lists.find(key);
  if (it != g_redo_lists.end()) return it->second;
  void* ptr = nullptr;
  if (cudaMalloc(&ptr, redo_bytes()) != cudaSuccess) return nullptr;
  if (cudaMemsetAsync(ptr, 0, redo_bytes(), stream) != cudaSuccess) {
    cudaFree(ptr);
    return nullptr;
  }
  g_redo_lists[key] = static_cast<unsigned int*>(ptr);
  return static_cast<unsigned int*>(ptr);
}

// Which kernel runs the fused pass: the single-CTA kernel (attn_fwd_kernel<0>)
// or the CTA-pair kernel (pair::attn_fwd_pair_kernel), which computes the
// same items and passes the same parity tests but measured slower on B200
// (793 vs 1003 TFLOP/s at B=64, S=8192, causal).
constexpr bool kPairFusedPass = false;

// the kernel checks 1 KiB alignment of the dynamic shared memory base
size_t fwd_smem_bytes(int D = kHeadDim) {
  return D == 64 ? sizeof(SharedFwdT<64>) : sizeof(SharedFwdT<128>);
}
size_t pair_smem_bytes() { return sizeof(pair::SharedPair); }

// The fused-pass kernels of one head dimension, indexed by variant
// (kEmuChoices[variant] FMA-pipe exponentials per 8 column pairs).
using FwdKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                           const FwdParams);
template <int kD, int... kV>
std::array<FwdKernel, sizeof...(kV)> fused_kernels(std::integer_sequence<int, kV...>) {
  return {{&attn_fwd_kernel<0, kD, kEmuChoices[kV]>...}};
}
template <int kD>
FwdKernel fused_kernel(int variant) {
  static const std::array<FwdKernel, kNumVariants> table =
      fused_kernels<kD>(std::make_integer_sequence<int, kNumVariants>{});
  return table[variant];
}

// Measured choice of fused-pass variant per shape class: rules
// (D, causal, smallest Sk, largest Sk, variant), first match wins, no match
// -> variant 0.  The rows are written by the package's tuner from timings of
// every variant on B200.
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

template <int kD>
bool set_smem_attributes() {
  const int bytes = static_cast<int>(fwd_smem_bytes(kD));
  for (int v = 0; v < kNumVariants; ++v)
    if (cudaFuncSetAttribute(fused_kernel<kD>(v), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess)
      return false;
  return cudaFuncSetAttribute(attn_fwd_kernel<1, kD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              bytes) == cudaSuccess;
}

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
        cudaSuccess)
      return ATTN_ERR_CUDA;
    if (!set_smem_attributes<128>() || !set_smem_attributes<64>() ||
        cudaFuncSetAttribute(pair::attn_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(pair_smem_bytes())) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (kPairFusedPass) {
      // a persistent grid of as many CTA pairs as can be resident together
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (g_dev_sms[dev] / 2));
      cfg.blockDim = dim3(pair::kThreads);
      cfg.dynamicSmemBytes = pair_smem_bytes();
      int pairs = 0;
      if (cudaOccupancyMaxActiveClusters(&pairs, pair::attn_fwd_pair_kernel, &cfg) !=
              cudaSuccess ||
          pairs < 1)
        return ATTN_ERR_CUDA;
      g_dev_pairs[dev] = pairs;
    }
    g_dev_state[dev].store(1, std::memory_order_release);
  }
  return g_dev_state[dev].load() == 1 ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

// 2-D view [rows, D] fp16 of a dense [.., S, D] tensor; 64 x box_rows boxes
// (one 128-byte swizzle panel).
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

// Streams of attn_fwd_host's copy / compute pipeline, created once per device
// (non-blocking, so they do not serialize with the legacy default stream).
constexpr int kHostChunks = 16;
struct HostPipe {
  cudaStream_t up, comp, down;
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

attn_status validate_sizes(int B, int Hq, int Hkv, int S, int D, int Sk = -1, int causal = 0) {
  if (Sk < 0) Sk = S;
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || Sk < 1 || D < 1) return ATTN_ERR_SHAPE;
  if (Hq % Hkv != 0) return ATTN_ERR_SHAPE;
  // a causal query with no visible key (Sq > Sk) has no softmax
  if (causal && S > Sk) return ATTN_ERR_SHAPE;
  if (static_cast<int64_t>(B) * Hkv * Sk >= (int64_t(1) << 31)) return ATTN_ERR_SHAPE;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  // row indices are 32-bit signed in the kernel and in TMA coordinates
  const int64_t q_rows = static_cast<int64_t>(B) * Hq * S;
  if (q_rows >= (int64_t(1) << 31)) return ATTN_ERR_SHAPE;
  if (Hq > 65535 || B > 65535) return ATTN_ERR_SHAPE;  // grid y / z limits
  return ATTN_OK;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Kernel parameters of one call (Sq query rows over Sk keys).
FwdParams make_params(void* o, float* lse, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                      int causal) {
  FwdParams p;
  p.o = static_cast<__half*>(o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = Sq;
  p.Sk = Sk;
  p.causal = causal ? 1 : 0;
  p.off = causal ? Sk - Sq : 0;
  p.n_qb = (Sq + kBlockM - 1) / kBlockM;
  p.n_kb = (Sk + kBlockN - 1) / kBlockN;
  p.s_tail = Sq - (p.n_qb - 1) * kBlockM;
  p.n_qb2 = (p.n_qb + 1) / 2;
  p.group = Hq / Hkv;
  p.n_items = B * Hq * p.n_qb2;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  p.timeout_ns = g_timeout_ns.load();
  return p;
}

// Tensor maps of one call: Q and V in 128-row boxes, K in 64-row boxes (the
// pair pass loads half a key block per CTA) and 128-row boxes (redo pass).
struct CallMaps {
  CUtensorMap q, k, k_half, v;
};

bool encode_call_maps(CallMaps* m, const void* q, const void* k, const void* v, int B, int Hq,
                      int Hkv, int Sq, int Sk, int D) {
  const uint64_t q_rows = static_cast<uint64_t>(B) * Hq * Sq;
  const uint64_t kv_rows = static_cast<uint64_t>(B) * Hkv * Sk;
  return encode_rows_map(&m->q, q, q_rows, D) && encode_rows_map(&m->k, k, kv_rows, D) &&
         encode_rows_map(&m->k_half, k, kv_rows, D, kBlockM / 2) &&
         encode_rows_map(&m->v, v, kv_rows, D);
}

// The fused pass over every item (in the given variant), then the hi+lo pass
// over the items it listed.
template <int kD>
attn_status launch_passes_d(const CallMaps& m, const FwdParams& p, int variant, int dev,
                            cudaStream_t cs) {
  const int sms = g_dev_sms[dev];
  // the pair kernel takes D = 128, Sq == Sk and whole 128-row blocks only
  if (kPairFusedPass && kD == 128 && p.S == p.Sk && p.s_tail == kBlockM) {
    const int pairs = p.n_items < g_dev_pairs[dev] ? p.n_items : g_dev_pairs[dev];
    pair::attn_fwd_pair_kernel<<<2 * pairs, pair::kThreads, pair_smem_bytes(), cs>>>(
        m.q, m.k_half, m.v, p);
  } else {
    fused_kernel<kD>(variant)<<<p.n_items < sms ? p.n_items : sms, kThreads, fwd_smem_bytes(kD),
                                cs>>>(m.q, m.k, m.v, p);
  }
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  attn_fwd_kernel<1, kD><<<sms, kThreads, fwd_smem_bytes(kD), cs>>>(m.q, m.k, m.v, p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

attn_status launch_passes(const CallMaps& m, const FwdParams& p, int D, int variant, int dev,
                          cudaStream_t cs) {
  return D == 64 ? launch_passes_d<64>(m, p, variant, dev, cs)
                 : launch_passes_d<128>(m, p, variant, dev, cs);
}

}  // namespace
}  // namespace attn_b200

using namespace attn_b200;

extern "C" {

int attn_version(void) { return (1 << 16) | 0; }

const char* attn_status_string(attn_status s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_NULL: return "ATTN_ERR_NULL: a required pointer is NULL";
    case ATTN_ERR_SHAPE: return "ATTN_ERR_SHAPE: invalid or too large sizes";
    case ATTN_ERR_ALIGN: return "ATTN_ERR_ALIGN: a device pointer is not 16-byte aligned";
    case ATTN_ERR_UNSUPPORTED:
      return "ATTN_ERR_UNSUPPORTED: needs D == 64 or 128 and an sm_100 device";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA: a CUDA call failed";
    case ATTN_ERR_DEVICE_TIMEOUT: return "ATTN_ERR_DEVICE_TIMEOUT: a kernel wait ran out";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE: device workspace too small";
    case ATTN_ERR_TOO_LARGE:
      return "ATTN_ERR_TOO_LARGE: B*Hq*ceil(S/256) exceeds attn_fwd_noalloc's fixed scratch "
             "(131072 work items)";
  }
  return "ATTN_ERR_UNKNOWN";
}

uint64_t attn_set_wait_timeout_ns(uint64_t ns) {
  if (ns < 1000000ull) ns = 1000000ull;
  return g_timeout_ns.exchange(ns);
}

int attn_variant_count(void) { return kNumVariants; }

const char* attn_variant_name(int variant) {
  static char names[kNumVariants][48];
  static std::once_flag once;
  std::call_once(once, [] {
    for (int v = 0; v < kNumVariants; ++v)
      std::snprintf(names[v], sizeof(names[v]), "fma_exp2_pairs=%d/8", kEmuChoices[v]);
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
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
  attn_status st = validate_sizes(B, Hq, Hkv, Sq, D, Sk, causal);
  if (st != ATTN_OK) return st;
  if (variant < 0 || variant >= kNumVariants) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return ATTN_ERR_ALIGN;
  int dev = 0;
  st = device_setup(&dev);
  if (st != ATTN_OK) return st;

  CallMaps maps;
  if (!encode_call_maps(&maps, q, k, v, B, Hq, Hkv, Sq, Sk, D)) return ATTN_ERR_CUDA;
  FwdParams p = make_params(o, lse, B, Hq, Hkv, Sq, Sk, D, causal);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  p.redo = redo_list(dev, cs);
  if (!p.redo) return ATTN_ERR_CUDA;
  p.redo_capacity = kRedoCapacity;

  return launch_passes(maps, p, D, variant, dev, cs);
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

attn_status attn_device_status(void* stream, uint32_t* site) {
  if (site) *site = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned int words[2] = {0, 0};
  if (cudaMemcpyFromSymbol(words, g_attn_status, sizeof(words)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (words[0] != 0 || words[1] != 0) {
    const unsigned int zero[2] = {0, 0};
    if (cudaMemcpyToSymbol(g_attn_status, zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (site) *site = words[1];
  if (words[0] & kStatusSmemAlign) return ATTN_ERR_CUDA;
  return (words[0] & kStatusTimeout) ? ATTN_ERR_DEVICE_TIMEOUT : ATTN_OK;
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
  st = attn_device_status(stream, nullptr);
  for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);
  return st;
}

}  // extern "C"

namespace attn_b200 {
// One thread waits, with the kernels' bounded wait, on an mbarrier that no
// one arrives on.
__global__ void selftest_wait_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_addr(&bar), 0, &abort_flag, timeout_ns, 0x501);
}
}  // namespace attn_b200

namespace attn_b200 {
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

extern "C" attn_status attn_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
  int dev = 0;
  attn_status st = device_setup(&dev);
  if (st != ATTN_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  return attn_device_status(stream, nullptr);
}

// ---------------------------------------------------------------------------
// attn_fwd_noalloc: the same two launches as attn_fwd, with the redo list in
// a fixed array of this file instead of memory from cudaMalloc.
// ---------------------------------------------------------------------------
namespace attn_b200 {
namespace {

constexpr unsigned int kNoAllocMaxItems = 1u << 17;  // 131072 items: 512 KiB of ids

// Header {count, done, -, -} then up to kNoAllocMaxItems item ids.  Every
// device that loads the library holds one copy until the process exits.
static __device__ __align__(256) unsigned int g_noalloc_redo[kRedoHeaderWords + kNoAllocMaxItems];

// Device address of g_noalloc_redo, looked up once per device with that
// device current (host code cannot use the symbol itself as an address).
unsigned int* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mutex;

unsigned int* noalloc_scratch(int dev) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_redo) != cudaSuccess || !ptr) return nullptr;
    g_noalloc_ptr[dev] = static_cast<unsigned int*>(ptr);
  }
  return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace attn_b200

extern "C" attn_status attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                        float* lse, int B, int Hq, int Hkv, int S, int D,
                                        int causal, void* stream) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
  attn_status st = validate_sizes(B, Hq, Hkv, S, D);
  if (st != ATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return ATTN_ERR_ALIGN;
  const int n_qb = (S + kBlockM - 1) / kBlockM;
  const int n_qb2 = (n_qb + 1) / 2;
  const long long n_items = static_cast<long long>(B) * Hq * n_qb2;
  if (n_items > kNoAllocMaxItems) return ATTN_ERR_TOO_LARGE;
  int dev = 0;
  st = device_setup(&dev);
  if (st != ATTN_OK) return st;
  unsigned int* scratch = noalloc_scratch(dev);
  if (!scratch) return ATTN_ERR_CUDA;

  CallMaps maps;
  if (!encode_call_maps(&maps, q, k, v, B, Hq, Hkv, S, S, D)) return ATTN_ERR_CUDA;

  FwdParams p = make_params(o, lse, B, Hq, Hkv, S, S, D, causal);
  p.redo = scratch;
  p.redo_capacity = kNoAllocMaxItems;  // >= n_items: the list cannot overflow
  cudaStream_t cs = static_cast<cudaStream_t>(stream);

  // the shared array keeps the previous call's header: start from an empty list
  if (cudaMemsetAsync(scratch, 0, kRedoHeaderWords * sizeof(unsigned int), cs) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return launch_passes(maps, p, D, select_variant(D, causal, S), dev, cs);
}
