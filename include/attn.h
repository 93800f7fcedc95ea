/*
 * attn.h -- C ABI of the B200 (sm_100a) fused attention forward library
 *           libattn_b200.so.
 *
 * Operation (attn_fwd).  Scaled dot-product attention with grouped-query
 * heads and an optional causal mask, computed in one fused pass that never
 * writes the S x S score matrix to memory.  This is the FlashAttention forward
 * that the PipeThreader pages evaluate on LLaMA3-8B/70B head shapes, SEQ
 * 512-8k and batch 1/64 (papers.lqhl.me "PipeThreader-OSDI25", section
 * 实验与结果, paper Sec. 6.2 / Fig. 12), and whose TMA-load / tensor-core /
 * CUDA-core task split those pages describe (section 核心方法, "sTask / sEU").
 * The pages do not print the formula; the textbook definition is used:
 *
 *   g          = hq / (Hq / Hkv)            (contiguous groups of query heads)
 *   s_ij       = <Q[b,hq,i,:], K[b,g,j,:]> / sqrt(D),  j in A(i)
 *   A(i)       = {0..i} if causal else {0..S-1}
 *   O[b,hq,i,:] = sum_j softmax_j(s_i.) V[b,g,j,:]
 *   LSE[b,hq,i] = ln sum_{j in A(i)} exp(s_ij)   (natural log, scaled logits)
 *
 * Precision: Q, K, V and O are IEEE fp16; products accumulate in fp32; the
 * probabilities feed the second product as fp16; LSE is fp32.
 *
 * Conventions shared by every entry point:
 *   - Layouts are dense row-major: Q, O [B, Hq, S, D]; K, V [B, Hkv, S, D];
 *     LSE [B, Hq, S].  "Device" pointers are CUDA device (or managed)
 *     addresses on the current device; "host" pointers are CPU addresses.
 *   - The caller owns every input and output buffer; the library keeps no
 *     pointer to them after returning.  Besides those, the kernels of a call
 *     write a 16-byte status block (error flags, the first wait that ran out,
 *     a count of recomputed work items).  The first call for each (device,
 *     stream) pair allocates that block with cudaMalloc and zeroes it on the
 *     stream; it is kept for later calls until the process exits.  The
 *     legacy default stream (NULL) is one stream for every host thread;
 *     cudaStreamPerThread is a different stream in each host thread, so it
 *     gets one block per (device, thread).  Nothing else allocates.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous with respect to the host unless stated otherwise.
 *   - Arguments are validated before anything is launched; a rejected call
 *     launches nothing and leaves the outputs untouched.
 *   - Every wait inside the kernels is bounded in time.  A wait that runs out
 *     makes the kernel stop early (without faulting) and records
 *     ATTN_ERR_DEVICE_TIMEOUT in the status block of the stream it ran on,
 *     read back with attn_device_status().
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_NULL = 1,           /* a required pointer is NULL */
  ATTN_ERR_SHAPE = 2,          /* B,Hq,Hkv,S < 1, Hq % Hkv != 0, or a size overflows */
  ATTN_ERR_ALIGN = 3,          /* q, k, v, o not 16-byte aligned, or lse not 4-byte aligned */
  ATTN_ERR_UNSUPPORTED = 4,    /* D not 64, 128 or 256, or not an sm_100 device */
  ATTN_ERR_CUDA = 5,           /* a CUDA runtime / driver call failed */
  ATTN_ERR_DEVICE_TIMEOUT = 6, /* a kernel wait ran out; results are invalid */
  ATTN_ERR_WORKSPACE = 7,      /* the device workspace given is too small */
  ATTN_ERR_TOO_LARGE = 8       /* more work than a fixed buffer holds (kept for ABI
                                  stability; no entry point of this version returns it) */
} attn_status;

/*
 * attn_fwd -- fused attention forward on device buffers.
 *   q   : device, fp16 [B, Hq, S, D], 16-byte aligned, read only.
 *   k, v: device, fp16 [B, Hkv, S, D], 16-byte aligned, read only.
 *   o   : device, fp16 [B, Hq, S, D], 16-byte aligned, written.
 *   lse : device, fp32 [B, Hq, S], 4-byte aligned, written (must not be NULL).
 *   B, Hq, Hkv, S, D: sizes; Hq % Hkv == 0; D == 64, 128 or 256; any S >= 1 (a
 *   last block of fewer than 128 rows is computed with the keys past S
 *   masked).
 *   causal: nonzero for the causal mask j <= i (square, Sq == Sk == S).
 *   stream: cudaStream_t to launch on.
 * Returns ATTN_OK once the kernel is enqueued; errors as listed above.  The
 * outputs must not overlap the inputs.  One kernel runs on `stream` (a call
 * with more than 2048 work items per SM is split into launches over batch
 * ranges).  Each CTA of it computes its work items (256 query rows: two
 * 128-row tiles of one head or of two heads of a group; or 128 rows) with
 * fp16 probabilities, then recomputes, with the probabilities split into two
 * fp16 parts, the 128-row tiles that have a row with max|O| >= 3.98, where
 * fp16 output rounding leaves almost no error budget;
 * attn_device_status_ex() reports how many items had such a tile.
 */
attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int Hq, int Hkv, int S, int D, int causal, void* stream);

/*
 * attn_fwd_qk -- attn_fwd with Sq query rows over Sk keys (Sq != Sk allowed).
 * Not in the pages, which evaluate Sq == Sk only: needed for a prefill over a
 * cached key prefix (Sq < Sk) and for non-causal cross attention.
 *   q, o: [B, Hq, Sq, D]; k, v: [B, Hkv, Sk, D]; lse: [B, Hq, Sq].
 *   causal: query i sees keys j <= i + (Sk - Sq) (aligned at the bottom right:
 *   the last query sees every key); requires Sq <= Sk (ATTN_ERR_SHAPE
 *   otherwise, as a query would see no key).  Non-causal: any Sq, Sk >= 1.
 * Everything else (pointers, alignment, D, streams, launches, errors) is as
 * for attn_fwd, which is attn_fwd_qk with Sq == Sk == S.
 */
attn_status attn_fwd_qk(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal,
                        void* stream);

/*
 * Fused-pass variants and their measured selection.  The pages' central idea
 * is that the best tiling / pipeline choice of an attention kernel is found by
 * profiling candidates on the target GPU (PipeThreader pages, sections 核心方法
 * and 设计取舍: a joint tile + pipeline search whose greedy choices are checked
 * by profiling); this library keeps that idea as a small build-time table.
 * The fused pass is compiled in attn_variant_count() variants, the product of
 * two axes.  The pipeline structure (variant v, structure v / 5):
 *   0 "pingpong,row_pairs"   two 128-row tiles of one query head (256 rows)
 *                            take turns on the tensor core, 128-key blocks;
 *   1 "pingpong,head_pairs"  the same schedule with the two tiles on the same
 *                            128 rows of two query heads of one group (falls
 *                            back to row pairs when Hq/Hkv is odd);
 *   2 "dbuf,softmax_split=1" one 128-row tile, S double-buffered in TMEM so
 *                            the softmax of one key block overlaps the MMAs
 *                            of the next (64-key blocks at D = 256);
 *   3 "dbuf,softmax_split=2" as 2, with two softmax warps per row, each on
 *                            half of a key block.
 * At D = 256 every structure runs as structure 2.  The second
 * axis, N = v % 5 ("fma_exp2_pairs=N/8"), is how many of every 16
 * exponentials of the softmax an FMA-pipe polynomial evaluates instead of the
 * MUFU unit (relative error 8e-5, well inside the fp16 rounding of P).  The
 * structures change the work order, not the arithmetic of a row.  The
 * package's tuner
 * (python -m dnn_compiler_pipelining_b200.tune) times every variant per
 * shape class on a B200 and writes the table compiled into the library;
 * attn_fwd, attn_fwd_qk, attn_fwd_host and attn_fwd_noalloc run the variant
 * the table picks.  The exact pass takes every exponential from the MUFU
 * unit in every variant.
 *
 * attn_variant_count -- number of compiled fused-pass variants (>= 1).
 * attn_variant_name  -- static, human-readable name of a variant; NULL when
 *                       `variant` is out of range.
 * attn_variant_select -- the variant the table picks for these sizes, or -1
 *                       when attn_fwd_qk would reject them (ATTN_ERR_SHAPE or
 *                       ATTN_ERR_UNSUPPORTED).  Pure host code: no device is
 *                       touched.
 * attn_fwd_variant   -- attn_fwd_qk running the given fused-pass variant
 *                       (0 <= variant < attn_variant_count(), else
 *                       ATTN_ERR_UNSUPPORTED, checked after the sizes); for
 *                       the tuner and tests.  Arguments, layouts and errors
 *                       otherwise as attn_fwd_qk.
 */
int attn_variant_count(void);
const char* attn_variant_name(int variant);
int attn_variant_select(int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal);
attn_status attn_fwd_variant(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int Hq, int Hkv, int Sq, int Sk, int D, int causal,
                             int variant, void* stream);

/*
 * attn_fwd_host_workspace_bytes -- size in bytes of the device workspace that
 * attn_fwd_host needs for these sizes (Q, K, V, O and LSE, each rounded up to
 * 256 bytes).  Returns 0 for invalid sizes.
 */
size_t attn_fwd_host_workspace_bytes(int B, int Hq, int Hkv, int S, int D);

/*
 * attn_fwd_host -- the same operation on HOST buffers, for callers whose data
 * live in CPU memory.  q_h, k_h, v_h (fp16, layouts as above) are copied into
 * the caller's device workspace, attn_fwd runs there, and O and LSE are
 * copied back into o_h (fp16) and lse_h (fp32).  The work runs as a pipeline
 * over up to 16 chunks of the batch on the library's own per-device streams
 * (uploads, kernels, downloads), so copies of one chunk overlap the kernels
 * of another; it starts after the work already enqueued on `stream`, `stream`
 * waits for it, and the call synchronizes `stream` before it returns, so the
 * host buffers hold the results on ATTN_OK.  Host buffers may be pageable or
 * pinned (pinned copies run asynchronously and faster).  The library creates
 * those three streams on its first call for each device and keeps them.
 * Concurrent calls on one device (from several host threads) run one after
 * another, so each call's status is its own.
 *   workspace: device, >= attn_fwd_host_workspace_bytes(...) bytes, 256-byte
 *              aligned; its contents are overwritten.
 * Also returns ATTN_ERR_DEVICE_TIMEOUT if the kernel reported one.
 */
attn_status attn_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* o_h,
                          float* lse_h, int B, int Hq, int Hkv, int S, int D, int causal,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_device_status -- synchronizes `stream`, then reads and clears the
 * status block of `stream` on the current device (per calling thread for
 * cudaStreamPerThread).  Returns ATTN_ERR_DEVICE_TIMEOUT if a kernel of this
 * library launched on that stream recorded a timed-out wait since the last
 * read, ATTN_ERR_CUDA if synchronizing or reading failed, else ATTN_OK.
 * Calls on other streams are not reported here.  `site`, if not NULL,
 * receives the first recorded wait site (0 when none).
 */
attn_status attn_device_status(void* stream, uint32_t* site);

/*
 * attn_device_status_ex -- attn_device_status, plus `exact_items` (if not
 * NULL): the number of work items (256 or 128 query rows of a head) of which
 * the kernels on `stream` recomputed at least one 128-row tile with two-part
 * probabilities since the last read.
 */
attn_status attn_device_status_ex(void* stream, uint32_t* site, uint64_t* exact_items);

/*
 * attn_set_wait_timeout_ns -- bound, in nanoseconds, on every wait inside the
 * kernels launched afterwards from this process (default 2e9 = 2 s; values
 * below 1e6 are raised to 1e6).  Returns the previous value.
 */
uint64_t attn_set_wait_timeout_ns(uint64_t ns);

/*
 * attn_selftest_wait_timeout -- launches one CTA that waits on an mbarrier
 * nothing will ever complete, with a bound of timeout_ns, using the same
 * bounded-wait routine as the attention kernels.  Synchronizes `stream` and
 * returns what attn_device_status() then reports (ATTN_ERR_DEVICE_TIMEOUT when
 * the bound works).  The GPU context stays usable afterwards.
 */
attn_status attn_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

/*
 * attn_fwd_noalloc -- attn_fwd for callers that must not allocate device
 * memory.  No counterpart in the paper: it exists for library users, not for
 * the method.  Besides the caller's buffers, the kernel of a call writes a
 * 16-byte status block; attn_fwd creates one per (device, stream) with
 * cudaMalloc on first use, and some callers cannot allow that: serving
 * engines that reserve all device memory up front for their caches,
 * frameworks whose own caching allocator must see every byte, or
 * latency-bound loops where cudaMalloc's implicit device synchronization or a
 * late out-of-memory failure is unacceptable.  This entry point uses a fixed
 * array inside the library instead (16 bytes per device, reserved when the
 * library is loaded and held until the process exits), and calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *   Arguments, layouts, results and errors: as attn_fwd; the same kernels
 *   run, so outputs are bit-identical to attn_fwd's.
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before capturing work into a stream graph.
 *   Sharing: every call on a device writes the same array, which accumulates
 *   until attn_noalloc_status() reads and clears it.  Calls that overlap on
 *   the GPU (different streams, or host threads without ordering) mix their
 *   reports there, so a timeout cannot be attributed to one of them.
 */
attn_status attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int Hq, int Hkv, int S, int D, int causal, void* stream);

/*
 * attn_noalloc_status -- synchronizes `stream`, then reads and clears the
 * fixed status array of attn_fwd_noalloc on the current device: status as
 * attn_device_status (ATTN_ERR_DEVICE_TIMEOUT if any such call timed out
 * since the last read), `site` and `exact_items` (if not NULL) as
 * attn_device_status_ex.  Allocates nothing.
 */
attn_status attn_noalloc_status(void* stream, uint32_t* site, uint64_t* exact_items);

/*
 * attn_selftest_exp2 -- evaluates, on the device, the polynomial 2^x that
 * the fused pass uses for part of its exponentials (so tests can check it
 * against a reference exp2).  x, y: device fp32 arrays of n elements
 * (y = 2^x for x <= 8; x below -126 gives a non-negative value below 2^-125).
 * Asynchronous on `stream`.
 */
attn_status attn_selftest_exp2(const float* x, float* y, int n, void* stream);

/*
 * attn_selftest_fastdiv -- the division by a launch-time constant that the
 * kernels use to decode their work items (a multiply-high and a shift in
 * place of the hardware divide; Granlund and Montgomery, "Division by
 * invariant integers using multiplication", PLDI 1994): q[i] = n[i] / d for
 * count values 0 <= n[i] < 2^31, d >= 1.  on_device = 0: n and q are host
 * arrays and the host evaluates the same arithmetic, synchronously;
 * on_device = 1: device arrays, evaluated by a kernel on `stream`
 * (asynchronous).  ATTN_ERR_SHAPE for d == 0 or count < 0.
 */
attn_status attn_selftest_fastdiv(uint32_t d, const uint32_t* n, uint32_t* q, int count,
                                  int on_device, void* stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char* attn_status_string(attn_status status);

/* Library ABI version: (major << 16) | minor. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
