/*
 * decoder_layer.h -- C ABI of the LLaMA3 single-decoder-layer forward proxy in
 *                    libattn_b200.so (the same library as attn.h).
 *
 * Operation.  The PipeThreader pages report, besides the attention operator,
 * an FP16 single decoder layer of LLaMA3-8B / 70B as a layer-level proxy
 * (papers.lqhl.me "PipeThreader-OSDI25", section 实验与结果, paper Sec. 6.3 /
 * Fig. 13).  The pages do not spell the layer out; the standard LLaMA3
 * pre-norm decoder layer is used, with causal self-attention over positions
 * 0..S-1 of each of the B sequences:
 *
 *   n1 = rmsnorm(x) * w_attn_norm         rmsnorm(r) = r / sqrt(mean(r^2) + eps)
 *   [q | k | v] = n1 W_qkv^T              (Hq, Hkv, Hkv heads of D columns)
 *   q, k <- rope(q), rope(k)              pair (i, i + D/2) at position s turns by
 *                                         s * rope_theta^(-2i/D), i < D/2
 *   o = attention(q, k, v), causal        (attn_fwd of attn.h, GQA)
 *   h = x + o W_o^T
 *   n2 = rmsnorm(h) * w_mlp_norm
 *   y = h + (silu(n2 W_gate^T) * (n2 W_up^T)) W_down^T,   silu(a) = a / (1 + e^-a)
 *
 * Precision: fp16 tensors between the steps (n1, q/k/v, o, h, n2, the
 * gate/up products, the SwiGLU output, y), each step computed in fp32 and
 * rounded once; GEMMs accumulate in fp32; the attention is attn_fwd's.
 *
 * Layouts (dense, row-major, fp16, 16-byte aligned):
 *   x, y        [B, S, hidden]                  token-major activations
 *   w_attn_norm, w_mlp_norm [hidden]
 *   w_qkv       [(Hq + 2*Hkv) * D, hidden]      rows: Hq query heads, then Hkv key
 *                                               heads, then Hkv value heads, D each
 *   w_o         [hidden, Hq * D]
 *   w_gate_up   [2 * inter, hidden]             rows: inter gate rows, then inter up rows
 *   w_down      [hidden, inter]
 * Sizes: B, S >= 1; hidden and inter multiples of 8; Hq % Hkv == 0; D 64 or
 * 128; eps >= 0; rope_theta > 1 (LLaMA3: eps 1e-5, theta 500000).
 *
 * The GEMMs are this library's tcgen05 kernel (2-SM tensor-core tiles of
 * 256 x 256, fp16 in, fp32 accumulation), with the element steps fused into
 * their epilogues: RoPE and the head split into the QKV projection, SwiGLU
 * into the gate/up projection, the residual adds into the O and down
 * projections; the O projection reads the attention output head-major when
 * S % 128 == 0 (otherwise a head-merge kernel runs first).  Each fused step
 * rounds where the unfused layer stores a tensor, so the stored values are
 * those of the sequence above.  RMSNorm is a separate kernel and the
 * attention is attn_fwd.  Each call launches them in order on `stream`.
 * Their bounded waits report into the stream's status block, like
 * attn_fwd's (read with attn_device_status()).
 */
#ifndef ATTN_B200_DECODER_LAYER_H
#define ATTN_B200_DECODER_LAYER_H

#include <stddef.h>

#include "attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * attn_decoder_layer_workspace_bytes -- bytes of device workspace that
 * attn_decoder_layer_fwd needs for these sizes (all intermediates: the rotary
 * table, RMSNorm outputs, Q/K/V/O head-major, LSE, the residual stream h and
 * the SwiGLU output; each region rounded up to 256 bytes).  Returns 0 for
 * sizes attn_decoder_layer_fwd rejects.
 */
size_t attn_decoder_layer_workspace_bytes(int B, int S, int hidden, int Hq, int Hkv, int D,
                                          int inter);

/*
 * attn_decoder_layer_fwd -- one LLaMA3 decoder layer forward on device buffers.
 *   x      : device, input activations (read only); y may equal x (in place).
 *   w_*    : device, weights as laid out above (read only).
 *   y      : device, output activations.
 *   workspace: device, >= attn_decoder_layer_workspace_bytes(...) bytes,
 *              256-byte aligned, not overlapping x, y or the weights; its
 *              contents are overwritten.
 *   stream : cudaStream_t to launch on (asynchronous).
 * Returns ATTN_OK once everything is enqueued; ATTN_ERR_NULL, ATTN_ERR_SHAPE
 * (sizes, eps, theta), ATTN_ERR_UNSUPPORTED (D), ATTN_ERR_ALIGN,
 * ATTN_ERR_WORKSPACE before launching anything; ATTN_ERR_CUDA when a launch
 * fails; the attention's status otherwise.  After a failure past validation,
 * earlier steps may already be enqueued: y and the workspace are then
 * undefined.  A timed-out wait in any of the kernels is reported by
 * attn_device_status() on `stream`.
 */
attn_status attn_decoder_layer_fwd(const void* x, const void* w_attn_norm, const void* w_qkv,
                                   const void* w_o, const void* w_mlp_norm, const void* w_gate_up,
                                   const void* w_down, void* y, int B, int S, int hidden, int Hq,
                                   int Hkv, int D, int inter, float eps, float rope_theta,
                                   void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_DECODER_LAYER_H */
