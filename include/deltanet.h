/* deltanet.h -- C ABI of libmoe.so's Gated DeltaNet decode step: one token of
 * the gated delta-rule recurrence for every sequence and value head.
 *
 * What it computes.  "Perplexity's Lily: A Breakthrough Local Inference
 * Engine Tailored Exclusively for Apple Silicon", section "The Model:
 * Qwen3.6-35B-A3B in Focus": besides its attention layers the model has 30
 * Gated DeltaNet layers whose recurrence keeps a fixed-size state.  The
 * pages give no formula; the step is the published gated delta rule (Yang,
 * Kautz and Hatamizadeh, "Gated Delta Networks: Improving Mamba2 with Delta
 * Rule"), for value head hv of sequence b with key head hk = hv / (Hv / Hk):
 *
 *   k^ = k / sqrt(|k|^2 + 1e-6),   q^ = q / sqrt(|q|^2 + 1e-6) / sqrt(dk),
 *   alpha = exp(g),
 *   S' = S (alpha (I - beta k^ k^T)) + beta v k^T     (S: dv x dk)
 *   o  = S' q^
 *
 * evaluated row by row as S'_i = alpha S_i + u_i k^ with
 * u_i = beta (v_i - alpha S_i . k^), and o_i = alpha S_i . q^ + u_i (k^ . q^)
 * (the same quantity; the state row is read once).
 *
 * Storage (DEVICE pointers; bf16 as 16-bit patterns):
 *   q, k    bf16 [B][Hk][dk]
 *   v       bf16 [B][Hv][dv]
 *   g, beta FP32 [B][Hv]    (g: log-decay, alpha = exp(g))
 *   state   FP32 [B][Hv][dv][dk], updated in place (row i of S is dk
 *           contiguous floats)
 *   out     bf16 [B][Hv][dv]
 *
 * Arithmetic: FP32 throughout (norms with IEEE square root and division,
 * dot products over dk in a fixed shuffle order); o rounded once to bf16.
 * Deterministic.
 *
 * Limits (else MOE_ERR_UNSUPPORTED): dk = 64, 128 or 256; dv a multiple of
 * 16; Hv a multiple of Hk; B <= 65535, Hv <= 65535.  state 16-byte aligned,
 * the other pointers 4-byte aligned (out 2-byte) (else MOE_ERR_INVALID_ARG).
 *
 * Asynchrony: enqueued on `stream` with programmatic dependent launch (global
 * memory is read only after the preceding work of the stream has completed).
 * No workspace, no device-side waits.
 */
#ifndef DELTANET_H_
#define DELTANET_H_

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One recurrence step (see above). */
MOE_API int gdn_decode_step(const moe_bf16* q, const moe_bf16* k, const moe_bf16* v, const float* g,
                            const float* beta, float* state, moe_bf16* out, int B, int Hk, int Hv, int dk, int dv,
                            moe_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* DELTANET_H_ */
