/* attn.h -- C ABI of libmoe.so's decode attention: one decode step of
 * grouped-query softmax attention over a fixed-block (paged) key/value cache.
 *
 * What it computes.  "Perplexity's Lily: A Breakthrough Local Inference
 * Engine Tailored Exclusively for Apple Silicon", section "The Model:
 * Qwen3.6-35B-A3B in Focus": the model's full-attention layers are
 * grouped-query attention with 16 query heads and 2 key/value heads; section
 * "How It Works: Prefill and Decode Strategies": decode attention packs the
 * query heads that share a key/value head (GQA packing) and keeps the cache in
 * fixed blocks, and making the cache reads compact and adjacent is what
 * decides long-context decode latency.  The pages give no formula; this is
 * the plain definition of one decode step, for every sequence b and query
 * head h (group = Hq / Hkv, key/value head g = h / group):
 *
 *   o[b, h] = sum_j softmax_j(scale * q[b, h] . K[b, g, j]) V[b, g, j],
 *             j = 0 .. ctx_len[b] - 1,
 *
 * where position j of sequence b is row j % block of physical block
 * block_table[b][j / block].  scale = 1/sqrt(D) unless given.
 *
 * Storage (all DEVICE pointers, bf16 as 16-bit patterns):
 *   q            [B][Hq][D]
 *   k_cache      [n_blocks][Hkv][block][D]   (one block of one head is a
 *   v_cache      [n_blocks][Hkv][block][D]    contiguous block x D tile)
 *   block_table  int32 [B][max_blocks]; entries past a sequence's last
 *                block are not read
 *   ctx_len      int32 [B]
 *   out          [B][Hq][D]
 *
 * Arithmetic.  Scores and the output accumulate in FP32 on the tensor cores
 * (bf16 q, k, v; the softmax weights are rounded to bf16 for the weighted sum
 * of the values, as flash-style kernels do); the output is rounded once to
 * bf16.  The weights use a running maximum per head, so no score overflows.
 *
 * Limits (else MOE_ERR_UNSUPPORTED): D = 128 or 256; Hq a multiple of Hkv
 * with Hq / Hkv <= 8; block a multiple of 16; n_blocks * Hkv * block < 2^31.
 * B <= 65535.  Alignment (else MOE_ERR_INVALID_ARG): the caches 16 bytes, q,
 * block_table and ctx_len 4 bytes, out 2 bytes.
 *
 * Degenerate and bad input on the device.  ctx_len[b] == 0 gives o[b] = 0.
 * A ctx_len above max_blocks * block, a negative one, or a block-table entry
 * the sequence needs that lies outside [0, n_blocks) records
 * MOE_ERR_DEVICE_INDEX in the workspace's status word (moe_get_status); the
 * out-of-range rows are not read, and the affected outputs are unspecified.
 *
 * Workspace.  attn_decode_workspace_size() bytes, 256-byte aligned, zero
 * before its first use (its first 256 bytes are the same control block as an
 * MoE workspace: moe_get_status reads and clears it).  It holds the partial
 * results of the key/value splits.  Two calls must not share a workspace
 * concurrently.
 *
 * Asynchrony.  attn_decode enqueues on `stream` and returns; both kernels are
 * launched with programmatic dependent launch (each reads global memory only
 * after the preceding work of the stream has completed).
 */
#ifndef ATTN_H_
#define ATTN_H_

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of workspace attn_decode needs for these sizes (0 if unsupported). */
MOE_API size_t attn_decode_workspace_size(int B, int Hkv, int D, int block, int max_blocks);

/* One decode step of grouped-query attention (see above).  scale <= 0 selects
 * 1/sqrt(D).  Work split: every (sequence, key/value head) pair is cut into
 * up to n_split contiguous ranges of 16-position chunks so that the grid
 * covers the SMs; each range's partial (running maximum, sum of weights,
 * weighted sum of values) is merged by a second kernel in fixed range order,
 * so results are deterministic. */
MOE_API int attn_decode(const moe_bf16* q, const moe_bf16* k_cache, const moe_bf16* v_cache,
                        const int32_t* block_table, const int32_t* ctx_len, int B, int Hq, int Hkv, int D,
                        int block, int max_blocks, int n_blocks, float scale, moe_bf16* out, void* workspace,
                        size_t workspace_bytes, moe_stream stream);

/* The work split attn_decode uses for these sizes: n_split ranges per
 * (sequence, key/value head), each of chunks_per_split 16-position chunks. */
MOE_API int attn_decode_plan(int B, int Hkv, int block, int max_blocks, int* n_split, int* chunks_per_split);

#ifdef __cplusplus
}
#endif
#endif /* ATTN_H_ */
