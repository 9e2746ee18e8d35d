// Device-side helpers shared by the MoE kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kGroup = 64;          // weights per affine 4-bit group
constexpr int kCodesPerWord = 8;    // 4-bit codes per uint32 word
constexpr int kMaxK = 8;            // largest supported experts-per-token
constexpr int kMaxE = 256;          // largest supported expert count

// Status codes written to the workspace status word (mirror moe_status).
constexpr int kStatusTimeout = -5;
constexpr int kStatusBadIndex = -6;

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Low / high bf16 of a packed pair, widened exactly to float.
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }
__device__ __forceinline__ float sigmoid(float z) { return 1.0f / (1.0f + expf(-z)); }

// Programmatic dependent launch (kernels.h, launch_pdl): pdl_wait() returns
// once the previous grid of the stream has completed and its writes are
// visible; pdl_launch_dependents() lets the next grid be scheduled (its CTAs
// then run their prologue and wait in their own pdl_wait()).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// One unit of grouped-GEMM work: `rows` consecutive rows of the grouped row
// space starting at `row0`, all owned by expert `e` (e == E: shared expert).
struct Chunk {
  int e;
  int row0;
  int rows;
  int pad;
};

}  // namespace moe

namespace moe {

// Order-preserving 32-bit key of a float (larger float -> larger key; every
// non-NaN float maps above 0).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = f == 0.f ? 0u : __float_as_uint(f);   // -0 and +0 are one value
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp top-k over E <= 256 logits in shared memory with the same order as
// the other routing kernels (larger logit first, equal logits -> lower expert
// index).  Lane i holds the keys of experts i, i + 32, ..., sorted once by a
// 19-comparator network on (key, expert) pairs, so its best candidate is
// always its head.  A pick is one redux.sync max over the heads and one min
// over the experts of the lanes holding that key; the winning lane pops its
// head.  Lanes j < k then form exp(l_j - l_0) in parallel and divide by their
// sum (a fixed shuffle tree).
__device__ __forceinline__ bool key_before(uint32_t ka, int ia, uint32_t kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}
__device__ __forceinline__ void cas(uint32_t (&key)[8], int (&ix)[8], int i, int j) {
  const bool keep = key_before(key[i], ix[i], key[j], ix[j]);
  const uint32_t ki = keep ? key[i] : key[j], kj = keep ? key[j] : key[i];
  const int ii = keep ? ix[i] : ix[j], ij = keep ? ix[j] : ix[i];
  key[i] = ki;
  key[j] = kj;
  ix[i] = ii;
  ix[j] = ij;
}
__device__ __forceinline__ void topk_redux(const float* lg, int E, int k, int lane, int32_t* idx_out,
                                           float* w_out) {
  uint32_t key[8];
  int ix[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    ix[i] = lane + 32 * i;
    key[i] = ix[i] < E ? order_key(lg[ix[i]]) : 0u;
  }
  cas(key, ix, 0, 1); cas(key, ix, 2, 3); cas(key, ix, 4, 5); cas(key, ix, 6, 7);
  cas(key, ix, 0, 2); cas(key, ix, 1, 3); cas(key, ix, 4, 6); cas(key, ix, 5, 7);
  cas(key, ix, 1, 2); cas(key, ix, 5, 6);
  cas(key, ix, 0, 4); cas(key, ix, 1, 5); cas(key, ix, 2, 6); cas(key, ix, 3, 7);
  cas(key, ix, 2, 4); cas(key, ix, 3, 5);
  cas(key, ix, 1, 2); cas(key, ix, 3, 4); cas(key, ix, 5, 6);
  int mine = 0, first = 0;
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j < k) {
      const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
      const uint32_t win = __reduce_min_sync(0xffffffffu, key[0] == m ? static_cast<uint32_t>(ix[0]) : 0xffffffffu);
      if (static_cast<uint32_t>(ix[0]) == win) {   // pop the head
#pragma unroll
        for (int i = 0; i < 7; ++i) {
          key[i] = key[i + 1];
          ix[i] = ix[i + 1];
        }
        key[7] = 0u;
        ix[7] = 0x7fffffff;
      }
      if (lane == j) mine = static_cast<int>(win);
      if (j == 0) first = static_cast<int>(win);
    }
  }
  const float z = lane < k ? expf(lg[mine] - lg[first]) : 0.f;
  const float sum = warp_sum(z);
  if (lane < k) {
    idx_out[lane] = mine;
    w_out[lane] = z / sum;
  }
}

}  // namespace moe
