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

// Warp-cooperative top-k over E <= 256 logits held in shared memory.
// Order: larger logit first; equal logits go to the lower expert index (a
// strict total order, so every lane agrees on each pick).  Lane 0 writes the
// chosen experts and their weights exp(l_j - l_0) / sum_j' exp(l_j' - l_0).
__device__ __forceinline__ void select_topk_warp(const float* lg, int E, int k, int lane,
                                                 int32_t* idx_out, float* w_out) {
  float v[8];
  unsigned taken = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? lg[e] : 0.f;
    if (e >= E) taken |= 1u << i;
  }
  float selv[kMaxK];
  int seli[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j < k) {
      float bv = 0.f;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (!((taken >> i) & 1u) && (bi == 0x7fffffff || v[i] > bv || (v[i] == bv && e < bi))) {
          bv = v[i];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
          bv = ov;
          bi = oi;
        }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      selv[j] = bv;
      seli[j] = bi;
    }
  }
  if (lane == 0) {
    float z[kMaxK];
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k) {
        z[j] = expf(selv[j] - selv[0]);
        s += z[j];
      }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k) {
        idx_out[j] = seli[j];
        w_out[j] = z[j] / s;
      }
  }
}

}  // namespace moe
