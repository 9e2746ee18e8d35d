// Tensor-core dot products of 4-bit affine-quantised weights with bf16
// activations (warp-level mma.sync m16n8k16, bf16 in, FP32 accumulation),
// shared by the decode kernels.
//
// Per group of 64 inputs, A = 128 + q as exact bf16 values (one AND-OR per
// code pair, no scale applied) and B = the activations, so that
//   sum_i (s q_i + b) x_i = s * (sum_i (128 + q_i) x_i - 128 X) + b X,  X = sum_i x_i,
// is applied per group after the MMAs ("Perplexity's Lily: ...", section
// "How It Works: Prefill and Decode Strategies": the weights stay 4-bit in
// memory and are rebuilt next to the arithmetic).  Inside each group of 8
// inputs both operands use the order (0,4,1,5,2,6,3,7) in which the AND-OR
// yields code pairs; activations are staged in that order (interleave8).
#pragma once

#include "common.cuh"

namespace moe {

// D (16 rows x 8 tokens, FP32) += A (16 x 16, bf16) B (16 x 8, bf16).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t code_pair(uint32_t w, int shift) {   // bf16 pair (128 + q_i, 128 + q_{i+4})
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w >> shift), "r"(0x000F000Fu), "r"(0x43004300u));
  return d;
}

// 8 bf16 values (x0,x1)(x2,x3)(x4,x5)(x6,x7) in the interleaved K order
// (x0,x4)(x1,x5)(x2,x6)(x3,x7).
__device__ __forceinline__ uint4 interleave8(const uint4& v) {
  uint4 o;
  o.x = __byte_perm(v.x, v.z, 0x5410);
  o.y = __byte_perm(v.x, v.z, 0x7632);
  o.z = __byte_perm(v.y, v.w, 0x5410);
  o.w = __byte_perm(v.y, v.w, 0x7632);
  return o;
}

// One group of 64 inputs for rows g, g+8 of a 16-row weight tile (lane g =
// lane/4, t = lane%4): lane reads words 2t, 2t+1 of the group in both rows
// (qg, qg8: this lane's 8 bytes) and the 32 staged activations of token g at
// 8-groups 2t, 2t+1 (xb0, xb1; zero for tokens outside the unit).  d gets
// sum (128 + q) x for (row g, tokens 2t, 2t+1) and (row g+8, same tokens).
__device__ __forceinline__ void group_dot(float (&d)[4], const uint2& qg, const uint2& qg8, const uint4& xb0,
                                          const uint4& xb1) {
  float e[4] = {0.f, 0.f, 0.f, 0.f};   // two accumulation chains, summed at the end
  d[0] = d[1] = d[2] = d[3] = 0.f;
  mma16816(d, code_pair(qg.x, 0), code_pair(qg8.x, 0), code_pair(qg.x, 4), code_pair(qg8.x, 4), xb0.x, xb0.y);
  mma16816(e, code_pair(qg.x, 8), code_pair(qg8.x, 8), code_pair(qg.x, 12), code_pair(qg8.x, 12), xb0.z, xb0.w);
  mma16816(d, code_pair(qg.y, 0), code_pair(qg8.y, 0), code_pair(qg.y, 4), code_pair(qg8.y, 4), xb1.x, xb1.y);
  mma16816(e, code_pair(qg.y, 8), code_pair(qg8.y, 8), code_pair(qg.y, 12), code_pair(qg8.y, 12), xb1.z, xb1.w);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] += e[i];
}

}  // namespace moe
