// Deterministic gather-combine and the RMSNorm that links stacked layers.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// out_t = bf16( sum_{j=0..k-1} w[t,j] * Y[inv_perm[t*k+j]]  +  sigma_t * Y[T*k + t] )
// in FP32, in exactly that order, with no atomics: every token's sum is formed
// by one thread per 16 columns, so the result is bitwise reproducible.  Y (the
// experts' down-projection rows) is stored as bf16.  Each thread issues all
// 2 (k + 1) of its 16-byte loads before the first FMA, so a CTA keeps many
// DRAM requests in flight.
constexpr int kCombThreads = 128;

__device__ __forceinline__ void fma_bf16x8(float (&acc)[8], float w, const uint4& y) {
  acc[0] = fmaf(w, bf16_lo(y.x), acc[0]); acc[1] = fmaf(w, bf16_hi(y.x), acc[1]);
  acc[2] = fmaf(w, bf16_lo(y.y), acc[2]); acc[3] = fmaf(w, bf16_hi(y.y), acc[3]);
  acc[4] = fmaf(w, bf16_lo(y.z), acc[4]); acc[5] = fmaf(w, bf16_hi(y.z), acc[5]);
  acc[6] = fmaf(w, bf16_lo(y.w), acc[6]); acc[7] = fmaf(w, bf16_hi(y.w), acc[7]);
}

__global__ void __launch_bounds__(kCombThreads) combine_kernel(
    const uint16_t* __restrict__ Y, const int32_t* __restrict__ inv_perm, const float* __restrict__ topk_w,
    const float* __restrict__ sigma, int T, int k, int H, uint16_t* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x;
  int pos[kMaxK];
  float w[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    pos[j] = j < k ? __ldg(inv_perm + static_cast<size_t>(t) * k + j) : 0;
    w[j] = j < k ? __ldg(topk_w + static_cast<size_t>(t) * k + j) : 0.f;
  }
  const float sg = __ldg(sigma + t);
  const size_t shared_row = static_cast<size_t>(T) * k + t;
  for (int c = threadIdx.x * 16; c < H; c += kCombThreads * 16) {
    uint4 ya[kMaxK], yb[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        const uint4* row = reinterpret_cast<const uint4*>(Y + static_cast<size_t>(pos[j]) * H + c);
        ya[j] = __ldcs(row);
        yb[j] = __ldcs(row + 1);
      }
    }
    const uint4* srow = reinterpret_cast<const uint4*>(Y + shared_row * H + c);
    const uint4 sa = __ldcs(srow), sb = __ldcs(srow + 1);
    float a0[8], a1[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) a0[q] = a1[q] = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        fma_bf16x8(a0, w[j], ya[j]);
        fma_bf16x8(a1, w[j], yb[j]);
      }
    }
    fma_bf16x8(a0, sg, sa);
    fma_bf16x8(a1, sg, sb);
    uint4 o0, o1;
    o0.x = pack_bf16x2(a0[0], a0[1]); o0.y = pack_bf16x2(a0[2], a0[3]);
    o0.z = pack_bf16x2(a0[4], a0[5]); o0.w = pack_bf16x2(a0[6], a0[7]);
    o1.x = pack_bf16x2(a1[0], a1[1]); o1.y = pack_bf16x2(a1[2], a1[3]);
    o1.z = pack_bf16x2(a1[4], a1[5]); o1.w = pack_bf16x2(a1[6], a1[7]);
    uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H + c);
    dst[0] = o0;
    dst[1] = o1;
  }
}

// y_out = bf16(y / sqrt(mean(y^2) + eps)), one CTA per row, fixed reduction tree.
__global__ void __launch_bounds__(256) rmsnorm_kernel(const uint16_t* __restrict__ y, uint16_t* __restrict__ out,
                                                      int H, float eps) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float part[8];
  const size_t row = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(y + row * H);
  float ss = 0.f;
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    const uint4 v = src[c];
    const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
    for (int q = 0; q < 8; ++q) ss = fmaf(f[q], f[q], ss);
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += part[w];
  const float inv = 1.0f / sqrtf(tot / static_cast<float>(H) + eps);
  uint4* dst = reinterpret_cast<uint4*>(out + row * H);
  __syncthreads();   // y and out may alias: every read of the row is done
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    const uint4 v = src[c];
    uint4 o;
    o.x = pack_bf16x2(bf16_lo(v.x) * inv, bf16_hi(v.x) * inv);
    o.y = pack_bf16x2(bf16_lo(v.y) * inv, bf16_hi(v.y) * inv);
    o.z = pack_bf16x2(bf16_lo(v.z) * inv, bf16_hi(v.z) * inv);
    o.w = pack_bf16x2(bf16_lo(v.w) * inv, bf16_hi(v.w) * inv);
    dst[c] = o;
  }
}

// xg[R] = x[perm[R] / k] (R < T*k) or x[R - T*k] (the shared expert's rows),
// with every group of 8 elements in the order (0,4,1,5,2,6,3,7): the gate/up
// GEMM's token rows, contiguous per expert group, in its K order.  One warp
// per row: its lanes load all their 16-byte pieces of the row before storing.
constexpr int kGatherWarps = 8;
constexpr int kGatherPieces = 8;    // 16-byte pieces per lane per pass (H <= 8192: up to 4 passes)

__device__ __forceinline__ uint4 interleave_k8(const uint4& v) {   // (x0,x1)(x2,x3)(x4,x5)(x6,x7)
  uint4 o;
  o.x = __byte_perm(v.x, v.z, 0x5410);   // (x0, x4)
  o.y = __byte_perm(v.x, v.z, 0x7632);   // (x1, x5)
  o.z = __byte_perm(v.y, v.w, 0x5410);   // (x2, x6)
  o.w = __byte_perm(v.y, v.w, 0x7632);   // (x3, x7)
  return o;
}

__global__ void __launch_bounds__(kGatherWarps * 32) gather_k8_kernel(const uint4* __restrict__ x,
                                                                    const int32_t* __restrict__ perm, int Tk,
                                                                    int k, int h8, int rows,
                                                                    uint4* __restrict__ xg) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kGatherWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int t = row < Tk ? __ldg(perm + row) / k : row - Tk;
  const uint4* src = x + static_cast<size_t>(t) * h8;
  uint4* dst = xg + static_cast<size_t>(row) * h8;
  for (int c0 = 0; c0 < h8; c0 += 32 * kGatherPieces) {
    uint4 v[kGatherPieces];
#pragma unroll
    for (int i = 0; i < kGatherPieces; ++i) {
      const int c = c0 + i * 32 + lane;
      if (c < h8) v[i] = __ldg(src + c);
    }
#pragma unroll
    for (int i = 0; i < kGatherPieces; ++i) {
      const int c = c0 + i * 32 + lane;
      if (c < h8) dst[c] = interleave_k8(v[i]);
    }
  }
}

cudaError_t launch_gather_k8(const uint16_t* x, const int32_t* perm, int T, int k, int H, uint16_t* xg,
                             cudaStream_t s) {
  const int rows = T * k + T;
  return launch_pdl(gather_k8_kernel, dim3((rows + kGatherWarps - 1) / kGatherWarps), dim3(kGatherWarps * 32), 0,
                    s, reinterpret_cast<const uint4*>(x), perm, T * k, k, H / 8, rows, reinterpret_cast<uint4*>(xg));
}

cudaError_t launch_combine(const uint16_t* Y, const int32_t* inv_perm, const float* topk_w, const float* sigma,
                           int T, int k, int H, uint16_t* out, cudaStream_t s) {
  return launch_pdl(combine_kernel, dim3(T), dim3(kCombThreads), 0, s, Y, inv_perm, topk_w, sigma, T, k, H, out);
}

cudaError_t launch_rmsnorm(const uint16_t* y, uint16_t* out, int T, int H, float eps, cudaStream_t s) {
  return launch_pdl(rmsnorm_kernel, dim3(T), dim3(256), 0, s, y, out, H, eps);
}

}  // namespace moe
