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
//
// In a stack of layers the next layer's input is RMSNorm(out_t) (weight 1, no
// residual): with norm_out given, the CTA also sums the squares of the row's
// bf16 outputs (per thread in column order, then the warps' sums in a fixed
// tree) and writes norm_out_t = bf16(out_t / sqrt(mean(out_t^2) + eps)), the
// value the stand-alone RMSNorm computes from out_t, without another pass
// over the row.  out may be NULL when only the normalised row is wanted.
constexpr int kCombThreads = 128;
constexpr int kCombMaxIters = 4;    // 16-column pieces per thread: H <= 128 * 16 * 4 = 8192

__device__ __forceinline__ void fma_bf16x8(float (&acc)[8], float w, const uint4& y) {
  acc[0] = fmaf(w, bf16_lo(y.x), acc[0]); acc[1] = fmaf(w, bf16_hi(y.x), acc[1]);
  acc[2] = fmaf(w, bf16_lo(y.y), acc[2]); acc[3] = fmaf(w, bf16_hi(y.y), acc[3]);
  acc[4] = fmaf(w, bf16_lo(y.z), acc[4]); acc[5] = fmaf(w, bf16_hi(y.z), acc[5]);
  acc[6] = fmaf(w, bf16_lo(y.w), acc[6]); acc[7] = fmaf(w, bf16_hi(y.w), acc[7]);
}

__device__ __forceinline__ uint4 pack8(const float (&a)[8]) {
  uint4 o;
  o.x = pack_bf16x2(a[0], a[1]); o.y = pack_bf16x2(a[2], a[3]);
  o.z = pack_bf16x2(a[4], a[5]); o.w = pack_bf16x2(a[6], a[7]);
  return o;
}

__device__ __forceinline__ float sumsq8(const uint4& v, float ss) {
  ss = fmaf(bf16_lo(v.x), bf16_lo(v.x), ss); ss = fmaf(bf16_hi(v.x), bf16_hi(v.x), ss);
  ss = fmaf(bf16_lo(v.y), bf16_lo(v.y), ss); ss = fmaf(bf16_hi(v.y), bf16_hi(v.y), ss);
  ss = fmaf(bf16_lo(v.z), bf16_lo(v.z), ss); ss = fmaf(bf16_hi(v.z), bf16_hi(v.z), ss);
  ss = fmaf(bf16_lo(v.w), bf16_lo(v.w), ss); ss = fmaf(bf16_hi(v.w), bf16_hi(v.w), ss);
  return ss;
}

__device__ __forceinline__ uint4 scale8(const uint4& v, float s) {
  uint4 o;
  o.x = pack_bf16x2(bf16_lo(v.x) * s, bf16_hi(v.x) * s);
  o.y = pack_bf16x2(bf16_lo(v.y) * s, bf16_hi(v.y) * s);
  o.z = pack_bf16x2(bf16_lo(v.z) * s, bf16_hi(v.z) * s);
  o.w = pack_bf16x2(bf16_lo(v.w) * s, bf16_hi(v.w) * s);
  return o;
}

__global__ void __launch_bounds__(kCombThreads) combine_kernel(
    const uint16_t* __restrict__ Y, const int32_t* __restrict__ inv_perm, const float* __restrict__ topk_w,
    const float* __restrict__ sigma, int T, int k, int H, uint16_t* __restrict__ out,
    uint16_t* __restrict__ norm_out, float eps, const int* status) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float part[kCombThreads / 32];
  const int t = blockIdx.x;
  // the status word is read together with the routing of the token; a
  // recorded error means inv_perm may hold entries no kernel wrote: skip
  const int st = *reinterpret_cast<volatile const int*>(status);
  int pos[kMaxK];
  float w[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    pos[j] = j < k ? __ldg(inv_perm + static_cast<size_t>(t) * k + j) : 0;
    w[j] = j < k ? __ldg(topk_w + static_cast<size_t>(t) * k + j) : 0.f;
  }
  const float sg = __ldg(sigma + t);
  if (st != 0) return;
  const size_t shared_row = static_cast<size_t>(T) * k + t;
  uint4 keep[2 * kCombMaxIters];      // this thread's bf16 outputs, kept for the normalisation
  float ss = 0.f;
#pragma unroll
  for (int it = 0; it < kCombMaxIters; ++it) {
    const int c = (it * kCombThreads + threadIdx.x) * 16;
    if (c >= H) break;
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
    const uint4 o0 = pack8(a0), o1 = pack8(a1);
    if (out) {
      uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H + c);
      dst[0] = o0;
      dst[1] = o1;
    }
    keep[2 * it] = o0;
    keep[2 * it + 1] = o1;
    ss = sumsq8(o1, sumsq8(o0, ss));
  }
  if (norm_out == nullptr) return;
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w8 = 0; w8 < kCombThreads / 32; ++w8) tot += part[w8];
  const float inv = 1.0f / sqrtf(tot / static_cast<float>(H) + eps);
#pragma unroll
  for (int it = 0; it < kCombMaxIters; ++it) {
    const int c = (it * kCombThreads + threadIdx.x) * 16;
    if (c >= H) break;
    uint4* dst = reinterpret_cast<uint4*>(norm_out + static_cast<size_t>(t) * H + c);
    dst[0] = scale8(keep[2 * it], inv);
    dst[1] = scale8(keep[2 * it + 1], inv);
  }
}

// y_out = bf16(y / sqrt(mean(y^2) + eps)), one CTA per row, fixed reduction tree.
// y and out may be the same buffer (no __restrict__): each thread reads its
// columns of the row before any thread writes them back.
__global__ void __launch_bounds__(256) rmsnorm_kernel(const uint16_t* y, uint16_t* out,
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
                                                                    uint4* __restrict__ xg, const int* status) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kGatherWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  // the status word is read together with the row's token; a recorded error
  // means perm may hold entries no kernel wrote: skip
  const int st = *reinterpret_cast<volatile const int*>(status);
  const int t = row < Tk ? __ldg(perm + row) / k : row - Tk;
  if (st != 0) return;
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
                             const int* status, cudaStream_t s) {
  const int rows = T * k + T;
  return launch_pdl(gather_k8_kernel, dim3((rows + kGatherWarps - 1) / kGatherWarps), dim3(kGatherWarps * 32), 0,
                    s, reinterpret_cast<const uint4*>(x), perm, T * k, k, H / 8, rows, reinterpret_cast<uint4*>(xg),
                    status);
}

cudaError_t launch_combine(const uint16_t* Y, const int32_t* inv_perm, const float* topk_w, const float* sigma,
                           int T, int k, int H, uint16_t* out, uint16_t* norm_out, float eps, const int* status,
                           cudaStream_t s) {
  if (H % 16 || H > kCombThreads * 16 * kCombMaxIters) return cudaErrorInvalidValue;
  return launch_pdl(combine_kernel, dim3(T), dim3(kCombThreads), 0, s, Y, inv_perm, topk_w, sigma, T, k, H, out,
                    norm_out, eps, status);
}

cudaError_t launch_rmsnorm(const uint16_t* y, uint16_t* out, int T, int H, float eps, cudaStream_t s) {
  return launch_pdl(rmsnorm_kernel, dim3(T), dim3(256), 0, s, y, out, H, eps);
}

}  // namespace moe
