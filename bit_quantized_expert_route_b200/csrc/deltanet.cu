// Gated DeltaNet decode step: one token of the gated delta-rule recurrence
// for every sequence and value head ("Perplexity's Lily: ...", section "The
// Model: Qwen3.6-35B-A3B in Focus": 30 Gated DeltaNet layers with a
// fixed-size recurrence; the rule itself is the published one, Yang, Kautz
// and Hatamizadeh, "Gated Delta Networks").
//
// The step is a streaming pass over the FP32 state: each row S_i (dk floats)
// is read once and written once, and needs two dot products with the
// normalised key and query.  With dk = 128 a row is 512 B of reads and 512 B
// of writes against ~8 FLOP per element, so the kernel is bound by HBM and
// the dot products stay on the CUDA cores (warp shuffles), not the tensor
// cores.
//
// Layout of the work: grid (dv / 16, Hv, B); a CTA of 4 warps owns 16 rows
// of one head's state, 4 rows per warp; lane l holds elements
// [l dk/32, (l+1) dk/32) of every row, of k^ and of q^ (vector loads, the
// warp's row access is one contiguous 512 B for dk = 128).  All of a warp's
// state loads are issued before the key and query arithmetic, so their
// memory latency overlaps it.  Row update (FP32):
//   sk = S_i . k^, sq = S_i . q^          (shuffle trees, fixed order)
//   u  = beta (v_i - alpha sk)
//   S'_i = alpha S_i + u k^               (fmaf per element)
//   o_i  = alpha sq + u (k^ . q^)
#include <math.h>

#include "common.cuh"
#include "deltanet.h"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kGRows = 16;                    // state rows per CTA
constexpr int kGWarps = 4;
constexpr int kGRowsPerWarp = kGRows / kGWarps;
constexpr int kGThreads = kGWarps * 32;

struct GdnArgs {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const float* g;
  const float* beta;
  float* state;
  uint16_t* out;
  int Hk, Hv, dv;
};

template <int PER>
struct Vec {   // PER consecutive floats / bf16 of one lane
  static __device__ __forceinline__ void load_f(float (&x)[PER], const float* p) {
    if constexpr (PER == 2) {
      const float2 t = __ldcg(reinterpret_cast<const float2*>(p));
      x[0] = t.x, x[1] = t.y;
    } else {
#pragma unroll
      for (int i = 0; i < PER; i += 4) {
        const float4 t = __ldcg(reinterpret_cast<const float4*>(p + i));
        x[i] = t.x, x[i + 1] = t.y, x[i + 2] = t.z, x[i + 3] = t.w;
      }
    }
  }
  static __device__ __forceinline__ void store_f(float* p, const float (&x)[PER]) {
    if constexpr (PER == 2) {
      *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    } else {
#pragma unroll
      for (int i = 0; i < PER; i += 4)
        *reinterpret_cast<float4*>(p + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
    }
  }
  static __device__ __forceinline__ void load_bf16(float (&x)[PER], const uint16_t* p) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(p);
#pragma unroll
    for (int i = 0; i < PER / 2; ++i) {
      const uint32_t t = __ldg(w + i);
      x[2 * i] = bf16_lo(t);
      x[2 * i + 1] = bf16_hi(t);
    }
  }
};

template <int DK>
__global__ void __launch_bounds__(kGThreads) gdn_step_kernel(const GdnArgs a) {
  constexpr int PER = DK / 32;
  const int hv = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hk = hv / (a.Hv / a.Hk);
  const size_t head = static_cast<size_t>(b) * a.Hv + hv;
  const int row0 = blockIdx.x * kGRows + warp * kGRowsPerWarp;
  pdl_wait();   // the state and the token's inputs come from earlier work of the stream

  float s[kGRowsPerWarp][PER];
  float* srow = a.state + (head * a.dv + row0) * DK + lane * PER;
#pragma unroll
  for (int r = 0; r < kGRowsPerWarp; ++r) Vec<PER>::load_f(s[r], srow + r * DK);

  float kk[PER], qq[PER];
  const size_t kh = (static_cast<size_t>(b) * a.Hk + hk) * DK + lane * PER;
  Vec<PER>::load_bf16(kk, a.k + kh);
  Vec<PER>::load_bf16(qq, a.q + kh);
  float vv[kGRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kGRowsPerWarp; ++r) vv[r] = bf16_bits_to_float(__ldg(a.v + head * a.dv + row0 + r));
  const float alpha = expf(__ldg(a.g + head)), beta = __ldg(a.beta + head);

  float kss = 0.f, qss = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    kss = fmaf(kk[i], kk[i], kss);
    qss = fmaf(qq[i], qq[i], qss);
  }
  kss = warp_sum(kss);
  qss = warp_sum(qss);
  const float kn = 1.0f / sqrtf(kss + 1e-6f);
  const float qn = 1.0f / sqrtf(qss + 1e-6f) / sqrtf(static_cast<float>(DK));
  float kq = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    kk[i] *= kn;
    qq[i] *= qn;
    kq = fmaf(kk[i], qq[i], kq);
  }
  kq = warp_sum(kq);

#pragma unroll
  for (int r = 0; r < kGRowsPerWarp; ++r) {
    float sk = 0.f, sq = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      sk = fmaf(s[r][i], kk[i], sk);
      sq = fmaf(s[r][i], qq[i], sq);
    }
    sk = warp_sum(sk);
    sq = warp_sum(sq);
    const float u = beta * (vv[r] - alpha * sk);
#pragma unroll
    for (int i = 0; i < PER; ++i) s[r][i] = fmaf(alpha, s[r][i], u * kk[i]);
    Vec<PER>::store_f(srow + r * DK, s[r]);
    if (lane == 0) a.out[head * a.dv + row0 + r] = float_to_bf16_bits(fmaf(alpha, sq, u * kq));
  }
  pdl_launch_dependents();
}

template <int DK>
int launch(const GdnArgs& a, int B, cudaStream_t s) {
  const dim3 grid(a.dv / kGRows, a.Hv, B);
  return launch_pdl(gdn_step_kernel<DK>, grid, dim3(kGThreads), 0, s, a) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

MOE_API int gdn_decode_step(const moe_bf16* q, const moe_bf16* k, const moe_bf16* v, const float* g,
                            const float* beta, float* state, moe_bf16* out, int B, int Hk, int Hv, int dk, int dv,
                            moe_stream stream) {
  if (!q || !k || !v || !g || !beta || !state || !out) return MOE_ERR_INVALID_ARG;
  auto aligned = [](const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0; };
  if (!aligned(state, 16) || !aligned(q, 4) || !aligned(k, 4) || !aligned(v, 2) || !aligned(g, 4) ||
      !aligned(beta, 4) || !aligned(out, 2))
    return MOE_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || Hk < 1 || Hv < Hk || Hv % Hk || Hv > 65535) return MOE_ERR_UNSUPPORTED;
  if ((dk != 64 && dk != 128 && dk != 256) || dv < kGRows || dv % kGRows) return MOE_ERR_UNSUPPORTED;
  GdnArgs a{q, k, v, g, beta, state, out, Hk, Hv, dv};
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dk == 64) return launch<64>(a, B, s);
  if (dk == 128) return launch<128>(a, B, s);
  return launch<256>(a, B, s);
}

}  // extern "C"
