// Decode path (T <= 64): the layer as bandwidth-bound GEMVs over the active
// experts only.  Batch-1 decoding barely reuses a weight, so every packed
// weight byte is read once with 128-bit coalesced loads and rebuilt in
// registers in FP32 ("Perplexity's Lily: ...", section "How It Works: Prefill
// and Decode Strategies", decode paragraph; "Frequently Asked Questions":
// decode is bound by moving weights, not by arithmetic).
//
// Dequantisation in FP32 without per-weight multiplies: for the 32 codes q_i
// of one 128-bit load (half a quantisation group: one scale s, one bias b)
//   sum_i (s q_i + b) x_i = 128 s * sum_i f_i x_i + (b - 128 s) * sum_i x_i,
//   f_i = 1 + q_i / 128,
// where f_i is built exactly by OR-ing the code into the mantissa of 1.0f
// (one shift + one LOP3), and sum_i x_i is computed once per token per
// segment when the activations are staged.  So a code costs about three
// instructions per token instead of a convert, a dequant FMA and a dot FMA.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDecWarps = 8;
constexpr int kRowsPerWarp = 4;                        // features per warp (each: gate row and up row)
constexpr int kDecFeat = kDecWarps * kRowsPerWarp;     // features per CTA
constexpr int kDownDims = 16;                          // output dims per CTA (8 warps x 2 half-warps)
constexpr int kDecTokMaxDecode = 8;                    // tokens per pass over an expert's weights

// Staged row strides (floats): whole interleave windows of 32 (gate/up) or
// 16 (down) lanes x 32 codes.
__host__ __device__ __forceinline__ int xstride_of(int H) { return (H + 1023) / 1024 * 1024; }
__host__ __device__ __forceinline__ int hstride_of(int I) { return (I + 511) / 512 * 512; }

__device__ __forceinline__ QMatPtr expert_qmat(const QMatPtr& stack, int e, size_t rows, size_t cols) {
  return QMatPtr{stack.q + static_cast<size_t>(e) * rows * (cols / 8),
                 stack.s + static_cast<size_t>(e) * rows * (cols / kGroup),
                 stack.b + static_cast<size_t>(e) * rows * (cols / kGroup)};
}

// f_i = 1 + q_i/128 for the eight codes of a word (code i in bits 4i..4i+3).
__device__ __forceinline__ void codes_plus_one(uint32_t w, float (&f)[8]) {
  const uint32_t M = 0x000F0000u, ONE = 0x3F800000u;
  f[0] = __uint_as_float(((w << 16) & M) | ONE);
  f[1] = __uint_as_float(((w << 12) & M) | ONE);
  f[2] = __uint_as_float(((w << 8) & M) | ONE);
  f[3] = __uint_as_float(((w << 4) & M) | ONE);
  f[4] = __uint_as_float((w & M) | ONE);
  f[5] = __uint_as_float(((w >> 4) & M) | ONE);
  f[6] = __uint_as_float(((w >> 8) & M) | ONE);
  f[7] = __uint_as_float(((w >> 12) & M) | ONE);
}

// sum_i f_i * x_i over the 32 codes of one 128-bit load; x comes from the
// lane-interleaved staging buffer: float4 j (codes 4j..4j+3) of this lane's
// segment at xl[j * stride4] (stride4 in float4 units).
__device__ __forceinline__ float dot32(const uint4& qv, const float4* __restrict__ xl, int stride4) {
  const uint32_t words[4] = {qv.x, qv.y, qv.z, qv.w};
  float a = 0.f;
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    float f[8];
    codes_plus_one(words[wd], f);
    const float4 x0 = xl[(2 * wd) * stride4];
    const float4 x1 = xl[(2 * wd + 1) * stride4];
    a = fmaf(f[0], x0.x, a); a = fmaf(f[1], x0.y, a); a = fmaf(f[2], x0.z, a); a = fmaf(f[3], x0.w, a);
    a = fmaf(f[4], x1.x, a); a = fmaf(f[5], x1.y, a); a = fmaf(f[6], x1.z, a); a = fmaf(f[7], x1.w, a);
  }
  return a;
}

// ---------------------------------------------------------------------------
// gate/up: CTA (active expert slot, block of 32 features).  Warp w owns
// features f0 + 4w .. +3; lane l owns the 128-bit load positions c = 32 v + l
// (v = 0 .. H/1024 - 1) of every row.  Activations of up to `kb` tokens at a
// time are staged as FP32 in a lane-interleaved layout:
//   element c*32 + i of token r at float index ((v*8 + i/4) * 32 + l) * 4 + i%4
// so that lane l's eight float4 reads are conflict-free, plus per-segment sums.
// ---------------------------------------------------------------------------
template <int NT>
__device__ __forceinline__ void gateup_warp(const QMatPtr& Wg, const QMatPtr& Wu, int H, int frow, int nf,
                                            const float* __restrict__ xs, const float* __restrict__ xsum,
                                            int nt, int lane, float (&res)[2][kRowsPerWarp][NT]) {
  const int xst = xstride_of(H);
  float acc[2][kRowsPerWarp][NT];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int f = 0; f < kRowsPerWarp; ++f)
#pragma unroll
      for (int r = 0; r < NT; ++r) acc[m][f][r] = 0.f;
  const int nv = xst / 1024;               // 128-bit positions per lane per row
  const int wpr = H / 8, gpr = H / kGroup;
  const int seg_per_tok = xst / 32;
  for (int v = 0; v < nv; ++v) {
    const int c = v * 32 + lane;
    if (c >= H / 32) break;
    uint4 q[2][kRowsPerWarp];
    float s[2][kRowsPerWarp], b[2][kRowsPerWarp];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const QMatPtr& W = m == 0 ? Wg : Wu;
#pragma unroll
      for (int f = 0; f < kRowsPerWarp; ++f) {
        const size_t row = static_cast<size_t>(frow + min(f, nf - 1));
        q[m][f] = __ldg(reinterpret_cast<const uint4*>(W.q + row * wpr) + c);
        s[m][f] = bf16_bits_to_float(__ldg(W.s + row * gpr + (c >> 1)));
        b[m][f] = bf16_bits_to_float(__ldg(W.b + row * gpr + (c >> 1)));
      }
    }
    const float4* xl = reinterpret_cast<const float4*>(xs) + (v * 8) * 32 + lane;
#pragma unroll
    for (int r = 0; r < NT; ++r) {
      if (r < nt) {
        const float4* xr = xl + static_cast<size_t>(r) * (xst / 4);
        const float X = xsum[r * seg_per_tok + c];
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int f = 0; f < kRowsPerWarp; ++f) {
            const float A = dot32(q[m][f], xr, 32);
            const float s128 = 128.f * s[m][f];
            acc[m][f][r] = fmaf(s128, A, fmaf(b[m][f] - s128, X, acc[m][f][r]));
          }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int f = 0; f < kRowsPerWarp; ++f)
#pragma unroll
      for (int r = 0; r < NT; ++r) res[m][f][r] = warp_sum(acc[m][f][r]);
}

template <int NT>
__device__ __forceinline__ void gateup_store(const QMatPtr& Wg, const QMatPtr& Wu, int H, int frow, int nf,
                                             const float* xs, const float* xsum, int nt, int lane,
                                             uint16_t* const* dst) {
  float res[2][kRowsPerWarp][NT];
  gateup_warp<NT>(Wg, Wu, H, frow, nf, xs, xsum, nt, lane, res);
#pragma unroll
  for (int f = 0; f < kRowsPerWarp; ++f)
#pragma unroll
    for (int r = 0; r < NT; ++r)
      if (lane == ((f * NT + r) & 31) && f < nf && r < nt)
        dst[r][frow + f] = float_to_bf16_bits(silu(res[0][f][r]) * res[1][f][r]);
}

// Stage `nt` activation rows (bf16) as FP32 in the lane-interleaved layout
// and their 32-element segment sums.
__device__ __forceinline__ void stage_rows(const uint16_t* const* rows, int nt, int H, int lanes, int stride,
                                           float* xs, float* xsum) {
  const int vec = H / 8;
  for (int i = threadIdx.x; i < nt * vec; i += blockDim.x) {
    const int r = i / vec, u = i - r * vec;           // u: 8-element chunk index
    const uint4 v = reinterpret_cast<const uint4*>(rows[r])[u];
    const int e0 = u * 8;                             // first element
    const int c = e0 >> 5, ii = e0 & 31;              // segment, offset in segment
    const int win = c / lanes, ln = c - win * lanes;
    float4* base = reinterpret_cast<float4*>(xs + static_cast<size_t>(r) * stride);
    base[((win * 8 + (ii >> 2)) * lanes) + ln] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
    base[((win * 8 + (ii >> 2) + 1) * lanes) + ln] =
        make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
  }
  __syncthreads();
  const int segs = H / 32, sstride = stride / 32;
  for (int i = threadIdx.x; i < nt * segs; i += blockDim.x) {
    const int r = i / segs, c = i - r * segs;
    const int win = c / lanes, ln = c - win * lanes;
    const float4* base = reinterpret_cast<const float4*>(xs + static_cast<size_t>(r) * stride);
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 q = base[(win * 8 + j) * lanes + ln];
      sum += (q.x + q.y) + (q.z + q.w);
    }
    xsum[r * sstride + c] = sum;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(256) decode_gateup_kernel(
    Geometry g, LayerPtr L, const uint16_t* __restrict__ x, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ perm, const int32_t* __restrict__ active, const int32_t* __restrict__ n_active,
    uint16_t* __restrict__ h, uint16_t* __restrict__ h_s, int kb) {
  extern __shared__ float sm[];
  const int slot = blockIdx.x;
  if (slot >= *n_active) return;
  const int e = active[slot];
  const bool shared = e >= g.E;
  const int Ie = shared ? g.Is : g.I;
  const int i0 = blockIdx.y * kDecFeat;
  if (i0 >= Ie) return;
  const QMatPtr Wg = shared ? L.sh_gate : expert_qmat(L.gate, e, g.I, g.H);
  const QMatPtr Wu = shared ? L.sh_up : expert_qmat(L.up, e, g.I, g.H);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int frow = i0 + warp * kRowsPerWarp;
  const int nf = max(0, min(kRowsPerWarp, Ie - frow));
  // warm this warp's first weight bytes before the token-list dependency chain
  if (nf > 0) {
    const int wpr = g.H / 8;
#pragma unroll
    for (int f = 0; f < kRowsPerWarp; ++f) {
      const size_t row = static_cast<size_t>(frow + min(f, nf - 1));
      asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const uint4*>(Wg.q + row * wpr) + lane));
      asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const uint4*>(Wu.q + row * wpr) + lane));
    }
  }
  const int pos0 = shared ? 0 : offsets[e];
  const int ntok = shared ? g.T : offsets[e + 1] - pos0;
  const int xst = xstride_of(g.H);
  float* xs = sm;                                        // [kb][xst]
  float* xsum = sm + static_cast<size_t>(kb) * xst;      // [kb][xst/32]
  for (int tb = 0; tb < ntok; tb += kb) {
    const int nt = min(kb, ntok - tb);
    const uint16_t* rows[kDecTokMaxDecode];
    uint16_t* dst[kDecTokMaxDecode];
#pragma unroll
    for (int r = 0; r < kDecTokMaxDecode; ++r) {
      const int rr = min(r, nt - 1);
      const int tok = shared ? (tb + rr) : perm[pos0 + tb + rr] / g.k;
      rows[r] = x + static_cast<size_t>(tok) * g.H;
      dst[r] = shared ? h_s + static_cast<size_t>(tb + rr) * g.Is : h + static_cast<size_t>(pos0 + tb + rr) * g.I;
    }
    __syncthreads();
    stage_rows(rows, nt, g.H, 32, xst, xs, xsum);
    if (nf > 0) {
      if (nt == 1)
        gateup_store<1>(Wg, Wu, g.H, frow, nf, xs, xsum, nt, lane, dst);
      else if (nt == 2)
        gateup_store<2>(Wg, Wu, g.H, frow, nf, xs, xsum, nt, lane, dst);
      else if (nt <= 4)
        gateup_store<4>(Wg, Wu, g.H, frow, nf, xs, xsum, nt, lane, dst);
      else
        gateup_store<8>(Wg, Wu, g.H, frow, nf, xs, xsum, nt, lane, dst);
    }
  }
}

__device__ __forceinline__ float halfwarp_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// down + combine: CTA (token t, block of 16 output dims); half-warp per dim.
//   out[t, d] = bf16( sum_j w[t,j] * (W_d[idx_j][d,:] . h_{t,j})  +  sigma_t * (W_sd[d,:] . hs_t) )
// The k + 1 terms are added in slot order, then the shared term.  The h rows
// are staged as FP32 with 16-lane interleaving (both half-warps read the same
// addresses) plus segment sums.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) decode_down_combine_kernel(
    Geometry g, LayerPtr L, const uint16_t* __restrict__ h, const uint16_t* __restrict__ h_s,
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, const int32_t* __restrict__ inv_perm,
    const float* __restrict__ sigma, uint16_t* __restrict__ out) {
  extern __shared__ float sm[];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hl = lane & 15;
  const int d = blockIdx.y * kDownDims + warp * 2 + (lane >> 4);
  const bool live = d < g.H;
  const int dd = min(d, g.H - 1);
  const int Imax = max(g.I, g.Is);
  const int hst = hstride_of(Imax);
  const int nterm = g.k + 1;
  float* hs = sm;                                          // [k+1][hst]
  float* hsum = sm + static_cast<size_t>(nterm) * hst;     // [k+1][hst/32]
  const uint16_t* rows[kMaxK + 1];
  for (int j = 0; j < nterm; ++j)
    rows[j] = j < g.k ? h + static_cast<size_t>(inv_perm[t * g.k + j]) * g.I : h_s + static_cast<size_t>(t) * g.Is;
  // stage h rows (routed rows have I columns, the shared row Is; Imax stride)
  {
    const int vec = Imax / 8;
    for (int i = threadIdx.x; i < nterm * vec; i += blockDim.x) {
      const int j = i / vec, u = i - j * vec;
      const int Ij = j < g.k ? g.I : g.Is;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (u * 8 < Ij) v = reinterpret_cast<const uint4*>(rows[j])[u];
      const int e0 = u * 8, c = e0 >> 5, ii = e0 & 31;
      const int win = c >> 4, ln = c & 15;
      float4* base = reinterpret_cast<float4*>(hs + static_cast<size_t>(j) * hst);
      base[(win * 8 + (ii >> 2)) * 16 + ln] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
      base[(win * 8 + (ii >> 2) + 1) * 16 + ln] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
    }
    __syncthreads();
    const int segs = Imax / 32;
    for (int i = threadIdx.x; i < nterm * segs; i += blockDim.x) {
      const int j = i / segs, c = i - j * segs;
      const int win = c >> 4, ln = c & 15;
      const float4* base = reinterpret_cast<const float4*>(hs + static_cast<size_t>(j) * hst);
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 f4 = base[(win * 8 + q) * 16 + ln];
        sum += (f4.x + f4.y) + (f4.z + f4.w);
      }
      hsum[j * (hst / 32) + c] = sum;
    }
    __syncthreads();
  }
  float acc = 0.f;
  for (int j = 0; j < nterm; ++j) {
    const bool sh = j == g.k;
    const int Ie = sh ? g.Is : g.I;
    const QMatPtr W = sh ? L.sh_down : expert_qmat(L.down, topk_idx[t * g.k + j], g.H, g.I);
    const int nv = hst / 512;
    float p = 0.f;
    for (int v = 0; v < nv; ++v) {
      const int c = v * 16 + hl;
      if (c < Ie / 32) {
        const size_t row = static_cast<size_t>(dd);
        const uint4 qv = __ldg(reinterpret_cast<const uint4*>(W.q + row * (Ie / 8)) + c);
        const float s = bf16_bits_to_float(__ldg(W.s + row * (Ie / kGroup) + (c >> 1)));
        const float b = bf16_bits_to_float(__ldg(W.b + row * (Ie / kGroup) + (c >> 1)));
        const float4* hl4 = reinterpret_cast<const float4*>(hs + static_cast<size_t>(j) * hst) + (v * 8) * 16 + hl;
        const float A = dot32(qv, hl4, 16);
        const float X = hsum[j * (hst / 32) + c];
        const float s128 = 128.f * s;
        p = fmaf(s128, A, fmaf(b - s128, X, p));
      }
    }
    p = halfwarp_sum(p);
    const float coef = sh ? sigma[t] : topk_w[t * g.k + j];
    acc = fmaf(coef, p, acc);
  }
  if (live && hl == 0) out[static_cast<size_t>(t) * g.H + d] = float_to_bf16_bits(acc);
}

int decode_tokens_per_pass(int H) {
  const int per_tok = xstride_of(H) * 4 + xstride_of(H) / 8;
  return max(1, min(kDecTokMaxDecode, 98304 / per_tok));
}

cudaError_t launch_decode_gateup(const Geometry& g, const LayerPtr& L, const uint16_t* x,
                                 const int32_t* offsets, const int32_t* perm,
                                 const int32_t* active, const int32_t* n_active,
                                 uint16_t* h, uint16_t* h_s, cudaStream_t s) {
  const int slots = min(g.E, g.T * g.k) + 1;
  const int fblocks = (max(g.I, g.Is) + kDecFeat - 1) / kDecFeat;
  const int kb = min(decode_tokens_per_pass(g.H), g.T);
  const int smem = kb * (xstride_of(g.H) * 4 + (xstride_of(g.H) / 32) * 4);
  const cudaError_t e = ensure_smem(reinterpret_cast<const void*>(decode_gateup_kernel), smem);
  if (e != cudaSuccess) return e;
  decode_gateup_kernel<<<dim3(slots, fblocks), 256, smem, s>>>(g, L, x, offsets, perm, active, n_active, h, h_s,
                                                               kb);
  return cudaGetLastError();
}

cudaError_t launch_decode_down_combine(const Geometry& g, const LayerPtr& L, const uint16_t* h,
                                       const uint16_t* h_s, const int32_t* topk_idx, const float* topk_w,
                                       const int32_t* inv_perm, const float* sigma, uint16_t* out,
                                       cudaStream_t s) {
  const int hst = hstride_of(max(g.I, g.Is));
  const int smem = (g.k + 1) * (hst * 4 + (hst / 32) * 4);
  const cudaError_t e = ensure_smem(reinterpret_cast<const void*>(decode_down_combine_kernel), smem);
  if (e != cudaSuccess) return e;
  decode_down_combine_kernel<<<dim3(g.T, (g.H + kDownDims - 1) / kDownDims), 256, smem, s>>>(
      g, L, h, h_s, topk_idx, topk_w, inv_perm, sigma, out);
  return cudaGetLastError();
}

}  // namespace moe
