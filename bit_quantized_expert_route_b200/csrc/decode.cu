// Decode path (T <= 64): the layer as bandwidth-bound GEMVs over the active
// experts only.  Batch-1 decoding barely reuses a weight, so every packed
// weight byte is read once with 128-bit coalesced loads and rebuilt in
// registers in FP32 ("Perplexity's Lily: ...", section "How It Works: Prefill
// and Decode Strategies", decode paragraph; "Frequently Asked Questions":
// decode is bound by moving weights, not by arithmetic).
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDecFeat = 32;    // intermediate features per CTA (8 warps x 4)
constexpr int kDecTokMax = 8;   // tokens per pass over the weights
constexpr int kDownDims = 16;   // output dims per CTA in down+combine (8 warps x 2)

__device__ __forceinline__ QMatPtr expert_qmat(const QMatPtr& stack, int e, size_t rows, size_t cols) {
  return QMatPtr{stack.q + static_cast<size_t>(e) * rows * (cols / 8),
                 stack.s + static_cast<size_t>(e) * rows * (cols / kGroup),
                 stack.b + static_cast<size_t>(e) * rows * (cols / kGroup)};
}

// One warp, 4 features x {gate, up} x NT tokens, over the full hidden size.
template <int NT>
__device__ __forceinline__ void gateup_pass(const QMatPtr& Wg, const QMatPtr& Wu, int H, int f_base, int nf,
                                            const uint4* __restrict__ xs, int vec, int lane, float (&res)[2][4][NT]) {
  float acc[2][4][NT];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int f = 0; f < 4; ++f)
#pragma unroll
      for (int r = 0; r < NT; ++r) acc[m][f][r] = 0.f;
  const int qvec = H / 32;          // uint4 of codes per weight row
  const int words_per_row = H / 8;
  const int groups_per_row = H / kGroup;
  for (int c = lane; c < qvec; c += 32) {
    uint4 qv[2][4];
    float sc[2][4], bi[2][4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const QMatPtr& W = m == 0 ? Wg : Wu;
#pragma unroll
      for (int f = 0; f < 4; ++f) {
        if (f < nf) {
          const size_t row = static_cast<size_t>(f_base + f);
          qv[m][f] = __ldg(reinterpret_cast<const uint4*>(W.q + row * words_per_row) + c);
          sc[m][f] = bf16_bits_to_float(__ldg(W.s + row * groups_per_row + c / 2));
          bi[m][f] = bf16_bits_to_float(__ldg(W.b + row * groups_per_row + c / 2));
        } else {
          qv[m][f] = make_uint4(0u, 0u, 0u, 0u);
          sc[m][f] = 0.f;
          bi[m][f] = 0.f;
        }
      }
    }
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      float xv[NT][8];
#pragma unroll
      for (int r = 0; r < NT; ++r) {
        const uint4 v = xs[r * vec + c * 4 + wd];
        xv[r][0] = bf16_lo(v.x); xv[r][1] = bf16_hi(v.x); xv[r][2] = bf16_lo(v.y); xv[r][3] = bf16_hi(v.y);
        xv[r][4] = bf16_lo(v.z); xv[r][5] = bf16_hi(v.z); xv[r][6] = bf16_lo(v.w); xv[r][7] = bf16_hi(v.w);
      }
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int f = 0; f < 4; ++f) {
          const uint32_t word = wd == 0 ? qv[m][f].x : wd == 1 ? qv[m][f].y : wd == 2 ? qv[m][f].z : qv[m][f].w;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float w = fmaf(sc[m][f], static_cast<float>((word >> (4 * q)) & 0xFu), bi[m][f]);
#pragma unroll
            for (int r = 0; r < NT; ++r) acc[m][f][r] = fmaf(w, xv[r][q], acc[m][f][r]);
          }
        }
    }
  }
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int f = 0; f < 4; ++f)
#pragma unroll
      for (int r = 0; r < NT; ++r) res[m][f][r] = warp_sum(acc[m][f][r]);
}

template <int NT>
__device__ __forceinline__ void gateup_tokens(const QMatPtr& Wg, const QMatPtr& Wu, int H, int f_base, int nf,
                                              const uint4* xs, int vec, int lane, int nt, uint16_t* const* dst,
                                              int f_col) {
  float res[2][4][NT];
  gateup_pass<NT>(Wg, Wu, H, f_base, nf, xs, vec, lane, res);
#pragma unroll
  for (int f = 0; f < 4; ++f)
#pragma unroll
    for (int r = 0; r < NT; ++r)
      if (lane == ((f * NT + r) & 31) && f < nf && r < nt)
        dst[r][f_col + f] = float_to_bf16_bits(silu(res[0][f][r]) * res[1][f][r]);
}

__global__ void __launch_bounds__(256) decode_gateup_kernel(
    Geometry g, LayerPtr L, const uint16_t* __restrict__ x, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ perm, const int32_t* __restrict__ active, const int32_t* __restrict__ n_active,
    uint16_t* __restrict__ h, uint16_t* __restrict__ h_s) {
  extern __shared__ uint4 xs[];   // [kDecTokMax][H/8]
  const int slot = blockIdx.x;
  if (slot >= *n_active) return;
  const int e = active[slot];
  const bool shared = e >= g.E;
  const int Ie = shared ? g.Is : g.I;
  const int i0 = blockIdx.y * kDecFeat;
  if (i0 >= Ie) return;
  const int pos0 = shared ? 0 : offsets[e];
  const int ntok = shared ? g.T : offsets[e + 1] - pos0;
  const QMatPtr Wg = shared ? L.sh_gate : expert_qmat(L.gate, e, g.I, g.H);
  const QMatPtr Wu = shared ? L.sh_up : expert_qmat(L.up, e, g.I, g.H);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vec = g.H / 8;
  const int f_col = i0 + warp * 4;
  const int nf = max(0, min(4, Ie - f_col));

  for (int tb = 0; tb < ntok; tb += kDecTokMax) {
    const int nt = min(kDecTokMax, ntok - tb);
    __syncthreads();
    for (int i = threadIdx.x; i < kDecTokMax * vec; i += blockDim.x) {
      const int r = i / vec, c = i - r * vec;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < nt) {
        const int tok = shared ? (tb + r) : perm[pos0 + tb + r] / g.k;
        v = reinterpret_cast<const uint4*>(x + static_cast<size_t>(tok) * g.H)[c];
      }
      xs[i] = v;
    }
    __syncthreads();
    if (nf == 0) continue;
    uint16_t* dst[kDecTokMax];
#pragma unroll
    for (int r = 0; r < kDecTokMax; ++r) {
      const int rr = min(r, nt - 1);
      dst[r] = shared ? h_s + static_cast<size_t>(tb + rr) * g.Is : h + static_cast<size_t>(pos0 + tb + rr) * g.I;
    }
    if (nt == 1)
      gateup_tokens<1>(Wg, Wu, g.H, f_col, nf, xs, vec, lane, nt, dst, f_col);
    else if (nt == 2)
      gateup_tokens<2>(Wg, Wu, g.H, f_col, nf, xs, vec, lane, nt, dst, f_col);
    else if (nt <= 4)
      gateup_tokens<4>(Wg, Wu, g.H, f_col, nf, xs, vec, lane, nt, dst, f_col);
    else
      gateup_tokens<8>(Wg, Wu, g.H, f_col, nf, xs, vec, lane, nt, dst, f_col);
  }
}

__device__ __forceinline__ float halfwarp_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// out[t, d] = bf16( sum_j w[t,j] * (W_d[idx_j][d,:] . h_{t,j})  +  sigma_t * (W_sd[d,:] . hs_t) )
// One half-warp per output dim; the k + 1 terms are added in slot order.
__global__ void __launch_bounds__(256) decode_down_combine_kernel(
    Geometry g, LayerPtr L, const uint16_t* __restrict__ h, const uint16_t* __restrict__ h_s,
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, const int32_t* __restrict__ inv_perm,
    const float* __restrict__ sigma, uint16_t* __restrict__ out) {
  extern __shared__ uint4 hsm[];   // [k + 1][Imax / 8]
  const int t = blockIdx.x;
  const int Imax = max(g.I, g.Is);
  const int hv = Imax / 8;
  for (int i = threadIdx.x; i < (g.k + 1) * hv; i += blockDim.x) {
    const int j = i / hv, c = i - j * hv;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j < g.k) {
      if (c < g.I / 8) v = reinterpret_cast<const uint4*>(h + static_cast<size_t>(inv_perm[t * g.k + j]) * g.I)[c];
    } else if (c < g.Is / 8) {
      v = reinterpret_cast<const uint4*>(h_s + static_cast<size_t>(t) * g.Is)[c];
    }
    hsm[i] = v;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hl = lane & 15;
  const int d = blockIdx.y * kDownDims + warp * 2 + (lane >> 4);
  const bool live = d < g.H;
  float acc = 0.f;
  for (int j = 0; j <= g.k; ++j) {
    const bool sh = j == g.k;
    const int Ie = sh ? g.Is : g.I;
    const QMatPtr W = sh ? L.sh_down : expert_qmat(L.down, topk_idx[t * g.k + j], g.H, g.I);
    const int qvec = Ie / 32;
    float p = 0.f;
    if (live) {
      const size_t row = static_cast<size_t>(d);
      for (int c = hl; c < qvec; c += 16) {
        const uint4 qv = __ldg(reinterpret_cast<const uint4*>(W.q + row * (Ie / 8)) + c);
        const float sc = bf16_bits_to_float(__ldg(W.s + row * (Ie / kGroup) + c / 2));
        const float bi = bf16_bits_to_float(__ldg(W.b + row * (Ie / kGroup) + c / 2));
        const uint32_t words[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          const uint4 hh = hsm[j * hv + c * 4 + wd];
          const float hf[8] = {bf16_lo(hh.x), bf16_hi(hh.x), bf16_lo(hh.y), bf16_hi(hh.y),
                               bf16_lo(hh.z), bf16_hi(hh.z), bf16_lo(hh.w), bf16_hi(hh.w)};
#pragma unroll
          for (int q = 0; q < 8; ++q)
            p = fmaf(fmaf(sc, static_cast<float>((words[wd] >> (4 * q)) & 0xFu), bi), hf[q], p);
        }
      }
    }
    p = halfwarp_sum(p);
    const float coef = sh ? sigma[t] : topk_w[t * g.k + j];
    acc = fmaf(coef, p, acc);
  }
  if (live && hl == 0) out[static_cast<size_t>(t) * g.H + d] = float_to_bf16_bits(acc);
}

cudaError_t launch_decode_gateup(const Geometry& g, const LayerPtr& L, const uint16_t* x,
                                 const int32_t* offsets, const int32_t* perm,
                                 const int32_t* active, const int32_t* n_active,
                                 uint16_t* h, uint16_t* h_s, cudaStream_t s) {
  const int slots = min(g.E, g.T * g.k) + 1;
  const int fblocks = (max(g.I, g.Is) + kDecFeat - 1) / kDecFeat;
  const int smem = kDecTokMax * g.H * 2;
  cudaFuncSetAttribute(decode_gateup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  decode_gateup_kernel<<<dim3(slots, fblocks), 256, smem, s>>>(g, L, x, offsets, perm, active, n_active, h, h_s);
  return cudaGetLastError();
}

cudaError_t launch_decode_down_combine(const Geometry& g, const LayerPtr& L, const uint16_t* h,
                                       const uint16_t* h_s, const int32_t* topk_idx, const float* topk_w,
                                       const int32_t* inv_perm, const float* sigma, uint16_t* out,
                                       cudaStream_t s) {
  const int smem = (g.k + 1) * max(g.I, g.Is) * 2;
  decode_down_combine_kernel<<<dim3(g.T, (g.H + kDownDims - 1) / kDownDims), 256, smem, s>>>(
      g, L, h, h_s, topk_idx, topk_w, inv_perm, sigma, out);
  return cudaGetLastError();
}

}  // namespace moe
