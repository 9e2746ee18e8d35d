// Grouped expert GEMMs with the affine 4-bit weights rebuilt tile by tile
// (SIMT FP32 version).  Work comes from the device chunk list: a unit is one
// chunk of an expert's rows times one 64-wide block of output features.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kChunkRows = 128;   // rows per chunk of the grouped row space
constexpr int kBK = 64;           // K tile = one quantisation group
constexpr int kBF = 64;           // output features per unit

int gemm_chunk_rows() { return kChunkRows; }

// Dequantise a [64 features][64 k] tile of a q-matrix into smem as FP32,
// transposed to w_s[k][feature].  q: [rows, K/8] words, s/b: [rows, K/64].
__device__ __forceinline__ void dequant_tile_t(const uint32_t* __restrict__ q, const uint16_t* __restrict__ s,
                                               const uint16_t* __restrict__ b, int K, int f0, int nf, int k0,
                                               float* __restrict__ w_s) {
  const int wpr = K / 8;
  for (int i = threadIdx.x; i < kBF * 8; i += blockDim.x) {
    const int f = i >> 3, w = i & 7;
    float vals[8];
    if (f < nf) {
      const size_t row = static_cast<size_t>(f0 + f);
      const uint32_t word = __ldg(q + row * wpr + k0 / 8 + w);
      const float sc = bf16_bits_to_float(__ldg(s + row * (K / kGroup) + k0 / kGroup));
      const float bi = bf16_bits_to_float(__ldg(b + row * (K / kGroup) + k0 / kGroup));
#pragma unroll
      for (int c = 0; c < 8; ++c) vals[c] = fmaf(sc, static_cast<float>((word >> (4 * c)) & 0xFu), bi);
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) vals[c] = 0.f;
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) w_s[(w * 8 + c) * kBF + f] = vals[c];
  }
}

// ---------------------------------------------------------------------------
// gate/up: for unit (chunk, feature block f0):  g = x W_g^T, u = x W_u^T over
// the chunk's rows, h = bf16(silu(g) * u).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gateup_simt_kernel(
    Geometry g, LayerPtr L, const uint16_t* __restrict__ x, const int32_t* __restrict__ perm,
    const Chunk* __restrict__ chunks, const int32_t* __restrict__ n_chunks_ptr,
    uint16_t* __restrict__ h, uint16_t* __restrict__ h_s) {
  extern __shared__ float sm[];
  float* xs = sm;                          // [kBK][kChunkRows]
  float* wg = xs + kBK * kChunkRows;       // [kBK][kBF]
  float* wu = wg + kBK * kBF;              // [kBK][kBF]
  const int nfb = (max(g.I, g.Is) + kBF - 1) / kBF;
  const int n_units = *n_chunks_ptr * nfb;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int Tk = g.T * g.k;

  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const Chunk ch = chunks[unit / nfb];
    const int f0 = (unit % nfb) * kBF;
    const bool shared = ch.e >= g.E;
    const int Ie = shared ? g.Is : g.I;
    if (f0 >= Ie) continue;
    const int nf = min(kBF, Ie - f0);
    const QMatPtr Wg = shared ? L.sh_gate : QMatPtr{L.gate.q + static_cast<size_t>(ch.e) * g.I * (g.H / 8),
                                                     L.gate.s + static_cast<size_t>(ch.e) * g.I * (g.H / kGroup),
                                                     L.gate.b + static_cast<size_t>(ch.e) * g.I * (g.H / kGroup)};
    const QMatPtr Wu = shared ? L.sh_up : QMatPtr{L.up.q + static_cast<size_t>(ch.e) * g.I * (g.H / 8),
                                                   L.up.s + static_cast<size_t>(ch.e) * g.I * (g.H / kGroup),
                                                   L.up.b + static_cast<size_t>(ch.e) * g.I * (g.H / kGroup)};
    float ag[8][4], au[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) ag[r][c] = au[r][c] = 0.f;

    for (int k0 = 0; k0 < g.H; k0 += kBK) {
      __syncthreads();
      for (int i = threadIdx.x; i < kChunkRows * 8; i += blockDim.x) {
        const int r = i >> 3, v = i & 7;
        float vals[8];
        if (r < ch.rows) {
          const int R = ch.row0 + r;
          const int tok = shared ? (R - Tk) : (perm[R] / g.k);
          const uint4 xv = *reinterpret_cast<const uint4*>(x + static_cast<size_t>(tok) * g.H + k0 + v * 8);
          vals[0] = bf16_lo(xv.x); vals[1] = bf16_hi(xv.x); vals[2] = bf16_lo(xv.y); vals[3] = bf16_hi(xv.y);
          vals[4] = bf16_lo(xv.z); vals[5] = bf16_hi(xv.z); vals[6] = bf16_lo(xv.w); vals[7] = bf16_hi(xv.w);
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) vals[c] = 0.f;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) xs[(v * 8 + c) * kChunkRows + r] = vals[c];
      }
      dequant_tile_t(Wg.q, Wg.s, Wg.b, g.H, f0, nf, k0, wg);
      dequant_tile_t(Wu.q, Wu.s, Wu.b, g.H, f0, nf, k0, wu);
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < kBK; ++kk) {
        const float4 a0 = *reinterpret_cast<const float4*>(xs + kk * kChunkRows + ty * 8);
        const float4 a1 = *reinterpret_cast<const float4*>(xs + kk * kChunkRows + ty * 8 + 4);
        const float4 bg = *reinterpret_cast<const float4*>(wg + kk * kBF + tx * 4);
        const float4 bu = *reinterpret_cast<const float4*>(wu + kk * kBF + tx * 4);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bgv[4] = {bg.x, bg.y, bg.z, bg.w};
        const float buv[4] = {bu.x, bu.y, bu.z, bu.w};
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            ag[r][c] = fmaf(a[r], bgv[c], ag[r][c]);
            au[r][c] = fmaf(a[r], buv[c], au[r][c]);
          }
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int rr = ty * 8 + r;
      if (rr >= ch.rows) continue;
      const int R = ch.row0 + rr;
      uint16_t* dst = shared ? (h_s + static_cast<size_t>(R - Tk) * g.Is) : (h + static_cast<size_t>(R) * g.I);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int f = tx * 4 + c;
        if (f < nf) dst[f0 + f] = float_to_bf16_bits(silu(ag[r][c]) * au[r][c]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// down: for unit (chunk, output block d0): Y[R, d] = h_R . W_d[e][d, :]
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) down_simt_kernel(
    Geometry g, LayerPtr L, const uint16_t* __restrict__ h, const uint16_t* __restrict__ h_s,
    const Chunk* __restrict__ chunks, const int32_t* __restrict__ n_chunks_ptr, float* __restrict__ Y) {
  extern __shared__ float sm[];
  float* hs = sm;                          // [kBK][kChunkRows]
  float* wd = hs + kBK * kChunkRows;       // [kBK][kBF]
  const int nfb = g.H / kBF;
  const int n_units = *n_chunks_ptr * nfb;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int Tk = g.T * g.k;

  for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const Chunk ch = chunks[unit / nfb];
    const int d0 = (unit % nfb) * kBF;
    const bool shared = ch.e >= g.E;
    const int Ie = shared ? g.Is : g.I;
    const QMatPtr Wd = shared ? L.sh_down : QMatPtr{L.down.q + static_cast<size_t>(ch.e) * g.H * (g.I / 8),
                                                     L.down.s + static_cast<size_t>(ch.e) * g.H * (g.I / kGroup),
                                                     L.down.b + static_cast<size_t>(ch.e) * g.H * (g.I / kGroup)};
    float acc[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
    for (int k0 = 0; k0 < Ie; k0 += kBK) {
      __syncthreads();
      for (int i = threadIdx.x; i < kChunkRows * 8; i += blockDim.x) {
        const int r = i >> 3, v = i & 7;
        float vals[8];
        if (r < ch.rows) {
          const int R = ch.row0 + r;
          const uint16_t* src = shared ? (h_s + static_cast<size_t>(R - Tk) * g.Is) : (h + static_cast<size_t>(R) * g.I);
          const uint4 hv = *reinterpret_cast<const uint4*>(src + k0 + v * 8);
          vals[0] = bf16_lo(hv.x); vals[1] = bf16_hi(hv.x); vals[2] = bf16_lo(hv.y); vals[3] = bf16_hi(hv.y);
          vals[4] = bf16_lo(hv.z); vals[5] = bf16_hi(hv.z); vals[6] = bf16_lo(hv.w); vals[7] = bf16_hi(hv.w);
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) vals[c] = 0.f;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) hs[(v * 8 + c) * kChunkRows + r] = vals[c];
      }
      dequant_tile_t(Wd.q, Wd.s, Wd.b, Ie, d0, kBF, k0, wd);
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < kBK; ++kk) {
        const float4 a0 = *reinterpret_cast<const float4*>(hs + kk * kChunkRows + ty * 8);
        const float4 a1 = *reinterpret_cast<const float4*>(hs + kk * kChunkRows + ty * 8 + 4);
        const float4 b = *reinterpret_cast<const float4*>(wd + kk * kBF + tx * 4);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], bv[c], acc[r][c]);
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int rr = ty * 8 + r;
      if (rr >= ch.rows) continue;
      float4 o = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
      *reinterpret_cast<float4*>(Y + static_cast<size_t>(ch.row0 + rr) * g.H + d0 + tx * 4) = o;
    }
  }
}

cudaError_t launch_gateup(const Geometry& g, const LayerPtr& L, const uint16_t* x, const int32_t* perm,
                          const Chunk* chunks, const int32_t* n_chunks, int max_chunks,
                          uint16_t* h, uint16_t* h_s, int* status, cudaStream_t s) {
  (void)status;
  const int smem = (kBK * kChunkRows + 2 * kBK * kBF) * 4;
  cudaFuncSetAttribute(gateup_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int nfb = (max(g.I, g.Is) + kBF - 1) / kBF;
  const int grid = min(max_chunks * nfb, 148 * 3);
  gateup_simt_kernel<<<grid, 256, smem, s>>>(g, L, x, perm, chunks, n_chunks, h, h_s);
  return cudaGetLastError();
}

cudaError_t launch_down(const Geometry& g, const LayerPtr& L, const uint16_t* h, const uint16_t* h_s,
                        const Chunk* chunks, const int32_t* n_chunks, int max_chunks,
                        float* Y, int* status, cudaStream_t s) {
  (void)status;
  const int smem = (kBK * kChunkRows + kBK * kBF) * 4;
  cudaFuncSetAttribute(down_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int grid = min(max_chunks * (g.H / kBF), 148 * 4);
  down_simt_kernel<<<grid, 256, smem, s>>>(g, L, h, h_s, chunks, n_chunks, Y);
  return cudaGetLastError();
}

}  // namespace moe
