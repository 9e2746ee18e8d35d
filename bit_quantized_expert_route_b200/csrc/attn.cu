// Decode attention: one step of grouped-query softmax attention over a
// fixed-block (paged) key/value cache ("Perplexity's Lily: ...", section "The
// Model: Qwen3.6-35B-A3B in Focus": 16 query heads share 2 key/value heads;
// section "How It Works: Prefill and Decode Strategies": decode attention
// packs the query heads of a key/value head and keeps the cache in fixed
// blocks).
//
// The step is bound by HBM: every cached key and value is read once, and the
// query heads of a group (up to 8) all use the same read (GQA packing).  For
// D = 256 a position costs 2 x 512 B per key/value head and 8 heads x 4 D
// FLOPs, ~8 FLOP per byte, so the dot products go to the tensor cores only so
// that they never become the limit.
//
// Design.
//   * Grid (n_split, Hkv, B): CTA (s, g, b) takes a contiguous range of
//     16-position chunks of sequence b's key/value head g.  Each chunk's keys
//     and values arrive by TMA tiled copies (D / 64 boxes of 16 rows x 128 B
//     per cache, 128-byte swizzle) in a ring of shared-memory stages (12 for
//     D = 256).  The four warps take the chunks in turn and each owns the
//     stages of its chunks (three): it computes on one while the next two
//     are in flight, and its lane 0 refills a stage as soon as the warp has
//     read it.  (A single producer thread feeding all stages through
//     empty/full barriers streamed at under 2.5 TB/s with the arithmetic
//     removed.)  Each warp keeps its own running maximum, weight sum and
//     output.
//   * Per chunk a warp computes S^T = K Q^T on mma.sync m16n8k16 with the 16
//     positions as M and the group's heads as the 8 columns, so
//     no tensor-core row is padding; the keys come from shared memory by
//     ldmatrix (the swizzle makes the 8 rows of a matrix hit 8 different
//     bank groups).  The weights P^T (bf16) become the B operand of
//     O^T += V^T P^T by one movmatrix transpose per 8x8 tile, the values by
//     ldmatrix.trans.
//   * The softmax runs in base 2 with scale * log2(e) folded into the scores;
//     rows past ctx_len get weight 0 and their values are zeroed in shared
//     memory (a cache row that was never written may hold any bits).
//   * At the end the CTA merges its four warps (fixed order) and writes either
//     the normalised output (one range per sequence and head) or its partial
//     (maximum, weight sum, unnormalised output), which attn_combine_kernel
//     merges over the ranges in range order.
#include <cuda.h>
#include <math.h>

#include <algorithm>

#include "attn.h"
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int kAChunk = 16;                     // positions per pipeline stage (one m16 tile)
constexpr int kAMT = kAChunk / 16;              // m16 tiles per stage
constexpr int kABoxCols = 64;                   // elements per swizzled box row (128 B)
constexpr int kABoxBytes = kAChunk * 128;       // one box: 16 rows x 128 B
constexpr int kAWarps = 4;                      // consumer warps
constexpr int kAThreads = kAWarps * 32;         // every warp consumes and refills its own stages
constexpr int kAMaxGroup = 8;                   // query heads per key/value head: the n8 columns
constexpr int kARingMax = 24;
constexpr int kACombThreads = 256;              // combine CTA: 32 dims x 8 warps over the ranges
constexpr int kAMaxSplit = 1024;                // ranges per (sequence, KV head) the combine takes
constexpr int kATabCache = 512;                 // block-table entries a CTA fetches up front

struct alignas(64) AttnArgs {
  CUtensorMap tk, tv;          // caches as [n_blocks * Hkv * block rows][D], box 16 rows x 64 cols, 128B swizzle
  const uint16_t* q;           // [B][Hq][D]
  const int32_t* table;        // [B][max_blocks]
  const int32_t* ctx;          // [B]
  uint16_t* out;               // [B][Hq][D]
  float* part_ml;              // [B][Hkv][n_split][8][2]: running maximum (base 2), weight sum
  float* part_o;               // [B][Hkv][n_split][8][D]: unnormalised output
  int* status;
  int Hq, Hkv, block, max_blocks, n_blocks, n_split, cps, ring;
  float scale_log2;            // scale * log2(e)
  long long wait_limit;
};

struct CombArgs {
  const float* part_ml;
  const float* part_o;
  uint16_t* out;
  int Hq, Hkv, n_split;
};

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transpose of an 8x8 bf16 matrix held as mma fragments (lane: row lane/4,
// columns 2 (lane%4), +1).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t v) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(v));
  return r;
}

// Shared-memory byte offset of (row, 16-byte column chunk c) of a chunk's
// cache tile: box c / 8, and inside the box the 128-byte swizzle of TMA
// (chunk c % 8 of row r is stored at position (c % 8) ^ (r % 8)).
__device__ __forceinline__ uint32_t tile_off(int row, int c) {
  return static_cast<uint32_t>((c >> 3) * kABoxBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kAWarps * 32) : "memory"); }

__device__ __forceinline__ float max_over_rows(float v) {   // over the 8 lanes of one column pair (lane / 4)
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
}
__device__ __forceinline__ float sum_over_rows(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 8);
  return v + __shfl_xor_sync(0xffffffffu, v, 16);
}

template <int D>
__global__ void __launch_bounds__(kAThreads, 1) attn_decode_kernel(const __grid_constant__ AttnArgs a) {
  constexpr int NB = D / kABoxCols;          // boxes per chunk and cache
  constexpr int HALF = NB * kABoxBytes;      // keys (or values) of one chunk
  constexpr int STAGE = 2 * HALF;
  constexpr int KS = D / 16;                 // k-steps of the scores; d-tiles of the output
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + a.ring * STAGE);
  int* bad = reinterpret_cast<int*>(full + kARingMax);      // [ring] stage skipped: block index out of range
  float* wml = reinterpret_cast<float*>(bad + kARingMax);   // [warps][8 heads][2]
  int* abort_i = reinterpret_cast<int*>(wml + kAWarps * kAMaxGroup * 2);
  volatile int* abort_flag = abort_i;
  int* s_tab = abort_i + 4;                                 // [kATabCache] this CTA's block-table entries

  const int sp = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int group = a.Hq / a.Hkv;
  if (threadIdx.x == 0) {
    for (int i = 0; i < a.ring; ++i) tc::mbar_init(&full[i], 1);
    *abort_i = 0;
    tc::fence_barrier_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(&a.tk) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&a.tv) : "memory");
  }
  __syncthreads();
  pdl_wait();   // q, the table, ctx_len and the caches are written by earlier work of the stream

  // this CTA's chunk range
  const int cap = a.max_blocks * a.block;
  const int ctx_raw = __ldg(a.ctx + b);
  const int ctx = min(max(ctx_raw, 0), cap);
  if (ctx != ctx_raw && sp == 0 && g == 0 && threadIdx.x == 0) atomicExch(a.status, kStatusBadIndex);
  const int n_chunks = (ctx + kAChunk - 1) / kAChunk;
  const int c0 = sp * a.cps;
  const int nc = max(min(c0 + a.cps, n_chunks) - c0, 0);
  pdl_launch_dependents();
  // the block-table entries of the CTA's whole range, fetched together and
  // without waiting for ctx_len (entries past the sequence are never used)
  const int blk0 = c0 * kAChunk / a.block;
  const int nblk = min((c0 + a.cps) * kAChunk - 1, cap - 1) / a.block - blk0 + 1;
  const int32_t* trow = a.table + static_cast<size_t>(b) * a.max_blocks;
  for (int j = threadIdx.x; j < min(nblk, kATabCache); j += kAThreads) s_tab[j] = __ldg(trow + blk0 + j);
  __syncthreads();

  // Chunk i goes to stage i % ring, and ring is a multiple of the warps, so
  // every stage belongs to one warp: the warp that consumes a stage also
  // refills it (lane 0 issues the copies right after the warp's reads), no
  // other warp touches it, and the warp waits on its phases in order.
  auto issue = [&](int i) {
    const int sl = i % a.ring;
    const int pos = (c0 + i) * kAChunk;
    const int jb = pos / a.block - blk0;
    const int phys = jb < kATabCache ? s_tab[jb] : __ldg(trow + blk0 + jb);
    if (phys < 0 || phys >= a.n_blocks) {
      bad[sl] = 1;                      // published by the arrival's release
      atomicExch(a.status, kStatusBadIndex);
      tc::mbar_arrive(&full[sl]);
    } else {
      bad[sl] = 0;
      const int y = (phys * a.Hkv + g) * a.block + pos % a.block;
      const uint32_t dst = tc::smem_u32(sm + sl * STAGE);
      tc::mbar_arrive_expect_tx(&full[sl], STAGE);
#pragma unroll
      for (int x = 0; x < NB; ++x) tc::tma_load_2d(dst + x * kABoxBytes, &a.tk, x * kABoxCols, y, &full[sl]);
#pragma unroll
      for (int x = 0; x < NB; ++x) tc::tma_load_2d(dst + HALF + x * kABoxBytes, &a.tv, x * kABoxCols, y, &full[sl]);
    }
  };
  if (lane == 0)
    for (int i = warp; i < min(nc, a.ring); i += kAWarps) issue(i);

  const int r8 = lane >> 2, t4 = lane & 3;   // fragment row / column pair
  // Q^T as the B operand: lane holds head r8, dims 16 ks + 2 t4 (+1) and +8
  uint32_t qf[KS][2];
  {
    const bool live = r8 < group;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        a.q + (static_cast<size_t>(b) * a.Hq + g * group + (live ? r8 : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qf[ks][0] = live ? __ldg(qrow + ks * 8 + t4) : 0u;
      qf[ks][1] = live ? __ldg(qrow + ks * 8 + 4 + t4) : 0u;
    }
  }
  // running state for heads 2 t4 and 2 t4 + 1 (the lane's two columns)
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[KS][4];
#pragma unroll
  for (int i = 0; i < KS; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  const uint32_t sbase = tc::smem_u32(sm);
  // ldmatrix lane roles: matrix mi = lane / 8, row mr = lane % 8
  const int mi = lane >> 3, mr = lane & 7;
  bool ok = true;
  int i = warp;
  for (; i < nc; i += kAWarps) {
    const int sl = i % a.ring;
    ok = __all_sync(0xffffffffu,
                    ok && tc::mbar_wait(&full[sl], (i / a.ring) & 1, abort_flag, a.status, a.wait_limit));
    if (!ok) break;
    const int nv = min(kAChunk, ctx - (c0 + i) * kAChunk);   // valid rows of the chunk (>= 1)
    if (!bad[sl]) {
      uint8_t* st = sm + sl * STAGE;
      if (nv < kAChunk) {
        // rows past the context: zero their values (their weights are 0, but 0 * NaN is not)
        for (int e = lane; e < (kAChunk - nv) * NB * 8; e += 32) {
          const int row = nv + e / (NB * 8), c = e % (NB * 8);
          *reinterpret_cast<uint4*>(st + HALF + tile_off(row, c)) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }
      const uint32_t kb = sbase + sl * STAGE, vb = kb + HALF;
      // S^T = K Q^T for the two 16-row tiles
      float s[kAMT][4];
#pragma unroll
      for (int mt = 0; mt < kAMT; ++mt) {
        float c4[4][4];   // k-steps mod 4 accumulate apart: four short dependency chains instead of one
#pragma unroll
        for (int c = 0; c < 4; ++c) c4[c][0] = c4[c][1] = c4[c][2] = c4[c][3] = 0.f;
        const int row = mt * 16 + mr + 8 * (mi & 1);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kb + tile_off(row, 2 * ks + (mi >> 1)), a0, a1, a2, a3);
          mma16816(c4[ks & 3], a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) s[mt][e] = (c4[0][e] + c4[1][e]) + (c4[2][e] + c4[3][e]);
      }
      // scale, mask, running maximum per head column
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < kAMT; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const bool live = mt * 16 + r8 + 8 * h < nv;
          s[mt][2 * h] = live ? s[mt][2 * h] * a.scale_log2 : -INFINITY;
          s[mt][2 * h + 1] = live ? s[mt][2 * h + 1] * a.scale_log2 : -INFINITY;
          mx0 = fmaxf(mx0, s[mt][2 * h]);
          mx1 = fmaxf(mx1, s[mt][2 * h + 1]);
        }
      mx0 = max_over_rows(mx0);
      mx1 = max_over_rows(mx1);
      const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);   // finite: row 0 of the chunk is valid
      const float al0 = exp2f(m0 - n0), al1 = exp2f(m1 - n1);
      m0 = n0;
      m1 = n1;
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int mt = 0; mt < kAMT; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          s[mt][2 * h] = exp2f(s[mt][2 * h] - n0);
          s[mt][2 * h + 1] = exp2f(s[mt][2 * h + 1] - n1);
          ps0 += s[mt][2 * h];
          ps1 += s[mt][2 * h + 1];
        }
      l0 = fmaf(l0, al0, ps0);
      l1 = fmaf(l1, al1, ps1);
#pragma unroll
      for (int dt = 0; dt < KS; ++dt) {
        o[dt][0] *= al0;
        o[dt][1] *= al1;
        o[dt][2] *= al0;
        o[dt][3] *= al1;
      }
      // O^T += V^T P^T, one 16-position k-step per score tile
#pragma unroll
      for (int mt = 0; mt < kAMT; ++mt) {
        const uint32_t b0 = movmatrix_t(pack_bf16x2(s[mt][0], s[mt][1]));
        const uint32_t b1 = movmatrix_t(pack_bf16x2(s[mt][2], s[mt][3]));
        const int row = mt * 16 + mr + 8 * (mi >> 1);
#pragma unroll
        for (int dt = 0; dt < KS; ++dt) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(vb + tile_off(row, 2 * dt + (mi & 1)), a0, a1, a2, a3);
          mma16816(o[dt], a0, a1, a2, a3, b0, b1);
        }
      }
    }
    // the stage's generic reads and writes precede its next TMA fill
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && i + a.ring < nc) issue(i + a.ring);
  }
  if (!ok && lane == 0)   // gave up: the copies this warp issued land before the CTA may exit
    for (int j = i; j < min(nc, i + a.ring); j += kAWarps) tc::mbar_wait_drain(&full[j % a.ring], (j / a.ring) & 1, a.status);

  // ---------------------------------------------- merge the four warps
  l0 = sum_over_rows(l0);
  l1 = sum_over_rows(l1);
  if (r8 == 0) {
    wml[(warp * kAMaxGroup + 2 * t4) * 2 + 0] = m0;
    wml[(warp * kAMaxGroup + 2 * t4) * 2 + 1] = l0;
    wml[(warp * kAMaxGroup + 2 * t4 + 1) * 2 + 0] = m1;
    wml[(warp * kAMaxGroup + 2 * t4 + 1) * 2 + 1] = l1;
  }
  consumers_sync();
  if (*abort_flag) return;   // every consumer read the same value after the barrier
  float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
  for (int w = 0; w < kAWarps; ++w) {
    M0 = fmaxf(M0, wml[(w * kAMaxGroup + 2 * t4) * 2]);
    M1 = fmaxf(M1, wml[(w * kAMaxGroup + 2 * t4 + 1) * 2]);
  }
  const float f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M0);
  const float f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M1);
  // every stage has been consumed (all issued copies landed): the ring is free
  float* red = reinterpret_cast<float*>(sm);   // [warps][8 heads][D]
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    const int d = dt * 16 + r8;
    red[(warp * kAMaxGroup + 2 * t4) * D + d] = o[dt][0] * f0;
    red[(warp * kAMaxGroup + 2 * t4 + 1) * D + d] = o[dt][1] * f1;
    red[(warp * kAMaxGroup + 2 * t4) * D + d + 8] = o[dt][2] * f0;
    red[(warp * kAMaxGroup + 2 * t4 + 1) * D + d + 8] = o[dt][3] * f1;
  }
  consumers_sync();
  const int tid = threadIdx.x;
  const size_t part = (static_cast<size_t>(b) * a.Hkv + g) * a.n_split + sp;
  for (int e = tid; e < group * D; e += kAWarps * 32) {
    const int h = e / D, d = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w) M = fmaxf(M, wml[(w * kAMaxGroup + h) * 2]);
    float acc = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w) {
      const float mw = wml[(w * kAMaxGroup + h) * 2];
      const float fw = mw == -INFINITY ? 0.f : exp2f(mw - M);
      L = fmaf(wml[(w * kAMaxGroup + h) * 2 + 1], fw, L);
      acc += red[(w * kAMaxGroup + h) * D + d];
    }
    if (a.n_split == 1) {
      a.out[(static_cast<size_t>(b) * a.Hq + g * group + h) * D + d] = float_to_bf16_bits(L > 0.f ? acc / L : 0.f);
    } else {
      a.part_o[(part * kAMaxGroup + h) * D + d] = acc;
      if (d == 0) {
        a.part_ml[(part * kAMaxGroup + h) * 2 + 0] = M;
        a.part_ml[(part * kAMaxGroup + h) * 2 + 1] = L;
      }
    }
  }
}

// Merge of the ranges' partials of one (sequence, query head), 32 dims per
// CTA: o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.  Ranges with no
// positions (l_s = 0) are skipped; all empty gives 0.  The ranges' (m, l) go
// to shared memory in one pass, warp 0 forms M, the factors and L (fixed
// order), then the 8 warps each sum every 8th range for the CTA's 32 dims
// (loads of different ranges in flight together) and the 8 partial sums are
// added in warp order.
template <int D>
__global__ void __launch_bounds__(kACombThreads) attn_combine_kernel(const CombArgs a) {
  __shared__ float s_f[kAMaxSplit], s_l[kAMaxSplit];
  __shared__ float s_acc[kACombThreads / 32][32];
  __shared__ float s_L;
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int h = blockIdx.y, b = blockIdx.z, d = blockIdx.x * 32 + lane;
  const int group = a.Hq / a.Hkv, g = h / group, j = h % group;
  const int ns = a.n_split;
  const size_t base = (static_cast<size_t>(b) * a.Hkv + g) * ns;
  const float* ml = a.part_ml + (base * kAMaxGroup + j) * 2;
  for (int s = tid; s < ns; s += kACombThreads) {
    const float l = __ldcg(ml + s * kAMaxGroup * 2 + 1);
    s_f[s] = l > 0.f ? __ldcg(ml + s * kAMaxGroup * 2) : -INFINITY;
    s_l[s] = l;
  }
  __syncthreads();
  if (w == 0) {
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, s_f[s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int s = lane; s < ns; s += 32) {
      const float f = s_l[s] > 0.f ? exp2f(s_f[s] - M) : 0.f;
      s_f[s] = f;
      L = fmaf(s_l[s], f, L);
    }
    L = warp_sum(L);
    if (lane == 0) s_L = L;
  }
  __syncthreads();
  const float* po = a.part_o + (base * kAMaxGroup + j) * D + d;
  constexpr int kW = kACombThreads / 32;
  float acc = 0.f;
  for (int s0 = w; s0 < ns; s0 += 8 * kW) {
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {   // eight ranges' loads in flight; an empty range's slot may hold anything
      const int s = s0 + q * kW;
      v[q] = s < ns ? __ldcg(po + static_cast<size_t>(s) * kAMaxGroup * D) : 0.f;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int s = s0 + q * kW;
      const float f = s < ns ? s_f[s] : 0.f;
      acc = f > 0.f ? fmaf(v[q], f, acc) : acc;
    }
  }
  s_acc[w][lane] = acc;
  __syncthreads();
  if (w == 0) {
    float o = 0.f;
#pragma unroll
    for (int q = 0; q < kACombThreads / 32; ++q) o += s_acc[q][lane];
    const float L = s_L;
    a.out[(static_cast<size_t>(b) * a.Hq + h) * D + d] = float_to_bf16_bits(L > 0.f ? o / L : 0.f);
  }
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

constexpr size_t kACtrl = 256;   // control block (status word) at the start of the workspace

struct Plan {
  int n_split, cps;
};

// Ranges per (sequence, key/value head): enough CTAs to cover the SMs once,
// at least 2 chunks per range.
Plan make_plan(int B, int Hkv, int block, int max_blocks, int sms) {
  const long long max_chunks = static_cast<long long>(max_blocks) * block / kAChunk;
  const long long pairs = static_cast<long long>(B) * Hkv;
  long long ns = (sms + pairs - 1) / pairs;
  ns = std::min<long long>(ns, (max_chunks + 1) / 2);
  ns = std::min<long long>(ns, kAMaxSplit);
  if (ns < 1) ns = 1;
  Plan p;
  p.cps = static_cast<int>((max_chunks + ns - 1) / ns);
  p.n_split = static_cast<int>((max_chunks + p.cps - 1) / p.cps);
  return p;
}

bool attn_sizes_ok(int B, int Hq, int Hkv, int D, int block, int max_blocks, int n_blocks) {
  if (B < 1 || B > 65535 || Hkv < 1 || Hq < Hkv || Hq % Hkv || Hq / Hkv > kAMaxGroup) return false;
  if (D != 128 && D != 256) return false;
  if (block < kAChunk || block % kAChunk || max_blocks < 1 || n_blocks < 1) return false;
  if (static_cast<long long>(n_blocks) * Hkv * block >= (1ll << 31)) return false;
  if (static_cast<long long>(max_blocks) * block >= (1ll << 31)) return false;
  return true;
}

size_t part_bytes(int B, int Hkv, int D, const Plan& p) {
  if (p.n_split == 1) return 0;
  const size_t n = static_cast<size_t>(B) * Hkv * p.n_split * kAMaxGroup;
  return (n * 2 * sizeof(float) + 255) / 256 * 256 + n * D * sizeof(float);
}

// Stages of the ring: a multiple of the consumer warps, so that stage i is
// always consumed by warp i % kAWarps and that warp waits on the stage's
// phases strictly in order (a parity wait cannot tell phase n from n + 2, so
// a stage shared by two warps in turn could be taken a fill early).
template <int D>
int ring_stages() {
  constexpr int stage = 2 * (D / kABoxCols) * kABoxBytes;
  int r = (200 * 1024) / stage;
  if (r > kARingMax) r = kARingMax;
  return r / kAWarps * kAWarps;
}
static_assert(kARingMax % kAWarps == 0, "the ring holds whole rounds of the consumer warps");

template <int D>
int smem_bytes(int ring) {
  constexpr int stage = 2 * (D / kABoxCols) * kABoxBytes;
  const int red = kAWarps * kAMaxGroup * D * 4;   // the merge reuses the ring
  const int body = (ring * stage > red ? ring * stage : red);
  return 1024 + body + kARingMax * 8 + kARingMax * 4 + kAWarps * kAMaxGroup * 2 * 4 + 16 + kATabCache * 4;
}

template <int D>
int launch(const AttnArgs& a, int B, cudaStream_t s) {
  const int smem = smem_bytes<D>(a.ring);
  if (ensure_smem(reinterpret_cast<const void*>(attn_decode_kernel<D>), smem) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_pdl(attn_decode_kernel<D>, dim3(a.n_split, a.Hkv, B), dim3(kAThreads), smem, s, a) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (a.n_split > 1) {
    CombArgs c{a.part_ml, a.part_o, a.out, a.Hq, a.Hkv, a.n_split};
    if (launch_pdl(attn_combine_kernel<D>, dim3(D / 32, a.Hq, B), dim3(kACombThreads), 0, s, c) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

MOE_API size_t attn_decode_workspace_size(int B, int Hkv, int D, int block, int max_blocks) {
  if (!attn_sizes_ok(B, Hkv, Hkv, D, block, max_blocks, 1)) return 0;
  return kACtrl + part_bytes(B, Hkv, D, make_plan(B, Hkv, block, max_blocks, num_sms()));
}

MOE_API int attn_decode_plan(int B, int Hkv, int block, int max_blocks, int* n_split, int* chunks_per_split) {
  if (!n_split || !chunks_per_split) return MOE_ERR_INVALID_ARG;
  if (!attn_sizes_ok(B, Hkv, Hkv, 128, block, max_blocks, 1)) return MOE_ERR_UNSUPPORTED;
  const Plan p = make_plan(B, Hkv, block, max_blocks, num_sms());
  *n_split = p.n_split;
  *chunks_per_split = p.cps;
  return MOE_OK;
}

MOE_API int attn_decode(const moe_bf16* q, const moe_bf16* k_cache, const moe_bf16* v_cache,
                        const int32_t* block_table, const int32_t* ctx_len, int B, int Hq, int Hkv, int D, int block,
                        int max_blocks, int n_blocks, float scale, moe_bf16* out, void* workspace,
                        size_t workspace_bytes, moe_stream stream) {
  if (!q || !k_cache || !v_cache || !block_table || !ctx_len || !out) return MOE_ERR_INVALID_ARG;
  auto aligned = [](const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0; };
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q, 4) || !aligned(out, 2) ||
      !aligned(block_table, 4) || !aligned(ctx_len, 4))
    return MOE_ERR_INVALID_ARG;
  if (!attn_sizes_ok(B, Hq, Hkv, D, block, max_blocks, n_blocks)) return MOE_ERR_UNSUPPORTED;
  const Plan p = make_plan(B, Hkv, block, max_blocks, num_sms());
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < kACtrl + part_bytes(B, Hkv, D, p))
    return MOE_ERR_WORKSPACE;
  AttnArgs a{};
  const uint64_t rows = static_cast<uint64_t>(n_blocks) * Hkv * block;
  if (!make_tmap_2d(&a.tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k_cache, D, rows, kABoxCols, kAChunk,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&a.tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v_cache, D, rows, kABoxCols, kAChunk,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return MOE_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t n = static_cast<size_t>(B) * Hkv * p.n_split * kAMaxGroup;
  a.q = q;
  a.table = block_table;
  a.ctx = ctx_len;
  a.out = out;
  a.part_ml = reinterpret_cast<float*>(ws + kACtrl);
  a.part_o = reinterpret_cast<float*>(ws + kACtrl + (n * 2 * sizeof(float) + 255) / 256 * 256);
  a.status = reinterpret_cast<int*>(ws);
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.block = block;
  a.max_blocks = max_blocks;
  a.n_blocks = n_blocks;
  a.n_split = p.n_split;
  a.cps = p.cps;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(D));
  a.scale_log2 = sc * 1.4426950408889634f;
  a.wait_limit = wait_limit_cycles();
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (D == 128) {
    a.ring = ring_stages<128>();
    return launch<128>(a, B, s);
  }
  a.ring = ring_stages<256>();
  return launch<256>(a, B, s);
}

}  // extern "C"
