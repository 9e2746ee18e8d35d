// Decode path for steps of up to 128 tokens that the fused kernel does not
// take: the tokens of the step spread over many experts with a few tokens
// each, so the layer is bound by streaming the active experts' packed weights
// ("Perplexity's Lily: ...", section "How It Works: Prefill and Decode
// Strategies", decode paragraph; "Frequently Asked Questions": decode moves
// weights, not arithmetic).  Two persistent kernels do the expert GEMVs on
// the tensor cores through warp-level mma.sync, the (up to) 8 tokens of an
// expert being the 8 columns of the n8 tile; the fixed-order combine kernel
// of the prefill path then adds each token's k + 1 terms.
//
// Work items.  An active expert slot with n tokens is cut into ceil(n/8)
// token tiles; an item is one token tile of one slot times one block of rows
// (gate/up: 128 features; down: 256 output dims).  A CTA of 8 warps takes
// items blockIdx.x, blockIdx.x + gridDim.x, ...; the items of one (slot, row
// block) are numbered consecutively over their token tiles, so the CTAs that
// read the same weights run side by side and all but the first read them
// from L2.  Per item the CTA stages the tile's activations in shared memory
// (bf16, in the interleaved order of mma_dq.cuh, plus per-group sums); each
// warp computes two 16-row tiles against it (gate/up: the gate and the up
// tile of the same 16 features, so SwiGLU needs no exchange; down: 32
// consecutive dims), so every activation fragment read from shared memory
// feeds two MMAs.
//
// Weight streaming.  The packed codes go from global memory straight into
// the MMA operand registers (8 bytes per lane per row and group): a warp
// holds the next block of B groups (B = 4, or 2 where a row has 2 mod 4
// groups or the scale stacks are only 4-byte aligned) of both tiles in
// flight (group j of the next block is loaded right after group j of the
// current block has been used), running on into the CTA's next item, whose
// weights do not depend on the activations; the scales and biases of the
// next block (one load per row) are loaded a block ahead, and L2 prefetches
// run a block further (deeper prefetches brought lines that were evicted
// before use: 309 MB read for 263 MB of weights at T=64, 3.5% slower).  Shared memory carries only the activations, read
// conflict-free: token rows are padded by 16 bytes and the group sums are
// stored token-minor, so a lane's two sums are one 8-byte read.  The kernels
// are issue-bound rather than memory-bound: the dequantising AND-OR/shift
// work and the MMA -> scale -> accumulate chains dominate.
#include <initializer_list>

#include "common.cuh"
#include "kernels.h"
#include "mma_dq.cuh"

namespace moe {

constexpr int kMWarps = 8;
constexpr int kMThreads = kMWarps * 32;
constexpr int kMGateUpRows = 16 * kMWarps;   // features of a gate/up item
constexpr int kMDownRows = 32 * kMWarps;     // output dims of a down item
constexpr int kMTok = 8;                     // tokens of an item: the n8 column tile

__device__ __forceinline__ QMatPtr expert_qmat(const QMatPtr& stack, int e, size_t rows, size_t cols) {
  return QMatPtr{stack.q + static_cast<size_t>(e) * rows * (cols / 8),
                 stack.s + static_cast<size_t>(e) * rows * (cols / kGroup),
                 stack.b + static_cast<size_t>(e) * rows * (cols / kGroup)};
}

// Items of every active slot, as an exclusive prefix in shared memory:
// start[s] = first item of slot s, start[n_act] = the total.  Slot s is
// expert active[s] (E: the shared expert, which sees all T tokens) with
// ceil(n/8) token tiles times `blocks_routed` (or `blocks_shared`) row blocks.
// Two slots per thread, so up to 2 * kMThreads slots.
__device__ int build_items(const Geometry& g, const int32_t* offsets, const int32_t* active, int n_act,
                           int blocks_routed, int blocks_shared, int* start, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int c[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int s = 2 * threadIdx.x + j;
    c[j] = 0;
    if (s < n_act) {
      const int e = active[s];
      const int n = e >= g.E ? g.T : offsets[e + 1] - offsets[e];
      c[j] = (n + kMTok - 1) / kMTok * (e >= g.E ? blocks_shared : blocks_routed);
    }
  }
  const int v = c[0] + c[1];
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kMWarps; ++w) {
    const int t = warp_tot[w];
    before += w < warp ? t : 0;
    total += t;
  }
  const int excl = before + incl - v;
  if (2 * threadIdx.x < n_act) start[2 * threadIdx.x] = excl;
  if (2 * threadIdx.x + 1 < n_act) start[2 * threadIdx.x + 1] = excl + c[0];
  if (threadIdx.x == 0) start[n_act] = total;
  __syncthreads();
  return total;
}

// Item `it` decoded: slot s = the last with start[s] <= it, its expert, the
// token tile (first grouped position pos0, tn tokens) and the row block.
struct Item {
  int e;        // expert (E: shared)
  bool sh;
  int blk;      // row block
  int tn;       // tokens in the tile (1..8)
  int pos0;     // routed: first grouped position; shared: first token
};

__device__ __forceinline__ Item decode_item(const Geometry& g, const int* start, int n_act, const int32_t* offsets,
                                            const int32_t* active, int it) {
  int lo = 0, hi = n_act - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= it) lo = mid;
    else hi = mid - 1;
  }
  Item r;
  r.e = active[lo];
  r.sh = r.e >= g.E;
  const int nt = r.sh ? g.T : offsets[r.e + 1] - offsets[r.e];
  const int ntt = (nt + kMTok - 1) / kMTok;
  const int local = it - start[lo];
  r.blk = local / ntt;
  const int tt = local - r.blk * ntt;
  r.tn = min(kMTok, nt - tt * kMTok);
  r.pos0 = (r.sh ? 0 : offsets[r.e]) + tt * kMTok;
  return r;
}

// Stage `tn` activation rows of `cols` bf16 values (row r at row_of(r)) as
// xs[r][cols/8 + 1] uint4 in the interleaved order, and their sums per group
// of 64 (FP32) as xsum[group][8 tokens].  Each group's 8 uint4 are handled by
// 8 consecutive lanes, which add their partial sums with shuffles; each
// thread has kStageLoads loads in flight.
constexpr int kStageLoads = 4;
template <class RowOf>
__device__ __forceinline__ void stage_tile(RowOf row_of, int tn, int cols, uint4* xs, float* xsum) {
  const int cpr = cols / 8;
  const int n = tn * cpr;
  // the loop bound is the warp's first index, so whole warps take part in the shuffles
  for (int base = threadIdx.x & ~31; base < n; base += kMThreads * kStageLoads) {
    const int i0 = base + (threadIdx.x & 31);
    uint4 v[kStageLoads];
#pragma unroll
    for (int j = 0; j < kStageLoads; ++j) {
      const int i = i0 + j * kMThreads;
      const int r = i / cpr, u = i - r * cpr;
      v[j] = i < n ? __ldg(reinterpret_cast<const uint4*>(row_of(r)) + u) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < kStageLoads; ++j) {
      const int i = i0 + j * kMThreads;
      const int r = i / cpr, u = i - r * cpr;
      float sm = ((bf16_lo(v[j].x) + bf16_hi(v[j].x)) + (bf16_lo(v[j].y) + bf16_hi(v[j].y))) +
                 ((bf16_lo(v[j].z) + bf16_hi(v[j].z)) + (bf16_lo(v[j].w) + bf16_hi(v[j].w)));
      sm += __shfl_xor_sync(0xffffffffu, sm, 1);
      sm += __shfl_xor_sync(0xffffffffu, sm, 2);
      sm += __shfl_xor_sync(0xffffffffu, sm, 4);
      if (i < n) {
        xs[r * (cpr + 1) + u] = interleave8(v[j]);
        if ((u & 7) == 0) xsum[(u >> 3) * kMTok + r] = sm;
      }
    }
  }
}

// The two 16-row tiles one warp computes for an item, as this lane's
// pointers: the codes of rows lg4 and lg4 + 8 of tile m start at q[m] and
// q[m] + 8 rs (rs = 32 ngr bytes per row; already offset by the lane's 8
// bytes of a group), the scales and biases of row lg4 at s[m] and b[m]
// (row lg4 + 8: + 8 ngr).
struct WTile {
  const uint8_t* q[2];
  const uint16_t* s[2];
  const uint16_t* b[2];
};

__device__ __forceinline__ WTile make_wtile(const QMatPtr& W0, size_t row0, const QMatPtr& W1, size_t row1, int ngr,
                                            int lg4, int lt) {
  const size_t rs = static_cast<size_t>(ngr) * 32;
  WTile w;
  w.q[0] = reinterpret_cast<const uint8_t*>(W0.q) + (row0 + lg4) * rs + lt * 8;
  w.q[1] = reinterpret_cast<const uint8_t*>(W1.q) + (row1 + lg4) * rs + lt * 8;
  w.s[0] = W0.s + (row0 + lg4) * ngr;
  w.b[0] = W0.b + (row0 + lg4) * ngr;
  w.s[1] = W1.s + (row1 + lg4) * ngr;
  w.b[1] = W1.b + (row1 + lg4) * ngr;
  return w;
}

// Codes of group G of both tiles (rows lg4 and lg4 + 8) into registers.
__device__ __forceinline__ void load_group(uint2 (&a)[2][2], const WTile& w, int ngr, int G) {
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int r = 0; r < 2; ++r)
      a[m][r] = __ldg(reinterpret_cast<const uint2*>(w.q[m] + static_cast<size_t>(r) * 8 * ngr * 32 + G * 32));
}

// Scales and biases of groups G0 .. G0 + B - 1 (B bf16 per row and tile,
// two per word).
template <int B>
struct BlockS {
  uint32_t s[2][2][B / 2], b[2][2][B / 2];   // [tile][row][word]
};
template <int B>
__device__ __forceinline__ void load_scales(BlockS<B>& S, const WTile& w, int ngr, int G0) {
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const uint16_t* sp = w.s[m] + r * 8 * ngr + G0;
      const uint16_t* bp = w.b[m] + r * 8 * ngr + G0;
      if constexpr (B == 4) {
        const uint2 sv = __ldg(reinterpret_cast<const uint2*>(sp)), bv = __ldg(reinterpret_cast<const uint2*>(bp));
        S.s[m][r][0] = sv.x; S.s[m][r][1] = sv.y;
        S.b[m][r][0] = bv.x; S.b[m][r][1] = bv.y;
      } else {
        S.s[m][r][0] = __ldg(reinterpret_cast<const uint32_t*>(sp));
        S.b[m][r][0] = __ldg(reinterpret_cast<const uint32_t*>(bp));
      }
    }
}

// Group G (position j of its block) of both tiles against the staged token
// tile: y[m][r][c] += s * sum (128 + q) x + (b - 128 s) X for row lg4 + 8r
// of tile m and token column 2lt + c.
template <int B>
__device__ __forceinline__ void group_step(float (&y)[2][2][2], const uint2 (&a)[2][2], const BlockS<B>& S, int j,
                                           const uint4* xr, const float* xsum, int G, int lt) {
  const uint4 xb0 = xr[G * 8], xb1 = xr[G * 8 + 1];
  const float2 X = *reinterpret_cast<const float2*>(xsum + G * kMTok + 2 * lt);
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    float d[4];
    group_dot(d, a[m][0], a[m][1], xb0, xb1);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const uint32_t sp = S.s[m][r][j >> 1];
      const uint32_t bp = S.b[m][r][j >> 1];
      const float sc = (j & 1) ? bf16_hi(sp) : bf16_lo(sp);
      const float cb = fmaf(-128.f, sc, (j & 1) ? bf16_hi(bp) : bf16_lo(bp));
      y[m][r][0] = fmaf(cb, X.x, fmaf(sc, d[2 * r], y[m][r][0]));
      y[m][r][1] = fmaf(cb, X.y, fmaf(sc, d[2 * r + 1], y[m][r][1]));
    }
  }
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// The body both kernels share.  tile_of(item, warp, row, lt) -> WTile: the
// warp's two tiles as seen by a lane that reads row `row` (and row + 8) at
// byte 8 lt of each group; k_of(item): inputs per row (a multiple of 64 B);
// row_of(item) -> a function r -> activation row r of the token tile;
// store(item, warp, y, lg4, lt): the epilogue.  Shared memory: the staged
// token tile.
//
// Three walks over the same block sequence: the computation; the register
// loads one block ahead of it (group j of block n + 1 right after group j of
// block n has been used); and L2 prefetches kPrefetchBlocks ahead, the
// line of one row per lane and block (lane = tile * 16 + row), so the
// register loads find their lines in L2.
constexpr int kPrefetchBlocks = 1;
template <int B, class TileOf, class KOf, class RowOf, class Store>
__device__ __forceinline__ void mid_body(const Geometry& g, const int32_t* offsets, const int32_t* active,
                                         const int32_t* n_active, int blocks_routed, int blocks_shared, int kmax,
                                         uint8_t* msm, TileOf tile_of, KOf k_of, RowOf row_of, Store store) {
  __shared__ int s_start[2 * kMThreads + 1];
  __shared__ int s_wt[kMWarps];
  const int n_act = *n_active;
  const int total = build_items(g, offsets, active, n_act, blocks_routed, blocks_shared, s_start, s_wt);
  if (static_cast<int>(blockIdx.x) >= total) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, lg4 = lane >> 2, lt = lane & 3;
  uint4* xs = reinterpret_cast<uint4*>(msm);
  float* xsum = reinterpret_cast<float*>(xs + kMTok * (kmax / 8 + 1));

  // The load walk (this lane's operand pointers lw for item lk, block lb)
  // and the prefetch walk (the line of row lane % 16 of tile lane / 16 at
  // pq, for item pk, block pb).  Both step through the same sequence.
  Item I = decode_item(g, s_start, n_act, offsets, active, blockIdx.x);
  WTile lw = tile_of(I, warp, lg4, lt);
  int lngr = k_of(I) / kGroup;
  int lk = 0, lb = 0, lnbat = lngr / B;
  bool lvalid = true;
  const uint8_t* pq;
  {
    const WTile w = tile_of(I, warp, lane & 15, 0);
    pq = (lane >> 4) ? w.q[1] : w.q[0];
  }
  int pk = 0, pb = 0, pnbat = lnbat;
  bool pvalid = true;

  uint2 A[B][2][2];
  BlockS<B> S;
#pragma unroll
  for (int j = 0; j < B; ++j) load_group(A[j], lw, lngr, j);
  load_scales<B>(S, lw, lngr, 0);
#define MID_STEP_LOAD()                                                             \
  do {                                                                              \
    if (lvalid && ++lb == lnbat) {                                                  \
      lb = 0;                                                                       \
      const int it_ = blockIdx.x + (++lk) * gridDim.x;                              \
      lvalid = it_ < total;                                                         \
      if (lvalid) {                                                                 \
        const Item n_ = decode_item(g, s_start, n_act, offsets, active, it_);       \
        lw = tile_of(n_, warp, lg4, lt);                                            \
        lngr = k_of(n_) / kGroup;                                                   \
        lnbat = lngr / B;                                                           \
      }                                                                             \
    }                                                                               \
  } while (0)
#define MID_STEP_PREFETCH()                                                         \
  do {                                                                              \
    if (pvalid && ++pb == pnbat) {                                                  \
      pb = 0;                                                                       \
      const int it_ = blockIdx.x + (++pk) * gridDim.x;                              \
      pvalid = it_ < total;                                                         \
      if (pvalid) {                                                                 \
        const Item n_ = decode_item(g, s_start, n_act, offsets, active, it_);       \
        const WTile w_ = tile_of(n_, warp, lane & 15, 0);                           \
        pq = (lane >> 4) ? w_.q[1] : w_.q[0];                                       \
        pnbat = k_of(n_) / kGroup / B;                                              \
      }                                                                             \
    }                                                                               \
    if (pvalid) prefetch_l2(pq + pb * (B * 32));                                    \
  } while (0)
  MID_STEP_LOAD();
  for (int i = 0; i < kPrefetchBlocks; ++i) MID_STEP_PREFETCH();

  for (int k = 0;; ++k) {
    const int K = k_of(I);
    const int ngr = K / kGroup, nbat = ngr / B;
    if (k > 0) __syncthreads();   // every warp is done with the previous item's staged tile
    stage_tile(row_of(I), I.tn, K, xs, xsum);
    __syncthreads();
    float y[2][2][2] = {{{0.f, 0.f}, {0.f, 0.f}}, {{0.f, 0.f}, {0.f, 0.f}}};
    const uint4* xr = xs + lg4 * (K / 8 + 1) + lt * 2;
    for (int b = 0; b < nbat; ++b) {
      MID_STEP_PREFETCH();
      const bool lv = lvalid;
      const int lG0 = lb * B;
      BlockS<B> NS = S;
      if (lv) load_scales<B>(NS, lw, lngr, lG0);
#pragma unroll
      for (int j = 0; j < B; ++j) {
        group_step<B>(y, A[j], S, j, xr, xsum, b * B + j, lt);
        if (lv) load_group(A[j], lw, lngr, lG0 + j);
      }
      S = NS;
      MID_STEP_LOAD();
    }
    store(I, warp, y, lg4, lt);
    const int nit = blockIdx.x + (k + 1) * gridDim.x;
    if (nit >= total) break;
    I = decode_item(g, s_start, n_act, offsets, active, nit);
  }
#undef MID_STEP_LOAD
#undef MID_STEP_PREFETCH
}

// ---------------------------------------------------------------------------
// gate/up + SwiGLU: h[pos] = bf16(silu(W_g x_t) * (W_u x_t)) for every routed
// entry pos (token t = perm[pos] / k) and h_s[t] for the shared expert.
// Warp w: the gate and up rows of features blk * 128 + 16 w .. + 15.
// ---------------------------------------------------------------------------
template <int B>
__global__ void __launch_bounds__(kMThreads, 2) mid_gateup_kernel(
    Geometry g, LayerPtr L, const uint16_t* __restrict__ x, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ perm, const int32_t* __restrict__ active, const int32_t* __restrict__ n_active,
    uint16_t* __restrict__ h, uint16_t* __restrict__ h_s) {
  extern __shared__ __align__(16) uint8_t msm[];
  pdl_wait();
  pdl_launch_dependents();
  const int ngr = g.H / kGroup;
  auto tile_of = [&](const Item& I, int warp, int lg4, int lt) {
    const size_t f0 = static_cast<size_t>(I.blk) * kMGateUpRows + warp * 16;
    const QMatPtr Wg = I.sh ? L.sh_gate : expert_qmat(L.gate, I.e, g.I, g.H);
    const QMatPtr Wu = I.sh ? L.sh_up : expert_qmat(L.up, I.e, g.I, g.H);
    return make_wtile(Wg, f0, Wu, f0, ngr, lg4, lt);
  };
  auto k_of = [&](const Item&) { return g.H; };
  auto row_of = [&](const Item& I) {
    return [&, I](int r) { return x + static_cast<size_t>(I.sh ? I.pos0 + r : perm[I.pos0 + r] / g.k) * g.H; };
  };
  auto store = [&](const Item& I, int warp, float (&y)[2][2][2], int lg4, int lt) {
    const int Ie = I.sh ? g.Is : g.I;
    const int f0 = I.blk * kMGateUpRows + warp * 16;
    uint16_t* dst = I.sh ? h_s : h;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int col = 2 * lt + c;
      if (col < I.tn)
#pragma unroll
        for (int r = 0; r < 2; ++r)
          dst[static_cast<size_t>(I.pos0 + col) * Ie + f0 + lg4 + 8 * r] =
              float_to_bf16_bits(silu(y[0][r][c]) * y[1][r][c]);
    }
  };
  mid_body<B>(g, offsets, active, n_active, g.I / kMGateUpRows, g.Is / kMGateUpRows, g.H, msm, tile_of, k_of, row_of,
           store);
}

// ---------------------------------------------------------------------------
// down: Y[pos] = bf16(W_d[e] h[pos]) for every routed entry (rows in the
// grouped order, as the prefill path's down GEMM writes them) and
// Y[T*k + t] = bf16(W_sd h_s[t]); the combine kernel then forms
// out_t = sum_j w[t,j] Y[inv_perm[t*k+j]] + sigma_t Y[T*k+t] in that order.
// Warp w: dims blk * 256 + 32 w .. + 31 (two tiles of 16).
// ---------------------------------------------------------------------------
template <int B>
__global__ void __launch_bounds__(kMThreads, 2) mid_down_kernel(
    Geometry g, LayerPtr L, const uint16_t* __restrict__ h, const uint16_t* __restrict__ h_s,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ active, const int32_t* __restrict__ n_active,
    uint16_t* __restrict__ Y) {
  extern __shared__ __align__(16) uint8_t msm[];
  pdl_wait();
  pdl_launch_dependents();
  const int blocks = g.H / kMDownRows;
  auto tile_of = [&](const Item& I, int warp, int lg4, int lt) {
    const size_t d0 = static_cast<size_t>(I.blk) * kMDownRows + warp * 32;
    const QMatPtr W = I.sh ? L.sh_down : expert_qmat(L.down, I.e, g.H, g.I);
    return make_wtile(W, d0, W, d0 + 16, (I.sh ? g.Is : g.I) / kGroup, lg4, lt);
  };
  auto k_of = [&](const Item& I) { return I.sh ? g.Is : g.I; };
  auto row_of = [&](const Item& I) {
    return [&, I](int r) { return (I.sh ? h_s : h) + static_cast<size_t>(I.pos0 + r) * (I.sh ? g.Is : g.I); };
  };
  auto store = [&](const Item& I, int warp, float (&y)[2][2][2], int lg4, int lt) {
    const int d0 = I.blk * kMDownRows + warp * 32;
    const size_t row0 = I.sh ? static_cast<size_t>(g.T) * g.k + I.pos0 : static_cast<size_t>(I.pos0);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int col = 2 * lt + c;
      if (col < I.tn)
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int r = 0; r < 2; ++r)
            Y[(row0 + col) * g.H + d0 + 16 * m + lg4 + 8 * r] = float_to_bf16_bits(y[m][r][c]);
    }
  };
  mid_body<B>(g, offsets, active, n_active, blocks, blocks, max(g.I, g.Is), msm, tile_of, k_of, row_of, store);
}

namespace {

// Resident CTAs of a mid-size kernel on this device (cached per kernel
// instance, device and shared-memory size).
int resident_ctas(int which, const void* func, int smem) {
  static int cache[4][16] = {};
  static int cache_smem[4][16] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return 0;
  if (cache[which][dev] > 0 && cache_smem[which][dev] == smem) return cache[which][dev];
  int sms = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, func, kMThreads, smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (per_sm < 1) return 0;
  cache[which][dev] = sms * per_sm;
  cache_smem[which][dev] = smem;
  return cache[which][dev];
}

// An upper bound of the items of a call: every routed entry may open its own
// token tile, and the active slots add at most one partial tile each.
int max_items(const Geometry& g, int blocks_routed, int blocks_shared) {
  const int n = g.T * g.k;
  const int slots = min(g.E, n);
  return (n / kMTok + slots) * blocks_routed + (g.T + kMTok - 1) / kMTok * blocks_shared;
}

// Shared memory: the staged token tile for rows of up to kmax inputs.
int mid_smem(int kmax) { return kMTok * (kmax / 8 + 1) * 16 + kMTok * (kmax / kGroup) * 4; }

bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

// Blocks of 4 groups when every row of the launch has a multiple of 4 groups
// and the scale/bias stacks allow 8-byte loads (rows and expert strides are
// then multiples of 8 bytes too), else blocks of 2.
bool blocks_of_4(std::initializer_list<int> ngrs, std::initializer_list<const QMatPtr*> mats) {
  for (int n : ngrs)
    if (n % 4) return false;
  for (const QMatPtr* m : mats)
    if (!aligned8(m->s) || !aligned8(m->b)) return false;
  return true;
}

template <int B>
cudaError_t launch_gateup_b(int which, const Geometry& g, const LayerPtr& L, const uint16_t* x,
                            const int32_t* offsets, const int32_t* perm, const int32_t* active,
                            const int32_t* n_active, uint16_t* h, uint16_t* h_s, cudaStream_t s) {
  const int smem = mid_smem(g.H);
  const void* fn = reinterpret_cast<const void*>(mid_gateup_kernel<B>);
  cudaError_t e = ensure_smem(fn, smem);
  if (e != cudaSuccess) return e;
  const int res = resident_ctas(which, fn, smem);
  if (res <= 0) return cudaErrorInvalidConfiguration;
  const int grid = max(1, min(res, max_items(g, g.I / kMGateUpRows, g.Is / kMGateUpRows)));
  return launch_pdl(mid_gateup_kernel<B>, dim3(grid), dim3(kMThreads), smem, s, g, L, x, offsets, perm, active,
                    n_active, h, h_s);
}

template <int B>
cudaError_t launch_down_b(int which, const Geometry& g, const LayerPtr& L, const uint16_t* h, const uint16_t* h_s,
                          const int32_t* offsets, const int32_t* active, const int32_t* n_active, uint16_t* Y,
                          cudaStream_t s) {
  const int smem = mid_smem(max(g.I, g.Is));
  const void* fn = reinterpret_cast<const void*>(mid_down_kernel<B>);
  cudaError_t e = ensure_smem(fn, smem);
  if (e != cudaSuccess) return e;
  const int res = resident_ctas(which, fn, smem);
  if (res <= 0) return cudaErrorInvalidConfiguration;
  const int blocks = g.H / kMDownRows;
  const int grid = max(1, min(res, max_items(g, blocks, blocks)));
  return launch_pdl(mid_down_kernel<B>, dim3(grid), dim3(kMThreads), smem, s, g, L, h, h_s, offsets, active,
                    n_active, Y);
}

}  // namespace

bool mid_decode_supported(const Geometry& g) {
  return g.T >= 1 && g.T <= 128 && g.H % kMDownRows == 0 && g.I % kMGateUpRows == 0 && g.Is % kMGateUpRows == 0 &&
         g.H <= 8192 && g.I <= 2048 && g.Is <= 2048;
}

cudaError_t launch_mid_gateup(const Geometry& g, const LayerPtr& L, const uint16_t* x, const int32_t* offsets,
                              const int32_t* perm, const int32_t* active, const int32_t* n_active, uint16_t* h,
                              uint16_t* h_s, cudaStream_t s) {
  if (blocks_of_4({g.H / kGroup}, {&L.gate, &L.up, &L.sh_gate, &L.sh_up}))
    return launch_gateup_b<4>(0, g, L, x, offsets, perm, active, n_active, h, h_s, s);
  return launch_gateup_b<2>(1, g, L, x, offsets, perm, active, n_active, h, h_s, s);
}

cudaError_t launch_mid_down(const Geometry& g, const LayerPtr& L, const uint16_t* h, const uint16_t* h_s,
                            const int32_t* offsets, const int32_t* active, const int32_t* n_active, uint16_t* Y,
                            cudaStream_t s) {
  if (blocks_of_4({g.I / kGroup, g.Is / kGroup}, {&L.down, &L.sh_down}))
    return launch_down_b<4>(2, g, L, h, h_s, offsets, active, n_active, Y, s);
  return launch_down_b<2>(3, g, L, h, h_s, offsets, active, n_active, Y, s);
}

}  // namespace moe
