// Fused decode layer for T <= 2: router, top-k, grouping, gate/up + SwiGLU,
// down projection and the fixed-order combine in ONE cooperative launch of
// one CTA per SM ("Perplexity's Lily: ...", section "How It Works: Prefill
// and Decode Strategies": batch-1 decode streams the active experts' packed
// weights, so the layer is bound by how fast those bytes arrive).
//
// Why one launch: at T = 1 the active weights are ~16 MB, about 2.5 us of HBM
// time.  As separate launches the layer pays several launch latencies, and no
// weight load can start before the routing kernel has finished.  Here the
// phases are separated by two grid-wide barriers (all CTAs are co-resident:
// cooperative launch), and every CTA issues ALL of its weight tiles as
// asynchronous bulk copies the moment routing is known, so the memory system
// sees the whole working set at once:
//
//   A  router logits: CTA c scores rows c, c+G, ... of [W_r; w_sg] for every
//      token and stores them; CTAs that own a shared-expert unit already
//      start that unit's copy (it does not depend on routing).
//   -- grid barrier --
//   B  every CTA reads the T x (E+1) logits and repeats the (tiny, exact and
//      deterministic) top-k, shared gate and counting sort, so it knows the
//      active experts without another barrier; CTA 0 also writes the routing
//      outputs.
//   C  gate/up units: (expert slot, 16 features) -> h = bf16(silu(g) * u),
//      one feature per consumer warp.
//   -- grid barrier (h complete) --  the producer warp keeps copying the down
//      tiles meanwhile: they depend on the routing, not on h.
//   D  down units: (16 output dims, up to 8 expert slots), one dim per
//      consumer warp; then the combine of each token's k + 1 terms in slot
//      order, then the shared term, exactly as the unfused decode kernels.
//
// Weight tiles stream through a ring of shared-memory slots filled by one
// producer thread (cp.async.bulk, completion on the slot's "full" mbarrier)
// and released by the 16 consumer warps ("empty" mbarrier, count 16).  All
// waits are bounded; a timeout records MOE_ERR_DEVICE_TIMEOUT in the status
// word and the kernel returns.
//
// Dot products on the tensor cores (warp-level mma.sync, bf16 in, FP32
// accumulation): per group of 64 inputs, with A = 128 + q as exact bf16 values
// (one AND-OR per code pair, no scale applied) and B = the activations,
//   sum_i (s q_i + b) x_i = s * (sum_i (128 + q_i) x_i - 128 X) + b X,  X = sum_i x_i,
// applied per group after the MMAs.  Inside each group of 8 inputs both
// operands use the order (0,4,1,5,2,6,3,7) in which the AND-OR yields code
// pairs; the activations are staged in that order, so no permutes are
// needed.  The integer work per code drops from ~2 (nibble to float) to ~1
// instruction per code pair.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int kFWarps = 16;                     // consumer warps
constexpr int kFThreads = (kFWarps + 1) * 32;   // + the producer warp
constexpr int kFFeat = 16;                      // features per gate/up unit (one per consumer warp)
constexpr int kFDims = 16;                      // output dims per down block (one per consumer warp)
constexpr int kFMaxSpd = 8;                     // expert slots per down unit
constexpr int kFRingMax = 8;
constexpr int kFMaxT = 2;
constexpr int kFRouterRows = 2;                 // router rows per CTA with loads in flight together

struct FusedArgs {
  Geometry g;
  LayerPtr L;
  const uint16_t* x;
  uint16_t* out;
  RoutingPtrs r;
  int32_t* active;
  int32_t* n_active;
  float* logits;          // [T, E+1]
  uint16_t* h;            // [T*k, I]
  uint16_t* h_s;          // [T, Is]
  unsigned* bar;          // [0] arrivals, [1] generation
  int* status;
  int ring, slot_bytes, spd;
  long long wait_limit;   // cycles before a bounded wait gives up
  int off_bar, off_xs, off_xsum, off_hs, off_hsum, off_lg, off_rt, off_y;
};

// Routing state every CTA rebuilds in shared memory.  Expert slots in down
// order: slot 0 is the shared expert (its rows are h rows T*k .. T*k+T-1),
// slots 1..n_act the routed active experts ascending (rows off .. off+cnt-1).
struct RouteSmem {
  int32_t idx[kFMaxT * kMaxK];
  float w[kFMaxT * kMaxK];
  float sigma[kFMaxT];
  int32_t perm[kFMaxT * kMaxK];
  int32_t inv_perm[kFMaxT * kMaxK];
  int32_t slot_e[kFMaxT * kMaxK + 1];
  int32_t slot_cnt[kFMaxT * kMaxK + 1];
  int32_t slot_off[kFMaxT * kMaxK + 1];
  int32_t n_act;               // routed active experts
  int32_t abort;
};


// 8 bf16 values (x0,x1)(x2,x3)(x4,x5)(x6,x7) in the interleaved K order
// (x0,x4)(x1,x5)(x2,x6)(x3,x7).
__device__ __forceinline__ uint4 interleave8(const uint4& v) {   // (x0,x1)(x2,x3)(x4,x5)(x6,x7)
  uint4 o;
  o.x = __byte_perm(v.x, v.z, 0x5410);
  o.y = __byte_perm(v.x, v.z, 0x7632);
  o.z = __byte_perm(v.y, v.w, 0x5410);
  o.w = __byte_perm(v.y, v.w, 0x7632);
  return o;
}

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

// One group of 64 inputs for rows g, g+8 of a 16-row weight tile (lane g =
// lane/4, t = lane%4): lane reads words 2t, 2t+1 of the group in both rows
// (qg, qg8: this lane's 8 bytes) and the 32 staged activations of token g at
// 8-groups 2t, 2t+1 (xb0, xb1; zero for padding tokens).  d gets
// sum (128 + q) x for (row g, tokens 2t, 2t+1) and (row g+8, same tokens).
__device__ __forceinline__ void group_dot(float (&d)[4], const uint2& qg, const uint2& qg8, const uint4& xb0,
                                          const uint4& xb1) {
  d[0] = d[1] = d[2] = d[3] = 0.f;
  mma16816(d, code_pair(qg.x, 0), code_pair(qg8.x, 0), code_pair(qg.x, 4), code_pair(qg8.x, 4), xb0.x, xb0.y);
  mma16816(d, code_pair(qg.x, 8), code_pair(qg8.x, 8), code_pair(qg.x, 12), code_pair(qg8.x, 12), xb0.z, xb0.w);
  mma16816(d, code_pair(qg.y, 0), code_pair(qg8.y, 0), code_pair(qg.y, 4), code_pair(qg8.y, 4), xb1.x, xb1.y);
  mma16816(d, code_pair(qg.y, 8), code_pair(qg8.y, 8), code_pair(qg.y, 12), code_pair(qg8.y, 12), xb1.z, xb1.w);
}

// Order-preserving 32-bit key of a float (larger float -> larger key; every
// non-NaN float maps above 0).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = f == 0.f ? 0u : __float_as_uint(f);   // -0 and +0 are one value
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp top-k over E <= 256 logits in shared memory with the same order as
// the other routing kernels (larger logit first, equal logits -> lower expert
// index): each pick is a lane-local scan of 8 keys and two warp reductions
// (redux.sync max of the key, then min of the expert index among the lanes
// holding that key).  Lane 0 writes the experts and exp(l_j - l_0) / sum.
__device__ __forceinline__ void topk_redux(const float* lg, int E, int k, int lane, int32_t* idx_out,
                                           float* w_out) {
  uint32_t key[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? order_key(lg[e]) : 0u;
  }
  int sel[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j < k) {
      uint32_t best = 0u;
      int bi = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (key[i] > best) {        // strictly greater: the lowest index among equal keys
          best = key[i];
          bi = i;
        }
      const uint32_t m = __reduce_max_sync(0xffffffffu, best);
      const uint32_t cand = (best == m && m != 0u) ? static_cast<uint32_t>(lane + 32 * bi) : 0xffffffffu;
      const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
      if (static_cast<int>(win & 31u) == lane) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (i == static_cast<int>(win >> 5)) key[i] = 0u;
      }
      sel[j] = static_cast<int>(win);
    }
  }
  if (lane == 0) {
    float z[kMaxK];
    float sum = 0.f;
    const float l0 = lg[sel[0]];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k) {
        z[j] = expf(lg[sel[j]] - l0);
        sum += z[j];
      }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k) {
        idx_out[j] = sel[j];
        w_out[j] = z[j] / sum;
      }
  }
}

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kFWarps * 32) : "memory"); }

// Grid-wide barrier n (1, 2, ...) of one launch, called by one thread per
// CTA after a CTA barrier (all CTAs are co-resident).  bar[0] counts arrivals
// over the whole launch: each CTA adds 1 with release semantics (publishing
// what its threads wrote before the CTA barrier) and polls, bounded, until
// the count reaches n * nblocks, then acquires.  No arriver has to reset or
// publish anything, so the barrier costs one release-add and the polls.
// bar[0] starts every launch at zero: grid_exit resets it.
__device__ bool grid_barrier(unsigned* bar, unsigned target, int* status, long long limit) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(bar) : "memory");
  const long long deadline = clock64() + limit;
  for (;;) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
    if (v >= target) break;
    if (clock64() > deadline) {
      if (status) atomicExch(status, kStatusTimeout);
      return false;
    }
  }
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
  return true;
}

// Called once per CTA by the thread that polls the barrier, after its last
// grid_barrier (or after giving up on one): the last CTA to get here resets
// both words for the next launch on the same workspace.  Every CTA has then
// finished polling bar[0].
__device__ void grid_exit(unsigned* bar, unsigned nblocks) {
  if (atomicAdd(bar + 1, 1u) == nblocks - 1) {
    bar[0] = 0u;
    bar[1] = 0u;
  }
}

// Unit schedule of one CTA: its gate/up units u = c, c+G, ... over the
// global list [shared-expert units | routed units], then its down units
// (dim blocks c, c+G, ..., each split into parts of at most spd_max slots,
// balanced).
struct Sched {
  int n_gu_units;      // global gate/up units
  int n_sh_units;      // of which shared-expert units (first)
  int units_per_exp;   // I / 16
  int n_slots;         // down slots: shared + routed active
  int n_down_parts;    // down units per dim block
  int spd;             // slots per down unit (the last may have fewer)
  int n_blocks;        // dim blocks (H / 16)
  int my_gu, my_blocks;
};

__device__ __forceinline__ Sched make_sched(const FusedArgs& a, int n_act) {
  Sched s;
  s.n_sh_units = a.g.Is / kFFeat;
  s.units_per_exp = a.g.I / kFFeat;
  s.n_gu_units = s.n_sh_units + n_act * s.units_per_exp;
  s.n_slots = n_act + 1;
  s.n_down_parts = (s.n_slots + a.spd - 1) / a.spd;
  s.spd = (s.n_slots + s.n_down_parts - 1) / s.n_down_parts;
  s.n_blocks = a.g.H / kFDims;
  const int G = gridDim.x, c = blockIdx.x;
  s.my_gu = s.n_gu_units > c ? (s.n_gu_units - c + G - 1) / G : 0;
  s.my_blocks = s.n_blocks > c ? (s.n_blocks - c + G - 1) / G : 0;
  return s;
}

// Gate/up unit u: expert slot (0 = shared) and first feature.
__device__ __forceinline__ void gu_unit(const Sched& s, int u, int& slot, int& f0) {
  const bool sh = u < s.n_sh_units;
  slot = sh ? 0 : 1 + (u - s.n_sh_units) / s.units_per_exp;
  f0 = (sh ? u : (u - s.n_sh_units) % s.units_per_exp) * kFFeat;
}

// Issue the bulk copies of unit i of this CTA into ring slot `dst`.
// gate/up layout: [q gate 16 rows][q up 16 rows][s gate][b gate][s up][b up];
// down layout: per expert slot jj at jj * 9 Kmax: [q 16 rows][s][b].
__device__ void issue_unit(const FusedArgs& a, const RouteSmem& rt, const Sched& s, int i, uint32_t dst,
                           uint64_t* full) {
  const Geometry& g = a.g;
  if (i < s.my_gu) {
    int slot, f0;
    gu_unit(s, blockIdx.x + i * gridDim.x, slot, f0);
    const bool sh = slot == 0;
    const size_t row0 = static_cast<size_t>(sh ? 0 : rt.slot_e[slot] * g.I) + f0;
    const QMatPtr Wg = sh ? a.L.sh_gate : a.L.gate;
    const QMatPtr Wu = sh ? a.L.sh_up : a.L.up;
    const uint32_t qb = kFFeat * g.H / 2, sb = kFFeat * g.H / 32;
    tc::mbar_arrive_expect_tx(full, 2 * qb + 4 * sb);
    tc::bulk_load(dst, Wg.q + row0 * (g.H / 8), qb, full);
    tc::bulk_load(dst + qb, Wu.q + row0 * (g.H / 8), qb, full);
    tc::bulk_load(dst + 2 * qb, Wg.s + row0 * (g.H / kGroup), sb, full);
    tc::bulk_load(dst + 2 * qb + sb, Wg.b + row0 * (g.H / kGroup), sb, full);
    tc::bulk_load(dst + 2 * qb + 2 * sb, Wu.s + row0 * (g.H / kGroup), sb, full);
    tc::bulk_load(dst + 2 * qb + 3 * sb, Wu.b + row0 * (g.H / kGroup), sb, full);
    return;
  }
  const int di = i - s.my_gu;
  const int blk = blockIdx.x + (di / s.n_down_parts) * gridDim.x;
  const int j0 = (di % s.n_down_parts) * s.spd, nj = min(s.spd, s.n_slots - j0);
  const int Kmax = max(g.I, g.Is);
  uint32_t bytes = 0;
  for (int jj = 0; jj < nj; ++jj) {
    const int K = j0 + jj == 0 ? g.Is : g.I;
    bytes += kFDims * K / 2 + 2 * (kFDims * K / 32);
  }
  tc::mbar_arrive_expect_tx(full, bytes);
  for (int jj = 0; jj < nj; ++jj) {
    const bool sh = j0 + jj == 0;
    const int K = sh ? g.Is : g.I;
    const QMatPtr W = sh ? a.L.sh_down : a.L.down;
    const size_t row0 = static_cast<size_t>(sh ? 0 : rt.slot_e[j0 + jj] * g.H) + blk * kFDims;
    const uint32_t base = dst + jj * (9 * Kmax);
    const uint32_t qb = kFDims * K / 2, sb = kFDims * K / 32;
    tc::bulk_load(base, W.q + row0 * (K / 8), qb, full);
    tc::bulk_load(base + 8 * Kmax, W.s + row0 * (K / kGroup), sb, full);
    tc::bulk_load(base + 8 * Kmax + Kmax / 2, W.b + row0 * (K / kGroup), sb, full);
  }
}

template <int NT>
__global__ void __launch_bounds__(kFThreads, 1) decode_fused_kernel(const __grid_constant__ FusedArgs a) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = g.T, k = g.k, E = g.E, E1 = g.E + 1;
  const uint32_t ring0 = tc::smem_u32(fsm);
  uint64_t* full = reinterpret_cast<uint64_t*>(fsm + a.off_bar);
  uint64_t* empty = full + kFRingMax;
  uint16_t* xs = reinterpret_cast<uint16_t*>(fsm + a.off_xs);   // [T][H] bf16, interleaved K order
  float* xsum = reinterpret_cast<float*>(fsm + a.off_xsum);      // [T][H/64] group sums
  uint16_t* hs = reinterpret_cast<uint16_t*>(fsm + a.off_hs);   // [T*k + T][Kmax] bf16, interleaved K order
  float* hsum = reinterpret_cast<float*>(fsm + a.off_hsum);      // [T*k + T][Kmax/64] group sums
  float* lg = reinterpret_cast<float*>(fsm + a.off_lg);       // [T][E1], also the router partials
  RouteSmem& rt = *reinterpret_cast<RouteSmem*>(fsm + a.off_rt);
  float* ys = reinterpret_cast<float*>(fsm + a.off_y);        // [T*k + T][my_blocks][16]
  volatile int* abort_flag = &rt.abort;
  const int Kmax = max(g.I, g.Is);
  const bool producer = warp == kFWarps;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.ring; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kFWarps);
    }
    rt.abort = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();

  // ---------------------------------------------------------------- phase A
  // The first unit of a CTA whose first gate/up unit is a shared-expert unit
  // does not depend on routing: start its copy now.
  const bool early = static_cast<int>(blockIdx.x) < g.Is / kFFeat;
  if (producer && lane == 0 && early) {
    Sched s0{};
    s0.n_sh_units = g.Is / kFFeat;
    s0.units_per_exp = g.I / kFFeat;
    s0.n_gu_units = s0.n_sh_units;
    s0.my_gu = 1;
    issue_unit(a, rt, s0, 0, ring0, &full[0]);
  }
  if (!producer) {
    const int tid = threadIdx.x, nthr = kFWarps * 32;
    // router rows r = c, c + G, ...: thread tid owns the inputs [4 tid, 4 tid + 4)
    // of every row and token.  x and the first rows are requested before any
    // of them is used, so they arrive in one memory round trip; x is then
    // staged from the same registers.
    const int nrows = (E1 - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x;
    const int c = 4 * tid;
    const bool live = c < g.H;
    uint2 xv[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t)
      xv[t] = (live && t < T) ? __ldg(reinterpret_cast<const uint2*>(a.x + static_cast<size_t>(t) * g.H + c))
                              : make_uint2(0u, 0u);
    float* part = lg;   // [nrows][kFWarps][NT] partials (lg is free until phase B)
    for (int r0 = 0; r0 < nrows; r0 += kFRouterRows) {
      uint2 wv[kFRouterRows];
#pragma unroll
      for (int q = 0; q < kFRouterRows; ++q) {
        const int row = blockIdx.x + (r0 + q) * gridDim.x;
        const uint16_t* wrow = row < E ? a.L.w_router + static_cast<size_t>(row) * g.H : a.L.w_sg;
        wv[q] = (live && r0 + q < nrows) ? __ldg(reinterpret_cast<const uint2*>(wrow + c)) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int q = 0; q < kFRouterRows; ++q) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          float s = fmaf(bf16_lo(xv[t].x), bf16_lo(wv[q].x), 0.f);
          s = fmaf(bf16_hi(xv[t].x), bf16_hi(wv[q].x), s);
          s = fmaf(bf16_lo(xv[t].y), bf16_lo(wv[q].y), s);
          s = fmaf(bf16_hi(xv[t].y), bf16_hi(wv[q].y), s);
          s = warp_sum(s);
          if (lane == 0 && r0 + q < nrows && t < T) part[((r0 + q) * kFWarps + warp) * NT + t] = s;
        }
      }
    }
    // x in the interleaved K order: threads 2i, 2i+1 hold the halves of 8-group i
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      uint2 p;
      p.x = __shfl_xor_sync(0xffffffffu, xv[t].x, 1);
      p.y = __shfl_xor_sync(0xffffffffu, xv[t].y, 1);
      if (live && t < T) {
        const uint32_t lo = (tid & 1) ? p.y : xv[t].x, hi = (tid & 1) ? xv[t].y : p.x;
        reinterpret_cast<uint2*>(xs + static_cast<size_t>(t) * g.H)[tid] =
            make_uint2(__byte_perm(lo, hi, 0x5410), __byte_perm(lo, hi, 0x7632));
      }
    }
    consumers_sync();
    for (int i = tid; i < T * (g.H / 64); i += nthr) {     // sums over groups of 64 (fixed order)
      const uint4* r4 = reinterpret_cast<const uint4*>(xs) + i * 8;
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 v = r4[j];
        sum += ((bf16_lo(v.x) + bf16_hi(v.x)) + (bf16_lo(v.y) + bf16_hi(v.y))) +
               ((bf16_lo(v.z) + bf16_hi(v.z)) + (bf16_lo(v.w) + bf16_hi(v.w)));
      }
      xsum[i] = sum;
    }
    if (tid < nrows * T) {
      const int rr = tid / T, t = tid % T;
      const int row = blockIdx.x + rr * gridDim.x;
      float v = 0.f;
      for (int w = 0; w < kFWarps; ++w) v += part[(rr * kFWarps + w) * NT + t];
      if (row < E && a.L.router_bias) v += a.L.router_bias[row];
      __stcg(a.logits + static_cast<size_t>(t) * E1 + row, v);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && !grid_barrier(a.bar, gridDim.x, a.status, a.wait_limit)) {
    rt.abort = 1;
    grid_exit(a.bar, gridDim.x);
  }
  __syncthreads();
  if (rt.abort) {
    if (producer && lane == 0 && early) tc::mbar_wait_drain(&full[0], 0, a.status);
    return;
  }

  // ---------------------------------------------------------------- phase B
  // Every CTA rebuilds the routing from the logits (top-k by warp reductions,
  // then a one-warp counting sort of the n = T*k <= 16 entries), so no
  // further barrier is needed before the expert weights can be requested.
  for (int i = threadIdx.x; i < T * E1; i += blockDim.x) lg[i] = __ldcg(a.logits + i);
  __syncthreads();
  if (warp < T) {
    topk_redux(lg + warp * E1, E, k, lane, rt.idx + warp * k, rt.w + warp * k);
    if (lane == 0) rt.sigma[warp] = sigmoid(lg[warp * E1 + E]);
  }
  __syncthreads();
  const int n = T * k;
  const int Tk = n;
  if (warp == 0) {
    const bool live = lane < n;
    const int e_i = live ? rt.idx[lane] : -1 - lane;          // distinct dummies for idle lanes
    const unsigned peers = __match_any_sync(0xffffffffu, e_i);
    const int rank = __popc(peers & lanemask_lt());           // same expert, earlier (token, slot)
    const bool first = live && rank == 0;
    const unsigned firsts = __ballot_sync(0xffffffffu, first);
    int below = 0, abelow = 0;                                // entries / active experts with a smaller expert
    for (int j = 0; j < n; ++j) {
      const int ej = __shfl_sync(0xffffffffu, e_i, j);
      below += ej < e_i ? 1 : 0;
      abelow += (((firsts >> j) & 1u) && ej < e_i) ? 1 : 0;
    }
    if (live) {
      const int pos = below + rank;
      rt.perm[pos] = lane;
      rt.inv_perm[lane] = pos;
      if (first) {
        rt.slot_e[1 + abelow] = e_i;
        rt.slot_cnt[1 + abelow] = __popc(peers);
        rt.slot_off[1 + abelow] = below;
      }
    }
    if (lane == 0) {
      rt.n_act = __popc(firsts);
      rt.slot_e[0] = E;
      rt.slot_cnt[0] = T;
      rt.slot_off[0] = Tk;
    }
  }
  __syncthreads();
  const Sched s = make_sched(a, rt.n_act);
  const int n_units = s.my_gu + s.my_blocks * s.n_down_parts;

  if (producer) {
    // ------------------------------------------------------- producer warp
    if (lane == 0) {
      int last[kFRingMax];
      for (int sl = 0; sl < kFRingMax; ++sl) last[sl] = -1;
      if (early) last[0] = 0;
      for (int i = early ? 1 : 0; i < n_units; ++i) {
        const int sl = i % a.ring;
        if (!tc::mbar_wait(&empty[sl], ((i / a.ring) & 1u) ^ 1u, abort_flag, a.status, a.wait_limit)) break;
        tc::fence_proxy_async_smem();   // consumers' generic reads of the slot precede the refill
        issue_unit(a, rt, s, i, ring0 + sl * a.slot_bytes, &full[sl]);
        last[sl] = i;
      }
      // every copy this thread issued has landed before the CTA may exit
      for (int sl = 0; sl < a.ring; ++sl)
        if (last[sl] >= 0) tc::mbar_wait_drain(&full[sl], (last[sl] / a.ring) & 1u, a.status);
    }
    __syncwarp();
    return;
  }

  // ------------------------------------------------------ consumer warps
  // gate/up, one unit at a time (its compute overlaps the next unit's
  // arrival): warp w owns the 16-row tile w % 2 (gate or up) for the K eighth
  // w / 2; per group of 64 inputs four mma.sync, then the group's scale and
  // bias.
  bool ok = true;
  float* red = lg;   // [2 tiles][8 K eighths][16 rows][NT] partial sums (logits are no longer needed)
  const int lg4 = lane >> 2, lt = lane & 3;
  const uint32_t qb = kFFeat * g.H / 2, sb = kFFeat * g.H / 32;
  const int ngrp = g.H / kGroup;
  {
    const int m = warp & 1, ke = warp >> 1;
    const int ge = ngrp / 8;                       // groups per K eighth
    for (int i = 0; i < s.my_gu && ok; ++i) {
      const int sl = i % a.ring;
      if (!tc::mbar_wait(&full[sl], (i / a.ring) & 1u, abort_flag, a.status, a.wait_limit)) {
        ok = false;
        break;
      }
      int slot, f0;
      gu_unit(s, blockIdx.x + i * gridDim.x, slot, f0);
      unsigned tmask = 0;                            // tokens of this unit's expert
      if (slot == 0)
        tmask = (1u << T) - 1u;
      else
        for (int r = 0; r < rt.slot_cnt[slot]; ++r) tmask |= 1u << (rt.perm[rt.slot_off[slot] + r] / k);
      const uint8_t* base = fsm + sl * a.slot_bytes;
      const uint8_t* qrow = base + m * qb + lg4 * (g.H / 2) + lt * 8;         // rows lg4, lg4 + 8
      const uint16_t* srow = reinterpret_cast<const uint16_t*>(base + 2 * qb + m * 2 * sb);
      const uint16_t* brow = srow + sb / 2;
      const bool tok_live = lg4 < T && ((tmask >> lg4) & 1u);
      const uint4* xrow = reinterpret_cast<const uint4*>(xs + (tok_live ? lg4 : 0) * g.H) + lt * 2;
      float y[2][NT];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t) y[r][t] = 0.f;
      for (int G = ke * ge; G < (ke + 1) * ge; ++G) {
        const uint2 qa = *reinterpret_cast<const uint2*>(qrow + G * 32);
        const uint2 qc = *reinterpret_cast<const uint2*>(qrow + 8 * (g.H / 2) + G * 32);
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        const uint4 xb0 = tok_live ? xrow[G * 8] : z, xb1 = tok_live ? xrow[G * 8 + 1] : z;
        float d[4];
        group_dot(d, qa, qc, xb0, xb1);
        if (lt == 0) {   // columns 0, 1 = tokens 0, 1
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int row = lg4 + 8 * r;
            const float sc = bf16_bits_to_float(srow[row * ngrp + G]);
            const float bi = bf16_bits_to_float(brow[row * ngrp + G]);
#pragma unroll
            for (int t = 0; t < NT; ++t)
              if (t < T) {
                const float X = xsum[t * ngrp + G];
                y[r][t] = fmaf(sc, d[2 * r + t] - 128.f * X, fmaf(bi, X, y[r][t]));
              }
          }
        }
      }
      // every read of the unit's slot is done: release it
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[sl]);
      if (lt == 0)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int t = 0; t < NT; ++t) red[((m * 8 + ke) * 16 + lg4 + 8 * r) * NT + t] = y[r][t];
      consumers_sync();
      // h = bf16(silu(g) * u) for (feature, token); K eighths summed in order
      if (threadIdx.x < kFFeat * T) {
        const int f = threadIdx.x / T, t = threadIdx.x % T;
        bool member = slot == 0;
        int pos = t;
        for (int r = 0; r < (slot == 0 ? 0 : rt.slot_cnt[slot]); ++r)
          if (rt.perm[rt.slot_off[slot] + r] / k == t) {
            member = true;
            pos = rt.slot_off[slot] + r;
          }
        if (member) {
          float gs = 0.f, us = 0.f;
#pragma unroll
          for (int e8 = 0; e8 < 8; ++e8) {
            gs += red[((0 * 8 + e8) * 16 + f) * NT + t];
            us += red[((1 * 8 + e8) * 16 + f) * NT + t];
          }
          const uint16_t hv = float_to_bf16_bits(silu(gs) * us);
          if (slot == 0)
            a.h_s[static_cast<size_t>(t) * g.Is + f0 + f] = hv;
          else
            a.h[static_cast<size_t>(pos) * g.I + f0 + f] = hv;
        }
      }
      consumers_sync();   // red is reused by the next unit
    }
  }
  // Every h row is written: grid barrier (consumer thread 0 of each CTA).
  consumers_sync();
  if (threadIdx.x == 0) {
    if (!ok || !grid_barrier(a.bar, 2u * gridDim.x, a.status, a.wait_limit)) rt.abort = 1;
    grid_exit(a.bar, gridDim.x);
  }
  consumers_sync();
  if (rt.abort) return;

  if (s.my_blocks > 0) {
    // stage every h row (routed rows I wide, shared rows Is wide) in the
    // interleaved K order, and its sums over groups of 64
    const int tid = threadIdx.x, nthr = kFWarps * 32;
    const int vmax = Kmax / 8;
    for (int i = tid; i < (Tk + T) * vmax; i += nthr) {
      const int r = i / vmax, u = i - r * vmax;
      const bool shr = r >= Tk;
      if (u * 8 >= (shr ? g.Is : g.I)) continue;
      const uint16_t* src = shr ? a.h_s + static_cast<size_t>(r - Tk) * g.Is : a.h + static_cast<size_t>(r) * g.I;
      reinterpret_cast<uint4*>(hs + static_cast<size_t>(r) * Kmax)[u] =
          interleave8(__ldcg(reinterpret_cast<const uint4*>(src) + u));
    }
    consumers_sync();
    const int kg = Kmax / kGroup;
    for (int i = tid; i < (Tk + T) * kg; i += nthr) {
      const int r = i / kg, G = i % kg;
      const int K = r >= Tk ? g.Is : g.I;
      if (G * kGroup < K) {
        const uint4* r4 = reinterpret_cast<const uint4*>(hs + static_cast<size_t>(r) * Kmax) + G * 8;
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 v = r4[j];
          sum += ((bf16_lo(v.x) + bf16_hi(v.x)) + (bf16_lo(v.y) + bf16_hi(v.y))) +
                 ((bf16_lo(v.z) + bf16_hi(v.z)) + (bf16_lo(v.w) + bf16_hi(v.w)));
        }
        hsum[i] = sum;
      }
    }
    consumers_sync();
  }
  // down units: warp w owns expert slot w % 8 of the unit (16 dims x K) for
  // the K half w / 8; lanes hold rows (dims) lg4, lg4 + 8 and tokens 0, 1
  {
    const int jj = warp & 7, kh = warp >> 3;
    const int kg = Kmax / kGroup;
    float* redd = lg;   // [8 slots][2 K halves][16 dims][NT]
    for (int di = 0; di < s.my_blocks * s.n_down_parts && ok; ++di) {
      const int i = s.my_gu + di;
      const int sl = i % a.ring;
      if (!tc::mbar_wait(&full[sl], (i / a.ring) & 1u, abort_flag, a.status, a.wait_limit)) {
        ok = false;
        break;
      }
      const int bl = di / s.n_down_parts;
      const int j0 = (di % s.n_down_parts) * s.spd, nj = min(s.spd, s.n_slots - j0);
      const bool live = jj < nj;
      const int j = j0 + jj;
      const int K = j == 0 ? g.Is : g.I;
      const int ng = K / kGroup, gh = ng / 2;       // groups, groups per K half
      const int nt = live ? rt.slot_cnt[j] : 0;
      const int pos0 = live ? rt.slot_off[j] : 0;
      float y[2][NT];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t) y[r][t] = 0.f;
      if (live) {
        const uint8_t* base = fsm + sl * a.slot_bytes + jj * (9 * Kmax);
        const uint8_t* qrow = base + lg4 * (K / 2) + lt * 8;
        const uint16_t* srow = reinterpret_cast<const uint16_t*>(base + 8 * Kmax);
        const uint16_t* brow = reinterpret_cast<const uint16_t*>(base + 8 * Kmax + Kmax / 2);
        const bool tok_live = lg4 < nt;
        const int hr = pos0 + (tok_live ? lg4 : 0);
        const uint4* hrow = reinterpret_cast<const uint4*>(hs + static_cast<size_t>(hr) * Kmax) + lt * 2;
        for (int G = kh * gh; G < (kh + 1) * gh; ++G) {
          const uint2 qa = *reinterpret_cast<const uint2*>(qrow + G * 32);
          const uint2 qc = *reinterpret_cast<const uint2*>(qrow + 8 * (K / 2) + G * 32);
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
          const uint4 hb0 = tok_live ? hrow[G * 8] : z, hb1 = tok_live ? hrow[G * 8 + 1] : z;
          float d[4];
          group_dot(d, qa, qc, hb0, hb1);
          if (lt == 0) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const int row = lg4 + 8 * r;
              const float sc = bf16_bits_to_float(srow[row * ng + G]);
              const float bi = bf16_bits_to_float(brow[row * ng + G]);
#pragma unroll
              for (int t = 0; t < NT; ++t)
                if (t < nt) {
                  const float X = hsum[(pos0 + t) * kg + G];
                  y[r][t] = fmaf(sc, d[2 * r + t] - 128.f * X, fmaf(bi, X, y[r][t]));
                }
            }
          }
        }
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[sl]);
      if (lt == 0)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int t = 0; t < NT; ++t) redd[((jj * 2 + kh) * 16 + lg4 + 8 * r) * NT + t] = y[r][t];
      consumers_sync();
      // y rows of this unit's slots: both K halves summed in order
      for (int q = threadIdx.x; q < nj * kFDims * NT; q += kFWarps * 32) {
        const int js = q / (kFDims * NT), d = (q / NT) % kFDims, t = q % NT;
        const int jx = j0 + js;
        if (t < rt.slot_cnt[jx])
          ys[((rt.slot_off[jx] + t) * s.my_blocks + bl) * kFDims + d] =
              redd[((js * 2 + 0) * 16 + d) * NT + t] + redd[((js * 2 + 1) * 16 + d) * NT + t];
      }
      consumers_sync();
    }
  }
  if (!ok) return;
  // combine: out[t, d] = bf16( sum_j w[t,j] * y[inv_perm[t k + j]][d] + sigma_t * y[T k + t][d] )
  for (int i = threadIdx.x; i < T * s.my_blocks * kFDims; i += kFWarps * 32) {
    const int t = i / (s.my_blocks * kFDims), rem = i % (s.my_blocks * kFDims);
    const int bl = rem / kFDims, d = rem % kFDims;
    float acc = 0.f;
    for (int j = 0; j < k; ++j)
      acc = fmaf(rt.w[t * k + j], ys[(rt.inv_perm[t * k + j] * s.my_blocks + bl) * kFDims + d], acc);
    acc = fmaf(rt.sigma[t], ys[((Tk + t) * s.my_blocks + bl) * kFDims + d], acc);
    const int blk = blockIdx.x + bl * gridDim.x;
    a.out[static_cast<size_t>(t) * g.H + blk * kFDims + d] = float_to_bf16_bits(acc);
  }
  if (blockIdx.x == 0) {
    // routing outputs (off the other CTAs' critical path)
    for (int i = threadIdx.x; i < n; i += kFWarps * 32) {
      a.r.topk_idx[i] = rt.idx[i];
      a.r.topk_w[i] = rt.w[i];
      a.r.perm[i] = rt.perm[i];
      a.r.inv_perm[i] = rt.inv_perm[i];
    }
    for (int e = threadIdx.x; e <= E; e += kFWarps * 32) {
      int c = 0, below = 0;
      for (int i = 0; i < n; ++i) {
        c += rt.idx[i] == e ? 1 : 0;
        below += rt.idx[i] < e ? 1 : 0;
      }
      if (e < E) a.r.counts[e] = c;
      a.r.offsets[e] = below;
    }
    for (int jx = threadIdx.x; jx < rt.n_act; jx += kFWarps * 32) a.active[jx] = rt.slot_e[1 + jx];
    if (threadIdx.x < T) a.r.sigma[threadIdx.x] = rt.sigma[threadIdx.x];
    if (threadIdx.x == 0) {
      a.active[rt.n_act] = E;
      *a.n_active = rt.n_act + 1;
    }
  }
}

int fused_grid() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  }
  return n;
}

}  // namespace

bool decode_fused_supported(const Geometry& g) {
  if (g.T < 1 || g.T > kFMaxT) return false;
  if (g.H % 1024 || g.H > 2048) return false;
  if (g.I % kFFeat || g.Is % kFFeat) return false;
  const int Kmax = g.I > g.Is ? g.I : g.Is;
  return 9 * Kmax <= 18 * g.H;   // at least one expert slot per down unit
}

cudaError_t launch_decode_fused(const Geometry& g, const LayerPtr& L, const uint16_t* x, uint16_t* out,
                                const RoutingPtrs& r, int32_t* active, int32_t* n_active, float* logits,
                                uint16_t* h, uint16_t* h_s, unsigned* bar, int* status, cudaStream_t s) {
  FusedArgs a{};
  a.g = g;
  a.L = L;
  a.x = x;
  a.out = out;
  a.r = r;
  a.active = active;
  a.n_active = n_active;
  a.logits = logits;
  a.h = h;
  a.h_s = h_s;
  a.bar = bar;
  a.status = status;
  a.wait_limit = wait_limit_cycles();
  const int G = fused_grid();
  const int Kmax = g.I > g.Is ? g.I : g.Is;
  a.slot_bytes = 18 * g.H;                                   // one gate/up unit
  a.spd = a.slot_bytes / (9 * Kmax);
  if (a.spd > kFMaxSpd) a.spd = kFMaxSpd;
  const int rows = g.T * g.k + g.T;
  const int blocks_per_cta = (g.H / kFDims + G - 1) / G;
  auto al = [](int v) { return (v + 127) / 128 * 128; };
  int off = 0;
  auto take = [&](int bytes) {
    const int o = off;
    off += al(bytes);
    return o;
  };
  // lg: logits, then the router partials, then the dot-product reductions
  const int lg_floats = max(max(g.T * (g.E + 1), (g.E + 1 + G - 1) / G * kFWarps * kFMaxT), 16 * 16 * kFMaxT);
  const int fixed = al(2 * kFRingMax * 8) + al(g.T * g.H * 2) + al(g.T * (g.H / kGroup) * 4) + al(rows * Kmax * 2) +
                    al(rows * (Kmax / kGroup) * 4) + al(lg_floats * 4) +
                    al(static_cast<int>(sizeof(RouteSmem))) + al(rows * blocks_per_cta * kFDims * 4);
  const int budget = 227 * 1024 - fixed;
  a.ring = budget / a.slot_bytes;
  if (a.ring > kFRingMax) a.ring = kFRingMax;
  if (a.ring < 2 || a.spd < 1) return cudaErrorInvalidValue;
  take(a.ring * a.slot_bytes);
  a.off_bar = take(2 * kFRingMax * 8);
  a.off_xs = take(g.T * g.H * 2);
  a.off_xsum = take(g.T * (g.H / kGroup) * 4);
  a.off_hs = take(rows * Kmax * 2);
  a.off_hsum = take(rows * (Kmax / kGroup) * 4);
  a.off_lg = take(lg_floats * 4);
  a.off_rt = take(static_cast<int>(sizeof(RouteSmem)));
  a.off_y = take(rows * blocks_per_cta * kFDims * 4);
  const int smem = off;
  const void* fn = g.T == 1 ? reinterpret_cast<const void*>(decode_fused_kernel<1>)
                            : reinterpret_cast<const void*>(decode_fused_kernel<2>);
  cudaError_t e = ensure_smem(fn, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (g.T == 1) return cudaLaunchKernelEx(&cfg, decode_fused_kernel<1>, a);
  return cudaLaunchKernelEx(&cfg, decode_fused_kernel<2>, a);
}

}  // namespace moe
