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
// Dequantisation and dot products follow the decode kernels (decode.cu):
//   sum_i (s q_i + b) x_i = 128 s * sum_i (1 + q_i/128) x_i + (b - 128 s) * sum_i x_i.
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

__host__ __device__ __forceinline__ int fx_stride(int H) { return (H + 1023) / 1024 * 1024; }   // 32-lane windows
__host__ __device__ __forceinline__ int fh_stride(int I) { return (I + 511) / 512 * 512; }      // 16-lane windows

__device__ __forceinline__ void codes_f(uint32_t w, float (&f)[8]) {
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

// Stage one bf16 row of n elements as FP32 in the `lanes`-interleaved layout
// (element 32c + i at float4 ((c/lanes)*8 + i/4)*lanes + c%lanes).  Called by
// `nthr` threads with index `tid`.
__device__ __forceinline__ void stage_row_f(const uint16_t* src, int n, int lanes, float* dst, int tid, int nthr) {
  float4* d4 = reinterpret_cast<float4*>(dst);
  for (int u = tid; u < n / 8; u += nthr) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[u];
    const int e0 = u * 8, c = e0 >> 5, ii = e0 & 31;
    const int win = c / lanes, ln = c - win * lanes;
    d4[(win * 8 + (ii >> 2)) * lanes + ln] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
    d4[(win * 8 + (ii >> 2) + 1) * lanes + ln] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
  }
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

// Grid-wide barrier, called by one thread per CTA after a CTA barrier (all
// CTAs co-resident).  bar[0] counts arrivals with acquire-release adds (each
// arrival publishes its CTA's writes; the last arriver acquires them all),
// the last arriver resets it and bumps the generation bar[1] with a release
// store; the others spin (bounded) on an acquire load of the generation.
__device__ bool grid_barrier(unsigned* bar, unsigned nblocks, int* status) {
  const unsigned gen = tc::ld_acquire_gpu(bar + 1);
  if (tc::atom_add_acq_rel_gpu(bar, 1u) == nblocks - 1) {
    atomicExch(bar, 0u);
    tc::st_release_gpu(bar + 1, gen + 1);
    return true;
  }
  const long long deadline = clock64() + (1ll << 32);
  while (tc::ld_acquire_gpu(bar + 1) == gen) {
    if (clock64() > deadline) {
      if (status) atomicExch(status, kStatusTimeout);
      return false;
    }
  }
  return true;
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

// Sum over the warp of v[r(lane)] with r(lane) = 4*bit4 + 2*bit3 + bit2 of
// the lane: a transposing butterfly (9 shuffles for 8 values).
__device__ __forceinline__ float warp_reduce8(const float (&v)[8], int lane) {
  const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4;
  float a4[4], a2[2];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    a4[j] = (h16 ? v[j + 4] : v[j]) + __shfl_xor_sync(0xffffffffu, h16 ? v[j] : v[j + 4], 16);
#pragma unroll
  for (int j = 0; j < 2; ++j)
    a2[j] = (h8 ? a4[j + 2] : a4[j]) + __shfl_xor_sync(0xffffffffu, h8 ? a4[j] : a4[j + 2], 8);
  float r = (h4 ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, h4 ? a2[0] : a2[1], 4);
  r += __shfl_xor_sync(0xffffffffu, r, 2);
  r += __shfl_xor_sync(0xffffffffu, r, 1);
  return r;
}

// Sum over each half-warp of v[r(lane)] with r(lane) = 2*bit3 + bit2.
__device__ __forceinline__ float halfwarp_reduce4(const float (&v)[4], int lane) {
  const bool h8 = lane & 8, h4 = lane & 4;
  float a2[2];
#pragma unroll
  for (int j = 0; j < 2; ++j)
    a2[j] = (h8 ? v[j + 2] : v[j]) + __shfl_xor_sync(0xffffffffu, h8 ? v[j] : v[j + 2], 8);
  float r = (h4 ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, h4 ? a2[0] : a2[1], 4);
  r += __shfl_xor_sync(0xffffffffu, r, 2);
  r += __shfl_xor_sync(0xffffffffu, r, 1);
  return r;
}

// sum_i (1 + q_i/128) * v_i for the 32 codes of qv against 32 staged values
// held in registers (v[0..31]), four partial sums.
__device__ __forceinline__ float dot32r(const uint4& qv, const float (&v)[32]) {
  const uint32_t words[4] = {qv.x, qv.y, qv.z, qv.w};
  float p[4];
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    float f[8];
    codes_f(words[wd], f);
    float acc = f[0] * v[8 * wd];
#pragma unroll
    for (int i = 1; i < 8; ++i) acc = fmaf(f[i], v[8 * wd + i], acc);
    p[wd] = acc;
  }
  return (p[0] + p[1]) + (p[2] + p[3]);
}

// Load one 32-element segment of a staged row (interleave `lanes`) into registers.
__device__ __forceinline__ void load_seg(const float* row, int c, int lanes, float (&v)[32]) {
  const float4* r4 = reinterpret_cast<const float4*>(row) + ((c / lanes) * 8) * lanes + (c % lanes);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 q = r4[j * lanes];
    v[4 * j] = q.x;
    v[4 * j + 1] = q.y;
    v[4 * j + 2] = q.z;
    v[4 * j + 3] = q.w;
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
  float* xs = reinterpret_cast<float*>(fsm + a.off_xs);       // [T][fx_stride(H)]
  float* xsum = reinterpret_cast<float*>(fsm + a.off_xsum);   // [T][fx_stride(H)/32]
  float* hs = reinterpret_cast<float*>(fsm + a.off_hs);       // [rows][fh_stride(Kmax)]
  float* hsum = reinterpret_cast<float*>(fsm + a.off_hsum);   // [rows][fh_stride(Kmax)/32]
  float* lg = reinterpret_cast<float*>(fsm + a.off_lg);       // [T][E1], also the router partials
  RouteSmem& rt = *reinterpret_cast<RouteSmem*>(fsm + a.off_rt);
  float* ys = reinterpret_cast<float*>(fsm + a.off_y);        // [T*k + T][my_blocks][16]
  volatile int* abort_flag = &rt.abort;
  const int xst = fx_stride(g.H);
  const int Kmax = max(g.I, g.Is);
  const int hst = fh_stride(Kmax);
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
    for (int t = 0; t < T; ++t) stage_row_f(a.x + static_cast<size_t>(t) * g.H, g.H, 32, xs + t * xst, tid, nthr);
    // router rows r = c, c + G, ...: warp w sums the K slice [w H/16, (w+1) H/16)
    const int nrows = (E1 - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x;
    const int kslice = g.H / kFWarps;
    float* part = lg;   // [nrows][kFWarps][NT] partials (lg is free until phase B)
    for (int rr = 0; rr < nrows; ++rr) {
      const int row = blockIdx.x + rr * gridDim.x;
      const uint16_t* wrow = row < E ? a.L.w_router + static_cast<size_t>(row) * g.H : a.L.w_sg;
      float acc[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t] = 0.f;
      for (int c = warp * kslice + lane * 4; c < (warp + 1) * kslice; c += 128) {
        const uint2 wv = __ldg(reinterpret_cast<const uint2*>(wrow + c));
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (t < T) {
            const uint2 xv = __ldg(reinterpret_cast<const uint2*>(a.x + static_cast<size_t>(t) * g.H + c));
            float s = acc[t];
            s = fmaf(bf16_lo(xv.x), bf16_lo(wv.x), s);
            s = fmaf(bf16_hi(xv.x), bf16_hi(wv.x), s);
            s = fmaf(bf16_lo(xv.y), bf16_lo(wv.y), s);
            s = fmaf(bf16_hi(xv.y), bf16_hi(wv.y), s);
            acc[t] = s;
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float v = warp_sum(acc[t]);
        if (lane == 0) part[(rr * kFWarps + warp) * NT + t] = v;
      }
    }
    consumers_sync();
    for (int i = tid; i < T * xst / 32; i += nthr) {
      const int t = i / (xst / 32), c = i % (xst / 32);
      if (c < g.H / 32) {
        const float4* r4 = reinterpret_cast<const float4*>(xs + t * xst);
        const int win = c >> 5, ln = c & 31;
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 q = r4[(win * 8 + j) * 32 + ln];
          sum += (q.x + q.y) + (q.z + q.w);
        }
        xsum[t * (xst / 32) + c] = sum;
      }
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
  if (threadIdx.x == 0 && !grid_barrier(a.bar, gridDim.x, a.status)) rt.abort = 1;
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
        if (!tc::mbar_wait(&empty[sl], ((i / a.ring) & 1u) ^ 1u, abort_flag, a.status)) break;
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
  // gate/up, two units at a time: warp pair p = warp / 2 owns 8 of the 64
  // rows (2 units x 16 features x {gate, up}); thread (p, c) keeps segment c
  // of every token's staged x in registers and runs 8 independent dot
  // products against it.
  bool ok = true;
  float* red = lg;   // [8 pairs][2 halves][8 rows][NT] partial sums (logits are no longer needed)
  const int pr = warp >> 1, half = warp & 1;
  const int nch = g.H / 32;
  const uint32_t qb = kFFeat * g.H / 2, sb = kFFeat * g.H / 32;
  for (int i0 = 0; i0 < s.my_gu && ok; i0 += 2) {
    const int nu = min(2, s.my_gu - i0);
    for (int ui = 0; ui < nu && ok; ++ui) {
      const int i = i0 + ui;
      if (!tc::mbar_wait(&full[i % a.ring], (i / a.ring) & 1u, abort_flag, a.status)) ok = false;
    }
    if (!ok) break;
    // this pair's rows: r = 8 pr + rr; unit r / 32, matrix (r / 16) & 1, feature r & 15
    const int ur = (8 * pr) >> 5;
    const bool rows_live = ur < nu;
    int slot = 0, f0 = 0;
    if (rows_live) gu_unit(s, blockIdx.x + (i0 + ur) * gridDim.x, slot, f0);
    const int m = ((8 * pr) >> 4) & 1, fb = (8 * pr) & 15;     // rows rr = 0..7: features fb .. fb+7
    const uint8_t* base = fsm + ((i0 + ur) % a.ring) * a.slot_bytes;
    const uint8_t* qrow0 = base + m * qb + fb * (g.H / 2);
    const uint16_t* srow0 = reinterpret_cast<const uint16_t*>(base + 2 * qb + m * 2 * sb) + fb * (g.H / kGroup);
    const uint16_t* brow0 = reinterpret_cast<const uint16_t*>(base + 2 * qb + m * 2 * sb + sb) + fb * (g.H / kGroup);
    // tokens of this unit's expert: routed slot -> its rows' tokens; shared -> 0..T-1
    unsigned tmask = 0;
    if (rows_live) {
      if (slot == 0)
        tmask = (1u << T) - 1u;
      else
        for (int r = 0; r < rt.slot_cnt[slot]; ++r) tmask |= 1u << (rt.perm[rt.slot_off[slot] + r] / k);
    }
    float acc[8][NT];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr)
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[rr][t] = 0.f;
    if (rows_live) {
      for (int c = half * 32 + lane; c < nch; c += 64) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if ((tmask >> t) & 1u) {
            float xv[32];
            load_seg(xs + t * xst, c, 32, xv);
            const float X = xsum[t * (xst / 32) + c];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
              const uint4 qv = reinterpret_cast<const uint4*>(qrow0 + rr * (g.H / 2))[c];
              const float s128 = 128.f * bf16_bits_to_float(srow0[rr * (g.H / kGroup) + (c >> 1)]);
              const float bb = bf16_bits_to_float(brow0[rr * (g.H / kGroup) + (c >> 1)]);
              acc[rr][t] = fmaf(s128, dot32r(qv, xv), fmaf(bb - s128, X, acc[rr][t]));
            }
          }
        }
      }
    }
    // every read of the pair's slots is done: release them
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0)
      for (int ui = 0; ui < nu; ++ui) tc::mbar_arrive(&empty[(i0 + ui) % a.ring]);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float v[8];
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) v[rr] = acc[rr][t];
      const float r = warp_reduce8(v, lane);
      if ((lane & 3) == 0) red[((pr * 2 + half) * 8 + (lane >> 2)) * NT + t] = r;
    }
    consumers_sync();
    // h = bf16(silu(g) * u) for (unit, feature, token)
    for (int q = threadIdx.x; q < nu * kFFeat * T; q += kFWarps * 32) {
      const int ui = q / (kFFeat * T), f = (q / T) % kFFeat, t = q % T;
      int uslot, uf0;
      gu_unit(s, blockIdx.x + (i0 + ui) * gridDim.x, uslot, uf0);
      bool member = uslot == 0;
      int pos = t;
      for (int r = 0; r < (uslot == 0 ? 0 : rt.slot_cnt[uslot]); ++r)
        if (rt.perm[rt.slot_off[uslot] + r] / k == t) {
          member = true;
          pos = rt.slot_off[uslot] + r;
        }
      if (!member) continue;
      const int rg = ui * 32 + f, ru = ui * 32 + 16 + f;      // gate and up rows of the pair
      const float gs = red[(((rg >> 3) * 2 + 0) * 8 + (rg & 7)) * NT + t] + red[(((rg >> 3) * 2 + 1) * 8 + (rg & 7)) * NT + t];
      const float us = red[(((ru >> 3) * 2 + 0) * 8 + (ru & 7)) * NT + t] + red[(((ru >> 3) * 2 + 1) * 8 + (ru & 7)) * NT + t];
      const uint16_t hv = float_to_bf16_bits(silu(gs) * us);
      if (uslot == 0)
        a.h_s[static_cast<size_t>(t) * g.Is + uf0 + f] = hv;
      else
        a.h[static_cast<size_t>(pos) * g.I + uf0 + f] = hv;
    }
    consumers_sync();   // red is reused by the next pair
  }
  // Every h row is written: grid barrier (consumer thread 0 of each CTA).
  consumers_sync();
  if (threadIdx.x == 0 && (!ok || !grid_barrier(a.bar, gridDim.x, a.status))) rt.abort = 1;
  consumers_sync();
  if (rt.abort) return;

  if (s.my_blocks > 0) {
    // stage every h row (routed rows I wide, shared rows Is wide; stride hst)
    const int tid = threadIdx.x, nthr = kFWarps * 32;
    const int vmax = Kmax / 8;
    for (int i = tid; i < (Tk + T) * vmax; i += nthr) {
      const int r = i / vmax, u = i - r * vmax;
      const bool shr = r >= Tk;
      if (u * 8 >= (shr ? g.Is : g.I)) continue;
      const uint16_t* src = shr ? a.h_s + static_cast<size_t>(r - Tk) * g.Is : a.h + static_cast<size_t>(r) * g.I;
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(src) + u);
      const int c = u >> 2, ii = (u & 3) * 8;
      float4* d4 = reinterpret_cast<float4*>(hs + r * hst);
      const int win = c >> 4, ln = c & 15;
      d4[(win * 8 + (ii >> 2)) * 16 + ln] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
      d4[(win * 8 + (ii >> 2) + 1) * 16 + ln] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
    }
    consumers_sync();
    for (int i = tid; i < (Tk + T) * (hst / 32); i += nthr) {
      const int r = i / (hst / 32), c = i % (hst / 32);
      const int K = r >= Tk ? g.Is : g.I;
      if (c < K / 32) {
        const float4* r4 = reinterpret_cast<const float4*>(hs + r * hst);
        const int win = c >> 4, ln = c & 15;
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 q = r4[(win * 8 + j) * 16 + ln];
          sum += (q.x + q.y) + (q.z + q.w);
        }
        hsum[r * (hst / 32) + c] = sum;
      }
    }
    consumers_sync();
  }
  // down units: half-warp hw = 2 warp + (lane >> 4) owns (slot jj = hw / 4,
  // dims 4 (hw % 4) .. +3) of the unit; lane hl = lane & 15 walks segments
  // c = hl, hl + 16, ... with the slot's staged h rows in registers.
  const int hl = lane & 15, hw = warp * 2 + (lane >> 4);
  const int jj = hw >> 2, dg = hw & 3;
  for (int di = 0; di < s.my_blocks * s.n_down_parts && ok; ++di) {
    const int i = s.my_gu + di;
    const int sl = i % a.ring;
    if (!tc::mbar_wait(&full[sl], (i / a.ring) & 1u, abort_flag, a.status)) {
      ok = false;
      break;
    }
    const int bl = di / s.n_down_parts;
    const int j0 = (di % s.n_down_parts) * s.spd, nj = min(s.spd, s.n_slots - j0);
    const bool live = jj < nj;
    const int j = j0 + jj;
    const bool sh = j == 0;
    const int K = sh ? g.Is : g.I;
    const int nt = live ? rt.slot_cnt[j] : 0;
    const int pos0 = live ? rt.slot_off[j] : 0;
    const uint8_t* base = fsm + sl * a.slot_bytes + jj * (9 * Kmax);
    const uint8_t* qrow0 = base + (dg * 4) * (K / 2);
    const uint16_t* srow0 = reinterpret_cast<const uint16_t*>(base + 8 * Kmax) + (dg * 4) * (K / kGroup);
    const uint16_t* brow0 = reinterpret_cast<const uint16_t*>(base + 8 * Kmax + Kmax / 2) + (dg * 4) * (K / kGroup);
    float p[4][NT];
#pragma unroll
    for (int d = 0; d < 4; ++d)
#pragma unroll
      for (int t = 0; t < NT; ++t) p[d][t] = 0.f;
    if (live) {
      for (int c = hl; c < K / 32; c += 16) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (t < nt) {
            const int r = pos0 + t;
            float hv[32];
            load_seg(hs + r * hst, c, 16, hv);
            const float X = hsum[r * (hst / 32) + c];
#pragma unroll
            for (int d = 0; d < 4; ++d) {
              const uint4 qv = reinterpret_cast<const uint4*>(qrow0 + d * (K / 2))[c];
              const float s128 = 128.f * bf16_bits_to_float(srow0[d * (K / kGroup) + (c >> 1)]);
              const float bb = bf16_bits_to_float(brow0[d * (K / kGroup) + (c >> 1)]);
              p[d][t] = fmaf(s128, dot32r(qv, hv), fmaf(bb - s128, X, p[d][t]));
            }
          }
        }
      }
    }
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&empty[sl]);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float v[4];
#pragma unroll
      for (int d = 0; d < 4; ++d) v[d] = p[d][t];
      const float r = halfwarp_reduce4(v, lane);
      if ((hl & 3) == 0 && t < nt) ys[((pos0 + t) * s.my_blocks + bl) * kFDims + dg * 4 + (hl >> 2)] = r;
    }
  }
  consumers_sync();
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
  const int G = fused_grid();
  const int Kmax = g.I > g.Is ? g.I : g.Is;
  a.slot_bytes = 18 * g.H;                                   // one gate/up unit
  a.spd = a.slot_bytes / (9 * Kmax);
  if (a.spd > kFMaxSpd) a.spd = kFMaxSpd;
  const int xst = fx_stride(g.H), hst = fh_stride(Kmax);
  const int rows = g.T * g.k + g.T;
  const int blocks_per_cta = (g.H / kFDims + G - 1) / G;
  auto al = [](int v) { return (v + 127) / 128 * 128; };
  int off = 0;
  auto take = [&](int bytes) {
    const int o = off;
    off += al(bytes);
    return o;
  };
  const int lg_floats = max(g.T * (g.E + 1), (g.E + 1 + G - 1) / G * kFWarps * kFMaxT);
  const int fixed = al(2 * kFRingMax * 8) + al(g.T * xst * 4) + al(g.T * (xst / 32) * 4) + al(rows * hst * 4) +
                    al(rows * (hst / 32) * 4) + al(lg_floats * 4) +
                    al(static_cast<int>(sizeof(RouteSmem))) + al(rows * blocks_per_cta * kFDims * 4);
  const int budget = 227 * 1024 - fixed;
  a.ring = budget / a.slot_bytes;
  if (a.ring > kFRingMax) a.ring = kFRingMax;
  if (a.ring < 2 || a.spd < 1) return cudaErrorInvalidValue;
  take(a.ring * a.slot_bytes);
  a.off_bar = take(2 * kFRingMax * 8);
  a.off_xs = take(g.T * xst * 4);
  a.off_xsum = take(g.T * (xst / 32) * 4);
  a.off_hs = take(rows * hst * 4);
  a.off_hsum = take(rows * (hst / 32) * 4);
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
