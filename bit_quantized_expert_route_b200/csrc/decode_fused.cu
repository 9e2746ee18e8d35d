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

// Routing state every CTA rebuilds in shared memory.
struct RouteSmem {
  int32_t idx[kFMaxT * kMaxK];
  float w[kFMaxT * kMaxK];
  float sigma[kFMaxT];
  int32_t perm[kFMaxT * kMaxK];
  int32_t inv_perm[kFMaxT * kMaxK];
  int32_t counts[kMaxE];
  int32_t offsets[kMaxE + 1];
  int32_t active[kMaxE + 1];   // routed active experts ascending
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

// sum_i (1 + q_i/128) * v_i over the 32 codes of `qv`; v from an interleaved
// staging row: float4 j of this lane's segment at vl[j * lanes].
__device__ __forceinline__ float dot32f(const uint4& qv, const float4* __restrict__ vl, int lanes) {
  const uint32_t words[4] = {qv.x, qv.y, qv.z, qv.w};
  float a = 0.f;
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    float f[8];
    codes_f(words[wd], f);
    const float4 v0 = vl[(2 * wd) * lanes];
    const float4 v1 = vl[(2 * wd + 1) * lanes];
    a = fmaf(f[0], v0.x, a); a = fmaf(f[1], v0.y, a); a = fmaf(f[2], v0.z, a); a = fmaf(f[3], v0.w, a);
    a = fmaf(f[4], v1.x, a); a = fmaf(f[5], v1.y, a); a = fmaf(f[6], v1.z, a); a = fmaf(f[7], v1.w, a);
  }
  return a;
}

// Stage one bf16 row of n elements as FP32 in the `lanes`-interleaved layout
// (element 32c + i at float4 ((c/lanes)*8 + i/4)*lanes + c%lanes).  Called by
// `nthr` threads with index `tid`; l2_only reads through L2 (rows written by
// other CTAs of this launch).
__device__ __forceinline__ void stage_row_f(const uint16_t* src, int n, int lanes, float* dst, int tid, int nthr,
                                            bool l2_only) {
  float4* d4 = reinterpret_cast<float4*>(dst);
  for (int u = tid; u < n / 8; u += nthr) {
    const uint4 v = l2_only ? __ldcg(reinterpret_cast<const uint4*>(src) + u) : reinterpret_cast<const uint4*>(src)[u];
    const int e0 = u * 8, c = e0 >> 5, ii = e0 & 31;
    const int win = c / lanes, ln = c - win * lanes;
    d4[(win * 8 + (ii >> 2)) * lanes + ln] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
    d4[(win * 8 + (ii >> 2) + 1) * lanes + ln] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
  }
}

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kFWarps * 32) : "memory"); }

// Grid-wide barrier, called by one thread per CTA (all CTAs co-resident).
// bar[0] counts arrivals and is reset by the last arriver, which then bumps
// the generation bar[1] with release semantics; the others wait (bounded)
// for the generation to move.
__device__ bool grid_barrier(unsigned* bar, unsigned nblocks, int* status) {
  const unsigned gen = tc::ld_acquire_gpu(bar + 1);
  __threadfence();
  if (atomicAdd(bar, 1u) == nblocks - 1) {
    atomicExch(bar, 0u);
    __threadfence();
    tc::st_release_gpu(bar + 1, gen + 1);
    return true;
  }
  const long long deadline = clock64() + (1ll << 32);
  while (tc::ld_acquire_gpu(bar + 1) == gen) {
    if (clock64() > deadline) {
      if (status) atomicExch(status, kStatusTimeout);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// Unit schedule of one CTA: its gate/up units u = c, c+G, ... over the
// global list [shared-expert units | routed units], then its down units.
struct Sched {
  int n_gu_units;      // global gate/up units
  int n_sh_units;      // of which shared-expert units (first)
  int units_per_exp;   // I / 16
  int n_slots;         // down slots: shared + routed active
  int n_down_parts;    // down units per dim block
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
  s.n_blocks = a.g.H / kFDims;
  const int G = gridDim.x, c = blockIdx.x;
  s.my_gu = s.n_gu_units > c ? (s.n_gu_units - c + G - 1) / G : 0;
  s.my_blocks = s.n_blocks > c ? (s.n_blocks - c + G - 1) / G : 0;
  return s;
}

// Expert of down slot j: slot 0 is the shared expert (index E), then the
// routed active experts in ascending order.
__device__ __forceinline__ int slot_expert(const RouteSmem& rt, int E, int j) { return j == 0 ? E : rt.active[j - 1]; }

// Issue the bulk copies of unit i of this CTA into ring slot `dst`.
__device__ void issue_unit(const FusedArgs& a, const RouteSmem& rt, const Sched& s, int i, uint32_t dst,
                           uint64_t* full) {
  const Geometry& g = a.g;
  if (i < s.my_gu) {
    const int u = blockIdx.x + i * gridDim.x;
    const bool sh = u < s.n_sh_units;
    const int e = sh ? g.E : rt.active[(u - s.n_sh_units) / s.units_per_exp];
    const int f0 = (sh ? u : (u - s.n_sh_units) % s.units_per_exp) * kFFeat;
    const size_t row0 = static_cast<size_t>(sh ? 0 : e * g.I) + f0;
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
  const int part = di % s.n_down_parts;
  const int j0 = part * a.spd, nj = min(a.spd, s.n_slots - j0);
  const int Kmax = max(g.I, g.Is);
  uint32_t bytes = 0;
  for (int jj = 0; jj < nj; ++jj) {
    const bool sh = j0 + jj == 0;
    const int K = sh ? g.Is : g.I;
    bytes += kFDims * K / 2 + 2 * (kFDims * K / 32);
  }
  tc::mbar_arrive_expect_tx(full, bytes);
  for (int jj = 0; jj < nj; ++jj) {
    const int e = slot_expert(rt, g.E, j0 + jj);
    const bool sh = e == g.E;
    const int K = sh ? g.Is : g.I;
    const QMatPtr W = sh ? a.L.sh_down : a.L.down;
    const size_t row0 = static_cast<size_t>(sh ? 0 : e * g.H) + blk * kFDims;
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
    for (int t = 0; t < T; ++t) stage_row_f(a.x + static_cast<size_t>(t) * g.H, g.H, 32, xs + t * xst, tid, nthr, false);
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
  for (int i = threadIdx.x; i < T * E1; i += blockDim.x) lg[i] = __ldcg(a.logits + i);
  __syncthreads();
  if (warp < T) {
    select_topk_warp(lg + warp * E1, E, k, lane, rt.idx + warp * k, rt.w + warp * k);
    if (lane == 0) rt.sigma[warp] = sigmoid(lg[warp * E1 + E]);
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) rt.counts[e] = 0;
  __syncthreads();
  const int n = T * k;
  if (warp == 0) {
    // counting sort of the n <= 16 entries: counts, offsets, stable ranks
    for (int i = lane; i < n; i += 32) atomicAdd(&rt.counts[rt.idx[i]], 1);
    __syncwarp();
    int run = 0, nact = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int c = e < E ? rt.counts[e] : 0;
      int incl = c, act = c > 0 ? 1 : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        const int va = __shfl_up_sync(0xffffffffu, act, o);
        if (lane >= o) {
          incl += v;
          act += va;
        }
      }
      if (e < E) {
        rt.offsets[e] = run + incl - c;
        if (c > 0) rt.active[nact + act - 1] = e;
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
      nact += __shfl_sync(0xffffffffu, act, 31);
    }
    if (lane == 0) {
      rt.offsets[E] = run;
      rt.n_act = nact;
    }
    __syncwarp();
    if (lane == 0) {
      // stable scatter (entries in (token, slot) order)
      int cur[kFMaxT * kMaxK];
      for (int i = 0; i < n; ++i) {
        int r = 0;
        for (int j = 0; j < i; ++j) r += rt.idx[j] == rt.idx[i] ? 1 : 0;
        cur[i] = rt.offsets[rt.idx[i]] + r;
      }
      for (int i = 0; i < n; ++i) {
        rt.perm[cur[i]] = i;
        rt.inv_perm[i] = cur[i];
      }
    }
  }
  __syncthreads();
  const Sched s = make_sched(a, rt.n_act);
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      a.r.topk_idx[i] = rt.idx[i];
      a.r.topk_w[i] = rt.w[i];
      a.r.perm[i] = rt.perm[i];
      a.r.inv_perm[i] = rt.inv_perm[i];
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) a.r.counts[e] = rt.counts[e];
    for (int e = threadIdx.x; e <= E; e += blockDim.x) a.r.offsets[e] = rt.offsets[e];
    for (int j = threadIdx.x; j < rt.n_act; j += blockDim.x) a.active[j] = rt.active[j];
    if (threadIdx.x < T) a.r.sigma[threadIdx.x] = rt.sigma[threadIdx.x];
    if (threadIdx.x == 0) {
      a.active[rt.n_act] = E;
      *a.n_active = rt.n_act + 1;
    }
  }
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
  bool ok = true;
  const int Tk = T * k;
  for (int i = 0; i < s.my_gu && ok; ++i) {
    const int sl = i % a.ring;
    if (!tc::mbar_wait(&full[sl], (i / a.ring) & 1u, abort_flag, a.status)) {
      ok = false;
      break;
    }
    const int u = blockIdx.x + i * gridDim.x;
    const bool sh = u < s.n_sh_units;
    const int e = sh ? E : rt.active[(u - s.n_sh_units) / s.units_per_exp];
    const int f = (sh ? u : (u - s.n_sh_units) % s.units_per_exp) * kFFeat + warp;
    const int nt = sh ? T : rt.counts[e];
    const int pos0 = sh ? 0 : rt.offsets[e];
    const uint8_t* slot = fsm + sl * a.slot_bytes;
    const uint32_t qb = kFFeat * g.H / 2, sb = kFFeat * g.H / 32;
    const uint4* qg = reinterpret_cast<const uint4*>(slot + warp * (g.H / 2));
    const uint4* qu = reinterpret_cast<const uint4*>(slot + qb + warp * (g.H / 2));
    const uint16_t* sg = reinterpret_cast<const uint16_t*>(slot + 2 * qb) + warp * (g.H / kGroup);
    const uint16_t* bg = reinterpret_cast<const uint16_t*>(slot + 2 * qb + sb) + warp * (g.H / kGroup);
    const uint16_t* su = reinterpret_cast<const uint16_t*>(slot + 2 * qb + 2 * sb) + warp * (g.H / kGroup);
    const uint16_t* bu = reinterpret_cast<const uint16_t*>(slot + 2 * qb + 3 * sb) + warp * (g.H / kGroup);
    int tok[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) tok[t] = t < nt ? (sh ? t : rt.perm[pos0 + t] / k) : 0;
    float ag[NT], au[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) ag[t] = au[t] = 0.f;
    for (int c = lane; c < g.H / 32; c += 32) {
      const uint4 vg = qg[c], vu = qu[c];
      const float s_g = 128.f * bf16_bits_to_float(sg[c >> 1]), b_g = bf16_bits_to_float(bg[c >> 1]);
      const float s_u = 128.f * bf16_bits_to_float(su[c >> 1]), b_u = bf16_bits_to_float(bu[c >> 1]);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (t < nt) {
          const float4* xl = reinterpret_cast<const float4*>(xs + tok[t] * xst) + ((c >> 5) * 8) * 32 + (c & 31);
          const float X = xsum[tok[t] * (xst / 32) + c];
          ag[t] = fmaf(s_g, dot32f(vg, xl, 32), fmaf(b_g - s_g, X, ag[t]));
          au[t] = fmaf(s_u, dot32f(vu, xl, 32), fmaf(b_u - s_u, X, au[t]));
        }
      }
    }
    // the slot's words are consumed: release it (generic reads before the async refill)
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&empty[sl]);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float gs = warp_sum(ag[t]), us = warp_sum(au[t]);
      if (lane == 0 && t < nt) {
        const uint16_t hv = float_to_bf16_bits(silu(gs) * us);
        if (sh)
          a.h_s[static_cast<size_t>(t) * g.Is + f] = hv;
        else
          a.h[static_cast<size_t>(pos0 + t) * g.I + f] = hv;
      }
    }
  }
  // Every h row is written: grid barrier (consumer thread 0 of each CTA).
  consumers_sync();
  if (threadIdx.x == 0 && (!ok || !grid_barrier(a.bar, gridDim.x, a.status))) rt.abort = 1;
  consumers_sync();
  if (rt.abort) return;

  if (s.my_blocks > 0) {
    // stage every h row (routed rows I wide, shared rows Is wide; stride hst)
    const int tid = threadIdx.x, nthr = kFWarps * 32;
    for (int r = 0; r < Tk + T; ++r) {
      const bool shr = r >= Tk;
      const uint16_t* src = shr ? a.h_s + static_cast<size_t>(r - Tk) * g.Is : a.h + static_cast<size_t>(r) * g.I;
      stage_row_f(src, shr ? g.Is : g.I, 16, hs + r * hst, tid, nthr, true);
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
  const int hl = lane & 15, hh = lane >> 4;
  for (int di = 0; di < s.my_blocks * s.n_down_parts && ok; ++di) {
    const int i = s.my_gu + di;
    const int sl = i % a.ring;
    if (!tc::mbar_wait(&full[sl], (i / a.ring) & 1u, abort_flag, a.status)) {
      ok = false;
      break;
    }
    const int bl = di / s.n_down_parts;
    const int j0 = (di % s.n_down_parts) * a.spd, nj = min(a.spd, s.n_slots - j0);
    const uint8_t* slot = fsm + sl * a.slot_bytes;
    // warp = output dim of the block; half-warps take the unit's slots in pairs
    for (int jj0 = 0; jj0 < nj; jj0 += 2) {
      const int jj = jj0 + hh;
      const bool live = jj < nj;
      const int e = live ? slot_expert(rt, E, j0 + jj) : E;
      const bool sh = e == E;
      const int K = sh ? g.Is : g.I;
      const int nt = live ? (sh ? T : rt.counts[e]) : 0;
      const int pos0 = sh ? Tk : (live ? rt.offsets[e] : 0);
      const uint8_t* base = slot + jj * (9 * Kmax);
      const uint4* qrow = reinterpret_cast<const uint4*>(base + warp * (K / 2));
      const uint16_t* srow = reinterpret_cast<const uint16_t*>(base + 8 * Kmax) + warp * (K / kGroup);
      const uint16_t* brow = reinterpret_cast<const uint16_t*>(base + 8 * Kmax + Kmax / 2) + warp * (K / kGroup);
      float p[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) p[t] = 0.f;
      if (live) {
        for (int c = hl; c < K / 32; c += 16) {
          const uint4 qv = qrow[c];
          const float s128 = 128.f * bf16_bits_to_float(srow[c >> 1]), bb = bf16_bits_to_float(brow[c >> 1]);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            if (t < nt) {
              const int r = pos0 + t;
              const float4* hl4 = reinterpret_cast<const float4*>(hs + r * hst) + ((c >> 4) * 8) * 16 + (c & 15);
              const float X = hsum[r * (hst / 32) + c];
              p[t] = fmaf(s128, dot32f(qv, hl4, 16), fmaf(bb - s128, X, p[t]));
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float v = p[t];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (hl == 0 && t < nt) ys[((pos0 + t) * s.my_blocks + bl) * kFDims + warp] = v;
      }
    }
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&empty[sl]);
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
