// Fused decode for T <= 8 tokens: router, top-k, grouping, gate/up + SwiGLU,
// down projection and the fixed-order combine of a whole STACK of layers in
// ONE cooperative launch of one CTA per SM ("Perplexity's Lily: ...", section
// "How It Works: Prefill and Decode Strategies": decoding a few tokens streams
// the active experts' packed weights, so a layer is bound by how fast those
// bytes arrive, and the forward pass is one GPU submission with no CPU round
// trip).  A single moe_forward call is a stack of one layer.
//
// Why one launch for many layers: at T = 1 a layer's active weights are
// ~16 MB, about 2.5 us of HBM time, so launch latency, cold instruction
// caches and memory latency decide the layer time.  Inside one launch the
// code stays warm from layer to layer, nothing is launched between layers,
// and the producer warp fetches the next layer's router rows and first
// shared-expert tile while the current layer still computes.
//
// Each layer has three all-to-all exchanges between the CTAs (all CTAs are
// co-resident: cooperative launch).  None is a grid barrier: the values
// travel in tagged 64-bit words that a reader polls until they are current
// (see wait_words), so a CTA goes on the moment the data it needs is there.
//
//   A  input: layer 0 reads x; layer l > 0 reads the previous layer's output
//      y (bf16) and the CTAs' partial sums of its squares and applies
//      RMSNorm (weight 1): x = bf16(y / sqrt(mean(y^2) + eps)).  Router
//      logits: CTA c scores rows c, c+G, ... of [W_r; w_sg] (from shared
//      memory, copied there by the producer ahead of time) for every token
//      and publishes them.                               -- exchange: logits
//   B  every CTA reads the T x (E+1) logits and repeats the (tiny, exact and
//      deterministic) top-k, shared gate and counting sort, so it knows the
//      active experts without another exchange.
//   C  gate/up units: (expert slot, 16 features) -> h = bf16(silu(g) * u),
//      published pair by pair.                           -- exchange: h
//      The producer keeps copying the down tiles meanwhile: they depend on
//      the routing, not on h.
//   D  down units: (16 output dims, up to 8 expert slots); then the combine
//      of each token's k + 1 terms in slot order, then the shared term,
//      exactly as the other kernels; between layers the CTA publishes its
//      output dims and the partial sum of their squares.  -- exchange: y
//
// Weight tiles stream through a ring of shared-memory slots filled by one
// producer thread (cp.async.bulk, completion on the slot's "full" mbarrier)
// and released by the 16 consumer warps ("empty" mbarrier, one arrival per
// warp).  The ring position runs on across layers, so the producer can start
// the next layer's routing-independent tile as soon as a slot frees up.  All
// waits are bounded; a timeout records MOE_ERR_DEVICE_TIMEOUT in the status
// word and the kernel returns with every copy it issued landed.
//
// Dot products on the tensor cores (warp-level mma.sync, bf16 in, FP32
// accumulation; the T <= 8 tokens are the 8 columns of the n8 tile): per group
// of 64 inputs, with A = 128 + q as exact bf16 values (one AND-OR per code
// pair, no scale applied) and B = the activations,
//   sum_i (s q_i + b) x_i = s * (sum_i (128 + q_i) x_i - 128 X) + b X,  X = sum_i x_i,
// applied per group after the MMAs.  Inside each group of 8 inputs both
// operands use the order (0,4,1,5,2,6,3,7) in which the AND-OR yields code
// pairs; the activations are staged in that order, so no permutes are
// needed.
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "mma_dq.cuh"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int kFWarps = 16;                     // consumer warps
constexpr int kFThreads = (kFWarps + 1) * 32;   // + the producer warp
constexpr int kFFeat = 16;                      // features per gate/up unit
constexpr int kFDims = 16;                      // output dims per down block
constexpr int kFMaxSpd = 8;                     // expert slots per down unit (one per warp pair)
constexpr int kFRingMax = 8;
constexpr int kFMaxT = 8;                       // tokens: the n8 column tile of mma.sync
constexpr int kFRouterRows = 2;                 // router rows per CTA with loads in flight together
constexpr int kFMaxRouterRows = 4;              // router rows per CTA held in shared memory
constexpr int kFMaxLayers = 40;                 // layers per launch (kernel-parameter space)
constexpr int kFMaxGrid = 160;                  // CTAs (SMs) the RMSNorm partial sums are read for in one pass

struct FusedArgs {
  Geometry g;
  int n_layers;
  float eps;              // RMSNorm between layers
  const uint16_t* x;      // input of layer 0 [T, H]
  uint16_t* out;          // output of the last layer [T, H]
  uint16_t* trace;        // NULL or [n_layers][2][T][H]: layer inputs and outputs
  RoutingPtrs r;          // routing outputs of the last layer (topk_idx NULL: none)
  int32_t* active;
  int32_t* n_active;
  // tagged exchange words (workspace): payload in the low half
  unsigned long long* lgx;     // [T][E+1] logits (FP32 bits)
  unsigned long long* hx;      // [T*k + T][Kmax/2] h (two bf16), routed rows then shared rows
  unsigned long long* yx;      // [T][H/2] outputs of the layers before the last (two bf16)
  unsigned long long* ssx;     // [G][kFMaxT] each CTA's sum of squares of its outputs (FP32 bits)
  unsigned* bar;          // [1] exit counter, [2] epoch
  int* status;
  int ring, slot_bytes, spd, rows_per_cta;
  int rs_gu, rs_dn, dslot;   // staged row strides of gate/up and down codes; bytes per down expert slot
  long long wait_limit;   // cycles before a bounded wait gives up
  int off_bar, off_wr, off_xs, off_xsum, off_lg, off_rt, off_y, off_nrm;
  LayerPtr layers[kFMaxLayers];
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
  int32_t first[kFMaxT * kMaxK];   // entry i is its expert's first occurrence
  int32_t n_act;               // routed active experts
  int32_t abort;
  uint32_t epoch;              // the launch's epoch (tags of layer l: (epoch + 1) * 64 + l)
};

// One warp's share of a 16-row weight tile: groups g0 .. g0 + ng - 1 (ng <=
// NG) of 64 inputs.  Lane (lg4, lt) holds rows lg4 and lg4 + 8 (codes at
// qrow and qrow + 8 rs, already offset by the lane's 8 bytes) and token
// columns 2 lt, 2 lt + 1 (valid below tn; activations at xrow, in uint4 units
// already offset by the lane; group sums at xsum[t * xs + G]); scales and
// biases are rows of ngr groups.  The scales and biases of all the warp's
// groups are loaded up front, then each group adds
// s (sum (128 + q) x - 128 X) + b X to y[row][column].
template <int NG>
__device__ __forceinline__ void tile_groups(float (&y)[2][2], const uint8_t* qrow, int rs, const uint16_t* srow,
                                            const uint16_t* brow, int ngr, int g0, int ng, const uint4* xrow,
                                            bool tok_live, const float* xsum, int xs, int tn, int lg4, int lt) {
  float sv[2][NG], bv[2][NG];
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    const int G = g0 + (q < ng ? q : 0);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      sv[r][q] = bf16_bits_to_float(srow[(lg4 + 8 * r) * ngr + G]);
      bv[r][q] = bf16_bits_to_float(brow[(lg4 + 8 * r) * ngr + G]);
    }
  }
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    if (q < ng) {
      const int G = g0 + q;
      const uint2 qa = *reinterpret_cast<const uint2*>(qrow + G * 32);
      const uint2 qc = *reinterpret_cast<const uint2*>(qrow + 8 * rs + G * 32);
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      const uint4 xb0 = tok_live ? xrow[G * 8] : z, xb1 = tok_live ? xrow[G * 8 + 1] : z;
      float d[4];
      group_dot(d, qa, qc, xb0, xb1);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int t = 2 * lt + c;
        if (t < tn) {
          const float X = xsum[t * xs + G];
#pragma unroll
          for (int r = 0; r < 2; ++r) y[r][c] = fmaf(sv[r][q], d[2 * r + c] - 128.f * X, fmaf(bv[r][q], X, y[r][c]));
        }
      }
    }
  }
}


__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kFWarps * 32) : "memory"); }

// Exchanges between CTAs carry their own readiness: every value travels in a
// 64-bit word whose high half is a tag unique to (launch, layer), stored and
// loaded whole (an aligned 8-byte access is single-copy atomic).  A reader
// polls the words it needs until each carries the current tag -- one round
// trip through L2, no fence and no separate counter.  A word left from an
// earlier layer or launch carries another tag, so it is never taken for a
// current one.  Tag of layer l: (epoch + 1) * 64 + l, with the epoch read
// from the workspace at the start of a launch and advanced once by the last
// CTA to leave (launch_exit); 2^32 / 64 launches before it wraps.
__device__ __forceinline__ unsigned long long ld_word(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_word(unsigned long long* p, uint32_t tag, uint32_t payload) {
  const unsigned long long v = (static_cast<unsigned long long>(tag) << 32) | payload;
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// The payloads of up to N words once each carries `tag`: all N loads are in
// flight together, and only the words still stale are loaded again, so a
// thread pays one round trip through L2 for the batch rather than one per
// word (one at a time, staging h took 12 us at T = 8).  A NULL pointer is a
// slot with nothing to wait for (payload 0).  Bounded: gives up (ok = false,
// status recorded, the CTA's abort flag raised) after the deadline or as
// soon as another thread of the CTA has given up.
template <int N>
__device__ __forceinline__ void wait_words(const unsigned long long* const (&p)[N], uint32_t tag,
                                           uint32_t (&out)[N], long long deadline, volatile int* abort,
                                           int* status, bool& ok) {
  unsigned long long v[N];
#pragma unroll
  for (int i = 0; i < N; ++i) v[i] = p[i] ? ld_word(p[i]) : (static_cast<unsigned long long>(tag) << 32);
  for (uint32_t n = 0; ok; ++n) {
    bool all = true;
#pragma unroll
    for (int i = 0; i < N; ++i) all = all && static_cast<uint32_t>(v[i] >> 32) == tag;
    if (all) break;
    if ((n & 15u) == 15u && (*abort || clock64() > deadline)) {
      ok = false;
      if (!*abort) {
        *abort = 1;
        if (status) atomicExch(status, kStatusTimeout);
      }
      break;
    }
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (static_cast<uint32_t>(v[i] >> 32) != tag) v[i] = ld_word(p[i]);
  }
#pragma unroll
  for (int i = 0; i < N; ++i) out[i] = static_cast<uint32_t>(v[i]);
}

// Called once per CTA at its end: the last CTA to leave advances the epoch
// (bar[2]) for the next launch on the same workspace and resets its exit
// counter (bar[1]).  Every CTA read the epoch at its start.
__device__ void launch_exit(unsigned* bar, unsigned nblocks) {
  if (atomicAdd(bar + 1, 1u) == nblocks - 1) {
    bar[1] = 0u;
    bar[2] = bar[2] + 1u;
  }
}

// Unit schedule of one CTA in one layer: its gate/up units u = c, c+G, ...
// over the global list [shared-expert units | routed units], then its down
// units (dim blocks c, c+G, ..., each split into parts of at most spd_max
// slots, balanced).
struct Sched {
  int n_gu_units;      // global gate/up units
  int n_sh_units;      // of which shared-expert units (first)
  int units_per_exp;   // I / 16
  int n_slots;         // down slots: shared + routed active
  int n_down_parts;    // down units per dim block
  int spd;             // slots per down unit (the last may have fewer)
  int n_blocks;        // dim blocks (H / 16)
  int my_gu, my_blocks, n_units;
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
  s.n_units = s.my_gu + s.my_blocks * s.n_down_parts;
  return s;
}

// Gate/up unit u: expert slot (0 = shared) and first feature.
__device__ __forceinline__ void gu_unit(const Sched& s, int u, int& slot, int& f0) {
  const bool sh = u < s.n_sh_units;
  slot = sh ? 0 : 1 + (u - s.n_sh_units) / s.units_per_exp;
  f0 = (sh ? u : (u - s.n_sh_units) % s.units_per_exp) * kFFeat;
}

// Staged tiles: a few large contiguous copies per tile, issued by the
// producer warp's lanes together (lane 0 first raised the slot's transaction
// count; the caller's __syncwarp orders it).  One copy per code row into a
// padded row (so that the 8 rows one mma fragment reads start in different
// bank groups) made ~36 copies per gate/up unit and ~90 per down unit; the
// copies then reached the memory system so late that the tiles' arrival, not
// the bank conflicts, bound the layer.
//
// gate/up unit (expert e, features f0..f0+15):
//   [16 gate rows][16 up rows] (H/2 bytes each), then
//   [s gate][b gate][s up][b up] (16 x H/64 bf16 each).
__device__ __forceinline__ uint32_t gateup_bytes(const Geometry& g) {
  return 2 * kFFeat * (g.H / 2) + 4 * (kFFeat * g.H / 32);
}
__device__ void issue_gateup(const FusedArgs& a, const LayerPtr& L, int e, int f0, uint32_t dst, uint64_t* full,
                             int lane) {
  const Geometry& g = a.g;
  const bool sh = e >= g.E;
  const size_t row0 = static_cast<size_t>(sh ? 0 : e * g.I) + f0;
  const uint32_t qb = kFFeat * g.H / 2, sb = kFFeat * g.H / 32;
  if (lane < 2) {
    const QMatPtr& W = lane == 0 ? (sh ? L.sh_gate : L.gate) : (sh ? L.sh_up : L.up);
    tc::bulk_load(dst + lane * qb, W.q + row0 * (g.H / 8), qb, full);
  } else if (lane < 6) {
    const int j = lane - 2;
    const QMatPtr& V = j < 2 ? (sh ? L.sh_gate : L.gate) : (sh ? L.sh_up : L.up);
    tc::bulk_load(dst + 2 * qb + j * sb, ((j & 1) ? V.b : V.s) + row0 * (g.H / kGroup), sb, full);
  }
}

// down unit (16 output dims of dim block blk, expert slots j0..j0+nj-1): per
// slot jj at jj * dslot (dslot = 9 Kmax): [16 code rows of K/2 bytes,
// contiguous][s: 16 x K/64 at + 8 Kmax][b at + 8 Kmax + Kmax / 2], three
// copies per slot, lane jj issuing slot jj's.  (One copy per 256-byte row
// spread the rows over the banks but made ~90 copies per unit, and the
// producer then finished issuing a layer's tiles ~12 us after its routing
// was known.)  Returns the bytes to expect.
__device__ __forceinline__ uint32_t down_bytes(const Geometry& g, int j0, int nj) {
  uint32_t bytes = 0;
  for (int jj = 0; jj < nj; ++jj) {
    const int K = j0 + jj == 0 ? g.Is : g.I;
    bytes += kFDims * K / 2 + 2 * (kFDims * K / 32);
  }
  return bytes;
}
__device__ void issue_down(const FusedArgs& a, const LayerPtr& L, const RouteSmem& rt, int blk, int j0, int nj,
                           uint32_t dst, uint64_t* full, int lane) {
  const Geometry& g = a.g;
  const int Kmax = max(g.I, g.Is);
  if (lane < nj) {
    const int jj = lane;
    const bool sh = j0 + jj == 0;
    const int K = sh ? g.Is : g.I;
    const QMatPtr& W = sh ? L.sh_down : L.down;
    const size_t row0 = static_cast<size_t>(sh ? 0 : rt.slot_e[j0 + jj] * g.H) + blk * kFDims;
    const uint32_t base = dst + jj * a.dslot;
    const uint32_t qb = kFDims * K / 2, sb = kFDims * K / 32;
    tc::bulk_load(base, W.q + row0 * (K / 8), qb, full);
    tc::bulk_load(base + 8 * Kmax, W.s + row0 * (K / kGroup), sb, full);
    tc::bulk_load(base + 8 * Kmax + Kmax / 2, W.b + row0 * (K / kGroup), sb, full);
  }
}

// Issue unit i of this CTA (layer L) into ring slot `dst` (whole producer warp).
__device__ void issue_unit(const FusedArgs& a, const LayerPtr& L, const RouteSmem& rt, const Sched& s, int i,
                           uint32_t dst, uint64_t* full, int lane) {
  const Geometry& g = a.g;
  if (i < s.my_gu) {
    int slot, f0;
    gu_unit(s, blockIdx.x + i * gridDim.x, slot, f0);
    if (lane == 0) tc::mbar_arrive_expect_tx(full, gateup_bytes(g));
    __syncwarp();
    issue_gateup(a, L, rt.slot_e[slot], f0, dst, full, lane);
    return;
  }
  const int di = i - s.my_gu;
  const int blk = blockIdx.x + (di / s.n_down_parts) * gridDim.x;
  const int j0 = (di % s.n_down_parts) * s.spd, nj = min(s.spd, s.n_slots - j0);
  if (lane == 0) tc::mbar_arrive_expect_tx(full, down_bytes(g, j0, nj));
  __syncwarp();
  issue_down(a, L, rt, blk, j0, nj, dst, full, lane);
}

// This CTA's router rows of layer L (rows c, c+G, ... of [W_r; w_sg]) into
// the shared-memory row buffer; completes on `full`.
__device__ void issue_router_rows(const Geometry& g, const LayerPtr& L, int nrows, uint32_t dst, uint64_t* full) {
  const uint32_t rb = static_cast<uint32_t>(g.H) * 2;
  tc::mbar_arrive_expect_tx(full, nrows * rb);
  for (int rr = 0; rr < nrows; ++rr) {
    const int row = blockIdx.x + rr * gridDim.x;
    const uint16_t* src = row < g.E ? L.w_router + static_cast<size_t>(row) * g.H : L.w_sg;
    tc::bulk_load(dst + rr * rb, src, rb, full);
  }
}

template <int NT>
__global__ void __launch_bounds__(kFThreads, 1) decode_fused_kernel(const __grid_constant__ FusedArgs a) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = g.T, k = g.k, E = g.E, E1 = g.E + 1;
  const int G = static_cast<int>(gridDim.x);
  const uint32_t ring0 = tc::smem_u32(fsm);
  uint64_t* full = reinterpret_cast<uint64_t*>(fsm + a.off_bar);
  uint64_t* empty = full + kFRingMax;
  uint64_t* rfull = empty + kFRingMax;    // router rows of the current layer have landed
  uint64_t* rfree = rfull + 1;            // consumers are done with the router rows
  uint64_t* ready = rfree + 1;            // the layer's routing is in shared memory
  const uint16_t* wr = reinterpret_cast<const uint16_t*>(fsm + a.off_wr);   // [rows_per_cta][H]
  // x (phases A, C) and h (phase D) share one staging area, as do their group sums
  uint16_t* xs = reinterpret_cast<uint16_t*>(fsm + a.off_xs);   // [T][H] bf16, interleaved K order
  float* xsum = reinterpret_cast<float*>(fsm + a.off_xsum);      // [T][H/64] group sums
  uint16_t* hs = xs;                                             // [T*k + T][Kmax] bf16, interleaved K order
  float* hsum = xsum;                                            // [T*k + T][Kmax/64] group sums
  float* lg = reinterpret_cast<float*>(fsm + a.off_lg);          // logits; router partials; dot reductions
  RouteSmem& rt = *reinterpret_cast<RouteSmem*>(fsm + a.off_rt);
  float* ys = reinterpret_cast<float*>(fsm + a.off_y);           // [T*k + T][my_blocks][16]
  float* nrm = reinterpret_cast<float*>(fsm + a.off_nrm);        // [T] 1/rms of the layer input
  volatile int* abort_flag = &rt.abort;
  const int Kmax = max(g.I, g.Is);
  const int n = T * k, Tk = n;
  const int nrows = (E1 - static_cast<int>(blockIdx.x) + G - 1) / G;   // router rows of this CTA
  const bool producer = warp == kFWarps;
  const bool early = static_cast<int>(blockIdx.x) < g.Is / kFFeat;      // first unit is a shared-expert unit

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.ring; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kFWarps);
    }
    tc::mbar_init(rfull, 1);
    tc::mbar_init(rfree, 1);
    tc::mbar_init(ready, 1);
    rt.abort = 0;
    rt.epoch = *reinterpret_cast<volatile const unsigned*>(a.bar + 2);
    tc::fence_barrier_init();
  }
  __syncthreads();

  if (producer) {
    // ------------------------------------------------------- producer warp
    // Per layer: the routing-independent first unit (a shared-expert tile),
    // then, once the layer's routing is known, the next layer's router rows
    // and the rest of this layer's units.  Ring fills are numbered across
    // layers in the order the consumers take them.  The whole warp runs the
    // loop (its waits are made warp-uniform) and issues each tile's row
    // copies together.
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity, abort_flag, a.status, a.wait_limit));
    };
    uint32_t fill = 0;             // ring fills issued
    if (lane == 0) issue_router_rows(g, a.layers[0], nrows, tc::smem_u32(wr), rfull);
    uint32_t rfills = 1;
    bool ok = true;
    for (int l = 0; l < a.n_layers && ok; ++l) {
      const LayerPtr& L = a.layers[l];
      const uint32_t base = fill;
      if (early) {
        const int sl = static_cast<int>(fill % a.ring);
        if (!wait_all(&empty[sl], ((fill / a.ring) & 1u) ^ 1u)) break;
        tc::fence_proxy_async_smem();
        if (lane == 0) tc::mbar_arrive_expect_tx(&full[sl], gateup_bytes(g));
        __syncwarp();
        issue_gateup(a, L, E, static_cast<int>(blockIdx.x) * kFFeat, ring0 + sl * a.slot_bytes, &full[sl], lane);
        ++fill;
      }
      if (!wait_all(ready, static_cast<uint32_t>(l) & 1u)) break;
      const Sched s = make_sched(a, rt.n_act);
      if (l + 1 < a.n_layers) {
        // the consumers finished with this layer's router rows before its routing was ready
        if (!wait_all(rfree, static_cast<uint32_t>(l) & 1u)) break;
        tc::fence_proxy_async_smem();
        if (lane == 0) issue_router_rows(g, a.layers[l + 1], nrows, tc::smem_u32(wr), rfull);
        ++rfills;
      }
      for (uint32_t i = fill - base; i < static_cast<uint32_t>(s.n_units); ++i) {
        const int sl = static_cast<int>(fill % a.ring);
        if (!wait_all(&empty[sl], ((fill / a.ring) & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        tc::fence_proxy_async_smem();   // consumers' generic reads of the slot precede the refill
        issue_unit(a, L, rt, s, static_cast<int>(i), ring0 + sl * a.slot_bytes, &full[sl], lane);
        ++fill;
      }
    }
    // every copy this warp issued has landed before the CTA may exit
    if (lane == 0) {
      tc::drain_ring(full, static_cast<uint32_t>(a.ring), fill, a.status);
      tc::drain_ring(rfull, 1u, rfills, a.status);
    }
    __syncwarp();
    return;
  }

  // ------------------------------------------------------ consumer warps
  const int tid = threadIdx.x, nthr = kFWarps * 32;
  const int lg4 = lane >> 2, lt = lane & 3;
  const int ngrp = g.H / kGroup;
  const uint32_t sb = kFFeat * g.H / 32;   // bytes of one scale (or bias) block of a gate/up tile
  const size_t act = static_cast<size_t>(T) * g.H;
  uint32_t fill = 0;      // ring fills consumed
  // Abort handling: a wait that gives up raises rt.abort (and makes later
  // waits give up at once).  No consumer warp leaves a loop on its own: every
  // warp keeps taking the same CTA barriers, skipping the work, and the
  // decision to stop is read from rt.abort right after a CTA barrier, where
  // every thread sees the same value.
  for (int l = 0; l < a.n_layers; ++l) {
    const LayerPtr& L = a.layers[l];
    const bool last = l + 1 == a.n_layers;
    bool ok = true;

    // -------------------------------------------------------------- phase A
    // the layer input: x, or RMSNorm of the previous layer's output, read
    // from the exchange words as soon as every CTA has published its part
    const uint32_t tag = (rt.epoch + 1u) * 64u + static_cast<uint32_t>(l);
    // the router bias of the logit this thread will publish, fetched now so
    // that its memory latency overlaps the input exchange
    float my_bias = 0.f;
    if (tid < nrows * T && L.router_bias) {
      const int row = static_cast<int>(blockIdx.x) + (tid / T) * G;
      if (row < E) my_bias = __ldg(L.router_bias + row);
    }
    const int c4 = 4 * tid;
    const bool live = c4 < g.H;
    uint2 xv[NT];
    if (l == 0) {
#pragma unroll
      for (int t = 0; t < NT; ++t)
        xv[t] = (live && t < T) ? __ldcg(reinterpret_cast<const uint2*>(a.x + static_cast<size_t>(t) * g.H + c4))
                                : make_uint2(0u, 0u);
    } else {
      const long long deadline = clock64() + a.wait_limit;
      const unsigned long long* yrow = a.yx + tid * 2;
      const unsigned long long* yp[2 * NT];
      uint32_t yv[2 * NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const bool need = live && t < T;
        yp[2 * t] = need ? yrow + t * (g.H / 2) : nullptr;
        yp[2 * t + 1] = need ? yrow + t * (g.H / 2) + 1 : nullptr;
      }
      wait_words<2 * NT>(yp, tag - 1u, yv, deadline, abort_flag, a.status, ok);
#pragma unroll
      for (int t = 0; t < NT; ++t) xv[t] = make_uint2(yv[2 * t], yv[2 * t + 1]);
      // warp t sums the CTAs' partial sums of squares of token t: lane i
      // takes CTAs i, i+32, ..., then a fixed shuffle tree; the same order in
      // every CTA
      if (warp < T) {
        const unsigned long long* sp_[kFMaxGrid / 32];
        uint32_t part[kFMaxGrid / 32];
#pragma unroll
        for (int j = 0; j < kFMaxGrid / 32; ++j) {
          const int c = lane + 32 * j;
          sp_[j] = c < G ? a.ssx + c * kFMaxT + warp : nullptr;
        }
        wait_words<kFMaxGrid / 32>(sp_, tag - 1u, part, deadline, abort_flag, a.status, ok);
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < kFMaxGrid / 32; ++j) ss += __uint_as_float(part[j]);
        ss = warp_sum(ss);
        if (lane == 0) nrm[warp] = 1.0f / sqrtf(ss / static_cast<float>(g.H) + a.eps);
      }
      consumers_sync();
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (live && t < T) {
          const float s = nrm[t];
          xv[t].x = pack_bf16x2(bf16_lo(xv[t].x) * s, bf16_hi(xv[t].x) * s);
          xv[t].y = pack_bf16x2(bf16_lo(xv[t].y) * s, bf16_hi(xv[t].y) * s);
        }
      }
    }
    if (a.trace && blockIdx.x == 0)
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (live && t < T)
          *reinterpret_cast<uint2*>(a.trace + 2 * l * act + static_cast<size_t>(t) * g.H + c4) = xv[t];
    // router rows r = c, c + G, ... (staged by the producer): thread tid owns
    // the inputs [4 tid, 4 tid + 4) of every row and token
    // (wait outcomes are made warp-uniform: the work they guard uses warp-collective instructions)
    ok = __all_sync(0xffffffffu, ok && tc::mbar_wait(rfull, static_cast<uint32_t>(l) & 1u, abort_flag, a.status,
                                                     a.wait_limit));
    float* part = lg;   // [nrows][kFWarps][NT] partials (lg is free until phase B)
    if (ok) {
      for (int r0 = 0; r0 < nrows; r0 += kFRouterRows) {
#pragma unroll
        for (int q = 0; q < kFRouterRows; ++q) {
          const uint2 wv = (live && r0 + q < nrows)
                               ? *reinterpret_cast<const uint2*>(wr + static_cast<size_t>(r0 + q) * g.H + c4)
                               : make_uint2(0u, 0u);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            float s = fmaf(bf16_lo(xv[t].x), bf16_lo(wv.x), 0.f);
            s = fmaf(bf16_hi(xv[t].x), bf16_hi(wv.x), s);
            s = fmaf(bf16_lo(xv[t].y), bf16_lo(wv.y), s);
            s = fmaf(bf16_hi(xv[t].y), bf16_hi(wv.y), s);
            s = warp_sum(s);
            if (lane == 0 && r0 + q < nrows && t < T) part[((r0 + q) * kFWarps + warp) * NT + t] = s;
          }
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
    if (tid == 0) {
      tc::fence_proxy_async_smem();      // the row buffer's generic reads precede its next TMA refill
      tc::mbar_arrive(rfree);
    }
    if (ok && tid < nrows * T) {      // this CTA's logits go out first: every CTA waits for them
      const int rr = tid / T, t = tid % T;
      const int row = blockIdx.x + rr * G;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kFWarps; ++w) v += part[(rr * kFWarps + w) * NT + t];
      v += my_bias;
      st_word(a.lgx + static_cast<size_t>(t) * E1 + row, tag, __float_as_uint(v));
    }
    for (int i = tid; i < T * ngrp; i += nthr) {     // sums over groups of 64 (fixed order)
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
    consumers_sync();   // the partials in lg are consumed before phase B reuses it

    // -------------------------------------------------------------- phase B
    // Every CTA rebuilds the routing from all CTAs' logits (top-k by warp
    // reductions, then a counting sort of the n = T*k <= 64 entries), so no
    // further exchange is needed before the expert weights can be requested.
    {
      const long long deadline = clock64() + a.wait_limit;
      for (int i0 = tid; i0 < T * E1; i0 += 8 * nthr) {
        const unsigned long long* lp[8];
        uint32_t lv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) lp[j] = i0 + j * nthr < T * E1 ? a.lgx + i0 + j * nthr : nullptr;
        wait_words<8>(lp, tag, lv, deadline, abort_flag, a.status, ok);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (i0 + j * nthr < T * E1) lg[i0 + j * nthr] = __uint_as_float(lv[j]);
      }
    }
    consumers_sync();
    if (rt.abort) break;
    if (warp < T) {
      topk_redux(lg + warp * E1, E, k, lane, rt.idx + warp * k, rt.w + warp * k);
      if (lane == 0) rt.sigma[warp] = sigmoid(lg[warp * E1 + E]);
    }
    // one token: warp 0 selected and now groups, so a warp barrier suffices
    if (T > 1)
      consumers_sync();
    else
      __syncwarp();
    if (warp == 0) {
      // grouping by one warp, O(n) per entry: first occurrences, then each
      // entry's stable rank (entries with a smaller expert, then earlier
      // entries of the same expert) and the active experts below its own
      for (int i = lane; i < n; i += 32) {
        const int e = rt.idx[i];
        int f = 1;
        for (int j = 0; j < i; ++j) f &= rt.idx[j] != e ? 1 : 0;
        rt.first[i] = f;
      }
      __syncwarp();
      int nact = 0;
      for (int i = lane; i < n; i += 32) {
        const int e_i = rt.idx[i];
        int below = 0, rank = 0, abelow = 0, cnt = 0;
        for (int j = 0; j < n; ++j) {
          const int ej = rt.idx[j];
          below += ej < e_i ? 1 : 0;
          rank += (ej == e_i && j < i) ? 1 : 0;
          cnt += ej == e_i ? 1 : 0;
          abelow += (rt.first[j] && ej < e_i) ? 1 : 0;
        }
        const int pos = below + rank;
        rt.perm[pos] = i;
        rt.inv_perm[i] = pos;
        if (rt.first[i]) {
          rt.slot_e[1 + abelow] = e_i;
          rt.slot_cnt[1 + abelow] = cnt;
          rt.slot_off[1 + abelow] = below;
          ++nact;
        }
      }
      nact = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(nact)));
      if (lane == 0) {
        rt.n_act = nact;
        rt.slot_e[0] = E;
        rt.slot_cnt[0] = T;
        rt.slot_off[0] = Tk;
      }
      // the producer may now schedule this layer's units: the warp's writes
      // are ordered before lane 0's arrival (release) by the warp barrier
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(ready);
    }
    consumers_sync();
    const Sched s = make_sched(a, rt.n_act);

    // -------------------------------------------------------------- phase C
    // gate/up, two units at a time (their dot products are independent, so
    // their tensor-core chains overlap, and the pair shares one round of CTA
    // barriers): warp w owns the 16-row tile w % 2 (gate or up) for the K
    // eighth w / 2 of both units; per group of 64 inputs four mma.sync, then
    // the group's scale and bias for the lane's two token columns.
    float* red = lg;   // [2 units][2 tiles][8 K eighths][16 rows][NT] partial sums (logits are no longer needed)
    {
      const int m = warp & 1, ke = warp >> 1;
      const int ge = ngrp / 8;                       // groups per K eighth
      constexpr int kRedUnit = 2 * 8 * 16 * NT;
      for (int i = 0; i < s.my_gu; i += 2) {
        const int nu = min(2, s.my_gu - i);
        int slot[2], f0[2];
        float y[2][2][2] = {};                         // [unit][row lg4 / lg4 + 8][token 2 lt / 2 lt + 1]
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (u < nu) {
            const uint32_t f = fill + u;
            const int sl = static_cast<int>(f % a.ring);
            const bool got = __all_sync(
                0xffffffffu, tc::mbar_wait(&full[sl], (f / a.ring) & 1u, abort_flag, a.status, a.wait_limit));
            gu_unit(s, blockIdx.x + (i + u) * G, slot[u], f0[u]);
            unsigned tmask = 0;                        // tokens of this unit's expert
            if (slot[u] == 0)
              tmask = (1u << T) - 1u;
            else
              for (int r = 0; r < rt.slot_cnt[slot[u]]; ++r) tmask |= 1u << (rt.perm[rt.slot_off[slot[u]] + r] / k);
            const uint8_t* ub = fsm + sl * a.slot_bytes;
            const uint8_t* qrow = ub + (m * kFFeat + lg4) * a.rs_gu + lt * 8;     // rows lg4, lg4 + 8
            const uint16_t* srow = reinterpret_cast<const uint16_t*>(ub + 2 * kFFeat * a.rs_gu + m * 2 * sb);
            const uint16_t* brow = srow + sb / 2;
            const bool tok_live = lg4 < T && ((tmask >> lg4) & 1u);
            const uint4* xrow = reinterpret_cast<const uint4*>(xs + (tok_live ? lg4 : 0) * g.H) + lt * 2;
            tile_groups<4>(y[u], qrow, a.rs_gu, srow, brow, ngrp, ke * ge, got ? ge : 0, xrow, tok_live, xsum, ngrp,
                           T, lg4, lt);
            // every read of the unit's slot is done: release it (a slot that
            // never filled is not handed back: the producer is stopping as well)
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && got) tc::mbar_arrive(&empty[sl]);
          }
        }
        fill += nu;
#pragma unroll
        for (int u = 0; u < 2; ++u)
          if (u < nu)
#pragma unroll
            for (int c = 0; c < 2; ++c)
              if (2 * lt + c < T)
#pragma unroll
                for (int r = 0; r < 2; ++r)
                  red[u * kRedUnit + ((m * 8 + ke) * 16 + lg4 + 8 * r) * NT + 2 * lt + c] = y[u][r][c];
        consumers_sync();
        // h = bf16(silu(g) * u) for (unit, feature pair, token); K eighths
        // summed in order; each pair goes out as one exchange word of h row
        // `pos` (routed rows in expert order, then the shared expert's rows)
        if (tid < nu * (kFFeat / 2) * T && !rt.abort) {
          const int u = tid / ((kFFeat / 2) * T), rem = tid % ((kFFeat / 2) * T);
          const int fp = rem / T, t = rem % T;
          const int sl_u = u == 0 ? slot[0] : slot[1];
          const int f0_u = u == 0 ? f0[0] : f0[1];
          bool member = sl_u == 0;
          int pos = Tk + t;
          for (int r = 0; r < (sl_u == 0 ? 0 : rt.slot_cnt[sl_u]); ++r)
            if (rt.perm[rt.slot_off[sl_u] + r] / k == t) {
              member = true;
              pos = rt.slot_off[sl_u] + r;
            }
          if (member) {
            const float* ru = red + u * kRedUnit;
            uint32_t hv[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int f = 2 * fp + q;
              float gs = 0.f, us = 0.f;
#pragma unroll
              for (int e8 = 0; e8 < 8; ++e8) {
                gs += ru[((0 * 8 + e8) * 16 + f) * NT + t];
                us += ru[((1 * 8 + e8) * 16 + f) * NT + t];
              }
              hv[q] = float_to_bf16_bits(silu(gs) * us);
            }
            st_word(a.hx + static_cast<size_t>(pos) * (Kmax / 2) + (f0_u / 2 + fp), tag, hv[0] | (hv[1] << 16));
          }
        }
        consumers_sync();   // red is reused by the next pair
      }
    }
    consumers_sync();
    if (rt.abort) break;

    // -------------------------------------------------------------- phase D
    if (s.my_blocks > 0) {
      // stage every h row (routed rows I wide, shared rows Is wide) in the
      // interleaved K order, as each CTA's gate/up units publish it, and its
      // sums over groups of 64
      const long long deadline = clock64() + a.wait_limit;
      const int vmax = Kmax / 8;
      const int ng4 = (Tk + T) * vmax;
      for (int i0 = tid; i0 < ng4; i0 += 4 * nthr) {   // four 8-value groups (16 words) per batch
        const unsigned long long* hp[16];
        uint32_t hv16[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = i0 + q * nthr;
          const int r = i / vmax, u = i - r * vmax;
          const bool need = i < ng4 && u * 8 < (r >= Tk ? g.Is : g.I);
          const unsigned long long* w4 = a.hx + static_cast<size_t>(r) * (Kmax / 2) + u * 4;
#pragma unroll
          for (int e = 0; e < 4; ++e) hp[4 * q + e] = need ? w4 + e : nullptr;
        }
        wait_words<16>(hp, tag, hv16, deadline, abort_flag, a.status, ok);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = i0 + q * nthr;
          const int r = i / vmax, u = i - r * vmax;
          if (i < ng4 && u * 8 < (r >= Tk ? g.Is : g.I))
            reinterpret_cast<uint4*>(hs + static_cast<size_t>(r) * Kmax)[u] =
                interleave8(make_uint4(hv16[4 * q], hv16[4 * q + 1], hv16[4 * q + 2], hv16[4 * q + 3]));
        }
      }
      consumers_sync();
      const int kg = Kmax / kGroup;
      for (int i = tid; i < (Tk + T) * kg; i += nthr) {
        const int r = i / kg, G8 = i % kg;
        const int K = r >= Tk ? g.Is : g.I;
        if (G8 * kGroup < K) {
          const uint4* r4 = reinterpret_cast<const uint4*>(hs + static_cast<size_t>(r) * Kmax) + G8 * 8;
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
    // down units, two at a time as the gate/up units: warp w owns expert slot
    // w % 8 of each unit (16 dims x K) for the K half w / 8; lanes hold rows
    // (dims) lg4, lg4 + 8 and token columns 2 lt, 2 lt + 1
    {
      const int jj = warp & 7, kh = warp >> 3;
      const int kg = Kmax / kGroup;
      float* redd = lg;   // [2 units][8 slots][2 K halves][16 dims][NT]
      constexpr int kRedUnit = 8 * 2 * 16 * NT;
      const int n_du = s.my_blocks * s.n_down_parts;
      for (int di = 0; di < n_du; di += 2) {
        const int nu = min(2, n_du - di);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (u < nu) {
            const uint32_t f = fill + u;
            const int sl = static_cast<int>(f % a.ring);
            const bool got = __all_sync(
                0xffffffffu, tc::mbar_wait(&full[sl], (f / a.ring) & 1u, abort_flag, a.status, a.wait_limit));
            const int dd = di + u;
            const int j0 = (dd % s.n_down_parts) * s.spd, nj = min(s.spd, s.n_slots - j0);
            const bool jlive = got && jj < nj;
            const int j = j0 + jj;
            const int K = j == 0 ? g.Is : g.I;
            const int ng = K / kGroup, gh = ng / 2;       // groups, groups per K half
            const int nt = jlive ? rt.slot_cnt[j] : 0;
            const int pos0 = jlive ? rt.slot_off[j] : 0;
            float y[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
            if (jlive) {
              const uint8_t* ub = fsm + sl * a.slot_bytes + jj * a.dslot;
              const uint8_t* qrow = ub + lg4 * (K / 2) + lt * 8;
              const uint16_t* srow = reinterpret_cast<const uint16_t*>(ub + 8 * Kmax);
              const uint16_t* brow = reinterpret_cast<const uint16_t*>(ub + 8 * Kmax + Kmax / 2);
              const bool tok_live = lg4 < nt;
              const int hr = pos0 + (tok_live ? lg4 : 0);
              const uint4* hrow = reinterpret_cast<const uint4*>(hs + static_cast<size_t>(hr) * Kmax) + lt * 2;
              for (int gb = 0; gb < gh; gb += 4)
                tile_groups<4>(y, qrow, K / 2, srow, brow, ng, kh * gh + gb, min(4, gh - gb), hrow, tok_live,
                               hsum + pos0 * kg, kg, nt, lg4, lt);
            }
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && got) tc::mbar_arrive(&empty[sl]);
#pragma unroll
            for (int c = 0; c < 2; ++c)
              if (2 * lt + c < nt)
#pragma unroll
                for (int r = 0; r < 2; ++r)
                  redd[u * kRedUnit + ((jj * 2 + kh) * 16 + lg4 + 8 * r) * NT + 2 * lt + c] = y[r][c];
          }
        }
        fill += nu;
        consumers_sync();
        // y rows of these units' slots: both K halves summed in order
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (u < nu) {
            const int dd = di + u;
            const int bl = dd / s.n_down_parts;
            const int j0 = (dd % s.n_down_parts) * s.spd, nj = min(s.spd, s.n_slots - j0);
            const float* ru = redd + u * kRedUnit;
            for (int q = tid; q < nj * kFDims * NT; q += nthr) {
              const int js = q / (kFDims * NT), d = (q / NT) % kFDims, t = q % NT;
              const int jx = j0 + js;
              if (t < rt.slot_cnt[jx])
                ys[((rt.slot_off[jx] + t) * s.my_blocks + bl) * kFDims + d] =
                    ru[((js * 2 + 0) * 16 + d) * NT + t] + ru[((js * 2 + 1) * 16 + d) * NT + t];
            }
          }
        }
        consumers_sync();
      }
    }
    consumers_sync();
    if (rt.abort) break;
    // combine: out[t, d] = bf16( sum_j w[t,j] * y[inv_perm[t k + j]][d] + sigma_t * y[T k + t][d] ),
    // two adjacent dims per thread; between layers the outputs go out as
    // exchange words and the CTA also sums the squares of its bf16 outputs
    // per token (dim pairs in order)
    for (int i = tid; i < T * s.my_blocks * (kFDims / 2); i += nthr) {
      const int t = i / (s.my_blocks * (kFDims / 2)), rem = i % (s.my_blocks * (kFDims / 2));
      const int bl = rem / (kFDims / 2), d = 2 * (rem % (kFDims / 2));
      uint32_t ov[2];
      float sq = 0.f;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float acc = 0.f;
        for (int j = 0; j < k; ++j)
          acc = fmaf(rt.w[t * k + j], ys[(rt.inv_perm[t * k + j] * s.my_blocks + bl) * kFDims + d + q], acc);
        acc = fmaf(rt.sigma[t], ys[((Tk + t) * s.my_blocks + bl) * kFDims + d + q], acc);
        ov[q] = float_to_bf16_bits(acc);
        sq = fmaf(bf16_bits_to_float(ov[q]), bf16_bits_to_float(ov[q]), sq);
      }
      const int blk = blockIdx.x + bl * G;
      const size_t o = static_cast<size_t>(t) * g.H + blk * kFDims + d;
      const uint32_t pair = ov[0] | (ov[1] << 16);
      if (last)
        *reinterpret_cast<uint32_t*>(a.out + o) = pair;
      else
        st_word(a.yx + o / 2, tag, pair);
      if (a.trace) *reinterpret_cast<uint32_t*>(a.trace + (2 * l + 1) * act + o) = pair;
      lg[i] = sq;
    }
    if (!last) {
      consumers_sync();
      if (tid < T) {
        float ss = 0.f;
        for (int q = 0; q < s.my_blocks * (kFDims / 2); ++q) ss += lg[tid * s.my_blocks * (kFDims / 2) + q];
        st_word(a.ssx + blockIdx.x * kFMaxT + tid, tag, __float_as_uint(ss));
      }
    } else if (blockIdx.x == 0 && a.r.topk_idx) {
      // routing outputs of the last layer (off the other CTAs' critical path)
      for (int i = tid; i < n; i += nthr) {
        a.r.topk_idx[i] = rt.idx[i];
        a.r.topk_w[i] = rt.w[i];
        a.r.perm[i] = rt.perm[i];
        a.r.inv_perm[i] = rt.inv_perm[i];
      }
      for (int e = tid; e <= E; e += nthr) {
        int c = 0, below = 0;
        for (int i = 0; i < n; ++i) {
          c += rt.idx[i] == e ? 1 : 0;
          below += rt.idx[i] < e ? 1 : 0;
        }
        if (e < E) a.r.counts[e] = c;
        a.r.offsets[e] = below;
      }
      for (int jx = tid; jx < rt.n_act; jx += nthr) a.active[jx] = rt.slot_e[1 + jx];
      if (tid < T) a.r.sigma[tid] = rt.sigma[tid];
      if (tid == 0) {
        a.active[rt.n_act] = E;
        *a.n_active = rt.n_act + 1;
      }
    }
    // the next layer reads the outputs from the exchange words; its phase A
    // reuses shared memory the combine still reads
    consumers_sync();
  }
  // (after an abort, rt.abort also stops a producer still waiting for a
  // layer that will not come)
  if (tid == 0) launch_exit(a.bar, gridDim.x);
}

const void* fused_kernel_fn(int T) {
  return T == 1   ? reinterpret_cast<const void*>(decode_fused_kernel<1>)
         : T == 2 ? reinterpret_cast<const void*>(decode_fused_kernel<2>)
         : T <= 4 ? reinterpret_cast<const void*>(decode_fused_kernel<4>)
                  : reinterpret_cast<const void*>(decode_fused_kernel<8>);
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

// Shared-memory carve-up of one launch (identical for every layer).
struct FusedLayout {
  int ring, slot_bytes, spd, rows_per_cta, rs_gu, rs_dn, dslot;
  int off_bar, off_wr, off_xs, off_xsum, off_lg, off_rt, off_y, off_nrm, total;
};

FusedLayout fused_layout(const Geometry& g, int G) {
  FusedLayout f{};
  const int Kmax = g.I > g.Is ? g.I : g.Is;
  f.rs_gu = g.H / 2;
  f.rs_dn = Kmax / 2;                                       // down code rows are copied contiguously
  f.dslot = 9 * Kmax;                                        // codes (8 Kmax), then scales and biases
  f.slot_bytes = 2 * kFFeat * f.rs_gu + 4 * (kFFeat * g.H / 32);   // one gate/up unit
  f.spd = f.slot_bytes / f.dslot;
  if (f.spd > kFMaxSpd) f.spd = kFMaxSpd;
  f.rows_per_cta = (g.E + 1 + G - 1) / G;
  const int rows = g.T * g.k + g.T;
  const int blocks_per_cta = (g.H / kFDims + G - 1) / G;
  auto al = [](int v) { return (v + 127) / 128 * 128; };
  const int lg_floats = max(max(g.T * (g.E + 1), f.rows_per_cta * kFWarps * kFMaxT),
                            max(2 * 16 * 16 * kFMaxT, g.T * blocks_per_cta * kFDims));   // pairs of units
  const int stage_bytes = max(g.T * g.H * 2, rows * Kmax * 2);
  const int sums_bytes = max(g.T * (g.H / kGroup) * 4, rows * (Kmax / kGroup) * 4);
  const int fixed = al((2 * kFRingMax + 3) * 8) + al(f.rows_per_cta * g.H * 2) + al(stage_bytes) + al(sums_bytes) +
                    al(lg_floats * 4) + al(static_cast<int>(sizeof(RouteSmem))) +
                    al(rows * blocks_per_cta * kFDims * 4) + al(kFMaxT * 4);
  f.ring = (227 * 1024 - fixed) / f.slot_bytes;
  if (f.ring > kFRingMax) f.ring = kFRingMax;
  int off = 0;
  auto take = [&](int bytes) {
    const int o = off;
    off += al(bytes);
    return o;
  };
  take(f.ring * f.slot_bytes);
  f.off_bar = take((2 * kFRingMax + 3) * 8);
  f.off_wr = take(f.rows_per_cta * g.H * 2);
  f.off_xs = take(stage_bytes);
  f.off_xsum = take(sums_bytes);
  f.off_lg = take(lg_floats * 4);
  f.off_rt = take(static_cast<int>(sizeof(RouteSmem)));
  f.off_y = take(rows * blocks_per_cta * kFDims * 4);
  f.off_nrm = take(kFMaxT * 4);
  f.total = off;
  return f;
}

}  // namespace

bool decode_fused_supported(const Geometry& g) {
  if (g.T < 1 || g.T > kFMaxT) return false;
  if (g.H % 1024 || g.H > 2048) return false;
  if (g.I % kGroup || g.Is % kGroup) return false;      // whole groups: every staged row is 16-byte sized
  const int G = fused_grid();
  if (G > kFMaxGrid || G > kFusedMaxGrid) return false;
  // Every CTA must own a router row: a CTA's logits of layer l + 1 are
  // published only after it has read everything of layer l, and every
  // reader of layer l + 1's data first waits for all CTAs' logits, which is
  // what makes reusing the exchange words from layer to layer safe.
  if (G > g.E + 1) return false;
  if ((g.E + 1 + G - 1) / G > kFMaxRouterRows) return false;
  const FusedLayout f = fused_layout(g, G);
  if (f.spd < 1 || f.ring < 2 || f.total > 227 * 1024) return false;   // spd: at least one expert slot per down unit
  // the cooperative launch needs one resident CTA per SM (registers, shared
  // memory); checked once per kernel instance and shared-memory size
  struct Fit {
    int total = -1;
    bool ok = false;
  };
  static Fit fit[4];
  static std::mutex mu;
  const int slot = g.T == 1 ? 0 : g.T == 2 ? 1 : g.T <= 4 ? 2 : 3;
  std::lock_guard<std::mutex> lock(mu);
  if (fit[slot].total != f.total) {
    const void* fn = fused_kernel_fn(g.T);
    int per_sm = 0;
    fit[slot].ok = ensure_smem(fn, f.total) == cudaSuccess &&
                   cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kFThreads, f.total) == cudaSuccess &&
                   per_sm >= 1;
    (void)cudaGetLastError();   // a failed query leaves no sticky error for the caller's next check
    fit[slot].total = f.total;
  }
  return fit[slot].ok;
}

int decode_fused_max_layers() { return kFMaxLayers; }

cudaError_t launch_decode_fused(const Geometry& g, const LayerPtr* layers, int n_layers, const uint16_t* x,
                                uint16_t* out, uint16_t* trace, float eps, const RoutingPtrs& r, int32_t* active,
                                int32_t* n_active, const FusedExchange& xch, unsigned* bar, int* status,
                                cudaStream_t s) {
  if (n_layers < 1 || n_layers > kFMaxLayers || !decode_fused_supported(g)) return cudaErrorInvalidValue;
  FusedArgs a{};
  a.g = g;
  a.n_layers = n_layers;
  a.eps = eps;
  a.x = x;
  a.out = out;
  a.trace = trace;
  a.r = r;
  a.active = active;
  a.n_active = n_active;
  a.lgx = xch.logits;
  a.hx = xch.h;
  a.yx = xch.y;
  a.ssx = xch.sumsq;
  a.bar = bar;
  a.status = status;
  a.wait_limit = wait_limit_cycles();
  for (int l = 0; l < n_layers; ++l) a.layers[l] = layers[l];
  const int G = fused_grid();
  const FusedLayout f = fused_layout(g, G);
  a.ring = f.ring;
  a.slot_bytes = f.slot_bytes;
  a.spd = f.spd;
  a.rows_per_cta = f.rows_per_cta;
  a.rs_gu = f.rs_gu;
  a.rs_dn = f.rs_dn;
  a.dslot = f.dslot;
  a.off_bar = f.off_bar;
  a.off_wr = f.off_wr;
  a.off_xs = f.off_xs;
  a.off_xsum = f.off_xsum;
  a.off_lg = f.off_lg;
  a.off_rt = f.off_rt;
  a.off_y = f.off_y;
  a.off_nrm = f.off_nrm;
  const void* fn = fused_kernel_fn(g.T);
  cudaError_t e = ensure_smem(fn, f.total);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = f.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (g.T == 1) return cudaLaunchKernelEx(&cfg, decode_fused_kernel<1>, a);
  if (g.T == 2) return cudaLaunchKernelEx(&cfg, decode_fused_kernel<2>, a);
  if (g.T <= 4) return cudaLaunchKernelEx(&cfg, decode_fused_kernel<4>, a);
  return cudaLaunchKernelEx(&cfg, decode_fused_kernel<8>, a);
}

}  // namespace moe
