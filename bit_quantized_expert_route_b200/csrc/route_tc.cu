// Router for T > 64 on the tensor cores: logits, top-k with renormalised
// softmax weights, and the shared-expert gate.
//
// A cluster of S CTAs scores 128 tokens (S = 4 for 256 experts, 2 for
// 128..240, else 1).  CTA r of the cluster owns the C experts [r C, r C + C)
// (C = the padded expert count / S, a multiple of 16): D[128 tokens x C] =
// x W_r^T accumulates in tensor memory (tcgen05.mma, bf16 operands staged by
// TMA, FP32 accumulators), and CTA 0 adds a 16-column MMA against
// [w_sg; 0 ... 0] for x . w_sg.  Splitting the experts rather than the tokens
// keeps the MMA at M = 128 and spreads a 4096-token batch over 128 SMs; each
// CTA streams a quarter of W_r instead of all of it.
//
// Each token's TMEM lane is read by four threads, one per quarter of the
// CTA's columns; each keeps the P best (P = k rounded up to a power of two)
// of its quarter by insertion in expert order, the four sorted lists are
// merged, and the cluster's S lists meet in distributed shared memory: CTA r
// merges those of tokens [r 128/S, (r+1) 128/S), writes their experts and
// renormalised weights, and counts their experts in its own shared memory.
// Every list is sorted by (logit desc, expert index asc), the order the top-k
// follows; two sorted lists are merged by taking, position by position, the
// better of one list and the other reversed (the P best of the union, in
// bitonic order), then a bitonic merge.  Finally CTA r sums its share of the
// experts over the cluster's counts: the cluster's 128*k (token, slot)
// entries per expert, the first pass of the counting sort (one segment per
// cluster).  The lists are stored token-minor ([entry][token]) so that a
// warp's accesses are contiguous.
// ("Perplexity's Lily: ...", section "The Model": the router scores 256
// experts and keeps 8, plus one shared expert for every token.)
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int kRM = 128;                  // tokens per cluster (TMEM lanes)
constexpr int kRBK = 64;                  // inputs per stage
constexpr int kRStages = 4;
constexpr int kRMaxCols = 128;            // experts per CTA (MMA N)
constexpr int kREpiWarps = 16;            // 4 per TMEM lane quadrant: one column quarter each
constexpr int kRLoadWarp = kREpiWarps;    // one lane issues the TMA loads
constexpr int kRMmaWarp = kREpiWarps + 1; // TMEM + MMA
constexpr int kRThreads = (kRMmaWarp + 1) * 32;
constexpr int kA_BYTES = kRM * kRBK * 2;                  // 16 KB
constexpr int kG_BYTES = 16 * kRBK * 2;                   // 2 KB: w_sg row + 15 zero rows
constexpr int kB_BYTES = kRMaxCols * kRBK * 2;            // 16 KB
constexpr int kSTAGE = kA_BYTES + kB_BYTES + kG_BYTES;    // 34 KB (multiple of 1024)
constexpr int kBAR_OFF = kRStages * kSTAGE;
constexpr int kHIST_OFF = kBAR_OFF + 128;                 // [kMaxE] expert counts of this CTA's token slice
constexpr int kPART_OFF = kHIST_OFF + kMaxE * 4;          // quarter lists [3][kMaxK][128]: values, then indices
constexpr int kLIST_OFF = kPART_OFF + 3 * kRM * kMaxK * 8;   // merged lists [kMaxK][128] of (value, index)
constexpr int kRSMEM = kLIST_OFF + kRM * kMaxK * 8 + 1024;   // + alignment slack
constexpr uint32_t kRTmemCols = 256;
constexpr int kGateCol = kRMaxCols;       // accumulator column of x . w_sg (CTA 0)

__host__ __device__ constexpr int list_len(int K) { return K <= 1 ? 1 : K <= 2 ? 2 : K <= 4 ? 4 : 8; }

// The top-k order: larger logit first, then the lower expert index.
__device__ __forceinline__ bool ranks_before(float av, int ai, float bv, int bi) {
  return av > bv || (av == bv && ai < bi);
}

// a <- the P best of a and b (both sorted best first), sorted best first.
template <int P>
__device__ __forceinline__ void merge_best(float (&av)[P], int (&ai)[P], const float (&bv)[P], const int (&bi)[P]) {
#pragma unroll
  for (int j = 0; j < P; ++j) {
    const bool take = ranks_before(bv[P - 1 - j], bi[P - 1 - j], av[j], ai[j]);
    av[j] = take ? bv[P - 1 - j] : av[j];
    ai[j] = take ? bi[P - 1 - j] : ai[j];
  }
#pragma unroll
  for (int d = P / 2; d >= 1; d >>= 1) {
#pragma unroll
    for (int j = 0; j < P; ++j) {
      if ((j & d) == 0) {
        const bool sw = ranks_before(av[j + d], ai[j + d], av[j], ai[j]);
        const float tv = av[j];
        const int ti = ai[j];
        av[j] = sw ? av[j + d] : tv;
        ai[j] = sw ? ai[j + d] : ti;
        av[j + d] = sw ? tv : av[j + d];
        ai[j + d] = sw ? ti : ai[j + d];
      }
    }
  }
}

// Phase 1, one token (this thread's TMEM lane), quarter `part` of this CTA's
// columns [c_lo, c_hi) = experts e0 + c: the P best (+ bias) by insertion in
// expert order (a later expert displaces a kept one only if strictly larger,
// so equal logits keep the lower index first).  The four lists meet in a
// two-level tree through shared memory, and quarter 0 publishes the CTA's
// list of the token for the cluster.
template <int P>
__device__ __forceinline__ void router_phase1(uint32_t lane_base, int part, int c_lo, int c_hi, int e0, int E,
                                              const float* __restrict__ bias, int tl, float* pv, int* pi,
                                              uint2* list) {
  float bv[P];
  int bi[P];
#pragma unroll
  for (int j = 0; j < P; ++j) {
    bv[j] = -INFINITY;
    bi[j] = 0x7fffffff;
  }
  // rolled loops: this code runs once per CTA, so its size (instruction
  // fetch) rather than its issue count sets its time
#pragma unroll 1
  for (int c0 = c_lo; c0 < c_hi; c0 += 4) {
    float v[4];
    tc::tmem_ld4(lane_base + c0, v);
    tc::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = e0 + c0 + i;
      // branch-free insertion (no divergence between the warp's tokens)
      float cv = e < E ? v[i] + (bias ? __ldg(bias + e) : 0.f) : -INFINITY;
      int ci = e;
#pragma unroll
      for (int j = 0; j < P; ++j) {
        const bool take = cv > bv[j];
        const float tv = bv[j];
        const int ti = bi[j];
        bv[j] = take ? cv : tv;
        bi[j] = take ? ci : ti;
        cv = take ? tv : cv;
        ci = take ? ti : ci;
      }
    }
  }
  // tree merge through slots of pv/pi: level 0, quarter 1 into 0 (slot 0) and
  // 3 into 2 (slot 2); level 1, quarter 2 into 0 (slot 1)
#pragma unroll 1
  for (int lvl = 0; lvl < 2; ++lvl) {
    const bool publish = lvl == 0 ? (part & 1) != 0 : part == 2;
    const int slot = lvl == 0 ? (part & ~1) : 1;
    if (publish) {
#pragma unroll
      for (int j = 0; j < P; ++j) {
        pv[(slot * kMaxK + j) * kRM + tl] = bv[j];
        pi[(slot * kMaxK + j) * kRM + tl] = bi[j];
      }
    }
    // level 0: all four quarters (barrier 2); level 1: quarters 0 and 2 (barrier 4)
    const uint32_t bar_id = lvl == 0 ? 2u : 4u, bar_n = lvl == 0 ? kREpiWarps * 32u : kREpiWarps * 16u;
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(bar_n) : "memory");
    if (publish || (lvl == 1 && part != 0)) return;
    float cv[P];
    int ci[P];
#pragma unroll
    for (int j = 0; j < P; ++j) {
      cv[j] = pv[(slot * kMaxK + j) * kRM + tl];
      ci[j] = pi[(slot * kMaxK + j) * kRM + tl];
    }
    merge_best<P>(bv, bi, cv, ci);
  }
#pragma unroll
  for (int j = 0; j < P; ++j) list[j * kRM + tl] = make_uint2(__float_as_uint(bv[j]), static_cast<uint32_t>(bi[j]));
}

// Phase 2, one token of this CTA's slice: merge the cluster's S lists (read
// from each CTA's shared memory), write the k experts and their renormalised
// softmax weights, and count the experts into this CTA's histogram.
template <int K>
__device__ __forceinline__ void router_phase2(uint32_t list_addr, int S, int tl, int t, int T, int E, int* hist,
                                              int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  constexpr int P = list_len(K);
  float bv[P];
  int bi[P];
  const uint32_t row = list_addr + static_cast<uint32_t>(tl * 8);   // entry j at + j * kRM * 8
  {
    const uint32_t remote = tc::mapa(row, 0);
#pragma unroll
    for (int j = 0; j < P; ++j) {
      const uint2 u = tc::ld_cluster_v2(remote + j * kRM * 8);
      bv[j] = __uint_as_float(u.x);
      bi[j] = static_cast<int>(u.y);
    }
  }
#pragma unroll 1
  for (int c = 1; c < S; ++c) {
    float cv[P];
    int ci[P];
    const uint32_t remote = tc::mapa(row, static_cast<uint32_t>(c));
#pragma unroll
    for (int j = 0; j < P; ++j) {
      const uint2 u = tc::ld_cluster_v2(remote + j * kRM * 8);
      cv[j] = __uint_as_float(u.x);
      ci[j] = static_cast<int>(u.y);
    }
    merge_best<P>(bv, bi, cv, ci);
  }
  if (t >= T) return;
  float z[K];
  float sum = 0.f;
#pragma unroll
  for (int j = 0; j < K; ++j) {
    z[j] = expf(bv[j] - bv[0]);
    sum += z[j];
  }
#pragma unroll
  for (int j = 0; j < K; ++j) {
    topk_idx[static_cast<size_t>(t) * K + j] = bi[j];
    topk_w[static_cast<size_t>(t) * K + j] = z[j] / sum;
    // counting is order-independent; an index outside [0, E) only follows a device timeout
    if (static_cast<unsigned>(bi[j]) < static_cast<unsigned>(E)) atomicAdd(&hist[bi[j]], 1);
  }
}

struct alignas(64) RouterMaps {
  CUtensorMap x;     // x [T, H], box 128 rows x 64 inputs, 128-B swizzle
  CUtensorMap w;     // W_r [E, H], box C rows x 64 inputs, 128-B swizzle
  CUtensorMap g;     // w_sg [1, H], box 1 row x 64 inputs
};

// Expert split of a cluster: S CTAs of C columns each.
struct RouterSplit {
  int S, C;
};
RouterSplit router_split(int E) {
  const int n_mma = max(16, (E + 15) & ~15);
  RouterSplit r;
  r.S = n_mma >= 256 ? 4 : (n_mma >= 128 ? 2 : 1);
  r.C = ((n_mma + r.S - 1) / r.S + 15) & ~15;
  return r;
}

__global__ void __launch_bounds__(kRThreads, 1) router_tc_kernel(
    const __grid_constant__ RouterMaps maps, const float* __restrict__ router_bias, int T, int H, int E, int k,
    int S, int C, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, float* __restrict__ sigma,
    int32_t* __restrict__ seg_counts, int* status, long long wait_limit) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  const uint32_t sbase = tc::smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBAR_OFF);
  uint64_t* empty = full + kRStages;
  uint64_t* acc_full = empty + kRStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* hist = reinterpret_cast<int*>(smem + kHIST_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_ctarank();           // = blockIdx.x % S
  const int t0 = (static_cast<int>(blockIdx.x) / S) * kRM;
  const int e0 = static_cast<int>(rank) * C;             // this CTA's first expert
  const bool with_gate = rank == 0;
  const int nks = H / kRBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(acc_full, 1);
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  // zero rows 1..15 of every stage's gate tile once (row 0 is reloaded per stage)
  constexpr int kEpiThreads = kREpiWarps * 32;
  if (warp < kREpiWarps) {
    for (int i = threadIdx.x; i < kMaxE; i += kEpiThreads) hist[i] = 0;
    if (with_gate) {
      for (int i = threadIdx.x; i < kRStages * 15 * 8; i += kEpiThreads) {
        const int s = i / 120, rr = 1 + (i % 120) / 8, c = i % 8;
        *reinterpret_cast<uint4*>(smem + s * kSTAGE + kA_BYTES + kB_BYTES + rr * 128 + c * 16) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      tc::fence_proxy_async_smem();
    }
  }
  if (warp == kRMmaWarp) tc::tmem_alloc(tmem_slot, kRTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the prologue touched only this CTA's shared and tensor memory
  pdl_wait();
  pdl_launch_dependents();

  if (warp == kRLoadWarp) {
    // ---------------------------------------------------------- loader
    // one thread streams the stages: x tile, this CTA's router rows, the gate row
    if (lane == 0) {
      const uint32_t tx = static_cast<uint32_t>(kA_BYTES + C * kRBK * 2 + (with_gate ? kRBK * 2 : 0));
      int ks = 0;
      for (; ks < nks; ++ks) {
        const int s = ks % kRStages;
        if (!tc::mbar_wait(&empty[s], ((ks / kRStages) & 1) ^ 1, abort_flag, status, wait_limit)) break;
        const uint32_t st = sbase + s * kSTAGE;
        tc::mbar_arrive_expect_tx(&full[s], tx);
        tc::tma_load_2d(st, &maps.x, ks * kRBK, t0, &full[s]);
        tc::tma_load_2d(st + kA_BYTES, &maps.w, ks * kRBK, e0, &full[s]);
        if (with_gate) tc::tma_load_2d(st + kA_BYTES + kB_BYTES, &maps.g, ks * kRBK, 0, &full[s]);
      }
      // every stage this thread requested has landed before the CTA may exit
      tc::drain_ring(full, kRStages, static_cast<uint32_t>(ks), status);
    }
    __syncwarp();
  } else if (warp < kREpiWarps) {
    // ------------------------------------------------- epilogue, phase 1
    // warp w reads TMEM lane quadrant w % 4 (its 32 tokens) and the column
    // quarter w / 4 of their logits
    const int q = warp & 3, part = warp >> 2, tl = q * 32 + lane;
    const int quarter = ((C / 4) + 15) & ~15;
    const int c_lo = min(part * quarter, C), c_hi = min(c_lo + quarter, C);
    const uint32_t got = tc::mbar_wait(acc_full, 0, abort_flag, status, wait_limit) ? 1u : 0u;
    uint32_t all_got;   // the epilogue threads agree before any of them enters its barriers
    asm volatile("{\n\t.reg .pred p, r;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred r, 3, %2, p;\n\t"
                 "selp.u32 %0, 1, 0, r;\n\t}"
                 : "=r"(all_got)
                 : "r"(got), "n"(kEpiThreads)
                 : "memory");
    if (all_got) {
      tc::tc_fence_after();
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
      float* pv = reinterpret_cast<float*>(smem + kPART_OFF);
      int* pi = reinterpret_cast<int*>(pv + 3 * kRM * kMaxK);
      uint2* list = reinterpret_cast<uint2*>(smem + kLIST_OFF);
      switch (list_len(k)) {   // list length fixed at compile time: the lists stay in registers
        case 1: router_phase1<1>(lane_base, part, c_lo, c_hi, e0, E, router_bias, tl, pv, pi, list); break;
        case 2: router_phase1<2>(lane_base, part, c_lo, c_hi, e0, E, router_bias, tl, pv, pi, list); break;
        case 4: router_phase1<4>(lane_base, part, c_lo, c_hi, e0, E, router_bias, tl, pv, pi, list); break;
        default: router_phase1<8>(lane_base, part, c_lo, c_hi, e0, E, router_bias, tl, pv, pi, list); break;
      }
      if (with_gate && part == 0) {
        float g[16];
        tc::tmem_ld16(lane_base + kGateCol, g);
        tc::tmem_wait_ld();
        if (t0 + tl < T) sigma[t0 + tl] = sigmoid(g[0]);
      }
    }
  } else if (warp == kRMmaWarp) {
    // -------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(kRM, C);
      const uint32_t idesc_g = tc::idesc_bf16(kRM, 16);
      bool ok = true;
      for (int ks = 0; ks < nks; ++ks) {
        const int s = ks % kRStages;
        if (!tc::mbar_wait(&full[s], (ks / kRStages) & 1, abort_flag, status, wait_limit)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t st = sbase + s * kSTAGE;
#pragma unroll
        for (int kk = 0; kk < kRBK / 16; ++kk) {
          const uint64_t adesc = tc::sdesc_sw128(st + kk * 32);
          const uint32_t accum = (ks > 0 || kk > 0) ? 1u : 0u;
          tc::mma_bf16_ss(tmem, adesc, tc::sdesc_sw128(st + kA_BYTES + kk * 32), idesc, accum);
          if (with_gate)
            tc::mma_bf16_ss(tmem + kGateCol, adesc, tc::sdesc_sw128(st + kA_BYTES + kB_BYTES + kk * 32), idesc_g,
                            accum);
        }
        tc::mma_commit(&empty[s]);
      }
      if (ok) tc::mma_commit(acc_full);
      tc::mma_commit(drain);
      tc::mbar_wait_drain(drain, 0, status);
    }
    __syncwarp();
  }
  // ------------------------------------------------------ phase 2 (cluster)
  // every CTA's lists are published; CTA `rank` finishes its slice of tokens
  __syncwarp();
  tc::cluster_sync();
  const int slice = kRM / S;
  if (threadIdx.x < slice) {
    const int tl = static_cast<int>(rank) * slice + threadIdx.x;
    const uint32_t list_addr = sbase + kLIST_OFF;
#define ROUTER_P2(K) router_phase2<K>(list_addr, S, tl, t0 + tl, T, E, hist, topk_idx, topk_w)
    switch (k) {   // k fixed at compile time
      case 1: ROUTER_P2(1); break;
      case 2: ROUTER_P2(2); break;
      case 3: ROUTER_P2(3); break;
      case 4: ROUTER_P2(4); break;
      case 5: ROUTER_P2(5); break;
      case 6: ROUTER_P2(6); break;
      case 7: ROUTER_P2(7); break;
      default: ROUTER_P2(8); break;
    }
#undef ROUTER_P2
  }
  // every slice is counted: CTA `rank` sums its share of the experts over the
  // cluster's histograms and writes the cluster's segment counts
  __syncwarp();
  tc::cluster_sync();
  {
    const int per = (E + S - 1) / S;
    const int e_lo = static_cast<int>(rank) * per, e_hi = min(e_lo + per, E);
    const int seg = static_cast<int>(blockIdx.x) / S;
    for (int e = e_lo + static_cast<int>(threadIdx.x); e < e_hi; e += kRThreads) {
      const uint32_t a = sbase + kHIST_OFF + static_cast<uint32_t>(e) * 4;
      uint32_t sum = 0;
      for (int c = 0; c < S; ++c) sum += tc::ld_cluster_u32(tc::mapa(a, static_cast<uint32_t>(c)));
      seg_counts[static_cast<size_t>(seg) * E + e] = static_cast<int32_t>(sum);
    }
  }
  __syncwarp();
  tc::cluster_sync();   // no CTA reads another's shared memory after this point
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == kRMmaWarp) tc::tmem_dealloc(tmem, kRTmemCols);
}

}  // namespace

cudaError_t launch_router(const uint16_t* x, const uint16_t* w_router, const float* router_bias,
                          const uint16_t* w_sg, int T, int H, int E, int k,
                          int32_t* topk_idx, float* topk_w, float* sigma, int32_t* seg_counts, int* status,
                          cudaStream_t s) {
  RouterMaps maps;
  const RouterSplit sp = router_split(E);
  if (!make_tmap_2d(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, H, T, kRBK, kRM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&maps.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_router, H, E, kRBK, sp.C,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&maps.g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_sg, H, 1, kRBK, 1, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(router_tc_kernel), kRSMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(((T + kRM - 1) / kRM) * sp.S));
  cfg.blockDim = dim3(kRThreads);
  cfg.dynamicSmemBytes = kRSMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(sp.S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // as launch_pdl
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, router_tc_kernel, maps, router_bias, T, H, E, k, sp.S, sp.C, topk_idx, topk_w,
                            sigma, seg_counts, status, wait_limit_cycles());
}

}  // namespace moe
