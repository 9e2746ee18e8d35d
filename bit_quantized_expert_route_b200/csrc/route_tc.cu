// Router for T > 64 on the tensor cores: logits, top-k with renormalised
// softmax weights, and the shared-expert gate in one kernel.
//
// One CTA scores 128 tokens: D[128 tokens x E experts] = x W_r^T accumulates
// in tensor memory (tcgen05.mma, bf16 operands in shared memory, FP32
// accumulators), and a second 16-column MMA against [w_sg; 0 ... 0] yields
// x . w_sg in column 256.  The epilogue gives each token four threads (one
// per quarter of the experts, all reading the token's TMEM lane): each keeps
// the k best of its quarter in registers by insertion in expert order, then
// the first thread merges the four sorted lists, which realises the order
// (logit desc, expert index asc).  The CTA also counts its 128*k (token,
// slot) entries per expert: the first pass of the counting sort (one segment
// per CTA).
// ("Perplexity's Lily: ...", section "The Model": the router scores 256
// experts and keeps 8, plus one shared expert for every token.)
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int kRM = 128;                  // tokens per CTA (TMEM lanes)
constexpr int kRBK = 64;                  // inputs per stage
constexpr int kRStages = 4;
constexpr int kREpiWarps = 16;            // 4 per TMEM lane quadrant: one expert quarter each
constexpr int kRLoadWarp = kREpiWarps;    // one lane issues the TMA loads
constexpr int kRMmaWarp = kREpiWarps + 1; // TMEM + MMA
constexpr int kRThreads = (kRMmaWarp + 1) * 32;
constexpr int kA_BYTES = kRM * kRBK * 2;                  // 16 KB
constexpr int kB_BYTES = kMaxE * kRBK * 2;                // 32 KB (up to 256 experts)
constexpr int kG_BYTES = 16 * kRBK * 2;                   // 2 KB: w_sg row + 15 zero rows
constexpr int kSTAGE = kA_BYTES + kB_BYTES + kG_BYTES;    // 50 KB (multiple of 1024)
constexpr int kBAR_OFF = kRStages * kSTAGE;
constexpr int kPART_OFF = kBAR_OFF + 128 + kMaxE * 4;       // per-token partial lists [3][128][2 x kMaxK]
constexpr int kRSMEM = kPART_OFF + 3 * kRM * 2 * kMaxK * 4 + 1024;   // + alignment slack
constexpr uint32_t kRTmemCols = 512;
constexpr int kGateCol = 256;             // accumulator column of x . w_sg

// One token's epilogue (this thread's TMEM lane), part `part` of 4: logits of
// experts [c_lo, c_hi) (+ bias) scanned in expert order, the K largest kept by
// insertion (a later expert replaces a kept one only if strictly larger, so
// equal logits keep the lower index first).  Parts 1-3 publish their sorted
// lists; part 0 merges them (ties go to the lower part, whose experts are
// lower), then writes the renormalised softmax weights, the shared gate and
// the token's contribution to the CTA's expert histogram.
template <int K>
__device__ __forceinline__ void router_epilogue(uint32_t lane_base, int part, int c_lo, int c_hi, int E,
                                                const float* __restrict__ bias, int tl, int t, int T,
                                                float* pv, int* pi, int32_t* __restrict__ topk_idx,
                                                float* __restrict__ topk_w, float* __restrict__ sigma, int* hist) {
  float bv[K];
  int bi[K];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    bv[j] = -INFINITY;
    bi[j] = 0x7fffffff;
  }
  for (int c0 = c_lo; c0 < c_hi; c0 += 16) {
    float v[16];
    tc::tmem_ld16(lane_base + c0, v);
    tc::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int e = c0 + i;
      // branch-free insertion (no divergence between the warp's tokens)
      float cv = e < E ? v[i] + (bias ? __ldg(bias + e) : 0.f) : -INFINITY;
      int ci = e;
#pragma unroll
      for (int j = 0; j < K; ++j) {
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
  if (part > 0) {
#pragma unroll
    for (int j = 0; j < K; ++j) {
      pv[((part - 1) * kRM + tl) * kMaxK + j] = bv[j];
      pi[((part - 1) * kRM + tl) * kMaxK + j] = bi[j];
    }
  }
  asm volatile("bar.sync 2, %0;" ::"n"(kREpiWarps * 32) : "memory");
  if (part > 0) return;
  // merge parts 1..3 into this thread's list; entries are inserted only if
  // strictly larger, so on ties the earlier (lower-expert) entry stays first
#pragma unroll 1
  for (int q = 0; q < 3; ++q) {
#pragma unroll
    for (int jj = 0; jj < K; ++jj) {
      float cv = pv[(q * kRM + tl) * kMaxK + jj];
      int ci = pi[(q * kRM + tl) * kMaxK + jj];
#pragma unroll
      for (int j = 0; j < K; ++j) {
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
  float g[16];
  tc::tmem_ld16(lane_base + kGateCol, g);
  tc::tmem_wait_ld();
  if (t < T) {
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
      atomicAdd(&hist[bi[j]], 1);      // counting is order-independent
    }
    sigma[t] = sigmoid(g[0]);
  }
}

struct alignas(64) RouterMaps {
  CUtensorMap x;     // x [T, H], box 128 rows x 64 inputs, 128-B swizzle
  CUtensorMap w;     // W_r [E, H], box n_mma rows x 64 inputs, 128-B swizzle
  CUtensorMap g;     // w_sg [1, H], box 1 row x 64 inputs
};

__global__ void __launch_bounds__(kRThreads, 1) router_tc_kernel(
    const __grid_constant__ RouterMaps maps, const float* __restrict__ router_bias, int T, int H, int E, int k,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, float* __restrict__ sigma,
    int32_t* __restrict__ seg_counts, int* status) {
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
  int* hist = reinterpret_cast<int*>(smem + kBAR_OFF + 128);       // [kMaxE] this CTA's expert counts

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRM;
  const int nks = H / kRBK;
  const int n_mma = max(16, (E + 15) & ~15);

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
    for (int i = threadIdx.x; i < kRStages * 15 * 8; i += kEpiThreads) {
      const int s = i / 120, rr = 1 + (i % 120) / 8, c = i % 8;
      *reinterpret_cast<uint4*>(smem + s * kSTAGE + kA_BYTES + kB_BYTES + rr * 128 + c * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    tc::fence_proxy_async_smem();
  }
  if (warp == kRMmaWarp) tc::tmem_alloc(tmem_slot, kRTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kRLoadWarp) {
    // ---------------------------------------------------------- loader
    // one thread streams the stages: x tile, router rows and the gate row
    if (lane == 0) {
      const uint32_t tx = static_cast<uint32_t>(kA_BYTES + n_mma * kRBK * 2 + kRBK * 2);
      for (int ks = 0; ks < nks; ++ks) {
        const int s = ks % kRStages;
        if (!tc::mbar_wait(&empty[s], ((ks / kRStages) & 1) ^ 1, abort_flag, status)) break;
        const uint32_t st = sbase + s * kSTAGE;
        tc::mbar_arrive_expect_tx(&full[s], tx);
        tc::tma_load_2d(st, &maps.x, ks * kRBK, t0, &full[s]);
        tc::tma_load_2d(st + kA_BYTES, &maps.w, ks * kRBK, 0, &full[s]);
        tc::tma_load_2d(st + kA_BYTES + kB_BYTES, &maps.g, ks * kRBK, 0, &full[s]);
      }
    }
    __syncwarp();
  } else if (warp < kREpiWarps) {
    // --------------------------------------------------------- epilogue
    // warp w reads TMEM lane quadrant w % 4 (its 32 tokens) and the expert
    // quarter w / 4 of their logits
    const int q = warp & 3, part = warp >> 2, tl = q * 32 + lane;
    const int quarter = ((n_mma / 4) + 15) & ~15;
    const int c_lo = min(part * quarter, n_mma), c_hi = min(c_lo + quarter, n_mma);
    const uint32_t got = tc::mbar_wait(acc_full, 0, abort_flag, status) ? 1u : 0u;
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
      const int t = t0 + tl;
#define ROUTER_EPI(K) router_epilogue<K>(lane_base, part, c_lo, c_hi, E, router_bias, tl, t, T, pv, pi, topk_idx, \
                                         topk_w, sigma, hist)
      switch (k) {   // k fixed at compile time: the candidate lists stay in registers
        case 1: ROUTER_EPI(1); break;
        case 2: ROUTER_EPI(2); break;
        case 3: ROUTER_EPI(3); break;
        case 4: ROUTER_EPI(4); break;
        case 5: ROUTER_EPI(5); break;
        case 6: ROUTER_EPI(6); break;
        case 7: ROUTER_EPI(7); break;
        default: ROUTER_EPI(8); break;
      }
#undef ROUTER_EPI
    }
    // this CTA's segment of the (token, slot) entries: expert counts for the sort
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
    for (int e = threadIdx.x; e < E; e += kEpiThreads) seg_counts[static_cast<size_t>(blockIdx.x) * E + e] = hist[e];
  } else if (warp == kRMmaWarp) {
    // -------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(kRM, n_mma);
      const uint32_t idesc_g = tc::idesc_bf16(kRM, 16);
      bool ok = true;
      for (int ks = 0; ks < nks; ++ks) {
        const int s = ks % kRStages;
        if (!tc::mbar_wait(&full[s], (ks / kRStages) & 1, abort_flag, status)) {
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
  const uint32_t n_mma = static_cast<uint32_t>(max(16, (E + 15) & ~15));
  if (!make_tmap_2d(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, H, T, kRBK, kRM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&maps.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_router, H, E, kRBK, n_mma,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&maps.g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_sg, H, 1, kRBK, 1, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(router_tc_kernel), kRSMEM);
  if (e != cudaSuccess) return e;
  router_tc_kernel<<<(T + kRM - 1) / kRM, kRThreads, kRSMEM, s>>>(maps, router_bias, T, H, E, k, topk_idx, topk_w,
                                                                   sigma, seg_counts, status);
  return cudaGetLastError();
}

}  // namespace moe
