// GPU-resident expert routing: router logits, top-k with renormalised softmax
// weights, the shared-expert gate, and the token-to-expert histogram, prefix
// sum and stable permutation.  Nothing here synchronises with the host: the
// group sizes stay on the device and later kernels read them from there
// ("Perplexity's Lily: ...", section "How It Works: Prefill and Decode
// Strategies": histogram, prefix scan, scatter and block maps live in one GPU
// submission with no CPU synchronisation between expert layers).
#include "common.cuh"
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------------------
// Router + top-k (SIMT).  One CTA scores TB tokens against all E experts.
//   l[t,e]   = x_t . W_r[e] + b_e                        (FP32 accumulation)
//   idx[t,:] = k best by (logit desc, expert index asc)
//   w[t,j]   = exp(l_j - l_0) / sum_j' exp(l_j' - l_0)
//   sigma_t  = sigmoid(x_t . w_sg)
// ---------------------------------------------------------------------------
template <int TB>
__global__ void __launch_bounds__(256) router_topk_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ w_router,
    const float* __restrict__ router_bias, const uint16_t* __restrict__ w_sg,
    int T, int H, int E, int k,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, float* __restrict__ sigma) {
  extern __shared__ uint4 smem_u4[];
  const int vec = H / 8;                                   // uint4 (8 bf16) per row
  uint4* xs = smem_u4;                                      // [TB][vec]
  float* lg = reinterpret_cast<float*>(xs + TB * vec);      // [TB][E]
  const int t0 = blockIdx.x * TB;
  const int nt = min(TB, T - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;

  for (int i = threadIdx.x; i < TB * vec; i += blockDim.x) {
    const int r = i / vec, c = i - r * vec;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < nt) v = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t0 + r) * H)[c];
    xs[i] = v;
  }
  __syncthreads();

  for (int e = warp; e < E; e += nwarps) {
    float acc[TB];
#pragma unroll
    for (int r = 0; r < TB; ++r) acc[r] = 0.f;
    const uint4* wr = reinterpret_cast<const uint4*>(w_router + static_cast<size_t>(e) * H);
    for (int c = lane; c < vec; c += 32) {
      const uint4 wv = __ldg(wr + c);
      const float w0 = bf16_lo(wv.x), w1 = bf16_hi(wv.x), w2 = bf16_lo(wv.y), w3 = bf16_hi(wv.y);
      const float w4 = bf16_lo(wv.z), w5 = bf16_hi(wv.z), w6 = bf16_lo(wv.w), w7 = bf16_hi(wv.w);
#pragma unroll
      for (int r = 0; r < TB; ++r) {
        const uint4 xv = xs[r * vec + c];
        float a = acc[r];
        a = fmaf(bf16_lo(xv.x), w0, a); a = fmaf(bf16_hi(xv.x), w1, a);
        a = fmaf(bf16_lo(xv.y), w2, a); a = fmaf(bf16_hi(xv.y), w3, a);
        a = fmaf(bf16_lo(xv.z), w4, a); a = fmaf(bf16_hi(xv.z), w5, a);
        a = fmaf(bf16_lo(xv.w), w6, a); a = fmaf(bf16_hi(xv.w), w7, a);
        acc[r] = a;
      }
    }
    const float b = router_bias ? router_bias[e] : 0.f;
#pragma unroll
    for (int r = 0; r < TB; ++r) {
      const float s = warp_sum(acc[r]);
      if (lane == 0) lg[r * E + e] = s + b;
    }
  }
  __syncthreads();

  for (int r = warp; r < nt; r += nwarps) {
    const int t = t0 + r;
    select_topk_warp(lg + r * E, E, k, lane, topk_idx + static_cast<size_t>(t) * k,
                     topk_w + static_cast<size_t>(t) * k);
    float a = 0.f;
    const uint4* ws = reinterpret_cast<const uint4*>(w_sg);
    for (int c = lane; c < vec; c += 32) {
      const uint4 wv = __ldg(ws + c);
      const uint4 xv = xs[r * vec + c];
      a = fmaf(bf16_lo(xv.x), bf16_lo(wv.x), a); a = fmaf(bf16_hi(xv.x), bf16_hi(wv.x), a);
      a = fmaf(bf16_lo(xv.y), bf16_lo(wv.y), a); a = fmaf(bf16_hi(xv.y), bf16_hi(wv.y), a);
      a = fmaf(bf16_lo(xv.z), bf16_lo(wv.z), a); a = fmaf(bf16_hi(xv.z), bf16_hi(wv.z), a);
      a = fmaf(bf16_lo(xv.w), bf16_lo(wv.w), a); a = fmaf(bf16_hi(xv.w), bf16_hi(wv.w), a);
    }
    a = warp_sum(a);
    if (lane == 0) sigma[t] = sigmoid(a);
  }
}

// ---------------------------------------------------------------------------
// Stable counting sort of the T*k (token, slot) entries by expert.
// Entries are cut into segments of kSeg; one warp owns one segment.
//   pass 1 (hist):    per-segment expert counts
//   pass 2 (scan):    counts, offsets, per-segment bases, chunk list
//   pass 3 (scatter): perm / inv_perm, ranks taken in entry order
// Integer atomics only count (order-independent); every position comes from
// the scan and an in-order rank, so the permutation is deterministic.
// ---------------------------------------------------------------------------
constexpr int kSeg = 1024;
constexpr int kSegWarps = 4;

__global__ void __launch_bounds__(32 * kSegWarps) hist_kernel(
    const int32_t* __restrict__ topk_idx, int n, int E, int32_t* __restrict__ seg_counts) {
  extern __shared__ int sh_hist[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = blockIdx.x * kSegWarps + warp;
  int* h = sh_hist + warp * E;
  for (int e = lane; e < E; e += 32) h[e] = 0;
  __syncwarp();
  const int nseg = (n + kSeg - 1) / kSeg;
  if (seg >= nseg) return;
  const int b = seg * kSeg, end = min(b + kSeg, n);
  for (int i = b + lane; i < end; i += 32) {
    const int e = topk_idx[i];
    if (e >= 0 && e < E) atomicAdd(&h[e], 1);
  }
  __syncwarp();
  for (int e = lane; e < E; e += 32) seg_counts[static_cast<size_t>(seg) * E + e] = h[e];
}

// Block-wide exclusive scan over blockDim.x (<= 1024) ints; returns the total.
__device__ int block_exclusive_scan(int v, int* scratch /*[32]*/, int* out_excl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int w = lane < nw ? scratch[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    scratch[lane] = wi - w;   // exclusive warp prefix
    if (lane == 31) scratch[32] = wi;
  }
  __syncthreads();
  *out_excl = scratch[warp] + incl - v;
  const int total = scratch[32];
  __syncthreads();
  return total;
}

// One CTA of kScanThreads (>= E + 1) threads.  Thread e < E owns routed
// expert e; thread E owns the shared expert (all T tokens).
constexpr int kScanThreads = 288;

__global__ void __launch_bounds__(kScanThreads) scan_kernel(
    int32_t* __restrict__ seg_counts, int nseg, int E, int T, int k, int chunk_rows,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    Chunk* __restrict__ chunks, int32_t* __restrict__ n_chunks,
    int32_t* __restrict__ active, int32_t* __restrict__ n_active) {
  __shared__ int scratch[33];
  const int e = threadIdx.x;
  int c = 0;
  if (e < E)
    for (int s = 0; s < nseg; ++s) c += seg_counts[static_cast<size_t>(s) * E + e];
  int off = 0;
  const int total = block_exclusive_scan(e < E ? c : 0, scratch, &off);
  if (e < E) {
    counts[e] = c;
    offsets[e] = off;
    int run = off;
    for (int s = 0; s < nseg; ++s) {
      const size_t i = static_cast<size_t>(s) * E + e;
      const int v = seg_counts[i];
      seg_counts[i] = run;     // becomes this segment's first position for expert e
      run += v;
    }
  }
  if (e == 0) offsets[E] = total;

  // Chunk list ("block map"): each expert's rows cut into near-equal pieces of
  // at most chunk_rows rows.  Row space: routed rows [0, T*k) in expert order,
  // then the shared expert's rows T*k + t.
  const int rows = (e < E) ? c : (e == E ? T : 0);
  const int base_row = (e < E) ? off : T * k;
  const int nch = (rows + chunk_rows - 1) / chunk_rows;
  int first = 0;
  const int nchunks = block_exclusive_scan(nch, scratch, &first);
  for (int q = 0; q < nch; ++q) {
    const int r0 = static_cast<int>((static_cast<long long>(rows) * q) / nch);
    const int r1 = static_cast<int>((static_cast<long long>(rows) * (q + 1)) / nch);
    Chunk ch;
    ch.e = e; ch.row0 = base_row + r0; ch.rows = r1 - r0; ch.pad = 0;
    chunks[first + q] = ch;
  }
  if (e == 0) *n_chunks = nchunks;

  // Active-expert list: routed experts with rows, ascending, then the shared one.
  int apos = 0;
  const int nact = block_exclusive_scan((e < E && c > 0) ? 1 : 0, scratch, &apos);
  if (e < E && c > 0) active[apos] = e;
  if (e == 0) {
    active[nact] = E;
    *n_active = nact + 1;
  }
}

__global__ void __launch_bounds__(32 * kSegWarps) scatter_kernel(
    const int32_t* __restrict__ topk_idx, int n, int E, const int32_t* __restrict__ seg_base,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm) {
  extern __shared__ int sh_cnt[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = blockIdx.x * kSegWarps + warp;
  const int nseg = (n + kSeg - 1) / kSeg;
  if (seg >= nseg) return;
  int* cnt = sh_cnt + warp * E;
  for (int e = lane; e < E; e += 32) cnt[e] = seg_base[static_cast<size_t>(seg) * E + e];
  __syncwarp();
  const int b = seg * kSeg, end = min(b + kSeg, n);
  for (int base = b; base < end; base += 32) {
    const int i = base + lane;
    const bool valid = i < end;
    int e = valid ? topk_idx[i] : -1;
    if (valid && (e < 0 || e >= E)) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lanemask_lt());
    const int start = (e >= 0) ? cnt[e] : 0;
    __syncwarp();
    if (e >= 0) {
      const int pos = start + rank;
      perm[pos] = i;
      inv_perm[i] = pos;
      if ((peers >> lane) == 1u) cnt[e] = start + __popc(peers);   // highest lane of the group
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
int router_smem_bytes(int tb, int H, int E) { return tb * H * 2 + tb * E * 4; }

cudaError_t launch_router(const uint16_t* x, const uint16_t* w_router, const float* router_bias,
                          const uint16_t* w_sg, int T, int H, int E, int k,
                          int32_t* topk_idx, float* topk_w, float* sigma, cudaStream_t s) {
  if (H <= 4096) {
    constexpr int TB = 16;
    const int smem = router_smem_bytes(TB, H, E);
    cudaFuncSetAttribute(router_topk_kernel<TB>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    router_topk_kernel<TB><<<(T + TB - 1) / TB, 256, smem, s>>>(x, w_router, router_bias, w_sg, T, H, E, k,
                                                                 topk_idx, topk_w, sigma);
  } else {
    constexpr int TB = 8;
    const int smem = router_smem_bytes(TB, H, E);
    cudaFuncSetAttribute(router_topk_kernel<TB>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    router_topk_kernel<TB><<<(T + TB - 1) / TB, 256, smem, s>>>(x, w_router, router_bias, w_sg, T, H, E, k,
                                                                 topk_idx, topk_w, sigma);
  }
  return cudaGetLastError();
}

int num_segments(int n_entries) { return (n_entries + kSeg - 1) / kSeg; }

cudaError_t launch_group(const int32_t* topk_idx, int T, int k, int E, int chunk_rows,
                         int32_t* seg_scratch, int32_t* counts, int32_t* offsets,
                         int32_t* perm, int32_t* inv_perm, Chunk* chunks, int32_t* n_chunks,
                         int32_t* active, int32_t* n_active, cudaStream_t s) {
  const int n = T * k;
  const int nseg = num_segments(n);
  const int grid = (nseg + kSegWarps - 1) / kSegWarps;
  const int smem = kSegWarps * E * static_cast<int>(sizeof(int));
  hist_kernel<<<grid, 32 * kSegWarps, smem, s>>>(topk_idx, n, E, seg_scratch);
  scan_kernel<<<1, kScanThreads, 0, s>>>(seg_scratch, nseg, E, T, k, chunk_rows, counts, offsets,
                                         chunks, n_chunks, active, n_active);
  scatter_kernel<<<grid, 32 * kSegWarps, smem, s>>>(topk_idx, n, E, seg_scratch, perm, inv_perm);
  return cudaGetLastError();
}

}  // namespace moe
