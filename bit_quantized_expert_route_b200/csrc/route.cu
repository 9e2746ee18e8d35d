// GPU-resident expert routing: the token-to-expert histogram, prefix sum and
// stable permutation, and (for T <= 64) a one-launch router + top-k + sort.
// The tensor-core router for larger T is in route_tc.cu.  Nothing here synchronises with the host: the
// group sizes stay on the device and later kernels read them from there
// ("Perplexity's Lily: ...", section "How It Works: Prefill and Decode
// Strategies": histogram, prefix scan, scatter and block maps live in one GPU
// submission with no CPU synchronisation between expert layers).
#include "common.cuh"
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------------------
// Stable counting sort of the T*k (token, slot) entries by expert.
// Segment s = the entries of tokens [128 s, 128 s + 128), i.e. of one router
// CTA, which already counted them per expert (pass 1).
//   pass 2 (scan):    counts, offsets, per-segment bases, chunk list
//   pass 3 (scatter): perm / inv_perm, ranks taken in entry order
// Integer atomics only count (order-independent); every position comes from
// the scan and an in-order rank, so the permutation is deterministic.
// ---------------------------------------------------------------------------
constexpr int kSegWarps = 4;   // scatter warps per 128-token segment (32 tokens each)

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
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int scratch[33];
  const int e = threadIdx.x;
  int c = 0;
  if (e < E)
    for (int s0 = 0; s0 < nseg; s0 += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (s0 + j < nseg) ? seg_counts[static_cast<size_t>(s0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) c += v[j];
    }
  int off = 0;
  const int total = block_exclusive_scan(e < E ? c : 0, scratch, &off);
  if (e < E) {
    counts[e] = c;
    offsets[e] = off;
    int run = off;
    for (int s0 = 0; s0 < nseg; s0 += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (s0 + j < nseg) ? seg_counts[static_cast<size_t>(s0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (s0 + j < nseg) {
          seg_counts[static_cast<size_t>(s0 + j) * E + e] = run;   // this segment's first position for expert e
          run += v[j];
        }
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
  // piece q starts at row floor(rows q / nch) = q base + floor(q rem / nch)
  // (rows = base nch + rem); q rem < nch^2 <= (T_max k / 128)^2 fits 32 bits
  const int base = nch > 0 ? rows / nch : 0, rem = nch > 0 ? rows % nch : 0;
  int r0 = 0;
  for (int q = 0; q < nch; ++q) {
    const int r1 = (q + 1) * base + ((q + 1) * rem) / nch;
    Chunk ch;
    ch.e = e; ch.row0 = base_row + r0; ch.rows = r1 - r0; ch.pad = 0;
    chunks[first + q] = ch;
    r0 = r1;
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

// One CTA per segment; warp w ranks the entries of the segment's tokens
// [32 w, 32 w + 32).  Each warp first counts its slice's experts, so warp w
// starts expert e at the segment's base plus the counts of slices 0..w-1;
// then it ranks its entries in order, 32 per round (at most k rounds).
__global__ void __launch_bounds__(32 * kSegWarps) scatter_kernel(
    const int32_t* __restrict__ topk_idx, int n, int seg_len, int E, const int32_t* __restrict__ seg_base,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ int sh_cnt[];   // [kSegWarps][E]: slice counts, then each slice's first positions
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = blockIdx.x;
  const int slice_len = seg_len / kSegWarps;
  const int b = seg * seg_len + warp * slice_len, end = min(b + slice_len, n);
  int* cnt = sh_cnt + warp * E;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  constexpr int kRounds = kRouteSegTokens * kMaxK / 32 / kSegWarps;   // 8 rounds of 32 entries at most
  int ex[kRounds];
#pragma unroll
  for (int j = 0; j < kRounds; ++j) {
    const int i = b + j * 32 + lane;
    const int e = (i < end) ? topk_idx[i] : -1;                     // every load issued before the first use
    ex[j] = (e >= 0 && e < E) ? e : -1;
  }
  __syncwarp();
#pragma unroll
  for (int j = 0; j < kRounds; ++j)
    if (ex[j] >= 0) atomicAdd(&cnt[ex[j]], 1);                       // counting is order-independent
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = seg_base[static_cast<size_t>(seg) * E + e];
    for (int w = 0; w < kSegWarps; ++w) {
      const int c = sh_cnt[w * E + e];
      sh_cnt[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kRounds; ++j) {
    if (b + j * 32 >= end) break;
    const int i = b + j * 32 + lane;
    const int e = ex[j];
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
// Passes 2 and 3 in one launch when the segments are few (T <= 64 * 128): CTA
// s recomputes, from the router's per-segment counts, every expert's total
// and the counts of the segments before s (nseg loads per thread, a few KB
// from L2), scans the totals into the offsets, and scatters its own segment
// as scatter_kernel does (8 warps of 16 tokens here).  CTA 0 also writes the
// counts, offsets, chunk list and active list exactly as scan_kernel does.
// One launch less, and no single-CTA pass on the critical path.
// ---------------------------------------------------------------------------
constexpr int kGroupThreads = 256;          // one routed expert per thread (E <= 256)
constexpr int kGroupWarps = kGroupThreads / 32;
constexpr int kGroupFuseSegs = 64;          // fused for up to 64 segments
constexpr int kGroupLoads = 16;             // segment counts per thread in flight together

__global__ void __launch_bounds__(kGroupThreads) group_fused_kernel(
    const int32_t* __restrict__ seg_counts, int nseg, int E, int T, int k, int chunk_rows,
    const int32_t* __restrict__ topk_idx, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    Chunk* __restrict__ chunks, int32_t* __restrict__ n_chunks, int32_t* __restrict__ active,
    int32_t* __restrict__ n_active, int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ int sh_cnt[];   // [kGroupWarps][E]: slice counts, then each slice's first positions
  __shared__ int scratch[33];
  __shared__ int seg_first[kMaxE];  // this segment's first position per expert
  const int e = threadIdx.x;
  const int seg = blockIdx.x;
  int c = 0, before = 0;
  if (e < E)
    for (int s0 = 0; s0 < nseg; s0 += kGroupLoads) {
      int v[kGroupLoads];
#pragma unroll
      for (int j = 0; j < kGroupLoads; ++j)
        v[j] = (s0 + j < nseg) ? seg_counts[static_cast<size_t>(s0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < kGroupLoads; ++j) {
        c += v[j];
        if (s0 + j < seg) before += v[j];
      }
    }
  int off = 0;
  const int total = block_exclusive_scan(e < E ? c : 0, scratch, &off);
  if (e < E) seg_first[e] = off + before;

  if (seg == 0) {
    // counts, offsets, chunk list (routed experts in order, then the shared
    // expert's rows T*k + t) and active list, as scan_kernel writes them
    if (e < E) {
      counts[e] = c;
      offsets[e] = off;
    }
    if (e == 0) offsets[E] = total;
    const int rows = e < E ? c : 0;
    const int nch = (rows + chunk_rows - 1) / chunk_rows;
    int first = 0;
    const int routed_chunks = block_exclusive_scan(nch, scratch, &first);
    {
      const int base = nch > 0 ? rows / nch : 0, rem = nch > 0 ? rows % nch : 0;
      int r0 = 0;
      for (int q = 0; q < nch; ++q) {
        const int r1 = (q + 1) * base + ((q + 1) * rem) / nch;
        Chunk ch;
        ch.e = e; ch.row0 = off + r0; ch.rows = r1 - r0; ch.pad = 0;
        chunks[first + q] = ch;
        r0 = r1;
      }
    }
    if (e == 0) {
      const int srows = T, snch = (T + chunk_rows - 1) / chunk_rows;
      const int base = srows / snch, rem = srows % snch;
      int r0 = 0;
      for (int q = 0; q < snch; ++q) {
        const int r1 = (q + 1) * base + ((q + 1) * rem) / snch;
        Chunk ch;
        ch.e = E; ch.row0 = T * k + r0; ch.rows = r1 - r0; ch.pad = 0;
        chunks[routed_chunks + q] = ch;
        r0 = r1;
      }
      *n_chunks = routed_chunks + snch;
    }
    int apos = 0;
    const int nact = block_exclusive_scan((e < E && c > 0) ? 1 : 0, scratch, &apos);
    if (e < E && c > 0) active[apos] = e;
    if (e == 0) {
      active[nact] = E;
      *n_active = nact + 1;
    }
  }

  // scatter this segment: warp w ranks the entries of tokens [16 w, 16 w + 16)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = T * k;
  const int seg_len = kRouteSegTokens * k;
  const int slice_len = seg_len / kGroupWarps;
  const int b = seg * seg_len + warp * slice_len, end = min(b + slice_len, n);
  int* cnt = sh_cnt + warp * E;
  for (int x = lane; x < E; x += 32) cnt[x] = 0;
  constexpr int kRounds = kRouteSegTokens * kMaxK / 32 / kGroupWarps;   // 4 rounds of 32 entries at most
  int ex[kRounds];
#pragma unroll
  for (int j = 0; j < kRounds; ++j) {
    const int i = b + j * 32 + lane;
    const int x = (i < end) ? topk_idx[i] : -1;
    ex[j] = (x >= 0 && x < E) ? x : -1;
  }
  __syncwarp();
#pragma unroll
  for (int j = 0; j < kRounds; ++j)
    if (ex[j] >= 0) atomicAdd(&cnt[ex[j]], 1);   // counting is order-independent
  __syncthreads();
  if (e < E) {
    int run = seg_first[e];
    for (int w = 0; w < kGroupWarps; ++w) {
      const int t = sh_cnt[w * E + e];
      sh_cnt[w * E + e] = run;
      run += t;
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kRounds; ++j) {
    if (b + j * 32 >= end) break;
    const int i = b + j * 32 + lane;
    const int x = ex[j];
    const unsigned peers = __match_any_sync(0xffffffffu, x);
    const int rank = __popc(peers & lanemask_lt());
    const int start = (x >= 0) ? cnt[x] : 0;
    __syncwarp();
    if (x >= 0) {
      const int pos = start + rank;
      perm[pos] = i;
      inv_perm[i] = pos;
      if ((peers >> lane) == 1u) cnt[x] = start + __popc(peers);   // highest lane of the group
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// Small-T routing (T <= 64): one launch does the router GEMV, top-k, shared
// gate and the whole counting sort.  CTA (b, y) scores the 16 rows e = 16b ..
// 16b + 15 of [W_r; w_sg] (row E: the shared-gate vector) for the 8 tokens of
// token group y on the tensor cores (mma.sync m16n8k16, bf16 operands, FP32
// accumulation); its 8 warps split K and add their partial tiles in shared
// memory in warp order.  The last CTA of a token group to finish (a counter
// per group in the workspace's control block) selects the experts of the
// group's tokens, one token per warp; the last group to finish (one more
// counter) sorts the T*k entries stably by expert and builds the
// active-expert list.  Each counter is reset by the CTA that saw it complete.
// ---------------------------------------------------------------------------
constexpr int kSmallWarps = 8;
constexpr int kSmallRows = 16;          // router rows per CTA (the MMA's M)
constexpr int kSmallLoads = 8;          // loads per thread in flight together
constexpr int kSmallKSteps = 8;         // 16-wide K steps whose loads are in flight together

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(256) router_small_kernel(
    const uint16_t* __restrict__ x, LayerPtr L, int T, int H, int E, int k,
    float* __restrict__ logits, unsigned* __restrict__ counter,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, float* __restrict__ sigma,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv_perm, int32_t* __restrict__ active, int32_t* __restrict__ n_active) {
  extern __shared__ uint4 smem_u4[];
  __shared__ int s_last;
  __shared__ int s_scan[33];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int E1 = E + 1;
  const int e0 = blockIdx.x * kSmallRows;
  const int t0 = blockIdx.y * kSmallTB;
  const int nt = min(kSmallTB, T - t0);

  // Lane (g, t) of the MMA holds rows e0 + g and e0 + g + 8 and token t0 + g.
  // Within each 16-wide K step the lane's logical K pairs (2t, 2t+1) and
  // (2t+8, 2t+9) are the four consecutive inputs 4t .. 4t+3 of the step, for
  // both operands, so each operand is one 8-byte load per step.
  auto row_of = [&](int e) -> const uint16_t* {
    return e < E ? L.w_router + static_cast<size_t>(e) * H : (e == E ? L.w_sg : nullptr);
  };
  const uint16_t* ra = row_of(e0 + g);
  const uint16_t* rb = row_of(e0 + g + 8);
  const uint16_t* xr = g < nt ? x + static_cast<size_t>(t0 + g) * H : nullptr;
  const int kw = H / kSmallWarps;              // inputs per warp (a multiple of 16)
  const int kbeg = warp * kw + 4 * t;
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  const uint2 z = make_uint2(0u, 0u);
  // The router rows do not depend on the previous kernel of the stream: the
  // first K steps' rows are requested before waiting for it (programmatic
  // dependent launch), x and every output after.
  uint2 a[kSmallKSteps], b[kSmallKSteps], xb[kSmallKSteps];
#pragma unroll
  for (int j = 0; j < kSmallKSteps; ++j) {
    const int kk = kbeg + 16 * j;
    const bool in = 16 * j < kw;
    a[j] = (in && ra) ? __ldg(reinterpret_cast<const uint2*>(ra + kk)) : z;
    b[j] = (in && rb) ? __ldg(reinterpret_cast<const uint2*>(rb + kk)) : z;
  }
  pdl_wait();
  pdl_launch_dependents();
  for (int ks0 = 0; ks0 < kw; ks0 += 16 * kSmallKSteps) {
    if (ks0 > 0) {
#pragma unroll
      for (int j = 0; j < kSmallKSteps; ++j) {
        const int kk = kbeg + ks0 + 16 * j;
        const bool in = ks0 + 16 * j < kw;
        a[j] = (in && ra) ? __ldg(reinterpret_cast<const uint2*>(ra + kk)) : z;
        b[j] = (in && rb) ? __ldg(reinterpret_cast<const uint2*>(rb + kk)) : z;
      }
    }
#pragma unroll
    for (int j = 0; j < kSmallKSteps; ++j) {
      const int kk = kbeg + ks0 + 16 * j;
      xb[j] = (ks0 + 16 * j < kw && xr) ? __ldg(reinterpret_cast<const uint2*>(xr + kk)) : z;
    }
#pragma unroll
    for (int j = 0; j < kSmallKSteps; ++j) mma_bf16_16816(d, a[j].x, b[j].x, a[j].y, b[j].y, xb[j].x, xb[j].y);
  }
  // partial tiles of the 8 K slices: part[warp][row][token], added in warp order
  float* part = reinterpret_cast<float*>(smem_u4);
  part[(warp * kSmallRows + g) * kSmallTB + 2 * t] = d[0];
  part[(warp * kSmallRows + g) * kSmallTB + 2 * t + 1] = d[1];
  part[(warp * kSmallRows + g + 8) * kSmallTB + 2 * t] = d[2];
  part[(warp * kSmallRows + g + 8) * kSmallTB + 2 * t + 1] = d[3];
  __syncthreads();
  if (threadIdx.x < kSmallRows * kSmallTB) {
    const int r = threadIdx.x / kSmallTB, c = threadIdx.x % kSmallTB;
    const int e = e0 + r;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kSmallWarps; ++w) sum += part[(w * kSmallRows + r) * kSmallTB + c];
    if (e <= E && c < nt) logits[static_cast<size_t>(t0 + c) * E1 + e] = sum + ((e < E && L.router_bias) ? L.router_bias[e] : 0.f);
  }

  // ---- the last CTA of this token group selects its tokens' experts ----
  unsigned* group_counter = counter + kSmallGroupCounter + blockIdx.y;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(group_counter, 1u) == gridDim.x - 1) ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x == 0) *group_counter = 0u;
  float* lg = reinterpret_cast<float*>(smem_u4);   // [8 tokens][E1], reuses the partial tiles
  for (int i0 = threadIdx.x; i0 < nt * E1; i0 += blockDim.x * kSmallLoads) {
    float v[kSmallLoads];
#pragma unroll
    for (int j = 0; j < kSmallLoads; ++j) {
      const int i = i0 + j * blockDim.x;
      v[j] = i < nt * E1 ? __ldcg(logits + static_cast<size_t>(t0) * E1 + i) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kSmallLoads; ++j)
      if (i0 + j * blockDim.x < nt * E1) lg[i0 + j * blockDim.x] = v[j];
  }
  __syncthreads();
  for (int r = warp; r < nt; r += kSmallWarps) {
    const int t = t0 + r;
    topk_redux(lg + r * E1, E, k, lane, topk_idx + t * k, topk_w + t * k);
    if (lane == 0) sigma[t] = sigmoid(lg[r * E1 + E]);
  }

  // ---- the last token group to finish groups the T*k entries ----
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(counter, 1u) == gridDim.y - 1) ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x == 0) *counter = 0u;

  // Stable counting sort of the n = T*k entries by expert.  Warp w owns the
  // entries [w*chunk, (w+1)*chunk): it counts them per expert (wcnt[w][e]),
  // one exclusive scan over the experts gives the offsets (and, packed in the
  // high half, the active-list positions), each expert's per-warp bases
  // follow in warp order, and every warp scatters its entries in order.
  int* wcnt = reinterpret_cast<int*>(smem_u4);       // [kSmallWarps][256]
  int* sel = wcnt + kSmallWarps * 256;               // [T*k] the selected experts
  const int n = T * k;
  const int chunk = (n + kSmallWarps - 1) / kSmallWarps;
  for (int i = threadIdx.x; i < kSmallWarps * 256; i += blockDim.x) wcnt[i] = 0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) sel[i] = __ldcg(topk_idx + i);
  __syncthreads();
  const int lo = warp * chunk, hi = min(n, lo + chunk);
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const int ex = i < hi ? sel[i] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, ex);
    if (ex >= 0 && (peers >> lane) == 1u) wcnt[warp * 256 + ex] += __popc(peers);   // one writer per expert
    __syncwarp();
  }
  __syncthreads();
  int c = 0;
  if (threadIdx.x < E)
    for (int w = 0; w < kSmallWarps; ++w) c += wcnt[w * 256 + threadIdx.x];
  int excl = 0;   // low 16 bits: entries before this expert; high 16 bits: active experts before it
  const int tot = block_exclusive_scan(c + ((c > 0) << 16), s_scan, &excl);
  const int off = excl & 0xFFFF, apos = excl >> 16, nact = tot >> 16;
  if (threadIdx.x < E) {
    counts[threadIdx.x] = c;
    offsets[threadIdx.x] = off;
    if (c > 0) active[apos] = threadIdx.x;
    int run = off;
    for (int w = 0; w < kSmallWarps; ++w) {
      const int t = wcnt[w * 256 + threadIdx.x];
      wcnt[w * 256 + threadIdx.x] = run;
      run += t;
    }
  }
  if (threadIdx.x == 0) {
    offsets[E] = tot & 0xFFFF;
    active[nact] = E;
    *n_active = nact + 1;
  }
  __syncthreads();
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const int ex = i < hi ? sel[i] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, ex);
    const int rank = __popc(peers & lanemask_lt());
    const int start = ex >= 0 ? wcnt[warp * 256 + ex] : 0;
    __syncwarp();
    if (ex >= 0) {
      perm[start + rank] = i;
      inv_perm[i] = start + rank;
      if ((peers >> lane) == 1u) wcnt[warp * 256 + ex] = start + __popc(peers);
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
int num_segments(int T) { return (T + kRouteSegTokens - 1) / kRouteSegTokens; }

cudaError_t launch_route_small(const uint16_t* x, const LayerPtr& L, int T, int H, int I, int Is, int E, int k,
                               float* logits, unsigned* counter, const RoutingPtrs& r, int32_t* active,
                               int32_t* n_active, cudaStream_t s) {
  (void)I;
  (void)Is;
  // one token group (one counter) per 8 tokens
  if (T > kSmallTB * kSmallMaxGroups || H % (16 * kSmallWarps)) return cudaErrorInvalidValue;
  const dim3 grid((E + 1 + kSmallRows - 1) / kSmallRows, (T + kSmallTB - 1) / kSmallTB);
  const int smem = max(kSmallWarps * kSmallRows * kSmallTB * 4, max(kSmallTB * (E + 1) * 4, (kSmallWarps * 256 + T * k) * 4));
  const cudaError_t e = ensure_smem(reinterpret_cast<const void*>(router_small_kernel), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(router_small_kernel, grid, dim3(256), smem, s, x, L, T, H, E, k, logits, counter, r.topk_idx,
                    r.topk_w, r.sigma, r.counts, r.offsets, r.perm, r.inv_perm, active, n_active);
}

cudaError_t launch_group(const int32_t* topk_idx, int T, int k, int E, int chunk_rows,
                         int32_t* seg_scratch, int32_t* counts, int32_t* offsets,
                         int32_t* perm, int32_t* inv_perm, Chunk* chunks, int32_t* n_chunks,
                         int32_t* active, int32_t* n_active, cudaStream_t s) {
  const int n = T * k;
  const int nseg = num_segments(T);
  if (nseg <= kGroupFuseSegs && E <= kGroupThreads) {
    const int fsmem = kGroupWarps * E * static_cast<int>(sizeof(int));
    return launch_pdl(group_fused_kernel, dim3(nseg), dim3(kGroupThreads), static_cast<size_t>(fsmem), s,
                      static_cast<const int32_t*>(seg_scratch), nseg, E, T, k, chunk_rows, topk_idx, counts, offsets,
                      chunks, n_chunks, active, n_active, perm, inv_perm);
  }
  const int grid = nseg;
  const int smem = kSegWarps * E * static_cast<int>(sizeof(int));
  cudaError_t e = launch_pdl(scan_kernel, dim3(1), dim3(kScanThreads), 0, s, seg_scratch, nseg, E, T, k, chunk_rows,
                             counts, offsets, chunks, n_chunks, active, n_active);
  if (e != cudaSuccess) return e;
  return launch_pdl(scatter_kernel, dim3(grid), dim3(32 * kSegWarps), static_cast<size_t>(smem), s, topk_idx, n,
                    kRouteSegTokens * k, E, static_cast<const int32_t*>(seg_scratch), perm, inv_perm);
}

}  // namespace moe
