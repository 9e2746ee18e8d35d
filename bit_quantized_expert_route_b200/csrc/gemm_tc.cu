// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a)
// with the affine 4-bit weights rebuilt tile by tile in shared memory.
//
// The write-ups this layer follows ("Perplexity's Lily: ...", sections "The
// Model" and "How It Works: Prefill and Decode Strategies") reconstruct the
// 4-bit weights one tile at a time inside the grouped expert GEMM, multiply in
// bf16 and accumulate in FP32, never writing dense weights to memory.  Here a
// tile is 128 weight rows x 64 inputs (exactly one quantisation group), the
// FP32 accumulators live in tensor memory, and the expert's tokens form the
// MMA's N dimension ("weights as M, tokens as N"), so a small expert group
// wastes little work.
//
// One persistent CTA per SM walks the device-built unit list:
//   unit = (chunk of <= 128 rows of one expert) x (block of 128 weight rows)
// Warp roles (288 threads):
//   warps 0-3  dequantise the packed tile of each stage into bf16 (128-byte
//              swizzled K-major layout) and, after a unit's last stage, run
//              the epilogue from tensor memory (lane quadrant = warp index);
//   warps 4-7  loaders: cp.async gathers of the unit's token rows (B operand),
//              the packed 4-bit words and the group scales / biases;
//   warp 8     allocates tensor memory; one lane issues tcgen05.mma.
// kGateUp = true: A = {W_gate, W_up} rows, two accumulators, epilogue
//   h = bf16(silu(g) * u).  kGateUp = false: A = W_down rows, one
//   accumulator, epilogue Y = acc (FP32).
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int BM = 128;    // weight rows per tile (MMA M)
constexpr int BN = 128;    // rows (tokens) per chunk: MMA N <= 128
constexpr int BK = 64;     // inputs per stage: one quantisation group, one 128-B swizzle row
constexpr int kThreads = 288;
constexpr int kMmaWarp = 8;
constexpr uint32_t kTmemCols = 256;

template <bool kGateUp>
struct Cfg {
  static constexpr int NA = kGateUp ? 2 : 1;              // weight matrices per stage
  static constexpr int STAGES = kGateUp ? 3 : 4;
  static constexpr int LAG = STAGES - 1;                   // loader cp.async groups in flight
  static constexpr int A_BYTES = BM * BK * 2;              // 16 KB bf16 tile
  static constexpr int B_BYTES = BN * BK * 2;              // 16 KB bf16 tile
  static constexpr int P_BYTES = BM * BK / 2;              // 4 KB packed words
  static constexpr int S_BYTES = BM * 4;                   // 2 groups of scale (or bias) per row
  static constexpr int STAGE_BYTES = NA * (A_BYTES + P_BYTES + 2 * S_BYTES) + B_BYTES;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;        // barriers + alignment slack
  // offsets inside a stage
  static constexpr int OFF_A = 0;                          // NA x A_BYTES
  static constexpr int OFF_B = NA * A_BYTES;
  static constexpr int OFF_P = OFF_B + B_BYTES;            // NA x P_BYTES
  static constexpr int OFF_S = OFF_P + NA * P_BYTES;       // NA x (scales, biases)
};

struct TcArgs {
  Geometry g;
  QMatPtr W0, W1;          // routed stacks: {gate, up} or {down, -}
  QMatPtr S0, S1;          // shared expert: {sh_gate, sh_up} or {sh_down, -}
  const uint16_t* x;       // gate/up: token rows [T, H]
  const int32_t* perm;
  const uint16_t* h;       // down: routed rows [T*k, I]
  const uint16_t* h_s;     // down: shared rows [T, Is]
  uint16_t* h_out;         // gate/up output, routed [T*k, I]
  uint16_t* hs_out;        // gate/up output, shared [T, Is]
  float* Y;                // down output [(T*k + T), H]
  const Chunk* chunks;
  const int32_t* n_chunks;
  int* status;
};

struct UnitInfo {
  bool skip;
  bool shared;
  int e, row0, rows, f0, K, nks;
};

template <bool kGateUp>
__device__ __forceinline__ UnitInfo unit_info(const TcArgs& a, int u, int nfb) {
  const Chunk ch = a.chunks[u / nfb];
  UnitInfo ui;
  ui.shared = ch.e >= a.g.E;
  ui.e = ch.e;
  ui.row0 = ch.row0;
  ui.rows = ch.rows;
  ui.f0 = (u % nfb) * BM;
  const int Ie = ui.shared ? a.g.Is : a.g.I;
  const int R = kGateUp ? Ie : a.g.H;          // weight rows of this expert's matrix
  ui.skip = ui.f0 >= R || ui.rows <= 0;
  ui.K = kGateUp ? a.g.H : Ie;
  ui.nks = ui.K / BK;
  return ui;
}

// Row pointer bases (packed words, scales, biases) of weight row `row` of
// matrix m of the unit.
struct RowPtr {
  const uint32_t* q;
  const uint16_t* s;
  const uint16_t* b;
};

template <bool kGateUp>
__device__ __forceinline__ RowPtr weight_row(const TcArgs& a, const UnitInfo& ui, int m, int row) {
  const QMatPtr& W = ui.shared ? (m == 0 ? a.S0 : a.S1) : (m == 0 ? a.W0 : a.W1);
  const int Ie = ui.shared ? a.g.Is : a.g.I;
  const size_t rows_per_expert = kGateUp ? static_cast<size_t>(a.g.I) : static_cast<size_t>(a.g.H);
  const size_t r = (ui.shared ? 0 : static_cast<size_t>(ui.e) * rows_per_expert) + row;
  (void)Ie;
  return RowPtr{W.q + r * (ui.K / 8), W.s + r * (ui.K / kGroup), W.b + r * (ui.K / kGroup)};
}

template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_tc_kernel(const TcArgs a) {
  using C = Cfg<kGateUp>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-B aligned base (the swizzle atoms must start on 1024 B)
  const uint32_t raw_u32 = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  const uint32_t sbase = tc::smem_u32(smem);

  uint64_t* full_ld = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);   // [STAGES]
  uint64_t* full_a = full_ld + C::STAGES;                                 // [STAGES]
  uint64_t* empty = full_a + C::STAGES;                                   // [STAGES]
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      tc::mbar_init(&full_ld[s], 128);
      tc::mbar_init(&full_a[s], 128);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(acc_full, 1);
    tc::mbar_init(acc_empty, 128);
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc(tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int nfb = (kGateUp ? max(a.g.I, a.g.Is) : a.g.H) / BM;
  const int n_units = *a.n_chunks * nfb;
  const int Tk = a.g.T * a.g.k;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ loaders
    const int r = threadIdx.x - 128;         // tile row owned by this thread
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const UnitInfo ui = unit_info<kGateUp>(a, u, nfb);
      if (ui.skip) continue;
      // B row source
      const uint16_t* brow = nullptr;
      if (r < ui.rows) {
        const int R = ui.row0 + r;
        if (kGateUp) {
          const int tok = ui.shared ? (R - Tk) : (a.perm[R] / a.g.k);
          brow = a.x + static_cast<size_t>(tok) * a.g.H;
        } else {
          brow = ui.shared ? a.h_s + static_cast<size_t>(R - Tk) * a.g.Is : a.h + static_cast<size_t>(R) * a.g.I;
        }
      }
      RowPtr wr[2];
#pragma unroll
      for (int m = 0; m < C::NA; ++m) wr[m] = weight_row<kGateUp>(a, ui, m, ui.f0 + r);
      for (int ks = 0; ks < ui.nks; ++ks, ++it) {
        const int s = it % C::STAGES;
        if (!tc::mbar_wait(&empty[s], ((it / C::STAGES) & 1u) ^ 1u, abort_flag, a.status)) {
          ok = false;
          break;
        }
        const uint32_t st = sbase + s * C::STAGE_BYTES;
        if (brow) {
          const uint32_t dst = st + C::OFF_B + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) tc::cp_async16(dst + ((c ^ (r & 7)) << 4), brow + ks * BK + c * 8);
        }
#pragma unroll
        for (int m = 0; m < C::NA; ++m) {
          const uint32_t pd = st + C::OFF_P + m * C::P_BYTES + r * 32;
          tc::cp_async16(pd, wr[m].q + ks * 8);
          tc::cp_async16(pd + 16, wr[m].q + ks * 8 + 4);
          const uint32_t sd = st + C::OFF_S + m * 2 * C::S_BYTES + r * 4;
          const int gpair = ks & ~1;
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sd), "l"(wr[m].s + gpair) : "memory");
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sd + C::S_BYTES), "l"(wr[m].b + gpair)
                       : "memory");
        }
        tc::cp_async_commit();
        if (it >= static_cast<uint32_t>(C::LAG)) {
          tc::cp_async_wait<C::LAG>();
          tc::fence_proxy_async_smem();
          tc::mbar_arrive(&full_ld[(it - C::LAG) % C::STAGES]);
        }
      }
    }
    tc::cp_async_wait_all();
    tc::fence_proxy_async_smem();
    if (ok) {
      const uint32_t first = it > static_cast<uint32_t>(C::LAG) ? it - C::LAG : 0u;
      for (uint32_t j = first; j < it; ++j) tc::mbar_arrive(&full_ld[j % C::STAGES]);
    }
  } else if (warp < 4) {
    // ------------------------------------------------- dequant + epilogue
    const int r = threadIdx.x;               // tile row == TMEM lane
    uint32_t it = 0, tt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const UnitInfo ui = unit_info<kGateUp>(a, u, nfb);
      if (ui.skip) continue;
      for (int ks = 0; ks < ui.nks; ++ks, ++it) {
        const int s = it % C::STAGES;
        if (!tc::mbar_wait(&full_ld[s], (it / C::STAGES) & 1u, abort_flag, a.status)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * C::STAGE_BYTES;
#pragma unroll
        for (int m = 0; m < C::NA; ++m) {
          const uint4* pk = reinterpret_cast<const uint4*>(st + C::OFF_P + m * C::P_BYTES + r * 32);
          const uint4 w0 = pk[0], w1 = pk[1];
          const uint16_t* sb = reinterpret_cast<const uint16_t*>(st + C::OFF_S + m * 2 * C::S_BYTES + r * 4);
          const uint16_t sv = sb[ks & 1];
          const uint16_t bv = sb[C::S_BYTES / 2 + (ks & 1)];
          __nv_bfloat162 s2, b2;
          *reinterpret_cast<uint32_t*>(&s2) = static_cast<uint32_t>(sv) | (static_cast<uint32_t>(sv) << 16);
          *reinterpret_cast<uint32_t*>(&b2) = static_cast<uint32_t>(bv) | (static_cast<uint32_t>(bv) << 16);
          const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          uint8_t* arow = st + C::OFF_A + m * C::A_BYTES + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(arow + ((c ^ (r & 7)) << 4)) = tc::dequant8(words[c], s2, b2);
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(&full_a[s]);
      }
      if (!ok) break;
      // epilogue: accumulators of this unit
      if (!tc::mbar_wait(acc_full, tt & 1u, abort_flag, a.status)) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
      const int feat = ui.f0 + r;
      for (int n0 = 0; n0 < ui.rows; n0 += 16) {
        float v0[16];
        tc::tmem_ld16(lane_base + n0, v0);
        if (kGateUp) {
          float v1[16];
          tc::tmem_ld16(lane_base + BN + n0, v1);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = n0 + j;
            if (n < ui.rows) {
              const int R = ui.row0 + n;
              uint16_t* dst = ui.shared ? a.hs_out + static_cast<size_t>(R - Tk) * a.g.Is
                                        : a.h_out + static_cast<size_t>(R) * a.g.I;
              dst[feat] = float_to_bf16_bits(silu(v0[j]) * v1[j]);
            }
          }
        } else {
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = n0 + j;
            if (n < ui.rows) a.Y[static_cast<size_t>(ui.row0 + n) * a.g.H + feat] = v0[j];
          }
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(acc_empty);
      ++tt;
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t it = 0, tt = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const UnitInfo ui = unit_info<kGateUp>(a, u, nfb);
        if (ui.skip) continue;
        const int n_mma = max(16, (ui.rows + 15) & ~15);
        const uint32_t idesc = tc::idesc_bf16(BM, n_mma);
        if (!tc::mbar_wait(acc_empty, (tt & 1u) ^ 1u, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        for (int ks = 0; ks < ui.nks; ++ks, ++it) {
          const int s = it % C::STAGES;
          const uint32_t par = (it / C::STAGES) & 1u;
          if (!tc::mbar_wait(&full_ld[s], par, abort_flag, a.status) ||
              !tc::mbar_wait(&full_a[s], par, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t st = sbase + s * C::STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bdesc = tc::sdesc_sw128(st + C::OFF_B + kk * 32);
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
#pragma unroll
            for (int m = 0; m < C::NA; ++m) {
              const uint64_t adesc = tc::sdesc_sw128(st + C::OFF_A + m * C::A_BYTES + kk * 32);
              tc::mma_bf16_ss(tmem + m * BN, adesc, bdesc, idesc, acc);
            }
          }
          tc::mma_commit(&empty[s]);
        }
        if (!ok) break;
        tc::mma_commit(acc_full);
        ++tt;
      }
      // every issued MMA has finished before tensor memory is released
      tc::mma_commit(drain);
      tc::mbar_wait_drain(drain, 0, a.status);
    }
    __syncwarp();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == kMmaWarp) tc::tmem_dealloc(tmem, kTmemCols);
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

}  // namespace

int gemm_chunk_rows() { return BN; }

cudaError_t launch_gateup(const Geometry& g, const LayerPtr& L, const uint16_t* x, const int32_t* perm,
                          const Chunk* chunks, const int32_t* n_chunks, int max_chunks,
                          uint16_t* h, uint16_t* h_s, int* status, cudaStream_t s) {
  TcArgs a{};
  a.g = g;
  a.W0 = L.gate;
  a.W1 = L.up;
  a.S0 = L.sh_gate;
  a.S1 = L.sh_up;
  a.x = x;
  a.perm = perm;
  a.h_out = h;
  a.hs_out = h_s;
  a.chunks = chunks;
  a.n_chunks = n_chunks;
  a.status = status;
  using C = Cfg<true>;
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM);
  if (e != cudaSuccess) return e;
  const int nfb = max(g.I, g.Is) / BM;
  const int grid = max(1, min(max_chunks * nfb, num_sms()));
  grouped_gemm_tc_kernel<true><<<grid, kThreads, C::SMEM, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_down(const Geometry& g, const LayerPtr& L, const uint16_t* h, const uint16_t* h_s,
                        const Chunk* chunks, const int32_t* n_chunks, int max_chunks,
                        float* Y, int* status, cudaStream_t s) {
  TcArgs a{};
  a.g = g;
  a.W0 = L.down;
  a.W1 = L.down;
  a.S0 = L.sh_down;
  a.S1 = L.sh_down;
  a.h = h;
  a.h_s = h_s;
  a.Y = Y;
  a.chunks = chunks;
  a.n_chunks = n_chunks;
  a.status = status;
  using C = Cfg<false>;
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM);
  if (e != cudaSuccess) return e;
  const int nfb = g.H / BM;
  const int grid = max(1, min(max_chunks * nfb, num_sms()));
  grouped_gemm_tc_kernel<false><<<grid, kThreads, C::SMEM, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
