// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a)
// with the affine 4-bit weights rebuilt tile by tile on chip.
//
// The write-ups this layer follows ("Perplexity's Lily: ...", sections "The
// Model" and "How It Works: Prefill and Decode Strategies") reconstruct the
// 4-bit weights one tile at a time inside the grouped expert GEMM, multiply in
// bf16 and accumulate in FP32, never writing dense weights to memory.  Here:
//
// * A tile is 128 weight rows x 64 inputs (exactly one quantisation group).
//   The packed words of each tile (128 rows x 32 B) arrive by TMA into a deep
//   shared-memory ring, the group scales / biases 8 groups at a time; dequant
//   warps rebuild bf16(scale * q + bias) and store the tile into tensor
//   memory, where the MMA reads it as its A operand.  The dense tile never
//   touches shared memory.
// * The expert's tokens are the MMA's N dimension (16..160 per chunk), staged
//   in shared memory in the 128-byte swizzled K-major layout by one 2-D TMA
//   per stage: the chunk's rows are contiguous (gate/up: a gather pass has
//   written x's rows in grouped order; down: h is produced in that order).
// * Inside every group of 8 inputs the K order of both operands is
//   (0,4,1,5,2,6,3,7): the order in which one AND-OR pulls code pairs out of
//   a packed word.  The gather pass writes x in that order and the gate/up
//   epilogue writes h in it, so the dequantiser needs no byte permutes.  A
//   dot product does not depend on the order of its terms.
// * FP32 accumulators live in tensor memory.  Epilogue warps read them, apply
//   the epilogue (gate/up: h = bf16(silu(g) * u); down: Y = bf16(acc)), stage
//   the tile in shared memory, release the accumulator, and only then write
//   the tile out with coalesced 16-byte stores, overlapping the next unit.
//
// One persistent CTA per SM walks the device-built unit list
//   unit = (chunk of <= 160 rows of one expert) x (block of 128 weight rows).
// Warp roles (864 threads):
//   warps 0-15  dequantisers in 4 sets of 4 (gate/up: set = stage parity x
//               matrix; down: set = stage mod 4); TMEM lane quadrant =
//               warp % 4 = row / 32
//   warps 16-23 epilogue, two per lane quadrant (warp % 4), taking alternate
//               16-column blocks of the accumulators
//   warp 24     token tiles: one lane issues a 2-D TMA per stage
//   warp 25     one lane issues the TMA loads of packed tiles and scales
//   warp 26     tensor-memory allocation; one lane issues tcgen05.mma
// Tensor memory (512 columns): gate/up = one accumulator pair (gate, up:
// 2 x 160 columns) + 3 A stages of 64 columns; down with two weight blocks
// per unit = two accumulators of 160 columns + 3 A stages of 64 columns;
// down with one block = a double-buffered 160-column accumulator + 6 A
// stages of 32 columns.
//
// Why chunks of up to 160 rows: a unit costs about the same whatever its N
// (the per-stage hand-offs between the roles, not the MMAs, set its length),
// so the number of units sets the kernel time.  With 128-row chunks an
// expert that receives a few more than 128 tokens (about half of them with
// uniform routing at T = 4096) paid for a second, nearly empty unit; 160 is
// the most tensor memory allows while keeping three A stages beside the
// gate/up accumulators.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int BM = 128;          // weight rows per tile = TMEM lanes (MMA M)
constexpr int BN = 160;          // rows (tokens) per chunk: MMA N <= 160
constexpr int BK = 64;           // inputs per stage: one quantisation group
constexpr int kBStagesMax = 5;   // token-tile ring
constexpr int kPStagesMax = 7;   // packed-tile ring
constexpr int kSBlock = 8;       // quantisation groups per scale block (16 B per row)
constexpr int kDqWarps = 16;     // dequantiser warps (4 sets of 4: one per TMEM lane quadrant)
constexpr int kEpiWarp0 = kDqWarps;
constexpr int kEpiWarps = 8;      // two per TMEM lane quadrant, alternate 16-column blocks
constexpr int kLoadWarp = kEpiWarp0 + kEpiWarps;   // token tiles
constexpr int kTmaWarp = kLoadWarp + 1;
constexpr int kMmaWarp = kTmaWarp + 1;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxCtaUnits = 256;   // chunk descriptors cached in shared memory per CTA
// token-tile box heights: a chunk loads the smallest box that covers its rows
constexpr int kTokenBoxes = 5;
__device__ __host__ constexpr int token_box(int i) { return i == 4 ? BN : 16 << i; }

// kNA: 128-row weight tiles per stage.  gate/up: 2 (the gate and up
// matrices, same rows); down: 2 (two consecutive 128-row blocks of the same
// matrix, which share every token tile: half the token-tile traffic per
// FLOP) or 1 (H not a multiple of 256).
template <bool kGateUp, int kNA>
struct Cfg {
  static constexpr int NA = kNA;                              // weight tiles per stage
  static constexpr int ACC_COLS = NA * BN;                    // one accumulator set
  static constexpr int ACC_BUFS = kNA == 2 ? 1 : 2;
  static constexpr int A_COLS = NA * BK / 2;                  // TMEM columns per A stage
  static constexpr int A_BASE = ACC_BUFS * ACC_COLS;
  static constexpr int A_STAGES = (static_cast<int>(kTmemCols) - A_BASE) / A_COLS;
  static constexpr int B_BYTES = BN * BK * 2;                 // 20 KB swizzled token tile
  static constexpr int P_BYTES = BM * 32;                     // 4 KB packed tile of one matrix
  static constexpr int S_BYTES = BM * kSBlock * 2;            // 2 KB: 8 groups of scales (or biases)
  static constexpr int S_SLOT = NA * 2 * S_BYTES;             // scales + biases of every matrix
  // Down with two blocks stages both output tiles at once, so the single
  // accumulator goes back to the MMA as soon as it is drained; the rings
  // give up one token stage and two packed stages to make room.
  static constexpr bool STAGE_ALL = !kGateUp && kNA == 2;
  static constexpr int OUT_TILES = STAGE_ALL ? kNA : 1;
  static constexpr int BST = STAGE_ALL ? kBStagesMax - 1 : kBStagesMax;
  static constexpr int PST = STAGE_ALL ? kPStagesMax - 2 : kPStagesMax;
  static constexpr int OUT_BYTES = OUT_TILES * BN * BM * 2;   // epilogue staging tiles (bf16)
  static constexpr int OFF_B = 0;
  static constexpr int OFF_P = OFF_B + BST * B_BYTES;
  static constexpr int OFF_S = OFF_P + PST * NA * P_BYTES;
  static constexpr int OFF_OUT = OFF_S + 2 * S_SLOT;
  static constexpr int BAR_OFF = OFF_OUT + OUT_BYTES;
  static constexpr int OFF_UNITS = BAR_OFF + 512;             // this CTA's chunk descriptors
  static constexpr int SMEM = OFF_UNITS + kMaxCtaUnits * 16 + 1024;   // + alignment slack
  static_assert(SMEM <= 227 * 1024, "dynamic shared memory of one CTA");
  static constexpr int DQ_PER_STAGE = kNA * 128;             // dequant threads consuming one stage
};

struct alignas(64) TcArgs {
  CUtensorMap tm_q[2][2];  // packed words: [routed, shared][matrix]
  CUtensorMap tm_s[2][2];  // scales:       [routed, shared][matrix] (valid when scales_tma)
  CUtensorMap tm_b[2][2];  // biases
  // token tiles: [gate/up: grouped x rows, - | down: routed h, shared h] x
  // box height [16, 32, 64, 128, 160 rows]: a chunk loads the smallest box that
  // covers its rows (a 3-row expert group needs 2 KB per stage, not 16 KB)
  CUtensorMap tm_h[2][kTokenBoxes];
  Geometry g;
  QMatPtr W0, W1;          // routed stacks: {gate, up} or {down, -}
  QMatPtr S0, S1;          // shared expert: {sh_gate, sh_up} or {sh_down, -}
  uint16_t* h_out;         // gate/up output, routed [T*k, I]
  uint16_t* hs_out;        // gate/up output, shared [T, Is]
  uint16_t* Y;             // down output, bf16 [(T*k + T), H]
  const Chunk* chunks;
  const int32_t* n_chunks;
  int* status;
  int scales_tma;          // scale rows are 16-B strided (K % 512 == 0): scales arrive by TMA
  long long wait_limit;    // cycles before a bounded wait gives up
};

struct UnitInfo {
  bool skip;
  bool shared;
  int e, row0, rows, f0, K, nks, wrow;   // wrow: first weight row of the tile in its matrix stack
};

template <bool kGateUp, int kNA>
__device__ __forceinline__ UnitInfo unit_info(const TcArgs& a, int u, int nfb, const Chunk* cache) {
  // this CTA's units are u = blockIdx.x + i * gridDim.x; their chunks were
  // copied to shared memory at the start, so the per-stage bookkeeping of
  // every role never waits on a global load
  const int i = (u - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x);
  const Chunk ch = i < kMaxCtaUnits ? cache[i] : a.chunks[u / nfb];
  UnitInfo ui;
  ui.shared = ch.e >= a.g.E;
  ui.e = ch.e;
  ui.row0 = ch.row0;
  ui.rows = ch.rows;
  ui.f0 = (u % nfb) * BM * (kGateUp ? 1 : kNA);   // first weight row (down: of the unit's kNA blocks)
  const int Ie = ui.shared ? a.g.Is : a.g.I;
  const int R = kGateUp ? Ie : a.g.H;          // weight rows of this expert's matrix
  ui.skip = ui.f0 >= R || ui.rows <= 0;
  ui.K = kGateUp ? a.g.H : Ie;
  ui.nks = ui.K / BK;
  ui.wrow = (ui.shared ? 0 : ui.e * (kGateUp ? a.g.I : a.g.H)) + ui.f0;
  return ui;
}

// Walks this CTA's stages in order: (unit, k-step) with global stage and
// scale-block counts (a scale block starts at every k-step multiple of 8).
template <bool kGateUp, int kNA>
struct StageCursor {
  int u, ks;
  uint32_t it, blk;
  bool done;
  UnitInfo ui;

  const Chunk* cache;
  __device__ __forceinline__ void seek_unit(const TcArgs& a, int from, int n_units, int nfb) {
    for (u = from; u < n_units; u += gridDim.x) {
      ui = unit_info<kGateUp, kNA>(a, u, nfb, cache);
      if (!ui.skip) {
        ks = 0;
        done = false;
        return;
      }
    }
    done = true;
  }
  __device__ __forceinline__ void begin(const TcArgs& a, int n_units, int nfb, const Chunk* units) {
    cache = units;
    it = 0;
    blk = 0;
    seek_unit(a, blockIdx.x, n_units, nfb);
  }
  __device__ __forceinline__ void next(const TcArgs& a, int n_units, int nfb) {
    ++it;
    if (++ks == ui.nks) seek_unit(a, u + gridDim.x, n_units, nfb);
    if (!done && ks % kSBlock == 0) ++blk;
  }
};

template <bool kGateUp, int kNA>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_tc_kernel(const __grid_constant__ TcArgs a) {
  using C = Cfg<kGateUp, kNA>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);   // 1024-B aligned swizzle atoms
  const uint32_t sbase = tc::smem_u32(smem);

  uint64_t* full_b = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);   // [C::BST]
  uint64_t* empty_b = full_b + C::BST;                                // [C::BST]
  uint64_t* full_p = empty_b + C::BST;                                // [C::PST]
  uint64_t* empty_p = full_p + C::PST;                                // [C::PST]
  uint64_t* full_s = empty_p + C::PST;                                // [2]
  uint64_t* empty_s = full_s + 2;                                       // [2]
  uint64_t* full_a = empty_s + 2;                                       // [A_STAGES]
  uint64_t* empty_a = full_a + C::A_STAGES;                             // [A_STAGES]
  uint64_t* acc_full = empty_a + C::A_STAGES;                           // [ACC_BUFS]
  uint64_t* acc_empty = acc_full + C::ACC_BUFS;                         // [ACC_BUFS]
  uint64_t* drain = acc_empty + C::ACC_BUFS;
  uint64_t* epi_sync = drain + 1;                                       // [2] staging written / copied out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_sync + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::BST; ++s) {
      tc::mbar_init(&full_b[s], 1);
      tc::mbar_init(&empty_b[s], 1);
    }
    for (int s = 0; s < C::PST; ++s) {
      tc::mbar_init(&full_p[s], 1);
      tc::mbar_init(&empty_p[s], C::DQ_PER_STAGE);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&full_s[s], 1);
      tc::mbar_init(&empty_s[s], kDqWarps * 32);   // every dequantiser releases every block once
    }
    for (int s = 0; s < C::A_STAGES; ++s) {
      tc::mbar_init(&full_a[s], C::DQ_PER_STAGE);
      tc::mbar_init(&empty_a[s], 1);
    }
    for (int b = 0; b < C::ACC_BUFS; ++b) {
      tc::mbar_init(&acc_full[b], 1);
      tc::mbar_init(&acc_empty[b], kEpiWarps * 32);
    }
    tc::mbar_init(drain, 1);
    tc::mbar_init(&epi_sync[0], kEpiWarps * 32);
    tc::mbar_init(&epi_sync[1], kEpiWarps * 32);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  // the barrier set-up above touched only shared memory
  pdl_wait();
  pdl_launch_dependents();
  // an error recorded in the status word (a bounded wait of this call's
  // router, or of an earlier call, gave up) means the chunk list may not
  // describe this call's tokens: do nothing (uniform over the CTA)
  if (*reinterpret_cast<volatile const int*>(a.status) != 0) return;
  const int nfb = (kGateUp ? max(a.g.I, a.g.Is) / BM : a.g.H / (BM * kNA));
  const int n_units = *a.n_chunks * nfb;
  const int Tk = a.g.T * a.g.k;
  Chunk* units = reinterpret_cast<Chunk*>(smem + C::OFF_UNITS);
  for (int i = threadIdx.x; i < kMaxCtaUnits; i += blockDim.x) {
    const int u = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    if (u < n_units) units[i] = a.chunks[u / nfb];
  }
  if (warp == kMmaWarp) tc::tmem_alloc(tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < kEpiWarp0) {
    // ------------------------------------------------------- dequantisers
    const int r = threadIdx.x & 127;                 // weight row of the tile == TMEM lane
    // 4 sets of 4 warps.  gate/up: set = (stage parity, matrix); down: set =
    // stage index mod 4.  Each stage is rebuilt by 128 threads per matrix, and
    // a warp works on every second (gate/up) or fourth (down) stage, so the
    // latency of one stage's loads, dequantisation and TMEM store overlaps the
    // other sets' work.
    const int set = warp >> 2;
    const int m = kNA == 2 ? (set & 1) : 0;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int psw = (r >> 2) & 1;                    // 32-byte swizzle of the packed tile rows
    auto mine = [&](uint32_t it) {
      return kNA == 2 ? static_cast<int>(it & 1u) == (set >> 1) : static_cast<int>(it & 3u) == set;
    };
    StageCursor<kGateUp, kNA> cur;
    cur.begin(a, n_units, nfb, units);
    while (!cur.done && !mine(cur.it)) cur.next(a, n_units, nfb);
    bool ok = true;
    uint32_t held_blk = 0xffffffffu;                 // scale block this thread still holds
    while (!cur.done && ok) {
      const uint32_t it = cur.it;
      const int ks = cur.ks;
      // scales of this stage: from the TMA'd block, or straight from global
      uint32_t sv, bv;
      if (a.scales_tma) {
        if (cur.blk != held_blk) {
          if (held_blk != 0xffffffffu) {
            tc::fence_proxy_async_smem();            // generic reads of the block before its TMA refill
            tc::mbar_arrive(&empty_s[held_blk & 1u]);
          }
          held_blk = cur.blk;
          if (!tc::mbar_wait(&full_s[held_blk & 1u], (held_blk >> 1) & 1u, abort_flag, a.status, a.wait_limit)) {
            ok = false;
            break;
          }
        }
        const uint16_t* sb = reinterpret_cast<const uint16_t*>(smem + C::OFF_S + (held_blk & 1u) * C::S_SLOT +
                                                               m * 2 * C::S_BYTES + r * 16);
        sv = sb[ks % kSBlock];
        bv = sb[C::S_BYTES / 2 + ks % kSBlock];
      } else {
        const QMatPtr& W = cur.ui.shared ? (m == 0 ? a.S0 : a.S1) : (m == 0 ? a.W0 : a.W1);
        const size_t row = static_cast<size_t>(cur.ui.wrow + (kGateUp ? 0 : m * BM) + r);
        sv = __ldg(W.s + row * (cur.ui.K / kGroup) + ks);
        bv = __ldg(W.b + row * (cur.ui.K / kGroup) + ks);
      }
      // packed words of this stage's tile row
      const int sp = static_cast<int>(it % C::PST);
      if (!tc::mbar_wait(&full_p[sp], (it / C::PST) & 1u, abort_flag, a.status, a.wait_limit)) {
        ok = false;
        break;
      }
      const uint8_t* prow = smem + C::OFF_P + (sp * C::NA + m) * C::P_BYTES + r * 32;
      const uint4 q0 = *reinterpret_cast<const uint4*>(prow + (psw << 4));
      const uint4 q1 = *reinterpret_cast<const uint4*>(prow + ((psw ^ 1) << 4));
      __nv_bfloat162 s2, b2;
      *reinterpret_cast<uint32_t*>(&s2) = sv | (sv << 16);
      *reinterpret_cast<uint32_t*>(&b2) = bv | (bv << 16);
      const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
      uint32_t cols[32];
#pragma unroll
      for (int wd = 0; wd < 8; ++wd) {
        const uint4 d = tc::dequant8(words[wd], s2, b2);
        cols[4 * wd + 0] = d.x;
        cols[4 * wd + 1] = d.y;
        cols[4 * wd + 2] = d.z;
        cols[4 * wd + 3] = d.w;
      }
      // Hand the slot back only once its words are consumed.  The next TMA
      // write into it is an async-proxy access following these generic-proxy
      // reads: the proxy fence orders the two (the mbarrier alone does not).
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&empty_p[sp]);
      const int sa = static_cast<int>(it % C::A_STAGES);
      if (!tc::mbar_wait(&empty_a[sa], ((it / C::A_STAGES) & 1u) ^ 1u, abort_flag, a.status, a.wait_limit)) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      tc::tmem_st32(lane_base + C::A_BASE + sa * C::A_COLS + m * 32, cols);
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::mbar_arrive(&full_a[sa]);
      cur.next(a, n_units, nfb);
      while (!cur.done && !mine(cur.it)) cur.next(a, n_units, nfb);
    }
    if (ok && a.scales_tma && held_blk != 0xffffffffu) {
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&empty_s[held_blk & 1u]);
    }
  } else if (warp < kLoadWarp) {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;                     // weight row == TMEM lane == output feature in tile
    const int rpos = kGateUp ? tc::k8_pos(r) : r;    // h is stored in the K order of the down GEMM
    const int et = threadIdx.x - kEpiWarp0 * 32;     // 0 .. kEpiWarps * 32 - 1
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    uint16_t* stage = reinterpret_cast<uint16_t*>(smem + C::OFF_OUT);   // [BN tokens][BM features]
    uint32_t tt = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      const UnitInfo ui = unit_info<kGateUp, kNA>(a, u, nfb, units);
      if (ui.skip) continue;
      const int buf = static_cast<int>(tt % C::ACC_BUFS);
      if (!tc::mbar_wait(&acc_full[buf], (tt / C::ACC_BUFS) & 1u, abort_flag, a.status, a.wait_limit)) break;
      tc::tc_fence_after();
      const uint32_t acc = lane_base + buf * C::ACC_COLS;
      // gate/up: one output tile (SwiGLU of the two accumulators); down: one
      // tile per 128-row block, staged and written out in turn, or (two
      // blocks) both staged before either is written, so that the single
      // accumulator is handed back as early as possible
      constexpr int kRounds = kGateUp ? 1 : kNA;
      constexpr bool kAll = C::STAGE_ALL;
      bool ok = true;
      for (int mm = 0; mm < kRounds && ok; ++mm) {
        uint16_t* st = stage + (kAll ? mm * BN * BM : 0);
        for (int n0 = 16 * ((warp - kEpiWarp0) >> 2); n0 < ui.rows; n0 += 32) {
          float v0[16];
          tc::tmem_ld16(acc + mm * BN + n0, v0);
          if (kGateUp) {
            float v1[16];
            tc::tmem_ld16(acc + BN + n0, v1);
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float g = v0[j];
              st[(n0 + j) * BM + rpos] = float_to_bf16_bits(__fdividef(g * v1[j], 1.0f + __expf(-g)));
            }
          } else {
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) st[(n0 + j) * BM + r] = float_to_bf16_bits(v0[j]);
          }
        }
        if (mm == kRounds - 1) {
          // accumulator drained: hand it back to the MMA before writing the tile out
          tc::tc_fence_before();
          tc::mbar_arrive(&acc_empty[buf]);
        }
        if (kAll && mm != kRounds - 1) continue;
        const uint32_t rr = kAll ? tt : tt * kRounds + mm;   // staging rounds so far: the epi_sync phases
        tc::mbar_arrive(&epi_sync[0]);
        if (!tc::mbar_wait(&epi_sync[0], rr & 1u, abort_flag, a.status, a.wait_limit)) {
          ok = false;
          break;
        }
        // coalesced copy-out: each token row of a tile is BM contiguous outputs (256 B)
        const int chunks = ui.rows * (BM / 8);
        for (int mo = kAll ? 0 : mm; mo <= mm; ++mo) {
          const uint16_t* so = stage + (kAll ? mo * BN * BM : 0);
          for (int i = et; i < chunks; i += kEpiWarps * 32) {
            const int n = i / (BM / 8), c = i % (BM / 8);
            const int R = ui.row0 + n;
            uint16_t* dst;
            if (kGateUp)
              dst = ui.shared ? a.hs_out + static_cast<size_t>(R - Tk) * a.g.Is
                              : a.h_out + static_cast<size_t>(R) * a.g.I;
            else
              dst = a.Y + static_cast<size_t>(R) * a.g.H;
            *reinterpret_cast<uint4*>(dst + ui.f0 + mo * BM + c * 8) =
                *reinterpret_cast<const uint4*>(so + n * BM + c * 8);
          }
        }
        tc::mbar_arrive(&epi_sync[1]);                     // the staging tiles are free again
        if (!tc::mbar_wait(&epi_sync[1], rr & 1u, abort_flag, a.status, a.wait_limit)) ok = false;
      }
      if (!ok) break;
      ++tt;
    }
  } else if (warp == kLoadWarp) {
    // ------------------------------------------------------- token tiles
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const UnitInfo ui = unit_info<kGateUp, kNA>(a, u, nfb, units);
        if (ui.skip) continue;
        // gate/up: rows of the grouped x (shared-expert rows follow the routed
        // ones); down: routed h or shared h
        int bsz = 0;
        while (bsz < kTokenBoxes - 1 && token_box(bsz) < ui.rows) ++bsz;
        const void* tm = &a.tm_h[(!kGateUp && ui.shared) ? 1 : 0][bsz];
        const uint32_t bbytes = static_cast<uint32_t>(token_box(bsz)) * BK * 2;   // rows x 64 inputs x bf16
        const int y = (!kGateUp && ui.shared) ? ui.row0 - Tk : ui.row0;
        for (int ks = 0; ks < ui.nks; ++ks, ++it) {
          const int s = static_cast<int>(it % C::BST);
          if (!tc::mbar_wait(&empty_b[s], ((it / C::BST) & 1u) ^ 1u, abort_flag, a.status, a.wait_limit)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&full_b[s], bbytes);
          tc::tma_load_2d(sbase + C::OFF_B + s * C::B_BYTES, tm, ks * BK, y, &full_b[s]);
        }
      }
      // every tile this thread requested has landed before the CTA may exit
      tc::drain_ring(full_b, C::BST, it, a.status);
    }
    __syncwarp();
  } else if (warp == kTmaWarp) {
    // ----------------------------------------- packed tiles and scales (TMA)
    if (lane == 0) {
      StageCursor<kGateUp, kNA> cur;
      cur.begin(a, n_units, nfb, units);
      uint32_t last_blk = 0xffffffffu;
      uint32_t p_fills = 0, s_fills = 0;   // packed-tile and scale-block fills issued
      while (!cur.done) {
        const int side = cur.ui.shared ? 1 : 0;
        if (a.scales_tma && cur.blk != last_blk) {
          last_blk = cur.blk;
          const int ss = static_cast<int>(cur.blk & 1u);
          if (!tc::mbar_wait(&empty_s[ss], ((cur.blk >> 1) & 1u) ^ 1u, abort_flag, a.status, a.wait_limit)) break;
          tc::fence_proxy_async_smem();
          ++s_fills;
          tc::mbar_arrive_expect_tx(&full_s[ss], C::S_SLOT);
          const uint32_t sdst = sbase + C::OFF_S + ss * C::S_SLOT;
#pragma unroll
          for (int mm = 0; mm < C::NA; ++mm) {
            tc::tma_load_2d(sdst + mm * 2 * C::S_BYTES, &a.tm_s[side][kGateUp ? mm : 0], cur.ks,
                            cur.ui.wrow + (kGateUp ? 0 : mm * BM), &full_s[ss]);
            tc::tma_load_2d(sdst + mm * 2 * C::S_BYTES + C::S_BYTES, &a.tm_b[side][kGateUp ? mm : 0], cur.ks,
                            cur.ui.wrow + (kGateUp ? 0 : mm * BM),
                            &full_s[ss]);
          }
        }
        const int sp = static_cast<int>(cur.it % C::PST);
        if (!tc::mbar_wait(&empty_p[sp], ((cur.it / C::PST) & 1u) ^ 1u, abort_flag, a.status, a.wait_limit)) break;
        tc::fence_proxy_async_smem();   // consumers' generic reads of the slot precede this async-proxy refill
        ++p_fills;
        tc::mbar_arrive_expect_tx(&full_p[sp], C::NA * C::P_BYTES);
#pragma unroll
        for (int mm = 0; mm < C::NA; ++mm)
          tc::tma_load_2d(sbase + C::OFF_P + (sp * C::NA + mm) * C::P_BYTES, &a.tm_q[side][kGateUp ? mm : 0],
                          cur.ks * 8, cur.ui.wrow + (kGateUp ? 0 : mm * BM), &full_p[sp]);
        cur.next(a, n_units, nfb);
      }
      // every copy this thread requested has landed before the CTA may exit
      tc::drain_ring(full_p, C::PST, p_fills, a.status);
      tc::drain_ring(full_s, 2, s_fills, a.status);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- MMA
    // The whole warp walks the schedule and waits on the barriers; one elected
    // lane issues.  Operand descriptors are formed once and advanced by adds
    // (the shared-memory address field counts 16-byte units).
    const bool leader = tc::elect_one_sync();
    const uint64_t bdesc0 = tc::sdesc_sw128(sbase + C::OFF_B);
    uint32_t it = 0, tt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const UnitInfo ui = unit_info<kGateUp, kNA>(a, u, nfb, units);
      if (ui.skip) continue;
      const int n_mma = max(16, (ui.rows + 15) & ~15);
      const uint32_t idesc = tc::idesc_bf16(BM, n_mma);
      const int buf = static_cast<int>(tt % C::ACC_BUFS);
      // (every wait's outcome is made warp-uniform so the lanes leave together)
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&acc_empty[buf], ((tt / C::ACC_BUFS) & 1u) ^ 1u, abort_flag,
                                                 a.status, a.wait_limit)))
        break;
      tc::tc_fence_after();
      const uint32_t acc = tmem + buf * C::ACC_COLS;
      for (int ks = 0; ks < ui.nks; ++ks, ++it) {
        const int sb = static_cast<int>(it % C::BST);
        const int sa = static_cast<int>(it % C::A_STAGES);
        const bool got = tc::mbar_wait(&full_b[sb], (it / C::BST) & 1u, abort_flag, a.status, a.wait_limit) &&
                         tc::mbar_wait(&full_a[sa], (it / C::A_STAGES) & 1u, abort_flag, a.status, a.wait_limit);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        if (leader) {
          const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(sb * (C::B_BYTES >> 4));
          const uint32_t ast = tmem + C::A_BASE + sa * C::A_COLS;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t accum = (ks > 0 || kk > 0) ? 1u : 0u;
#pragma unroll
            for (int mm = 0; mm < C::NA; ++mm)
              tc::mma_bf16_ts(acc + mm * BN, ast + mm * 32 + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc,
                              accum);
          }
          tc::mma_commit(&empty_a[sa]);
          tc::mma_commit(&empty_b[sb]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (leader) tc::mma_commit(&acc_full[buf]);
      __syncwarp();
      ++tt;
    }
    // every issued MMA has finished before tensor memory is released
    if (leader) {
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

// ----------------------------------------------------------------- host ---

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

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  return make_tmap_2d(m, dt, esize, base, cols, rows, box_cols, box_rows, sw);
}

// Token-tile maps of a bf16 [rows, K] matrix: 64-input boxes of 16, 32, 64,
// 128 and 160 rows, 128-byte swizzle (K-major, the UMMA B layout).
bool make_token_maps(CUtensorMap (&m)[kTokenBoxes], const void* base, int K, uint64_t rows) {
  for (int i = 0; i < kTokenBoxes; ++i)
    if (!make_map(&m[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, K, rows, BK, static_cast<uint32_t>(token_box(i)),
                  CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  return true;
}

// Maps of one affine 4-bit matrix stack [rows, K]: packed words (box 128 rows
// x 8 words, 32-B swizzle) and, when the scale rows are 16-B strided, scales
// and biases (box 128 rows x 8 groups).
bool make_qmat_maps(TcArgs& a, int side, int m, const QMatPtr& W, int rows, int K) {
  if (!make_map(&a.tm_q[side][m], CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, W.q, K / 8, rows, 8, BM,
                CU_TENSOR_MAP_SWIZZLE_32B))
    return false;
  if (a.scales_tma) {
    if (!make_map(&a.tm_s[side][m], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, W.s, K / kGroup, rows, kSBlock, BM,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&a.tm_b[side][m], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, W.b, K / kGroup, rows, kSBlock, BM,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  }
  return true;
}

}  // namespace

static_assert(BN == kGemmChunkRows, "the chunk list and the GEMM tile must agree");
int gemm_chunk_rows() { return BN; }

cudaError_t launch_gateup(const Geometry& g, const LayerPtr& L, const uint16_t* xg, const Chunk* chunks,
                          const int32_t* n_chunks, int max_chunks, uint16_t* h, uint16_t* h_s, int* status,
                          cudaStream_t s) {
  TcArgs a{};
  a.g = g;
  a.W0 = L.gate;
  a.W1 = L.up;
  a.S0 = L.sh_gate;
  a.S1 = L.sh_up;
  a.h_out = h;
  a.hs_out = h_s;
  a.chunks = chunks;
  a.n_chunks = n_chunks;
  a.status = status;
  a.wait_limit = wait_limit_cycles();
  a.scales_tma = (g.H % (kGroup * kSBlock)) == 0;
  const uint64_t rows = static_cast<uint64_t>(g.T) * g.k + g.T;
  if (!make_qmat_maps(a, 0, 0, L.gate, g.E * g.I, g.H) || !make_qmat_maps(a, 0, 1, L.up, g.E * g.I, g.H) ||
      !make_qmat_maps(a, 1, 0, L.sh_gate, g.Is, g.H) || !make_qmat_maps(a, 1, 1, L.sh_up, g.Is, g.H) ||
      !make_token_maps(a.tm_h[0], xg, g.H, rows))
    return cudaErrorInvalidValue;
  for (int i = 0; i < kTokenBoxes; ++i) a.tm_h[1][i] = a.tm_h[0][i];
  using C = Cfg<true, 2>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(grouped_gemm_tc_kernel<true, 2>), C::SMEM);
  if (e != cudaSuccess) return e;
  const int nfb = max(g.I, g.Is) / BM;
  const int grid = max(1, min(max_chunks * nfb, num_sms()));
  return launch_pdl(grouped_gemm_tc_kernel<true, 2>, dim3(grid), dim3(kThreads), C::SMEM, s, a);
}

cudaError_t launch_down(const Geometry& g, const LayerPtr& L, const uint16_t* h, const uint16_t* h_s,
                        const Chunk* chunks, const int32_t* n_chunks, int max_chunks,
                        uint16_t* Y, int* status, cudaStream_t s) {
  TcArgs a{};
  a.g = g;
  a.W0 = L.down;
  a.W1 = L.down;
  a.S0 = L.sh_down;
  a.S1 = L.sh_down;
  a.Y = Y;
  a.chunks = chunks;
  a.n_chunks = n_chunks;
  a.status = status;
  a.wait_limit = wait_limit_cycles();
  a.scales_tma = (g.I % (kGroup * kSBlock)) == 0 && (g.Is % (kGroup * kSBlock)) == 0;
  if (!make_qmat_maps(a, 0, 0, L.down, g.E * g.H, g.I) || !make_qmat_maps(a, 1, 0, L.sh_down, g.H, g.Is) ||
      !make_token_maps(a.tm_h[0], h, g.I, static_cast<uint64_t>(g.T) * g.k) ||
      !make_token_maps(a.tm_h[1], h_s, g.Is, g.T))
    return cudaErrorInvalidValue;
  if (g.H % (2 * BM) == 0) {   // two 128-row blocks per unit share each token tile
    using C = Cfg<false, 2>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(grouped_gemm_tc_kernel<false, 2>), C::SMEM);
    if (e != cudaSuccess) return e;
    const int nfb = g.H / (2 * BM);
    const int grid = max(1, min(max_chunks * nfb, num_sms()));
    return launch_pdl(grouped_gemm_tc_kernel<false, 2>, dim3(grid), dim3(kThreads), C::SMEM, s, a);
  }
  using C = Cfg<false, 1>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(grouped_gemm_tc_kernel<false, 1>), C::SMEM);
  if (e != cudaSuccess) return e;
  const int nfb = g.H / BM;
  const int grid = max(1, min(max_chunks * nfb, num_sms()));
  return launch_pdl(grouped_gemm_tc_kernel<false, 1>, dim3(grid), dim3(kThreads), C::SMEM, s, a);
}

}  // namespace moe
