// Host-side launchers of the MoE kernels (internal to libmoe.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

// Per-call geometry shared by the launchers.
struct Geometry {
  int T, H, I, Is, E, k;
};

// Device pointers of one layer (mirrors moe_layer_desc).
struct QMatPtr {
  const uint32_t* q;
  const uint16_t* s;
  const uint16_t* b;
};
struct LayerPtr {
  const uint16_t* w_router;
  const float* router_bias;
  QMatPtr gate, up, down, sh_gate, sh_up, sh_down;
  const uint16_t* w_sg;
};

// Routing outputs of one call.
struct RoutingPtrs {
  int32_t* topk_idx;
  float* topk_w;
  float* sigma;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv_perm;
};

// tmap.cu: 2-D TMA tensor map over a row-major [rows, cols] array of
// `esize`-byte elements with box [box_rows, box_cols]; false on failure.
bool make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, uint64_t cols, uint64_t rows,
                  uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw);

// Launch with programmatic dependent launch: the kernel may be scheduled
// while the previous kernel of the stream still runs, so its launch and
// prologue overlap that kernel's tail.  Every kernel launched this way calls
// pdl_wait() before its first global-memory access (its prologue touches only
// its own shared and tensor memory) and then pdl_launch_dependents().
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// api.cu: SM clock cycles after which the kernels' bounded device-side waits
// give up (moe_set_wait_limit; default tc::kDefaultWaitLimit, ~2 s).
long long wait_limit_cycles();

// api.cu: raise a kernel's dynamic shared-memory limit once per device (and
// again only if a launch needs more), keeping the attribute call off the
// per-launch path.
cudaError_t ensure_smem(const void* func, int bytes);

// route_tc.cu: tensor-core router + top-k + shared gate (any T >= 1); also
// writes seg_counts[ceil(T/128)][E], the expert counts of each 128-token
// segment of the (token, slot) entries.
constexpr int kRouteSegTokens = 128;
cudaError_t launch_router(const uint16_t* x, const uint16_t* w_router, const float* router_bias,
                          const uint16_t* w_sg, int T, int H, int E, int k,
                          int32_t* topk_idx, float* topk_w, float* sigma, int32_t* seg_counts, int* status,
                          cudaStream_t s);

// route.cu: small-T router (T <= kSmallTB * kSmallMaxGroups).  `counter`
// points at a zeroed control area of at least (kSmallGroupCounter +
// kSmallMaxGroups) words: word 0 counts finished token groups, word
// kSmallGroupCounter + y the finished CTAs of token group y.
constexpr int kSmallTB = 8;
constexpr int kSmallMaxGroups = 16;
constexpr int kSmallGroupCounter = 16;

// route.cu
int num_segments(int T);   // 128-token segments of the counting sort
// T <= 64: router + top-k + shared gate + counting sort + active list in one launch.
// logits: workspace [T, E+1] FP32; counter: the control area described above.
cudaError_t launch_route_small(const uint16_t* x, const LayerPtr& L, int T, int H, int I, int Is, int E, int k,
                               float* logits, unsigned* counter, const RoutingPtrs& r, int32_t* active,
                               int32_t* n_active, cudaStream_t s);
// Second and third pass of the counting sort (seg_scratch holds the router's
// per-segment counts and is turned into per-segment bases in place).
cudaError_t launch_group(const int32_t* topk_idx, int T, int k, int E, int chunk_rows,
                         int32_t* seg_scratch, int32_t* counts, int32_t* offsets,
                         int32_t* perm, int32_t* inv_perm, Chunk* chunks, int32_t* n_chunks,
                         int32_t* active, int32_t* n_active, cudaStream_t s);

// gemm_tc.cu: tcgen05 grouped expert GEMMs over the device chunk list.
// Rows per chunk of the chunk list (the GEMM tile's token count); moe.h states
// moe_route_static's scratch limit with this value.
constexpr int kGemmChunkRows = 160;
int gemm_chunk_rows();
// xg: the grouped token rows [T*k + T, H] (routed rows in expert order, then
// the shared expert's T rows), each group of 8 in the interleaved K order.
cudaError_t launch_gateup(const Geometry& g, const LayerPtr& L, const uint16_t* xg, const Chunk* chunks,
                          const int32_t* n_chunks, int max_chunks, uint16_t* h, uint16_t* h_s, int* status,
                          cudaStream_t s);
cudaError_t launch_down(const Geometry& g, const LayerPtr& L, const uint16_t* h, const uint16_t* h_s,
                        const Chunk* chunks, const int32_t* n_chunks, int max_chunks,
                        uint16_t* Y, int* status, cudaStream_t s);

// combine.cu
// xg[R] = row perm[R] / k of x for R < T*k, row R - T*k for the shared
// expert's rows, each group of 8 elements reordered (0,4,1,5,2,6,3,7): the
// B operand of the gate/up GEMM in its grouped order and K order.
// status: the call's status word; gather, combine and the grouped GEMMs do
// nothing while it holds an error (their index inputs may then be unwritten).
cudaError_t launch_gather_k8(const uint16_t* x, const int32_t* perm, int T, int k, int H, uint16_t* xg,
                             const int* status, cudaStream_t s);
// out (may be NULL) = the layer output; norm_out (may be NULL) = RMSNorm(out)
// with weight 1 and `eps`, the next stacked layer's input.
cudaError_t launch_combine(const uint16_t* Y, const int32_t* inv_perm, const float* topk_w, const float* sigma,
                           int T, int k, int H, uint16_t* out, uint16_t* norm_out, float eps, const int* status,
                           cudaStream_t s);
cudaError_t launch_rmsnorm(const uint16_t* y, uint16_t* out, int T, int H, float eps, cudaStream_t s);

// decode.cu: steps of up to 64 tokens outside the fused kernel's range.
// Persistent mma.sync GEMVs over the active experts; gate/up writes h (rows
// in the grouped order) and h_s, down writes Y in the layout combine_kernel
// reads (routed rows in the grouped order, then the T shared rows).
bool mid_decode_supported(const Geometry& g);
cudaError_t launch_mid_gateup(const Geometry& g, const LayerPtr& L, const uint16_t* x, const int32_t* offsets,
                              const int32_t* perm, const int32_t* active, const int32_t* n_active, uint16_t* h,
                              uint16_t* h_s, cudaStream_t s);
cudaError_t launch_mid_down(const Geometry& g, const LayerPtr& L, const uint16_t* h, const uint16_t* h_s,
                            const int32_t* offsets, const int32_t* active, const int32_t* n_active, uint16_t* Y,
                            cudaStream_t s);

// decode_fused.cu: a stack of 1..decode_fused_max_layers() decode layers
// (T <= 8, H = 1024 or 2048) in one cooperative launch; layer l > 0 takes
// RMSNorm(eps) of layer l-1's output.  The CTAs exchange logits, h and the
// layer outputs through tagged 64-bit words in the workspace (FusedExchange,
// sizes from fused_exchange_words).  bar: workspace words [1] exit counter
// and [2] epoch (zero in a new workspace); trace: NULL or
// [n_layers][2][T][H]; r.topk_idx NULL: no routing outputs (else those of
// the last layer).
constexpr int kFusedMaxGrid = 1024;
struct FusedExchange {
  unsigned long long* logits;   // [T][E+1]
  unsigned long long* h;        // [T*k + T][max(I, Is)/2]
  unsigned long long* y;        // [T][H/2]
  unsigned long long* sumsq;    // [kFusedMaxGrid][8]
};
inline size_t fused_exchange_words(int T, int H, int I, int Is, int E, int k, int which) {
  const int Kmax = I > Is ? I : Is;
  switch (which) {
    case 0: return static_cast<size_t>(T) * (E + 1);
    case 1: return static_cast<size_t>(T * k + T) * (Kmax / 2);
    case 2: return static_cast<size_t>(T) * (H / 2);
    default: return static_cast<size_t>(kFusedMaxGrid) * 8;
  }
}
bool decode_fused_supported(const Geometry& g);
int decode_fused_max_layers();
cudaError_t launch_decode_fused(const Geometry& g, const LayerPtr* layers, int n_layers, const uint16_t* x,
                                uint16_t* out, uint16_t* trace, float eps, const RoutingPtrs& r, int32_t* active,
                                int32_t* n_active, const FusedExchange& xch, unsigned* bar, int* status,
                                cudaStream_t s);

}  // namespace moe
