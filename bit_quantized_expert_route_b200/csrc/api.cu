// C ABI of libmoe.so: argument validation, workspace carving and the launch
// sequence of one MoE layer on the caller's stream.  No host synchronisation
// except in moe_get_status and moe_forward_host.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "moe.h"
#include "kernels.h"
#include "tc.cuh"

namespace moe {

cudaError_t ensure_smem(const void* func, int bytes) {
  struct Entry {
    const void* func;
    int dev;
    int bytes;
  };
  static std::mutex mu;
  static Entry table[128];
  static int n = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n; ++i)
    if (table[i].func == func && table[i].dev == dev) {
      if (table[i].bytes >= bytes) return cudaSuccess;
      e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e == cudaSuccess) table[i].bytes = bytes;
      return e;
    }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && n < 128) table[n++] = Entry{func, dev, bytes};
  return e;
}

namespace {
std::atomic<long long> g_wait_limit{tc::kDefaultWaitLimit};
}  // namespace

long long wait_limit_cycles() { return g_wait_limit.load(std::memory_order_relaxed); }

// Keeps the device busy for `ns` nanoseconds (bounded by construction), so
// that every launch a traced call enqueues is already queued when its first
// stage starts: stage times then measure kernels, not host launch gaps.
__global__ void busy_wait_kernel(unsigned long long ns) {
  unsigned long long t0, t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  do {
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  } while (t - t0 < ns);
}

}  // namespace moe

namespace {

using namespace moe;

constexpr int kDecodeMaxT = 64;
// Tokens the fused decode kernel takes: a stack of layers runs up to 40 of
// them per cooperative launch and wins up to T = 7 (T=4 28.4 vs 37.3 us per
// layer, T=6 35.7 vs 39.5, T=8 42.2 vs 40.6 on the mid-size path); a single
// layer pays the cooperative launch and the kernel's fixed phases every call,
// and the mid-size path is faster from T = 4 (T=3 38.9 vs 39.8 us, T=4 46.6
// vs 40.9, T=8 81.1 vs 59.1).
constexpr int kFusedMaxT = 3;       // single-layer calls
constexpr int kFusedMaxTStack = 7;  // moe_forward_stack
constexpr int kMidMaxT = 128;       // tokens the mid-size decode path takes (moe_forward)
constexpr int kMaxT = 65536;
constexpr int kMaxStackLayers = 1024;
constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte offsets of every workspace buffer for a call with T tokens.
struct WsLayout {
  size_t status, counter, grid_bar, topk_idx, topk_w, counts, offsets, perm, inv_perm, sigma, seg, chunks, n_chunks,
      active, n_active, logits, h, h_s, Y, x_stage, out_stage, xch[4], total;
  int max_chunks;
};

WsLayout ws_layout(const moe_layer_desc* d, int T) {
  WsLayout w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes);
    return o;
  };
  const size_t n = static_cast<size_t>(T) * d->k;
  const int cr = gemm_chunk_rows();
  w.max_chunks = static_cast<int>(n / cr + T / cr + d->E + 2);
  w.status = take(256);          // control block: status word, small-T routing counter, grid barrier
  w.counter = w.status + 4;
  w.grid_bar = w.status + 8;     // fused decode kernel: [unused, exit counter, epoch]
  w.topk_idx = take(n * 4);
  w.topk_w = take(n * 4);
  w.counts = take(static_cast<size_t>(d->E) * 4);
  w.offsets = take(static_cast<size_t>(d->E + 1) * 4);
  w.perm = take(n * 4);
  w.inv_perm = take(n * 4);
  w.sigma = take(static_cast<size_t>(T) * 4);
  w.seg = take(static_cast<size_t>(num_segments(T)) * d->E * 4);
  w.chunks = take(static_cast<size_t>(w.max_chunks) * sizeof(Chunk));
  w.n_chunks = take(4);
  w.active = take(static_cast<size_t>(d->E + 1) * 4);
  w.n_active = take(4);
  w.logits = take(static_cast<size_t>(T <= kMidMaxT ? T : 0) * (d->E + 1) * 4);
  w.h = take(n * d->I * 2);
  w.h_s = take(static_cast<size_t>(T) * d->I_shared * 2);
  w.Y = take((n + T) * d->H * 2);   // also holds the gate/up GEMM's grouped token rows before the down GEMM
  w.x_stage = take(static_cast<size_t>(T) * d->H * 2);
  w.out_stage = take(static_cast<size_t>(T) * d->H * 2);
  // the fused decode kernel's exchange words: logits, h, outputs between
  // stacked layers and the CTAs' sums of squares of them
  for (int i = 0; i < 4; ++i)
    w.xch[i] = take(T <= kFusedMaxTStack ? fused_exchange_words(T, d->H, d->I, d->I_shared, d->E, d->k, i) * 8 : 0);
  w.total = off;
  return w;
}

bool qmat_ok(const moe_qmat& m) {
  return m.q && m.scales && m.biases && aligned16(m.q) && (reinterpret_cast<uintptr_t>(m.scales) & 3u) == 0 &&
         (reinterpret_cast<uintptr_t>(m.biases) & 3u) == 0;
}

int validate_layer(const moe_layer_desc* d) {
  if (!d) return MOE_ERR_INVALID_ARG;
  if (d->bits != 4 || d->group_size != 64 || d->renorm != 1) return MOE_ERR_UNSUPPORTED;
  if (d->k < 1 || d->k > kMaxK || d->E < d->k || d->E > kMaxE) return MOE_ERR_UNSUPPORTED;
  if (d->H < 128 || d->H % 128 || d->H > 8192) return MOE_ERR_UNSUPPORTED;
  if (d->I < 128 || d->I % 128 || d->I > 2048) return MOE_ERR_UNSUPPORTED;
  if (d->I_shared < 128 || d->I_shared % 128 || d->I_shared > 2048) return MOE_ERR_UNSUPPORTED;
  if (!d->w_router || !aligned16(d->w_router)) return MOE_ERR_INVALID_ARG;
  if (d->router_bias && (reinterpret_cast<uintptr_t>(d->router_bias) & 3u)) return MOE_ERR_INVALID_ARG;
  if (!qmat_ok(d->gate) || !qmat_ok(d->up) || !qmat_ok(d->down)) return MOE_ERR_INVALID_ARG;
  if (!qmat_ok(d->sh_gate) || !qmat_ok(d->sh_up) || !qmat_ok(d->sh_down)) return MOE_ERR_INVALID_ARG;
  if (!d->w_shared_gate || !aligned16(d->w_shared_gate)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

int validate_ws(const moe_layer_desc* d, int T, void* ws, size_t ws_bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return MOE_ERR_WORKSPACE;
  if (ws_layout(d, T).total > ws_bytes) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

int validate_routing(const moe_routing* r) {
  if (!r) return MOE_OK;
  if (!r->topk_idx || !r->topk_w || !r->counts || !r->offsets || !r->perm || !r->inv_perm)
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

LayerPtr layer_ptrs(const moe_layer_desc* d) {
  auto qp = [](const moe_qmat& m) { return QMatPtr{m.q, m.scales, m.biases}; };
  return LayerPtr{d->w_router, d->router_bias, qp(d->gate), qp(d->up), qp(d->down),
                  qp(d->sh_gate), qp(d->sh_up), qp(d->sh_down), d->w_shared_gate};
}

// Resolved device buffers of one call.
struct Bufs {
  char* base;
  WsLayout w;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv_perm;
  float* sigma;
  template <class P>
  P* at(size_t off) const { return reinterpret_cast<P*>(base + off); }
};

Bufs resolve(const moe_layer_desc* d, int T, void* ws, const moe_routing* r) {
  Bufs b;
  b.base = static_cast<char*>(ws);
  b.w = ws_layout(d, T);
  b.topk_idx = r ? r->topk_idx : b.at<int32_t>(b.w.topk_idx);
  b.topk_w = r ? r->topk_w : b.at<float>(b.w.topk_w);
  b.counts = r ? r->counts : b.at<int32_t>(b.w.counts);
  b.offsets = r ? r->offsets : b.at<int32_t>(b.w.offsets);
  b.perm = r ? r->perm : b.at<int32_t>(b.w.perm);
  b.inv_perm = r ? r->inv_perm : b.at<int32_t>(b.w.inv_perm);
  b.sigma = (r && r->sigma) ? r->sigma : b.at<float>(b.w.sigma);
  return b;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Optional stage tracer: records ev[0] before the first stage and ev[i+1]
// after stage i on the call's stream.
struct Tracer {
  cudaEvent_t ev[8];
  int n = 0;
  void mark(cudaStream_t s) {
    if (n < 8) cudaEventRecord(ev[n++], s);
  }
};

inline void mark(Tracer* tr, cudaStream_t s) {
  if (tr) tr->mark(s);
}

// Routing of T tokens.  T <= 64 without `grouped` (T <= 128 for the
// mid-size decode path): one launch of the small-T router (routing outputs
// and active list only).  Otherwise the tensor-core router and the
// counting-sort passes, which also build the chunk list the grouped GEMMs
// walk.
int enqueue_route(const moe_layer_desc* d, const uint16_t* x, int T, const Bufs& b, cudaStream_t s,
                  Tracer* tr = nullptr, bool grouped = false, int small_max_t = kDecodeMaxT) {
  mark(tr, s);
  if (T <= small_max_t && !grouped) {
    const RoutingPtrs rp{b.topk_idx, b.topk_w, b.sigma, b.counts, b.offsets, b.perm, b.inv_perm};
    const cudaError_t e = launch_route_small(x, layer_ptrs(d), T, d->H, d->I, d->I_shared, d->E, d->k,
                                             b.at<float>(b.w.logits), b.at<unsigned>(b.w.counter), rp,
                                             b.at<int32_t>(b.w.active), b.at<int32_t>(b.w.n_active), s);
    mark(tr, s);
    return cuda_status(e);
  }
  cudaError_t e = launch_router(x, d->w_router, d->router_bias, d->w_shared_gate, T, d->H, d->E, d->k,
                                b.topk_idx, b.topk_w, b.sigma, b.at<int32_t>(b.w.seg), b.at<int>(b.w.status), s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  mark(tr, s);
  e = launch_group(b.topk_idx, T, d->k, d->E, gemm_chunk_rows(), b.at<int32_t>(b.w.seg), b.counts, b.offsets,
                   b.perm, b.inv_perm, b.at<Chunk>(b.w.chunks), b.at<int32_t>(b.w.n_chunks),
                   b.at<int32_t>(b.w.active), b.at<int32_t>(b.w.n_active), s);
  mark(tr, s);
  return cuda_status(e);
}

// n_layers (<= decode_fused_max_layers()) layers of one geometry through the
// fused decode kernel; with_routing: the last layer's routing goes to b's
// routing buffers.
cudaError_t launch_fused_layers(const Geometry& g, const LayerPtr* layers, int n_layers, const uint16_t* x,
                                uint16_t* out, uint16_t* trace, float eps, const Bufs& b, bool with_routing,
                                cudaStream_t s) {
  RoutingPtrs rp{b.topk_idx, b.topk_w, b.sigma, b.counts, b.offsets, b.perm, b.inv_perm};
  if (!with_routing) rp = RoutingPtrs{};
  const FusedExchange xch{b.at<unsigned long long>(b.w.xch[0]), b.at<unsigned long long>(b.w.xch[1]),
                          b.at<unsigned long long>(b.w.xch[2]), b.at<unsigned long long>(b.w.xch[3])};
  return launch_decode_fused(g, layers, n_layers, x, out, trace, eps, rp, b.at<int32_t>(b.w.active),
                             b.at<int32_t>(b.w.n_active), xch, b.at<unsigned>(b.w.grid_bar), b.at<int>(b.w.status),
                             s);
}

// Bulk copies of whole scale/bias tile rows need 16-byte aligned stacks.
bool fused_decode_ok(const moe_layer_desc* d, const Geometry& g) {
  const moe_qmat* m[6] = {&d->gate, &d->up, &d->down, &d->sh_gate, &d->sh_up, &d->sh_down};
  for (const moe_qmat* q : m)
    if (!aligned16(q->scales) || !aligned16(q->biases)) return false;
  return decode_fused_supported(g);
}

bool mid_decode_ok(const moe_layer_desc* d, const Geometry& g) {
  (void)d;
  return mid_decode_supported(g);
}

// The kernels one layer of T tokens runs on: the single-launch fused decode
// kernel where it applies (T <= 8), else for T <= kMidMaxT the mid-size
// decode path (small-T router, mma.sync GEMVs over the active experts,
// combine), else the tensor-core (tcgen05) grouped-GEMM path.
enum class Path { kFused, kMid, kPrefill };

Path layer_path(const moe_layer_desc* d, int T, bool stacked = false) {
  const Geometry g{T, d->H, d->I, d->I_shared, d->E, d->k};
  if (T <= (stacked ? kFusedMaxTStack : kFusedMaxT) && fused_decode_ok(d, g)) return Path::kFused;
  if (T <= kMidMaxT && mid_decode_ok(d, g)) return Path::kMid;
  return Path::kPrefill;
}

bool forward_uses_fused_decode(const moe_layer_desc* d, int T, bool stacked = false) {
  return layer_path(d, T, stacked) == Path::kFused;
}

// The fused decode kernel for one layer (routing outputs included).
int enqueue_fused(const moe_layer_desc* d, const uint16_t* x, int T, uint16_t* out, const Bufs& b,
                  cudaStream_t s, Tracer* tr = nullptr) {
  const Geometry g{T, d->H, d->I, d->I_shared, d->E, d->k};
  mark(tr, s);
  const LayerPtr L = layer_ptrs(d);
  const cudaError_t e = launch_fused_layers(g, &L, 1, x, out, nullptr, 0.f, b, true, s);
  mark(tr, s);
  return cuda_status(e);
}

// The mid-size decode path: router (one launch), gate/up, down, combine
// (which also writes RMSNorm(out) to norm_out when given; out may then be
// NULL).
int enqueue_mid(const moe_layer_desc* d, const uint16_t* x, int T, uint16_t* out, const Bufs& b, cudaStream_t s,
                Tracer* tr = nullptr, uint16_t* norm_out = nullptr, float eps = 0.f) {
  int st = enqueue_route(d, x, T, b, s, tr, /*grouped=*/false, kMidMaxT);
  if (st != MOE_OK) return st;
  const Geometry g{T, d->H, d->I, d->I_shared, d->E, d->k};
  const LayerPtr L = layer_ptrs(d);
  uint16_t* h = b.at<uint16_t>(b.w.h);
  uint16_t* h_s = b.at<uint16_t>(b.w.h_s);
  uint16_t* Y = b.at<uint16_t>(b.w.Y);
  const int32_t* active = b.at<int32_t>(b.w.active);
  const int32_t* n_active = b.at<int32_t>(b.w.n_active);
  cudaError_t e = launch_mid_gateup(g, L, x, b.offsets, b.perm, active, n_active, h, h_s, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  mark(tr, s);
  e = launch_mid_down(g, L, h, h_s, b.offsets, active, n_active, Y, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  mark(tr, s);
  e = launch_combine(Y, b.inv_perm, b.topk_w, b.sigma, T, d->k, d->H, out, norm_out, eps, b.at<int>(b.w.status), s);
  mark(tr, s);
  return cuda_status(e);
}

// out: the layer output (may be NULL when norm_out is given); norm_out (may
// be NULL): RMSNorm(out) with weight 1 and eps, fused into the combine.
int enqueue_prefill(const moe_layer_desc* d, const uint16_t* x, int T, uint16_t* out, const Bufs& b,
                    cudaStream_t s, Tracer* tr = nullptr, uint16_t* norm_out = nullptr, float eps = 0.f) {
  int st = enqueue_route(d, x, T, b, s, tr, /*grouped=*/true);
  if (st != MOE_OK) return st;
  const Geometry g{T, d->H, d->I, d->I_shared, d->E, d->k};
  const LayerPtr L = layer_ptrs(d);
  uint16_t* h = b.at<uint16_t>(b.w.h);
  uint16_t* h_s = b.at<uint16_t>(b.w.h_s);
  uint16_t* Y = b.at<uint16_t>(b.w.Y);
  int* status = b.at<int>(b.w.status);
  const Chunk* chunks = b.at<Chunk>(b.w.chunks);
  const int32_t* n_chunks = b.at<int32_t>(b.w.n_chunks);
  // the grouped token rows live in Y's storage until the down GEMM overwrites it
  cudaError_t e = launch_gather_k8(x, b.perm, T, d->k, d->H, Y, status, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  mark(tr, s);
  e = launch_gateup(g, L, Y, chunks, n_chunks, b.w.max_chunks, h, h_s, status, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  mark(tr, s);
  e = launch_down(g, L, h, h_s, chunks, n_chunks, b.w.max_chunks, Y, status, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  mark(tr, s);
  e = launch_combine(Y, b.inv_perm, b.topk_w, b.sigma, T, d->k, d->H, out, norm_out, eps, status, s);
  mark(tr, s);
  return cuda_status(e);
}

// One layer of a stack: out (may be NULL) receives the layer output and
// norm_out (may be NULL) its RMSNorm, the next layer's input.
int enqueue_layer(const moe_layer_desc* d, const uint16_t* x, int T, uint16_t* out, uint16_t* norm_out, float eps,
                  const Bufs& b, cudaStream_t s) {
  switch (layer_path(d, T, /*stacked=*/true)) {
    case Path::kPrefill: return enqueue_prefill(d, x, T, out, b, s, nullptr, norm_out, eps);
    case Path::kMid: return enqueue_mid(d, x, T, out, b, s, nullptr, norm_out, eps);
    default: break;
  }
  uint16_t* y = out ? out : norm_out;
  const int st = enqueue_fused(d, x, T, y, b, s);
  if (st != MOE_OK || !norm_out) return st;
  return cuda_status(launch_rmsnorm(y, norm_out, T, d->H, eps, s));   // in place when out is NULL
}

// One layer, output to out (the path layer_path picks).
int enqueue_forward(const moe_layer_desc* d, const uint16_t* x, int T, uint16_t* out, const Bufs& b, cudaStream_t s,
                    Tracer* tr = nullptr) {
  switch (layer_path(d, T)) {
    case Path::kFused: return enqueue_fused(d, x, T, out, b, s, tr);
    case Path::kMid: return enqueue_mid(d, x, T, out, b, s, tr);
    default: return enqueue_prefill(d, x, T, out, b, s, tr);
  }
}

int check_call(const moe_layer_desc* d, const void* x, int T, int T_limit, const void* out, const moe_routing* r,
               void* ws, size_t ws_bytes, bool need_out) {
  int st = validate_layer(d);
  if (st != MOE_OK) return st;
  if (T < 1 || T > T_limit) return MOE_ERR_INVALID_ARG;
  if (!x || !aligned16(x)) return MOE_ERR_INVALID_ARG;
  if (need_out && (!out || !aligned16(out))) return MOE_ERR_INVALID_ARG;
  st = validate_routing(r);
  if (st != MOE_OK) return st;
  return validate_ws(d, T, ws, ws_bytes);
}

}  // namespace

// Scratch of moe_route_static: one static device array per GPU that loads
// the library (a CUDA __device__ variable exists on every device of the
// context), so callers that cannot allocate need not pass a workspace.
constexpr size_t kRouteStaticBytes = 512u * 1024u;
// moe.h states the scratch limit with 128-token segments and 160-row chunks.
static_assert(moe::kGemmChunkRows == 160 && moe::kRouteSegTokens == 128,
              "update moe_route_static's documented limit");
static __device__ __align__(256) unsigned char g_route_static_scratch[kRouteStaticBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_route_static_mu;
void* g_route_static_ptr[kMaxDevices] = {};

// Device address of the static scratch on the current device; looked up once
// per device (host code cannot use the symbol itself as a device address).
int route_static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_route_static_mu);
  if (!g_route_static_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_static_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_route_static_ptr[dev] = p;
  }
  *out = g_route_static_ptr[dev];
  return MOE_OK;
}

// Pieces of the static scratch for one moe_route_static call: the same
// buffers a workspace provides to moe_route (control block first, which the
// zero-initialised array and every call leave zero except for a recorded
// error status), each rounded up to 256 bytes.
struct RouteStaticLayout {
  size_t status, counter, seg, chunks, n_chunks, active, n_active, logits, sigma, total;
};

RouteStaticLayout route_static_layout(const moe_layer_desc* d, int T, bool sigma_given) {
  RouteStaticLayout l{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes);
    return o;
  };
  l.status = take(256);   // status word, then the small-T routing counter
  l.counter = l.status + 4;
  if (T <= kDecodeMaxT) {
    l.logits = take(static_cast<size_t>(T) * (d->E + 1) * 4);
  } else {
    const size_t n = static_cast<size_t>(T) * d->k;
    const int cr = gemm_chunk_rows();
    const size_t max_chunks = n / cr + T / cr + d->E + 2;
    l.seg = take(static_cast<size_t>(num_segments(T)) * d->E * 4);
    l.chunks = take(max_chunks * sizeof(Chunk));
    l.n_chunks = take(4);
  }
  l.active = take(static_cast<size_t>(d->E + 1) * 4);
  l.n_active = take(4);
  l.sigma = sigma_given ? 0 : take(static_cast<size_t>(T) * 4);
  l.total = off;
  return l;
}

}  // namespace

extern "C" {

int moe_workspace_size(const moe_layer_desc* layer, int T_max, size_t* bytes) {
  if (!bytes) return MOE_ERR_INVALID_ARG;
  const int st = validate_layer(layer);
  if (st != MOE_OK) return st;
  if (T_max < 1 || T_max > kMaxT) return MOE_ERR_INVALID_ARG;
  // The layout grows with T inside each regime, but a smaller T can need
  // more: T <= 8 adds the fused kernel's exchange words and T <= 64 the small
  // router's logits.  A workspace must serve every T <= T_max.
  size_t need = ws_layout(layer, T_max).total;
  for (int t : {kFusedMaxTStack, kMidMaxT})
    if (t < T_max) need = std::max(need, ws_layout(layer, t).total);
  *bytes = need;
  return MOE_OK;
}

int moe_route(const moe_layer_desc* layer, const moe_bf16* x, int T, moe_routing* r, void* ws, size_t ws_bytes,
              moe_stream stream) {
  if (!r) return MOE_ERR_INVALID_ARG;
  const int st = check_call(layer, x, T, kMaxT, nullptr, r, ws, ws_bytes, false);
  if (st != MOE_OK) return st;
  return enqueue_route(layer, x, T, resolve(layer, T, ws, r), static_cast<cudaStream_t>(stream));
}

int moe_forward(const moe_layer_desc* layer, const moe_bf16* x, int T, moe_bf16* out, moe_routing* r, void* ws,
                size_t ws_bytes, moe_stream stream) {
  const int st = check_call(layer, x, T, kMaxT, out, r, ws, ws_bytes, true);
  if (st != MOE_OK) return st;
  const Bufs b = resolve(layer, T, ws, r);
  return enqueue_forward(layer, x, T, out, b, static_cast<cudaStream_t>(stream));
}

int moe_decode(const moe_layer_desc* layer, const moe_bf16* x, int T, moe_bf16* out, moe_routing* r, void* ws,
               size_t ws_bytes, moe_stream stream) {
  const int st = check_call(layer, x, T, kDecodeMaxT, out, r, ws, ws_bytes, true);
  if (st != MOE_OK) return st;
  return enqueue_forward(layer, x, T, out, resolve(layer, T, ws, r), static_cast<cudaStream_t>(stream));
}

int moe_forward_stack(const moe_layer_desc* layers, int n_layers, const moe_bf16* x, int T, moe_bf16* out,
                      moe_bf16* trace, float eps, void* ws, size_t ws_bytes, moe_stream stream) {
  if (!layers || n_layers < 1 || n_layers > kMaxStackLayers) return MOE_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || (trace && !aligned16(trace))) return MOE_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    const moe_layer_desc& d = layers[l];
    const int st = check_call(&d, x, T, kMaxT, out, nullptr, ws, ws_bytes, true);
    if (st != MOE_OK) return st;
    const moe_layer_desc& d0 = layers[0];
    if (d.H != d0.H || d.I != d0.I || d.I_shared != d0.I_shared || d.E != d0.E || d.k != d0.k)
      return MOE_ERR_UNSUPPORTED;
  }
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t act = static_cast<size_t>(T) * layers[0].H;
  const Bufs b0 = resolve(&layers[0], T, ws, nullptr);
  uint16_t* pingpong[2] = {b0.at<uint16_t>(b0.w.x_stage), b0.at<uint16_t>(b0.w.out_stage)};
  uint16_t* tr = reinterpret_cast<uint16_t*>(trace);
  bool fused = true;
  for (int l = 0; l < n_layers; ++l) fused = fused && forward_uses_fused_decode(&layers[l], T, /*stacked=*/true);
  if (fused) {
    // whole chunks of layers per launch of the fused decode kernel, which
    // applies the RMSNorm between its layers itself and writes the trace
    const moe_layer_desc& d0 = layers[0];
    const Geometry g{T, d0.H, d0.I, d0.I_shared, d0.E, d0.k};
    const int chunk = decode_fused_max_layers();
    LayerPtr lp[kMaxStackLayers];
    for (int l = 0; l < n_layers; ++l) lp[l] = layer_ptrs(&layers[l]);
    const uint16_t* xin = x;
    for (int l0 = 0, c = 0; l0 < n_layers; l0 += chunk, ++c) {
      const int nl = n_layers - l0 < chunk ? n_layers - l0 : chunk;
      const bool last = l0 + nl == n_layers;
      uint16_t* cout = last ? out : pingpong[c & 1];
      if (launch_fused_layers(g, lp + l0, nl, xin, cout, tr ? tr + 2 * l0 * act : nullptr, eps, b0, false, s) !=
          cudaSuccess)
        return MOE_ERR_CUDA;
      if (!last && launch_rmsnorm(cout, cout, T, d0.H, eps, s) != cudaSuccess) return MOE_ERR_CUDA;
      xin = cout;
    }
    return MOE_OK;
  }
  if (tr && cudaMemcpyAsync(tr, x, act * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return MOE_ERR_CUDA;
  const uint16_t* xin = x;
  for (int l = 0; l < n_layers; ++l) {
    const bool last = l == n_layers - 1;
    uint16_t* y = last ? out : (tr ? tr + (2 * l + 1) * act : nullptr);
    uint16_t* next = last ? nullptr : (tr ? tr + (2 * l + 2) * act : pingpong[l & 1]);
    const int st = enqueue_layer(&layers[l], xin, T, y, next, eps, resolve(&layers[l], T, ws, nullptr), s);
    if (st != MOE_OK) return st;
    xin = next;
  }
  if (tr && cudaMemcpyAsync(tr + (2 * n_layers - 1) * act, out, act * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_route_static(const moe_layer_desc* layer, const moe_bf16* x, int T, moe_routing* r, moe_stream stream) {
  if (!r) return MOE_ERR_INVALID_ARG;
  int st = validate_layer(layer);
  if (st != MOE_OK) return st;
  if (T < 1 || T > kMaxT || !x || !aligned16(x)) return MOE_ERR_INVALID_ARG;
  st = validate_routing(r);
  if (st != MOE_OK) return st;
  // carve the static scratch exactly as a workspace is carved for moe_route
  const RouteStaticLayout sl = route_static_layout(layer, T, r->sigma != nullptr);
  if (sl.total > kRouteStaticBytes) return MOE_ERR_WORKSPACE;
  void* base = nullptr;
  st = route_static_scratch(&base);
  if (st != MOE_OK) return st;
  char* b = static_cast<char*>(base);
  Bufs bufs;
  bufs.base = b;
  bufs.w = WsLayout{};
  bufs.w.status = sl.status;
  bufs.w.counter = sl.counter;
  bufs.w.seg = sl.seg;
  bufs.w.chunks = sl.chunks;
  bufs.w.n_chunks = sl.n_chunks;
  bufs.w.active = sl.active;
  bufs.w.n_active = sl.n_active;
  bufs.w.logits = sl.logits;
  bufs.topk_idx = r->topk_idx;
  bufs.topk_w = r->topk_w;
  bufs.counts = r->counts;
  bufs.offsets = r->offsets;
  bufs.perm = r->perm;
  bufs.inv_perm = r->inv_perm;
  bufs.sigma = r->sigma ? r->sigma : reinterpret_cast<float*>(b + sl.sigma);
  return enqueue_route(layer, x, T, bufs, static_cast<cudaStream_t>(stream));
}

static int forward_host_enqueue(const moe_layer_desc* layer, const moe_bf16* x_host, int T, moe_bf16* out_host,
                                void* ws, size_t ws_bytes, cudaStream_t s) {
  int st = validate_layer(layer);
  if (st != MOE_OK) return st;
  if (T < 1 || T > kMaxT || !x_host || !out_host) return MOE_ERR_INVALID_ARG;
  st = validate_ws(layer, T, ws, ws_bytes);
  if (st != MOE_OK) return st;
  const Bufs b = resolve(layer, T, ws, nullptr);
  uint16_t* xd = b.at<uint16_t>(b.w.x_stage);
  uint16_t* od = b.at<uint16_t>(b.w.out_stage);
  const size_t bytes = static_cast<size_t>(T) * layer->H * sizeof(uint16_t);
  if (cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return MOE_ERR_CUDA;
  st = enqueue_forward(layer, xd, T, od, b, s);
  if (st != MOE_OK) return st;
  if (cudaMemcpyAsync(out_host, od, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_forward_host_async(const moe_layer_desc* layer, const moe_bf16* x_host, int T, moe_bf16* out_host,
                           void* ws, size_t ws_bytes, moe_stream stream) {
  return forward_host_enqueue(layer, x_host, T, out_host, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int moe_forward_host(const moe_layer_desc* layer, const moe_bf16* x_host, int T, moe_bf16* out_host, void* ws,
                     size_t ws_bytes, moe_stream stream) {
  const cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  const int st = forward_host_enqueue(layer, x_host, T, out_host, ws, ws_bytes, s0);
  if (st != MOE_OK) return st;
  return cuda_status(cudaStreamSynchronize(s0));
}


int moe_rmsnorm(const moe_bf16* y, moe_bf16* y_out, int T, int H, float eps, moe_stream stream) {
  if (!y || !y_out || !aligned16(y) || !aligned16(y_out)) return MOE_ERR_INVALID_ARG;
  if (T < 1 || T > kMaxT || H < 8 || H % 8 || H > 65536 || !(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_rmsnorm(y, y_out, T, H, eps, static_cast<cudaStream_t>(stream)));
}

int moe_forward_profiled(const moe_layer_desc* layer, const moe_bf16* x, int T, moe_bf16* out, void* ws,
                         size_t ws_bytes, moe_stream stream, float* stage_ms, int* n_stages) {
  if (!stage_ms || !n_stages) return MOE_ERR_INVALID_ARG;
  int st = check_call(layer, x, T, kMaxT, out, nullptr, ws, ws_bytes, true);
  if (st != MOE_OK) return st;
  const Bufs b = resolve(layer, T, ws, nullptr);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  busy_wait_kernel<<<1, 32, 0, s>>>(300000ull);     // 0.3 ms: the host enqueues the stages meanwhile
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  Tracer tr;
  for (int i = 0; i < 8; ++i)
    if (cudaEventCreate(&tr.ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(tr.ev[j]);
      return MOE_ERR_CUDA;
    }
  st = enqueue_forward(layer, x, T, out, b, s, &tr);
  if (st == MOE_OK && cudaEventSynchronize(tr.ev[tr.n - 1]) != cudaSuccess) st = MOE_ERR_CUDA;
  *n_stages = 0;
  if (st == MOE_OK) {
    for (int i = 0; i + 1 < tr.n; ++i) cudaEventElapsedTime(&stage_ms[i], tr.ev[i], tr.ev[i + 1]);
    *n_stages = tr.n - 1;
  }
  for (int i = 0; i < 8; ++i) cudaEventDestroy(tr.ev[i]);
  return st;
}

int moe_get_status(void* ws, moe_stream stream) {
  if (!ws) {
    // the status word of moe_route_static's scratch on the current device
    const int st = route_static_scratch(&ws);
    if (st != MOE_OK) return st;
  }
  if (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) return MOE_ERR_WORKSPACE;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host = 0;
  if (cudaMemcpyAsync(&host, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  // a device timeout can leave the control block's counters mid-count: clear
  // them (the status word, the routing and exit counters, the small-T
  // router's token-group counters; not the fused kernel's epoch)
  if (host != MOE_OK && cudaMemsetAsync(ws, 0, 16, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (host != MOE_OK &&
      cudaMemsetAsync(static_cast<char*>(ws) + 4 * (1 + kSmallGroupCounter), 0, 4 * kSmallMaxGroups, s) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  return host;
}

int moe_set_wait_limit(long long cycles) {
  g_wait_limit.store(cycles > 0 ? cycles : tc::kDefaultWaitLimit, std::memory_order_relaxed);
  return MOE_OK;
}

const char* moe_strerror(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (NULL or misaligned pointer, or T out of range)";
    case MOE_ERR_UNSUPPORTED: return "unsupported layer (needs affine 4-bit, group 64, renorm, supported sizes)";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA runtime error or kernel launch failure";
    case MOE_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
    case MOE_ERR_DEVICE_INDEX: return "a device-side bounds check found an index out of range";
    default: return "unknown status";
  }
}

}  // extern "C"
