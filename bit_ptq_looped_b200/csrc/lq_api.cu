// C ABI of the lq library: argument checks, resident objects, dispatch and the
// loop driver (CUDA-graph replay of the T x L schedule).
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <cmath>
#include <map>
#include <memory>
#include <mutex>
#include <string>
#include <vector>

#include "lq_common.cuh"

namespace lq {

static thread_local std::string g_err;

void set_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
}

lq_status cuda_error(cudaError_t e, const char* what) {
  set_error("%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
  return LQ_ERR_CUDA;
}

}  // namespace lq

using namespace lq;

// Resident weights: only the packed 4-bit codes and their float32 steps.  The
// tensor-core GEMM reads an 8-bit operand copy (E4M3 or int8 bytes) and the
// steps transposed (G x N); both are expanded into the caller's workspace by
// each call that runs the GEMM (once per launch, which covers up to 8 loops).
struct lq_wq {
  int64_t N = 0, K = 0, G = 0;
  uint8_t* codes4 = nullptr;   // N x K/2 packed
  float* scales = nullptr;     // N x G
  int device = 0;
  int64_t bytes = 0;
};

struct lq_layer {
  uint64_t id = 0;
  const lq_wq* wq = nullptr;
  int a = 0, b = 0, T = 0, a_bits = 4;
  float* P1 = nullptr;  // device a x a
  float* P2 = nullptr;  // device b x b
  std::vector<float> las;
};

struct lq_cta {
  uint64_t id = 0;
  int64_t d = 0;
  int rank = 0, n_trans = 0;
  double* U8 = nullptr;  // device d x 8 float64, columns >= rank zero
  double* V8 = nullptr;  // device d x 8 float64
  float* a = nullptr;   // device n_trans x d
  float* b = nullptr;   // device n_trans x d
  std::vector<float> eta;
  int device = 0;
};

namespace {

std::atomic<uint64_t> g_layer_ids{1};

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
inline int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

lq_status check_bits_group(int bits, int group, bool allow8) {
  if (group != kGroup) {
    set_error("group size %d is not supported (only 32)", group);
    return LQ_ERR_UNSUPPORTED;
  }
  if (!(bits == 4 || (allow8 && bits == 8))) {
    set_error("bits=%d is not supported", bits);
    return LQ_ERR_UNSUPPORTED;
  }
  return LQ_OK;
}

lq_status check_kron(int64_t K, const float* P1, int a, const float* P2, int b, bool optional) {
  if (optional && P1 == nullptr && P2 == nullptr) {
    if (a != 0 || b != 0) {
      set_error("a and b must be 0 when no Kronecker factors are given");
      return LQ_ERR_ARG;
    }
    return LQ_OK;
  }
  if (P1 == nullptr || P2 == nullptr) {
    set_error("both Kronecker factors must be given");
    return LQ_ERR_ARG;
  }
  if (a <= 0 || b <= 0) {
    set_error("factor sizes must be positive (a=%d, b=%d)", a, b);
    return LQ_ERR_ARG;
  }
  if ((int64_t)a * b != K) {
    set_error("a*b = %d*%d != K = %lld", a, b, (long long)K);
    return LQ_ERR_SHAPE;
  }
  if (a % 16 || b % 8 || a > 128 || b > 128) {
    set_error("Kronecker factor sizes must be a multiple of 16 (a) and of 8 (b), at most 128 "
              "(a=%d, b=%d)", a, b);
    return LQ_ERR_UNSUPPORTED;
  }
  if (rotate_smem_bytes(a, b, nullptr) == 0) {
    set_error("Kronecker factors %dx%d, %dx%d exceed shared memory", a, a, b, b);
    return LQ_ERR_UNSUPPORTED;
  }
  return LQ_OK;
}

lq_status check_mk(int64_t M, int64_t K) {
  if (M < 0 || K <= 0) {
    set_error("invalid shape M=%lld K=%lld", (long long)M, (long long)K);
    return LQ_ERR_ARG;
  }
  if (K % kGroup) {
    set_error("K=%lld is not a multiple of 32", (long long)K);
    return LQ_ERR_SHAPE;
  }
  if (M * K >= (int64_t)1 << 40) {
    set_error("M*K too large");
    return LQ_ERR_SHAPE;
  }
  return LQ_OK;
}

// decode-sized M runs the weight-streaming GEMV while its activation fits in shared memory
bool use_gemv(int64_t M, int64_t K) {
  return M <= kGemvMaxM && K <= 8192 && (size_t)M * (K / kGroup) * 40 <= 200u * 1024u;
}

// workspace: codes (M x K bytes), steps (M x G fp32), and for the GEMV path the
// per-group code sums (M x G int32) and 256 bytes for the persistent chain
// kernel's grid barrier
int64_t ws_bytes_for(int64_t M, int64_t K) {
  const int64_t steps = round_up(M * (K / kGroup) * 4, 256);
  return round_up(M * K, 256) + steps + (use_gemv(M, K) ? steps + 256 : 0);
}

// the GEMM's weight operand in the workspace: N x K code bytes, then the
// steps transposed (G x N float32)
int64_t op_bytes_for(int64_t N, int64_t K) {
  return round_up(N * K, 256) + round_up(N * (K / kGroup) * 4, 256);
}

// workspace of one linear call: activation codes and steps, plus the weight
// operand when the call takes the tensor-core path
int64_t ws_bytes_linear(int64_t M, int64_t K, int64_t N) {
  return round_up(ws_bytes_for(M, K), 256) + (use_gemv(M, K) ? 0 : op_bytes_for(N, K));
}

// Graph cache of the loop driver: one instantiated graph per argument set.
struct GraphKey {
  const void* x;
  int32_t dtype;
  int64_t M;
  std::vector<uint64_t> layer_ids;
  int32_t T, mode;
  float* y;
  void* ws;
  int64_t ws_bytes;
  int device;
  uint64_t cta = 0;
  bool operator<(const GraphKey& o) const {
    if (cta != o.cta) return cta < o.cta;
    if (x != o.x) return x < o.x;
    if (dtype != o.dtype) return dtype < o.dtype;
    if (M != o.M) return M < o.M;
    if (layer_ids != o.layer_ids) return layer_ids < o.layer_ids;
    if (T != o.T) return T < o.T;
    if (mode != o.mode) return mode < o.mode;
    if (y != o.y) return y < o.y;
    if (ws != o.ws) return ws < o.ws;
    if (ws_bytes != o.ws_bytes) return ws_bytes < o.ws_bytes;
    return device < o.device;
  }
};

std::mutex g_graph_mu;
struct CachedGraph {
  cudaGraphExec_t exec;
  uint64_t last_use;
};
std::map<GraphKey, CachedGraph> g_graphs;
uint64_t g_graph_clock = 0;
// at most this many instantiated schedules stay cached (the least recently
// used goes first): callers that pass a new workspace or output buffer on
// every call would otherwise grow the cache without bound
constexpr size_t kMaxCachedGraphs = 64;
std::map<int, cudaStream_t> g_capture_streams;

void drop_graphs_of_layer(uint64_t id) {
  std::lock_guard<std::mutex> lk(g_graph_mu);
  for (auto it = g_graphs.begin(); it != g_graphs.end();) {
    bool uses = it->first.cta == id;
    for (uint64_t l : it->first.layer_ids) uses |= (l == id);
    if (uses) {
      cudaGraphExecDestroy(it->second.exec);
      it = g_graphs.erase(it);
    } else {
      ++it;
    }
  }
}

// Kernel timing probe (see lq_probe_enable): event pairs per kernel kind.
struct Probe {
  std::mutex mu;
  bool on = false;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending[LQ_PROBE_KINDS];
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
Probe g_probe;

enum ProbeKind {
  kProbeRotQuant = 0,
  kProbeQuant = 1,
  kProbeGemm = 2,
  kProbeGemv = 3,
  kProbeWeightOp = 4,
  kProbeChain = 5
};

struct ProbeScope {
  cudaEvent_t a = nullptr, b = nullptr;
  int kind;
  cudaStream_t s;
  ProbeScope(int k, cudaStream_t st) : kind(k), s(st) {
    std::lock_guard<std::mutex> lk(g_probe.mu);
    if (!g_probe.on) return;
    a = g_probe.get();
    b = g_probe.get();
    cudaEventRecord(a, s);
  }
  ~ProbeScope() {
    if (!a) return;
    cudaEventRecord(b, s);
    std::lock_guard<std::mutex> lk(g_probe.mu);
    g_probe.pending[kind].emplace_back(a, b);
  }
};

bool probe_on() {
  std::lock_guard<std::mutex> lk(g_probe.mu);
  return g_probe.on;
}

// Enqueue one looped linear (quantize, then GEMV or GEMM) for loops
// t .. t + nb - 1 of one layer: launch row r is row r % M of loop t + r / M,
// whose input starts x_stride elements after the previous loop's and whose
// output starts y_stride floats after it (nb = 1: one loop, strides unused).
// pdl_first: the quantizer may overlap the previous kernel of the same
// sequence (programmatic dependent launch); x_early: x was written before the
// sequence began.  The consumer kernel always overlaps the quantizer's tail.
lq_status enqueue_linear(const void* x, int32_t x_dtype, int64_t M, const lq_layer* L, int t,
                         float* y, void* ws, cudaStream_t s, bool pdl_first = false,
                         bool x_early = true, int nb = 1, int64_t x_stride = 0,
                         int64_t y_stride = 0) {
  const lq_wq* wq = L->wq;
  const int64_t K = wq->K, N = wq->N, Mt = M * nb;
  const bool gemv = use_gemv(Mt, K);
  const int opf = gemv ? kOpGemvAct : (L->a_bits == 4 ? kOpE4M3 : kOpInt8);
  uint8_t* codes = (uint8_t*)ws;
  float* scales = (float*)((char*)ws + round_up(Mt * K, 256));
  int* asum = gemv ? (int*)((char*)scales + round_up(Mt * (K / kGroup) * 4, 256)) : nullptr;
  if (nb > 1 && (L->P1 == nullptr || nb > kMaxLoopsPerLaunch)) {
    set_error("internal: loop batching needs the rotating quantizer");
    return LQ_ERR_ARG;
  }
  LoopSegs segs = one_loop(L->las[t]);
  if (nb > 1) {
    segs.seg_rows = M;
    segs.x_stride = x_stride;
    for (int j = 0; j < nb; ++j) segs.c[j] = L->las[t + j];
  }
  // no programmatic overlap while the probe brackets each kernel with events
  const bool pdl = !probe_on();
  cudaError_t e;
  {
    ProbeScope ps(kProbeRotQuant, s);
    e = launch_quantize(x, x_dtype, Mt, K, L->P1, L->a, L->P2, L->b, segs, L->a_bits,
                        (int8_t*)codes, opf, nullptr, scales, s, pdl && pdl_first, x_early, asum);
  }
  if (e != cudaSuccess) return cuda_error(e, "quantize launch");
  if (gemv) {
    ProbeScope ps(kProbeGemv, s);
    e = launch_group_gemv((const int8_t*)codes, asum, scales, wq->codes4, wq->scales, y, Mt, N, K,
                          s, pdl, nb > 1 ? M : INT64_MAX, y_stride);
    if (e != cudaSuccess) return cuda_error(e, "gemv launch");
  } else {
    // the weight operand for this launch, expanded from the resident 4-bit codes
    uint8_t* op = (uint8_t*)ws + round_up(ws_bytes_for(Mt, K), 256);
    float* sw_t = (float*)(op + round_up(N * K, 256));
    {
      ProbeScope pw(kProbeWeightOp, s);
      e = launch_weight_operand(wq->codes4, wq->scales, N, K, opf, op, sw_t, s, pdl);
    }
    if (e != cudaSuccess) return cuda_error(e, "weight operand launch");
    ProbeScope ps(kProbeGemm, s);
    const char* why = nullptr;
    e = launch_group_gemm(codes, scales, op, sw_t, y, Mt, N, K, opf, s, &why,
                          pdl, nb > 1 ? M : INT64_MAX, y_stride);
    if (e != cudaSuccess) {
      if (why) {
        set_error("gemm launch: %s", why);
        return LQ_ERR_CUDA;
      }
      return cuda_error(e, "gemm launch");
    }
  }
  return LQ_OK;
}

// Loops of one layer that open mode runs per launch with a workspace of
// ws_bytes.  Batching needs the rotating quantizer (its per-loop row
// segments); a decode-sized M stays on the GEMV path, so its batch is bounded
// by the GEMV's row limit, and each launch then streams the layer's weights
// once for all loops of the batch.
int loops_per_launch(const lq_layer* L, int64_t M, int T, int64_t ws_bytes) {
  const int64_t K = L->wq->K;
  if (L->P1 == nullptr) return 1;
  const bool gemv = use_gemv(M, K);
  int nb = std::min(T, kMaxLoopsPerLaunch);
  while (nb > 1 && ((gemv && !use_gemv(M * nb, K)) ||
                    ws_bytes_linear(M * nb, K, L->wq->N) > ws_bytes ||
                    M * nb > ((int64_t)1 << 31) - 256))
    --nb;
  return nb;
}

// Loops per GEMV launch of a decode-sized open-mode stack: the most loops of
// every layer whose rows still fit the GEMV path (1 when a layer does not
// rotate).
int decode_loops_per_launch(const std::vector<const lq_layer*>& tl, int64_t M, int T) {
  int nb = std::min(T, kMaxLoopsPerLaunch);
  for (const lq_layer* ly : tl) {
    if (ly->P1 == nullptr) return 1;
    while (nb > 1 && !use_gemv(M * nb, ly->wq->K)) --nb;
  }
  return nb;
}

// Decode-sized open-mode stacks: the (t, l) steps are independent, so they
// run as kDecodeBranches concurrent chains (quantize, then GEMV, each chain
// with its own slice of the workspace), forked from and joined back into the
// caller's stream.  Per device: the branch streams and the fork/join events.
constexpr int kDecodeBranches = 16;
struct BranchSet {
  cudaStream_t st[kDecodeBranches];
  cudaEvent_t fork;
  cudaEvent_t join[kDecodeBranches];
};
std::mutex g_branch_mu;
std::map<int, BranchSet> g_branch_sets;

lq_status branch_set(BranchSet** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  auto it = g_branch_sets.find(dev);
  if (it == g_branch_sets.end()) {
    BranchSet b{};
    for (int i = 0; i < kDecodeBranches; ++i) {
      if ((e = cudaStreamCreateWithFlags(&b.st[i], cudaStreamNonBlocking)) != cudaSuccess)
        return cuda_error(e, "create branch stream");
      if ((e = cudaEventCreateWithFlags(&b.join[i], cudaEventDisableTiming)) != cudaSuccess)
        return cuda_error(e, "create branch event");
    }
    if ((e = cudaEventCreateWithFlags(&b.fork, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_error(e, "create branch event");
    it = g_branch_sets.emplace(dev, b).first;
  }
  *out = &it->second;
  return LQ_OK;
}

// workspace slice of one decode branch (the largest layer's codes, steps and sums)
int64_t decode_branch_bytes(const std::vector<const lq_layer*>& tl, int64_t M) {
  int64_t per = 0;
  for (const lq_layer* ly : tl) per = std::max(per, round_up(ws_bytes_for(M, ly->wq->K), 256));
  return per;
}

// The work units of a decode-sized open-mode stack (tl: T x L handles): loops
// t .. t + w - 1 of layer l in one quantize and one GEMV launch, w = nbd when
// one handle serves all of those loops, else one unit per loop.
struct DecodeUnit {
  int t, l, w;
};
void decode_units(const std::vector<const lq_layer*>& tl, int L, int T, int nbd,
                  std::vector<DecodeUnit>* units) {
  units->clear();
  for (int t = 0; t < T; t += nbd) {
    const int nb = std::min(nbd, T - t);
    for (int l = 0; l < L; ++l) {
      bool same = true;
      for (int j = 1; j < nb; ++j) same = same && tl[(size_t)(t + j) * L + l] == tl[(size_t)t * L + l];
      if (same)
        units->push_back({t, l, nb});
      else
        for (int j = 0; j < nb; ++j) units->push_back({t + j, l, 1});
    }
  }
}

lq_status check_layer_call(const lq_layer* layer, int64_t M, int32_t x_dtype) {
  if (!layer) {
    set_error("null layer");
    return LQ_ERR_ARG;
  }
  if (x_dtype != LQ_F32 && x_dtype != LQ_BF16) {
    set_error("unsupported x dtype %d", x_dtype);
    return LQ_ERR_UNSUPPORTED;
  }
  if (M < 0) {
    set_error("negative M");
    return LQ_ERR_ARG;
  }
  const bool gemm = !use_gemv(M, layer->wq->K);
  if (gemm && layer->wq->K % 128) {
    set_error("K=%lld must be a multiple of 128 for the tensor-core path (M > %d)",
              (long long)layer->wq->K, kGemvMaxM);
    return LQ_ERR_SHAPE;
  }
  if (M > ((int64_t)1 << 31) - 256 || layer->wq->N > ((int64_t)1 << 30)) {
    set_error("M or N too large");
    return LQ_ERR_SHAPE;
  }
  return LQ_OK;
}

}  // namespace

extern "C" {

const char* lq_last_error(void) { return g_err.c_str(); }

int32_t lq_version(void) { return 100; }

int64_t lq_act_scale_bytes(int64_t M, int64_t K) { return M * (K / kGroup) * 4; }

lq_status lq_quantize_act(const void* d_x, int32_t x_dtype, int64_t M, int64_t K,
                          const float* d_P1, int32_t a, const float* d_P2, int32_t b,
                          float las_t, int32_t bits, int32_t group, int8_t* d_codes8,
                          uint8_t* d_codes4, float* d_scales, void* stream) {
  lq_status st;
  if ((st = check_mk(M, K)) != LQ_OK) return st;
  if ((st = check_bits_group(bits, group, true)) != LQ_OK) return st;
  if ((st = check_kron(K, d_P1, a, d_P2, b, true)) != LQ_OK) return st;
  if (x_dtype != LQ_F32 && x_dtype != LQ_BF16) {
    set_error("unsupported x dtype %d", x_dtype);
    return LQ_ERR_UNSUPPORTED;
  }
  if (!(las_t > 0.f) || !std::isfinite(las_t)) {
    set_error("LAS clip must be a positive finite number (got %g)", (double)las_t);
    return LQ_ERR_ARG;
  }
  if (M > 0 && (d_x == nullptr || d_scales == nullptr || (d_codes8 == nullptr && d_codes4 == nullptr))) {
    set_error("null input or output pointer");
    return LQ_ERR_ARG;
  }
  if (d_codes4 && bits != 4) {
    set_error("packed 4-bit output requested for bits=%d", bits);
    return LQ_ERR_UNSUPPORTED;
  }
  if (!aligned16(d_x) || !aligned16(d_codes8) || !aligned16(d_codes4) || !aligned16(d_scales)) {
    set_error("input and output pointers must be 16-byte aligned");
    return LQ_ERR_ALIGN;
  }
  cudaError_t e = launch_quantize(d_x, x_dtype, M, K, d_P1, a, d_P2, b, one_loop(las_t), bits,
                                  d_codes8, kOpInt8, d_codes4, d_scales, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_error(e, "quantize launch");
  return LQ_OK;
}

lq_status lq_fold_weights(const float* d_W, int64_t N, int64_t K, const float* d_Q1, int32_t a,
                          const float* d_Q2, int32_t b, float* d_W_out, void* stream) {
  lq_status st;
  if (N < 0 || K <= 0) {
    set_error("invalid shape");
    return LQ_ERR_ARG;
  }
  if (K % 8) {
    set_error("K must be a multiple of 8");
    return LQ_ERR_SHAPE;
  }
  if ((st = check_kron(K, d_Q1, a, d_Q2, b, false)) != LQ_OK) return st;
  if (N > 0 && (!d_W || !d_W_out)) {
    set_error("null pointer");
    return LQ_ERR_ARG;
  }
  if (!aligned16(d_W) || !aligned16(d_W_out)) {
    set_error("pointers must be 16-byte aligned");
    return LQ_ERR_ALIGN;
  }
  if (d_W == d_W_out && N > 0) {
    set_error("input and output may not alias");
    return LQ_ERR_ARG;
  }
  cudaError_t e = launch_rotate_store(d_W, N, K, d_Q1, a, d_Q2, b, d_W_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_error(e, "fold launch");
  return LQ_OK;
}

lq_status lq_inverse_transpose(const float* h_P, int32_t n, float* h_out) {
  if (!h_P || !h_out || n <= 0 || n > 4096) {
    set_error("invalid arguments");
    return LQ_ERR_ARG;
  }
  // Gauss-Jordan with partial pivoting on [P | I] in float64
  std::vector<double> A((size_t)n * n), I((size_t)n * n, 0.0);
  for (int i = 0; i < n * n; ++i) A[i] = h_P[i];
  for (int i = 0; i < n; ++i) I[(size_t)i * n + i] = 1.0;
  for (int col = 0; col < n; ++col) {
    int piv = col;
    for (int r = col + 1; r < n; ++r)
      if (std::fabs(A[(size_t)r * n + col]) > std::fabs(A[(size_t)piv * n + col])) piv = r;
    if (A[(size_t)piv * n + col] == 0.0) {
      set_error("matrix is singular");
      return LQ_ERR_ARG;
    }
    if (piv != col)
      for (int c = 0; c < n; ++c) {
        std::swap(A[(size_t)piv * n + c], A[(size_t)col * n + c]);
        std::swap(I[(size_t)piv * n + c], I[(size_t)col * n + c]);
      }
    const double d = A[(size_t)col * n + col];
    for (int c = 0; c < n; ++c) {
      A[(size_t)col * n + c] /= d;
      I[(size_t)col * n + c] /= d;
    }
    for (int r = 0; r < n; ++r) {
      if (r == col) continue;
      const double f = A[(size_t)r * n + col];
      if (f == 0.0) continue;
      for (int c = 0; c < n; ++c) {
        A[(size_t)r * n + c] -= f * A[(size_t)col * n + c];
        I[(size_t)r * n + c] -= f * I[(size_t)col * n + c];
      }
    }
  }
  // out = (P^-1)^T
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) h_out[(size_t)i * n + j] = (float)I[(size_t)j * n + i];
  return LQ_OK;
}

lq_status lq_quantize_weights(const float* d_W, int64_t N, int64_t K, int32_t bits, int32_t group,
                              int8_t* d_codes8, uint8_t* d_codes4, float* d_scales,
                              void* stream) {
  lq_status st;
  if ((st = check_mk(N, K)) != LQ_OK) return st;
  if ((st = check_bits_group(bits, group, false)) != LQ_OK) return st;
  if (N > 0 && (!d_W || !d_scales || (!d_codes8 && !d_codes4))) {
    set_error("null pointer");
    return LQ_ERR_ARG;
  }
  if (!aligned16(d_W) || !aligned16(d_codes8) || !aligned16(d_codes4) || !aligned16(d_scales)) {
    set_error("pointers must be 16-byte aligned");
    return LQ_ERR_ALIGN;
  }
  cudaError_t e = launch_quantize(d_W, LQ_F32, N, K, nullptr, 0, nullptr, 0, one_loop(1.0f), 4,
                                  d_codes8, kOpInt8, d_codes4, d_scales, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_error(e, "weight quantize launch");
  return LQ_OK;
}

lq_status lq_pack_weights(const float* d_W_folded, int64_t N, int64_t K, int32_t bits,
                          int32_t group, lq_wq** out, void* stream) {
  lq_status st;
  if (!out) {
    set_error("null output handle");
    return LQ_ERR_ARG;
  }
  *out = nullptr;
  if (N <= 0) {
    set_error("N must be positive");
    return LQ_ERR_ARG;
  }
  if ((st = check_mk(N, K)) != LQ_OK) return st;
  if ((st = check_bits_group(bits, group, false)) != LQ_OK) return st;
  if (!d_W_folded) {
    set_error("null weight pointer");
    return LQ_ERR_ARG;
  }
  if (!aligned16(d_W_folded)) {
    set_error("weight pointer must be 16-byte aligned");
    return LQ_ERR_ALIGN;
  }
  cudaStream_t s = (cudaStream_t)stream;
  lq_wq* w = new lq_wq();
  w->N = N;
  w->K = K;
  w->G = K / kGroup;
  cudaGetDevice(&w->device);
  cudaError_t e;
  const size_t b4 = (size_t)N * K / 2, bs = (size_t)N * w->G * 4;
  if ((e = cudaMalloc(&w->codes4, b4)) != cudaSuccess ||
      (e = cudaMalloc(&w->scales, bs)) != cudaSuccess) {
    lq_wq_free(w);
    set_error("cudaMalloc of %zu bytes failed: %s", b4 + bs, cudaGetErrorString(e));
    return LQ_ERR_NOMEM;
  }
  w->bytes = (int64_t)(b4 + bs);
  e = launch_quantize(d_W_folded, LQ_F32, N, K, nullptr, 0, nullptr, 0, one_loop(1.0f), 4,
                      nullptr, kOpInt8, w->codes4, w->scales, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    lq_wq_free(w);
    return cuda_error(e, "pack weights");
  }
  *out = w;
  return LQ_OK;
}

lq_status lq_wq_info(const lq_wq* wq, int64_t* N, int64_t* K, const uint8_t** d_codes4,
                     const float** d_scales, int64_t* device_bytes) {
  if (!wq) {
    set_error("null handle");
    return LQ_ERR_ARG;
  }
  if (N) *N = wq->N;
  if (K) *K = wq->K;
  if (d_codes4) *d_codes4 = wq->codes4;
  if (d_scales) *d_scales = wq->scales;
  if (device_bytes) *device_bytes = wq->bytes;
  return LQ_OK;
}

void lq_wq_free(lq_wq* wq) {
  if (!wq) return;
  cudaFree(wq->codes4);
  cudaFree(wq->scales);

  delete wq;
}

lq_status lq_layer_create(const lq_wq* wq, const float* d_P1, int32_t a, const float* d_P2,
                          int32_t b, const float* h_las, int32_t T, int32_t a_bits,
                          lq_layer** out) {
  if (!out) {
    set_error("null output handle");
    return LQ_ERR_ARG;
  }
  *out = nullptr;
  if (!wq || !h_las || T <= 0) {
    set_error("null weights, null LAS clips or T <= 0");
    return LQ_ERR_ARG;
  }
  lq_status st;
  if ((st = check_kron(wq->K, d_P1, a, d_P2, b, false)) != LQ_OK) return st;
  if (a_bits != 4 && a_bits != 8) {
    set_error("a_bits=%d is not supported", a_bits);
    return LQ_ERR_UNSUPPORTED;
  }
  for (int t = 0; t < T; ++t)
    if (!(h_las[t] > 0.f) || !std::isfinite(h_las[t])) {
      set_error("LAS clip %d is not a positive finite number", t);
      return LQ_ERR_ARG;
    }
  lq_layer* L = new lq_layer();
  L->id = g_layer_ids.fetch_add(1);
  L->wq = wq;
  L->a = a;
  L->b = b;
  L->T = T;
  L->a_bits = a_bits;
  L->las.assign(h_las, h_las + T);
  cudaError_t e;
  if ((e = cudaMalloc(&L->P1, (size_t)a * a * 4)) != cudaSuccess ||
      (e = cudaMalloc(&L->P2, (size_t)b * b * 4)) != cudaSuccess) {
    lq_layer_free(L);
    set_error("cudaMalloc failed: %s", cudaGetErrorString(e));
    return LQ_ERR_NOMEM;
  }
  if ((e = cudaMemcpy(L->P1, d_P1, (size_t)a * a * 4, cudaMemcpyDeviceToDevice)) != cudaSuccess ||
      (e = cudaMemcpy(L->P2, d_P2, (size_t)b * b * 4, cudaMemcpyDeviceToDevice)) != cudaSuccess) {
    lq_layer_free(L);
    return cuda_error(e, "copy Kronecker factors");
  }
  *out = L;
  return LQ_OK;
}

void lq_layer_free(lq_layer* layer) {
  if (!layer) return;
  drop_graphs_of_layer(layer->id);
  cudaFree(layer->P1);
  cudaFree(layer->P2);
  delete layer;
}

int64_t lq_workspace_bytes(const lq_layer* const* layers, int32_t L, int64_t M) {
  if (!layers || L <= 0 || M < 0) return -1;
  int64_t need = 0;
  for (int i = 0; i < L; ++i) {
    if (!layers[i]) return -1;
    need = std::max(need, ws_bytes_linear(M, layers[i]->wq->K, layers[i]->wq->N));
  }
  return need;
}

int64_t lq_stack_workspace_bytes(const lq_layer* const* layers, int32_t L, int64_t M,
                                 int32_t T) {
  if (!layers || L <= 0 || M < 0 || T <= 0) return -1;
  int64_t need = 0;
  for (int i = 0; i < L; ++i) {
    if (!layers[i]) return -1;
    const int64_t K = layers[i]->wq->K;
    const int nb = loops_per_launch(layers[i], M, T, INT64_MAX);
    need = std::max(need, ws_bytes_linear(M * nb, K, layers[i]->wq->N));
  }
  bool decode = (int64_t)T * L > 1;
  for (int i = 0; i < L; ++i) decode = decode && use_gemv(M, layers[i]->wq->K);
  const std::vector<const lq_layer*> tl(layers, layers + L);
  if (decode) {  // one workspace region per unit of a grouped round (covers the chains)
    const int nbd = decode_loops_per_launch(tl, M, T);
    const int64_t units = (int64_t)((T + nbd - 1) / nbd) * L;
    need = std::max(need, decode_branch_bytes(tl, M * nbd) *
                              std::min<int64_t>(std::max<int64_t>(kGroupMaxUnits, kDecodeBranches),
                                                units));
  }
  return need;
}

lq_status lq_loop_linear(const void* d_x, int32_t x_dtype, int64_t M, const lq_layer* layer,
                         int32_t t, float* d_y, void* d_ws, int64_t ws_bytes, void* stream) {
  lq_status st;
  if ((st = check_layer_call(layer, M, x_dtype)) != LQ_OK) return st;
  if (t < 0 || t >= layer->T) {
    set_error("loop index t=%d outside [0, %d)", t, layer->T);
    return LQ_ERR_SHAPE;
  }
  if (M == 0) return LQ_OK;
  if (!d_x || !d_y || !d_ws) {
    set_error("null pointer");
    return LQ_ERR_ARG;
  }
  if (!aligned16(d_x) || !aligned16(d_y) || ((uintptr_t)d_ws & 255u)) {
    set_error("x and y must be 16-byte aligned and the workspace 256-byte aligned");
    return LQ_ERR_ALIGN;
  }
  if (ws_bytes < ws_bytes_linear(M, layer->wq->K, layer->wq->N)) {
    set_error("workspace of %lld bytes is smaller than the %lld needed", (long long)ws_bytes,
              (long long)ws_bytes_linear(M, layer->wq->K, layer->wq->N));
    return LQ_ERR_WORKSPACE;
  }
  return enqueue_linear(d_x, x_dtype, M, layer, t, d_y, d_ws, (cudaStream_t)stream);
}

// The T x L schedule over a table of handles: step (t, l) applies tl[t * L + l].
static lq_status enqueue_stack(const void* d_x, int32_t x_dtype, int64_t M,
                               const std::vector<const lq_layer*>& tl, int32_t L, int32_t T,
                               int32_t mode, float* d_y, void* d_ws, int64_t ws_bytes,
                               cudaStream_t s, const lq_cta* cta = nullptr) {
  const size_t esz = x_dtype == LQ_BF16 ? 2 : 4;
  auto at = [&](int t, int l) { return tl[(size_t)t * L + l]; };
  if (mode == LQ_OPEN) {
    // step (t, l) reads x at element offset M * (t * sum_K + sum_{l' < l} K_l') and
    // writes y at M * (t * sum_N + sum_{l' < l} N_l'); loops of a layer are
    // independent, so consecutive loops that use the same handle share launches
    int64_t sum_k = 0, sum_n = 0;
    for (int l = 0; l < L; ++l) {
      sum_k += at(0, l)->wq->K;
      sum_n += at(0, l)->wq->N;
    }
    bool decode = T * L > 1;
    for (const lq_layer* ly : tl) decode = decode && use_gemv(M, ly->wq->K);
    if (decode) {
      // units of work: the loops t .. t + nbd - 1 of layer l in one quantize
      // and one GEMV launch (the weights streamed once for them) when the
      // same handle serves all of them, else one unit per loop
      std::vector<DecodeUnit> units;
      int nbd = decode_loops_per_launch(tl, M, T);
      decode_units(tl, L, T, nbd, &units);
      std::vector<int64_t> k_before(L, 0), n_before(L, 0);
      for (int l = 1; l < L; ++l) {
        k_before[l] = k_before[l - 1] + at(0, l - 1)->wq->K;
        n_before[l] = n_before[l - 1] + at(0, l - 1)->wq->N;
      }
      // all units in one quantize and one GEMV launch (per round of up to
      // kGroupMaxUnits units), when their shapes fit the grouped kernels and
      // the workspace holds a region per unit of a round
      {
        const int64_t per = decode_branch_bytes(tl, M * nbd);
        bool ok = ws_bytes >= per * std::min<int64_t>(kGroupMaxUnits, (int64_t)units.size());
        for (const DecodeUnit& u : units) {
          const lq_layer* ly = at(u.t, u.l);
          ok = ok && ly->P1 != nullptr && use_gemv(M * u.w, ly->wq->K) &&
               group_unit_ok(M * u.w, ly->wq->K, ly->a, ly->b);
        }
        if (ok) {
          const bool pdl = !probe_on();
          std::unique_ptr<GroupLaunch> P(new GroupLaunch());
          // rounds of equal size
          const size_t n_rounds = (units.size() + kGroupMaxUnits - 1) / kGroupMaxUnits;
          const size_t per_round = (units.size() + n_rounds - 1) / n_rounds;
          for (size_t r0 = 0; r0 < units.size(); r0 += per_round) {
            const int n = (int)std::min(per_round, units.size() - r0);
            P->n_units = n;
            for (int i = 0; i < n; ++i) {
              const DecodeUnit& u = units[r0 + i];
              const lq_layer* ly = at(u.t, u.l);
              const int64_t K = ly->wq->K, rows = M * u.w;
              GroupUnit& g = P->u[i];
              char* reg = (char*)d_ws + (size_t)i * per;
              g.x = (const char*)d_x + (size_t)(M * (u.t * sum_k + k_before[u.l])) * esz;
              g.P1 = ly->P1;
              g.P2 = ly->P2;
              g.w4 = ly->wq->codes4;
              g.sw = ly->wq->scales;
              g.y = d_y + M * (u.t * sum_n + n_before[u.l]);
              g.codes = (int8_t*)reg;
              g.scales = (float*)(reg + round_up(rows * K, 256));
              g.asum = (int*)((char*)g.scales + round_up(rows * (K / kGroup) * 4, 256));
              g.x_stride = M * sum_k;
              g.y_stride = M * sum_n;
              for (int j = 0; j < kMaxLoopsPerLaunch; ++j)
                g.c[j] = j < u.w ? ly->las[u.t + j] : 0.f;
              g.K = (int)K;
              g.N = (int)ly->wq->N;
              g.a = ly->a;
              g.b = ly->b;
              g.seg_rows = (int)M;
              g.rows = (int)rows;
              g.qmax = ly->a_bits == 8 ? 127 : 7;
              g.blk0 = 0;
            }
            cudaError_t e;
            {
              ProbeScope ps(kProbeRotQuant, s);
              e = launch_quantize_units(*P, x_dtype, s, pdl && r0 > 0);
            }
            if (e != cudaSuccess) return cuda_error(e, "grouped quantize launch");
            {
              ProbeScope ps(kProbeGemv, s);
              e = launch_gemv_units(*P, s, pdl);
            }
            if (e != cudaSuccess) return cuda_error(e, "grouped gemv launch");
          }
          return LQ_OK;
        }
      }
      int64_t per = decode_branch_bytes(tl, M * nbd);
      if (nbd > 1 && ws_bytes < 2 * per) {
        while (nbd > 1 && ws_bytes < 2 * per) per = decode_branch_bytes(tl, M * --nbd);
        decode_units(tl, L, T, nbd, &units);
      }
      const int nbr = (int)std::min(std::min((int64_t)kDecodeBranches, (int64_t)units.size()),
                                    ws_bytes / per);
      if (nbr >= 2) {
        std::lock_guard<std::mutex> lk(g_branch_mu);
        BranchSet* bs = nullptr;
        lq_status st = branch_set(&bs);
        if (st != LQ_OK) return st;
        cudaError_t e = cudaEventRecord(bs->fork, s);
        if (e != cudaSuccess) return cuda_error(e, "fork record");
        for (int b = 0; b < nbr; ++b)
          if ((e = cudaStreamWaitEvent(bs->st[b], bs->fork, 0)) != cudaSuccess)
            return cuda_error(e, "fork wait");
        for (size_t i = 0; i < units.size() && st == LQ_OK; ++i) {
          const DecodeUnit& u = units[i];
          const int b = (int)(i % nbr);
          const char* xin =
              (const char*)d_x + (size_t)(M * (u.t * sum_k + k_before[u.l])) * esz;
          float* yout = d_y + M * (u.t * sum_n + n_before[u.l]);
          st = enqueue_linear(xin, x_dtype, M, at(u.t, u.l), u.t, yout,
                              (char*)d_ws + (size_t)b * per, bs->st[b], i >= (size_t)nbr, true,
                              u.w, M * sum_k, M * sum_n);
        }
        // join every branch back (also after an error, so no capture is left unjoined)
        for (int b = 0; b < nbr; ++b) {
          cudaError_t e1 = cudaEventRecord(bs->join[b], bs->st[b]);
          cudaError_t e2 = e1 == cudaSuccess ? cudaStreamWaitEvent(s, bs->join[b], 0) : e1;
          if (e2 != cudaSuccess && st == LQ_OK) st = cuda_error(e2, "join");
        }
        return st;
      }
    }
    int nb_all = kMaxLoopsPerLaunch;
    for (const lq_layer* ly : tl) nb_all = std::min(nb_all, loops_per_launch(ly, M, T, ws_bytes));
    bool first = true;
    for (int t = 0; t < T; t += nb_all) {
      const int nb = std::min(nb_all, T - t);
      int64_t k_before = 0, n_before = 0;
      for (int l = 0; l < L; ++l) {
        const lq_layer* ly = at(t, l);
        bool same = true;  // one handle for every loop of the batch
        for (int j = 1; j < nb; ++j) same = same && at(t + j, l) == ly;
        for (int j = 0; j < nb; j += same ? nb : 1) {
          const int w = same ? nb : 1;
          const char* xin = (const char*)d_x + (size_t)(M * ((t + j) * sum_k + k_before)) * esz;
          float* yout = d_y + M * ((t + j) * sum_n + n_before);
          lq_status st = enqueue_linear(xin, x_dtype, M, at(t + j, l), t + j, yout, d_ws, s,
                                        !first, true, w, M * sum_k, M * sum_n);
          if (st != LQ_OK) return st;
          first = false;
        }
        k_before += ly->wq->K;
        n_before += ly->wq->N;
      }
    }
    return LQ_OK;
  }
  // decode-sized chain mode without CTA: every step in one persistent kernel
  // (launches of up to kChainMaxSteps steps)
  if (!cta && (int64_t)T * L > 1) {
    bool ok = true;
    size_t act = 0, fac = 0, wts = 0;
    int64_t kmax = 0;
    for (const lq_layer* ly : tl) {
      size_t a1 = 0, f1 = 0, w1 = 0;
      ok = ok && ly->P1 != nullptr && use_gemv(M, ly->wq->K) &&
           chain_decode_ok((int)M, (int)ly->wq->K, (int)ly->wq->N, ly->a, ly->b, &a1, &f1, &w1);
      act = std::max(act, a1);
      fac = std::max(fac, f1);
      wts = std::max(wts, w1);
      kmax = std::max(kmax, ly->wq->K);
    }
    const size_t smem = act + fac + wts;
    if (ok && smem <= 220u * 1024u && ws_bytes >= ws_bytes_for(M, kmax)) {
      std::unique_ptr<ChainLaunch> P(new ChainLaunch());
      const int64_t steps_b = round_up(M * (kmax / kGroup) * 4, 256);
      P->M = (int)M;
      P->act_bytes = (int)act;
      P->fac_bytes = (int)fac;
      P->codes = (int8_t*)d_ws;
      P->scales = (float*)((char*)d_ws + round_up(M * kmax, 256));
      P->asum = (int*)((char*)P->scales + steps_b);
      P->bar = (unsigned*)((char*)P->asum + steps_b);
      float* yc = d_y;
      const void* xin = d_x;
      bool x_bf16 = x_dtype == LQ_BF16;
      int n = 0;
      for (int t = 0; t < T; ++t) {
        for (int l = 0; l < L; ++l) {
          const lq_layer* ly = at(t, l);
          ChainStep& c = P->s[n++];
          c.x = xin;
          c.P1 = ly->P1;
          c.P2 = ly->P2;
          c.w4 = ly->wq->codes4;
          c.sw = ly->wq->scales;
          c.y = yc;
          c.c = ly->las[t];
          c.K = (int)ly->wq->K;
          c.N = (int)ly->wq->N;
          c.a = ly->a;
          c.b = ly->b;
          c.qmax = ly->a_bits == 8 ? 127 : 7;
          c.x_bf16 = x_bf16 ? 1 : 0;
          xin = yc;
          x_bf16 = false;
          yc += M * ly->wq->N;
          if (n == kChainMaxSteps || (t == T - 1 && l == L - 1)) {
            P->n_steps = n;
            cudaError_t e;
            {
              ProbeScope ps(kProbeChain, s);
              e = launch_chain_decode(*P, smem, s);
            }
            if (e != cudaSuccess) return cuda_error(e, "chain decode launch");
            n = 0;
          }
        }
      }
      return LQ_OK;
    }
  }
  float* ycur = d_y;
  const float* prev_y = nullptr;
  // CTA state (the adapted input of the next loop) after the codes and steps
  int64_t codes_ws = 0;
  for (const lq_layer* ly : tl)
    codes_ws = std::max(codes_ws, ws_bytes_linear(M, ly->wq->K, ly->wq->N));
  float* state = (float*)((char*)d_ws + round_up(codes_ws, 256));
  for (int t = 0; t < T; ++t) {
    for (int l = 0; l < L; ++l) {
      const lq_layer* ly = at(t, l);
      const void* xin = prev_y ? (const void*)prev_y : d_x;
      const int32_t dt = prev_y ? LQ_F32 : x_dtype;
      // every linear after the first overlaps its predecessor; its input is
      // the previous output, written inside the sequence
      const bool first = prev_y == nullptr;
      lq_status st = enqueue_linear(xin, dt, M, ly, t, ycur, d_ws, s, !first, first);
      if (st != LQ_OK) return st;
      prev_y = ycur;
      ycur += M * ly->wq->N;
    }
    if (cta && t + 1 < T) {  // loop transition t -> t + 1
      cudaError_t e = launch_cta_apply(prev_y, M, (int)cta->d, cta->U8, cta->V8,
                                       cta->a + (size_t)t * cta->d, cta->b + (size_t)t * cta->d,
                                       cta->eta[t], state, s, !probe_on());
      if (e != cudaSuccess) return cuda_error(e, "cta launch");
      prev_y = state;
    }
  }
  return LQ_OK;
}

// Checks, graph cache and launch of the schedule over a (t, l) table of handles.
static lq_status loop_stack_impl(const void* d_x, int32_t x_dtype, int64_t M,
                                 const std::vector<const lq_layer*>& tl, int32_t L, int32_t T,
                                 int32_t mode, float* d_y, void* d_ws, int64_t ws_bytes,
                                 void* stream, const lq_cta* cta = nullptr) {
  if (mode != LQ_OPEN && mode != LQ_CHAIN) {
    set_error("unknown mode %d", mode);
    return LQ_ERR_ARG;
  }
  lq_status st;
  int64_t need = 0;
  for (int t = 0; t < T; ++t) {
    for (int l = 0; l < L; ++l) {
      const lq_layer* ly = tl[(size_t)t * L + l];
      if ((st = check_layer_call(ly, M, x_dtype)) != LQ_OK) return st;
      if (ly->T <= t) {
        set_error("layer (t=%d, l=%d) has %d LAS clips", t, l, ly->T);
        return LQ_ERR_SHAPE;
      }
      const lq_layer* l0 = tl[l];
      if (ly->wq->K != l0->wq->K || ly->wq->N != l0->wq->N) {
        set_error("layer (t=%d, l=%d) is %lldx%lld, loop 0 has %lldx%lld", t, l,
                  (long long)ly->wq->N, (long long)ly->wq->K, (long long)l0->wq->N,
                  (long long)l0->wq->K);
        return LQ_ERR_SHAPE;
      }
      need = std::max(need, ws_bytes_linear(M, ly->wq->K, ly->wq->N));
    }
  }
  if (mode == LQ_CHAIN) {
    for (int l = 0; l < L; ++l) {
      const int64_t next_k = tl[(l + 1) % L]->wq->K;
      if (tl[l]->wq->N != next_k) {
        set_error("chain mode needs N_%d == K_%d", l, (l + 1) % L);
        return LQ_ERR_SHAPE;
      }
    }
  }
  if (cta) {
    if (mode != LQ_CHAIN) {
      set_error("transition alignment needs chain mode");
      return LQ_ERR_ARG;
    }
    if (cta->d != tl[L - 1]->wq->N) {
      set_error("CTA width %lld != state width %lld", (long long)cta->d,
                (long long)tl[L - 1]->wq->N);
      return LQ_ERR_SHAPE;
    }
    if (cta->n_trans < T - 1) {
      set_error("CTA has %d transitions, T=%d needs %d", cta->n_trans, T, T - 1);
      return LQ_ERR_SHAPE;
    }
    need = round_up(need, 256) + round_up(M * cta->d * 4, 256);
  }
  if (M == 0) return LQ_OK;
  if (!d_x || !d_y || !d_ws) {
    set_error("null pointer");
    return LQ_ERR_ARG;
  }
  if (!aligned16(d_x) || !aligned16(d_y) || ((uintptr_t)d_ws & 255u)) {
    set_error("x and y must be 16-byte aligned and the workspace 256-byte aligned");
    return LQ_ERR_ALIGN;
  }
  if (ws_bytes < need) {
    set_error("workspace too small");
    return LQ_ERR_WORKSPACE;
  }
  cudaStream_t s = (cudaStream_t)stream;
  // within a caller's own capture, record the kernels into it directly
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cap);
  if (e != cudaSuccess) return cuda_error(e, "stream query");
  if (cap != cudaStreamCaptureStatusNone || probe_on())
    return enqueue_stack(d_x, x_dtype, M, tl, L, T, mode, d_y, d_ws, ws_bytes, s, cta);

  GraphKey key;
  key.x = d_x;
  key.dtype = x_dtype;
  key.M = M;
  for (const lq_layer* ly : tl) key.layer_ids.push_back(ly->id);
  key.T = T;
  key.mode = mode;
  key.y = d_y;
  key.ws = d_ws;
  key.ws_bytes = ws_bytes;
  key.cta = cta ? cta->id : 0;
  cudaGetDevice(&key.device);

  std::lock_guard<std::mutex> lk(g_graph_mu);
  auto it = g_graphs.find(key);
  if (it == g_graphs.end()) {
    cudaStream_t cs;
    auto sit = g_capture_streams.find(key.device);
    if (sit == g_capture_streams.end()) {
      if ((e = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking)) != cudaSuccess)
        return cuda_error(e, "create capture stream");
      g_capture_streams[key.device] = cs;
    } else {
      cs = sit->second;
    }
    if ((e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal)) != cudaSuccess)
      return cuda_error(e, "begin capture");
    st = enqueue_stack(d_x, x_dtype, M, tl, L, T, mode, d_y, d_ws, ws_bytes, cs, cta);
    cudaGraph_t g = nullptr;
    e = cudaStreamEndCapture(cs, &g);
    if (st != LQ_OK) {
      if (g) cudaGraphDestroy(g);
      return st;
    }
    if (e != cudaSuccess) return cuda_error(e, "end capture");
    cudaGraphExec_t ge = nullptr;
    e = cudaGraphInstantiate(&ge, g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) return cuda_error(e, "instantiate graph");
    if (g_graphs.size() >= kMaxCachedGraphs) {
      auto old = g_graphs.begin();
      for (auto jt = g_graphs.begin(); jt != g_graphs.end(); ++jt)
        if (jt->second.last_use < old->second.last_use) old = jt;
      // a graph still running on some stream stays valid: destruction is deferred
      cudaGraphExecDestroy(old->second.exec);
      g_graphs.erase(old);
    }
    it = g_graphs.emplace(key, CachedGraph{ge, 0}).first;
  }
  it->second.last_use = ++g_graph_clock;
  e = cudaGraphLaunch(it->second.exec, s);
  if (e != cudaSuccess) return cuda_error(e, "graph launch");
  return LQ_OK;
}

lq_status lq_loop_stack(const void* d_x, int32_t x_dtype, int64_t M,
                        const lq_layer* const* layers, int32_t L, int32_t T, int32_t mode,
                        float* d_y, void* d_ws, int64_t ws_bytes, void* stream) {
  if (!layers || L <= 0 || T <= 0) {
    set_error("need at least one layer and one loop");
    return LQ_ERR_ARG;
  }
  for (int l = 0; l < L; ++l) {
    if (layers[l] && layers[l]->T < T) {
      set_error("layer %d has %d LAS clips but T=%d", l, layers[l]->T, T);
      return LQ_ERR_SHAPE;
    }
  }
  std::vector<const lq_layer*> tl((size_t)T * L);
  for (int t = 0; t < T; ++t)
    for (int l = 0; l < L; ++l) tl[(size_t)t * L + l] = layers[l];
  return loop_stack_impl(d_x, x_dtype, M, tl, L, T, mode, d_y, d_ws, ws_bytes, stream);
}

lq_status lq_loop_stack_slt(const void* d_x, int32_t x_dtype, int64_t M,
                            const lq_layer* const* layers_tl, int32_t L, int32_t T, int32_t mode,
                            float* d_y, void* d_ws, int64_t ws_bytes, void* stream) {
  if (!layers_tl || L <= 0 || T <= 0) {
    set_error("need at least one layer and one loop");
    return LQ_ERR_ARG;
  }
  std::vector<const lq_layer*> tl(layers_tl, layers_tl + (size_t)T * L);
  return loop_stack_impl(d_x, x_dtype, M, tl, L, T, mode, d_y, d_ws, ws_bytes, stream);
}

lq_status lq_cta_create(const float* d_U, const float* d_V, int64_t d, int32_t rank,
                        const float* d_a, const float* d_b, const float* h_eta, int32_t n_trans,
                        lq_cta** out) {
  if (!out || !d_U || !d_V || !d_a || !d_b || !h_eta) {
    set_error("null pointer");
    return LQ_ERR_ARG;
  }
  *out = nullptr;
  if (d <= 0 || d > (1 << 24) || rank <= 0 || rank > 8 || n_trans <= 0) {
    set_error("CTA needs d > 0, 1 <= rank <= 8 and at least one transition");
    return LQ_ERR_ARG;
  }
  for (int t = 0; t < n_trans; ++t) {
    if (!std::isfinite(h_eta[t])) {
      set_error("gate %d is not finite", t);
      return LQ_ERR_ARG;
    }
  }
  if (d % 32 || d > 6144) {
    set_error("CTA width d=%lld must be a multiple of 32 and at most 6144", (long long)d);
    return LQ_ERR_SHAPE;
  }
  lq_cta* c = new lq_cta();
  c->d = d;
  c->rank = rank;
  c->n_trans = n_trans;
  c->eta.assign(h_eta, h_eta + n_trans);
  cudaGetDevice(&c->device);
  // U, V to float64 d x 8 (zero columns past the rank), converted on the host
  std::vector<float> hu((size_t)d * rank), hv((size_t)d * rank);
  std::vector<double> u8((size_t)d * 8, 0.0), v8((size_t)d * 8, 0.0);
  const size_t b8 = u8.size() * sizeof(double), bt = (size_t)n_trans * d * sizeof(float);
  cudaError_t e = cudaMemcpy(hu.data(), d_U, hu.size() * sizeof(float), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess)
    e = cudaMemcpy(hv.data(), d_V, hv.size() * sizeof(float), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) {
    for (int64_t k = 0; k < d; ++k)
      for (int q = 0; q < rank; ++q) {
        u8[k * 8 + q] = hu[k * rank + q];
        v8[k * 8 + q] = hv[k * rank + q];
      }
  }
  if (e == cudaSuccess) e = cudaMalloc(&c->U8, b8);
  if (e == cudaSuccess) e = cudaMalloc(&c->V8, b8);
  if (e == cudaSuccess) e = cudaMalloc(&c->a, bt);
  if (e == cudaSuccess) e = cudaMalloc(&c->b, bt);
  if (e == cudaSuccess) e = cudaMemcpy(c->U8, u8.data(), b8, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(c->V8, v8.data(), b8, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(c->a, d_a, bt, cudaMemcpyDeviceToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(c->b, d_b, bt, cudaMemcpyDeviceToDevice);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    lq_cta_free(c);
    return cuda_error(e, "cta create");
  }
  c->id = g_layer_ids.fetch_add(1);
  *out = c;
  return LQ_OK;
}

void lq_cta_free(lq_cta* c) {
  if (!c) return;
  drop_graphs_of_layer(c->id);
  cudaFree(c->U8);
  cudaFree(c->V8);
  cudaFree(c->a);
  cudaFree(c->b);
  delete c;
}

lq_status lq_cta_apply(const float* d_h, int64_t M, const lq_cta* cta, int32_t t, float* d_out,
                       void* stream) {
  if (!cta) {
    set_error("null CTA");
    return LQ_ERR_ARG;
  }
  if (M < 0) {
    set_error("negative M");
    return LQ_ERR_ARG;
  }
  if (t < 0 || t >= cta->n_trans) {
    set_error("transition t=%d outside [0, %d)", t, cta->n_trans);
    return LQ_ERR_SHAPE;
  }
  if (M == 0) return LQ_OK;
  if (!d_h || !d_out) {
    set_error("null pointer");
    return LQ_ERR_ARG;
  }
  if (!aligned16(d_h) || !aligned16(d_out)) {
    set_error("h and out must be 16-byte aligned");
    return LQ_ERR_ALIGN;
  }
  cudaError_t e = launch_cta_apply(d_h, M, (int)cta->d, cta->U8, cta->V8,
                                   cta->a + (size_t)t * cta->d, cta->b + (size_t)t * cta->d,
                                   cta->eta[t], d_out, (cudaStream_t)stream, false);
  if (e != cudaSuccess) return cuda_error(e, "cta launch");
  return LQ_OK;
}

int64_t lq_cta_stack_workspace_bytes(const lq_layer* const* layers, int32_t L, int64_t M) {
  if (!layers || L <= 0 || M < 0 || !layers[L - 1]) return -1;
  const int64_t base = lq_workspace_bytes(layers, L, M);
  if (base < 0) return -1;
  return round_up(base, 256) + round_up(M * layers[L - 1]->wq->N * 4, 256);
}

lq_status lq_loop_stack_cta(const void* d_x, int32_t x_dtype, int64_t M,
                            const lq_layer* const* layers, int32_t L, int32_t T,
                            const lq_cta* cta, float* d_y, void* d_ws, int64_t ws_bytes,
                            void* stream) {
  if (!layers || L <= 0 || T <= 0 || !cta) {
    set_error("need layers, loops and a CTA");
    return LQ_ERR_ARG;
  }
  for (int l = 0; l < L; ++l) {
    if (layers[l] && layers[l]->T < T) {
      set_error("layer %d has %d LAS clips but T=%d", l, layers[l]->T, T);
      return LQ_ERR_SHAPE;
    }
  }
  std::vector<const lq_layer*> tl((size_t)T * L);
  for (int t = 0; t < T; ++t)
    for (int l = 0; l < L; ++l) tl[(size_t)t * L + l] = layers[l];
  return loop_stack_impl(d_x, x_dtype, M, tl, L, T, LQ_CHAIN, d_y, d_ws, ws_bytes, stream, cta);
}

int64_t lq_hessian_workspace_bytes(int64_t M, int64_t K, int32_t T) {
  if (M < 0 || K <= 0 || T <= 0) return -1;
  return round_up(K * hessian_rows_padded(M * T) * 2, 256);
}

lq_status lq_trajectory_hessian(const void* d_X, int32_t x_dtype, int64_t M, int64_t K,
                                int32_t T, float* d_H, int32_t accumulate, void* d_ws,
                                int64_t ws_bytes, void* stream) {
  if (x_dtype != LQ_BF16) {
    set_error("the trajectory Hessian takes bf16 inputs (products exact in float32)");
    return LQ_ERR_UNSUPPORTED;
  }
  if (M < 0 || K <= 0 || T <= 0) {
    set_error("invalid shape M=%lld K=%lld T=%d", (long long)M, (long long)K, T);
    return LQ_ERR_ARG;
  }
  if (K % 128 || K > 65536) {
    set_error("K=%lld must be a multiple of 128 and at most 65536", (long long)K);
    return LQ_ERR_SHAPE;
  }
  if (!d_H) {
    set_error("null H");
    return LQ_ERR_ARG;
  }
  if (!aligned16(d_H)) {
    set_error("H must be 16-byte aligned");
    return LQ_ERR_ALIGN;
  }
  cudaStream_t s = (cudaStream_t)stream;
  if (M == 0) {  // no rows: H = 0, or unchanged when accumulating
    if (accumulate) return LQ_OK;
    cudaError_t e = cudaMemsetAsync(d_H, 0, (size_t)K * K * sizeof(float), s);
    return e == cudaSuccess ? LQ_OK : cuda_error(e, "clear H");
  }
  if (!d_X || !d_ws) {
    set_error("null pointer");
    return LQ_ERR_ARG;
  }
  if (!aligned16(d_X) || ((uintptr_t)d_ws & 255u)) {
    set_error("X must be 16-byte aligned and the workspace 256-byte aligned");
    return LQ_ERR_ALIGN;
  }
  if (M * T > ((int64_t)1 << 31) - 64) {
    set_error("too many rows");
    return LQ_ERR_SHAPE;
  }
  if (ws_bytes < lq_hessian_workspace_bytes(M, K, T)) {
    set_error("workspace too small");
    return LQ_ERR_WORKSPACE;
  }
  const char* why = nullptr;
  cudaError_t e = launch_trajectory_hessian((const uint16_t*)d_X, M * T, K, (uint16_t*)d_ws, d_H,
                                            accumulate ? 1 : 0, s, &why);
  if (e != cudaSuccess) {
    if (why) {
      set_error("trajectory Hessian: %s", why);
      return LQ_ERR_CUDA;
    }
    return cuda_error(e, "trajectory Hessian launch");
  }
  return LQ_OK;
}

lq_status lq_probe_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_probe.mu);
  g_probe.on = on != 0;
  return LQ_OK;
}

lq_status lq_probe_read(double* h_ms, int64_t* h_count) {
  if (!h_ms || !h_count) {
    set_error("null output");
    return LQ_ERR_ARG;
  }
  std::lock_guard<std::mutex> lk(g_probe.mu);
  lq_status st = LQ_OK;
  for (int k = 0; k < LQ_PROBE_KINDS; ++k) {
    double tot = 0.0;
    for (auto& pr : g_probe.pending[k]) {
      cudaError_t e = cudaEventSynchronize(pr.second);
      float ms = 0.f;
      if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, pr.first, pr.second);
      if (e != cudaSuccess && st == LQ_OK) st = cuda_error(e, "probe event");
      tot += ms;
      g_probe.pool.push_back(pr.first);
      g_probe.pool.push_back(pr.second);
    }
    h_ms[k] = tot;
    h_count[k] = (int64_t)g_probe.pending[k].size();
    g_probe.pending[k].clear();
  }
  return st;
}

lq_status lq_selftest_bounded_wait(int64_t limit_us, void* stream) {
  if (limit_us <= 0 || limit_us > 10000000) {
    set_error("limit must be in (0, 10 s]");
    return LQ_ERR_ARG;
  }
  cudaError_t e = launch_wait_selftest((uint64_t)limit_us * 1000u, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_error(e, "self-test launch");
  return LQ_OK;
}

lq_status lq_selftest_grid_wait(int64_t limit_us, void* d_scratch, void* stream) {
  if (limit_us <= 0 || limit_us > 10000000) {
    set_error("limit must be in (0, 10 s]");
    return LQ_ERR_ARG;
  }
  if (!d_scratch || (uintptr_t)d_scratch % 4) {
    set_error("scratch must be 8 bytes of 4-byte aligned device memory");
    return LQ_ERR_ARG;
  }
  cudaError_t e = launch_grid_wait_selftest((uint64_t)limit_us * 1000u, (cudaStream_t)stream,
                                            (unsigned*)d_scratch);
  if (e != cudaSuccess) return cuda_error(e, "self-test launch");
  return LQ_OK;
}

lq_status lq_check_device(void* stream) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "pending CUDA error");
  lq_status st = read_and_clear_device_status((cudaStream_t)stream);
  if (st != LQ_OK) return st;
  // bounds-check build: an index a kernel found out of range (none otherwise)
  const char* files[4] = {"lq_quant.cu", "lq_gemm.cu", "lq_gemv.cu", "lq_cta.cu"};
  const unsigned long long v[4] = {bounds_fail_quant(), bounds_fail_gemm(), bounds_fail_gemv(),
                                   bounds_fail_cta()};
  for (int i = 0; i < 4; ++i)
    if (v[i]) {
      set_error("index out of range in %s line %llu (index %lld)", files[i], v[i] >> 40,
                (long long)(v[i] & 0xFFFFFFFFFFull));
      return LQ_ERR_DEVICE_BOUNDS;
    }
  return LQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// helpers for lq_loop_linear_noalloc (lq_noalloc.cu): the same checks and the
// same kernels as lq_loop_linear, with the workspace supplied by the caller
// of these helpers
// ---------------------------------------------------------------------------
namespace lq {

lq_status noalloc_check(const void* d_x, int32_t x_dtype, int64_t M, const lq_layer* layer,
                        int32_t t, float* d_y) {
  lq_status st;
  if ((st = check_layer_call(layer, M, x_dtype)) != LQ_OK) return st;
  if (t < 0 || t >= layer->T) {
    set_error("loop index t=%d outside [0, %d)", t, layer->T);
    return LQ_ERR_SHAPE;
  }
  if (M == 0) return LQ_OK;
  if (!d_x || !d_y) {
    set_error("null pointer");
    return LQ_ERR_ARG;
  }
  if (!aligned16(d_x) || !aligned16(d_y)) {
    set_error("x and y must be 16-byte aligned");
    return LQ_ERR_ALIGN;
  }
  return LQ_OK;
}

int64_t noalloc_ws_bytes(const lq_layer* layer, int64_t M) {
  return ws_bytes_linear(M, layer->wq->K, layer->wq->N);
}

lq_status noalloc_enqueue(const void* d_x, int32_t x_dtype, int64_t M, const lq_layer* layer,
                          int32_t t, float* d_y, void* d_ws, cudaStream_t s) {
  return enqueue_linear(d_x, x_dtype, M, layer, t, d_y, d_ws, s);
}

}  // namespace lq
