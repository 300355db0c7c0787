// lq_loop_linear_noalloc: lq_loop_linear for callers that cannot allocate
// device memory.  Its scratch (the activation codes and steps of one call)
// lives in a fixed, file-scope device array that every GPU loading this
// library holds until the process exits.
#include <mutex>

#include "lq_common.cuh"

namespace lq {

lq_status noalloc_check(const void* d_x, int32_t x_dtype, int64_t M, const lq_layer* layer,
                        int32_t t, float* d_y);
int64_t noalloc_ws_bytes(const lq_layer* layer, int64_t M);
lq_status noalloc_enqueue(const void* d_x, int32_t x_dtype, int64_t M, const lq_layer* layer,
                          int32_t t, float* d_y, void* d_ws, cudaStream_t s);

namespace {

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, not a device address: host code must go through scratch_address().
static __device__ __align__(256) unsigned char g_noalloc_scratch[LQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
struct ScratchEntry {
  void* ctx;  // the context the address belongs to
  void* ptr;
};
ScratchEntry g_scratch[kMaxDevices] = {};

using CtxGetCurrentFn = int (*)(void**);  // cuCtxGetCurrent(CUcontext*)

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the scratch on the current device, looked up with that
// device current and cached per device together with the context it belongs
// to: after a device reset (a new primary context, the module loaded again,
// possibly elsewhere) the address is looked up again.
lq_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("device index %d out of range", dev);
    return LQ_ERR_ARG;
  }
  e = cudaSetDevice(dev);  // the same device: makes its primary context current
  if (e != cudaSuccess) return cuda_error(e, "cudaSetDevice");
  CtxGetCurrentFn get = ctx_get_current();
  void* ctx = nullptr;
  if (get == nullptr || get(&ctx) != 0 || ctx == nullptr) {
    set_error("cannot query the current CUDA context");
    return LQ_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchEntry& ent = g_scratch[dev];
  if (ent.ptr == nullptr || ent.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress of the static scratch");
    ent.ctx = ctx;
    ent.ptr = p;
  }
  *out = ent.ptr;
  return LQ_OK;
}

}  // namespace
}  // namespace lq

extern "C" lq_status lq_loop_linear_noalloc(const void* d_x, int32_t x_dtype, int64_t M,
                                            const lq_layer* layer, int32_t t, float* d_y,
                                            void* stream) {
  using namespace lq;
  lq_status st = noalloc_check(d_x, x_dtype, M, layer, t, d_y);
  if (st != LQ_OK) return st;
  const int64_t need = noalloc_ws_bytes(layer, M);
  if (need > (int64_t)LQ_NOALLOC_SCRATCH_BYTES) {
    set_error("M=%lld needs %lld bytes of scratch but the static scratch holds %lld; "
              "split the call or use lq_loop_linear with a workspace",
              (long long)M, (long long)need, (long long)LQ_NOALLOC_SCRATCH_BYTES);
    return LQ_ERR_WORKSPACE;
  }
  if (M == 0) return LQ_OK;
  void* ws = nullptr;
  if ((st = scratch_address(&ws)) != LQ_OK) return st;
  // every byte the kernels read from the scratch is written earlier in the
  // same call (codes and steps of all M rows), so nothing needs clearing
  return noalloc_enqueue(d_x, x_dtype, M, layer, t, d_y, ws, (cudaStream_t)stream);
}
