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
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
lq_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("device index %d out of range", dev);
    return LQ_ERR_ARG;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress of the static scratch");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
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
