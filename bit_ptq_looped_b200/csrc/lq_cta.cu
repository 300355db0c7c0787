// Cross-loop transition alignment (CTA) at loop transitions (sm_100a).
//
//   h' = a_t * h + b_t + eta_t * (h V) U^T,   U, V: d x r (r <= 8), a_t, b_t: d
//
// ("paper_specification.yaml" of the LoopQ reproduction: cta, Section 4.3,
// Eq. (7); implementation_status lq5: an affine plus gated low-rank adapter
// applied only at loop transitions, U and V shared, a_t, b_t and eta_t
// loop-dependent, rank 8, identity at initialization.  Eq. (7) is not printed
// on the pages; this is the plainest reading of that description.)
//
// Every product and sum is float64 and the result is rounded once to float32,
// the precision of the carried state.  A warp takes 4 rows at a time: pass 1
// forms the r projections p = h V of each row (each lane over the columns
// lane, lane + 32, ..., then a butterfly over the warp), pass 2 writes
// a*h + b + eta * p U^T.  One load of a row of U or V serves the 4 rows.
// The kernel is memory-bound (h read twice from L2, written once; U, V, a, b
// from L1) plus 18 d float64 FMAs per row.
#include <algorithm>

#include "lq_common.cuh"

namespace lq {
namespace {

constexpr int kCtaThreads = 256;
constexpr int kCtaRowsPerWarp = 4;

__global__ void __launch_bounds__(kCtaThreads) k_cta_apply(
    const float* __restrict__ h, int64_t M, int d, const float* __restrict__ U8,
    const float* __restrict__ V8, const float* __restrict__ a, const float* __restrict__ b,
    float eta, float* __restrict__ out) {
  pdl_trigger();
  pdl_wait();  // h is the previous kernel's output
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * kCtaThreads + threadIdx.x) >> 5;
  const int64_t n_warps = ((int64_t)gridDim.x * kCtaThreads) >> 5;
  const double e = (double)eta;
  for (int64_t r0 = warp0 * kCtaRowsPerWarp; r0 < M; r0 += n_warps * kCtaRowsPerWarp) {
    const int nr = M - r0 < kCtaRowsPerWarp ? (int)(M - r0) : kCtaRowsPerWarp;
    // ---- pass 1: p[i][q] = sum_k h[r0 + i][k] V[k][q]
    double p[kCtaRowsPerWarp][8];
#pragma unroll
    for (int i = 0; i < kCtaRowsPerWarp; ++i)
#pragma unroll
      for (int q = 0; q < 8; ++q) p[i][q] = 0.0;
    for (int k = lane; k < d; k += 32) {
      const float4 v0 = __ldg(reinterpret_cast<const float4*>(V8 + (size_t)k * 8));
      const float4 v1 = __ldg(reinterpret_cast<const float4*>(V8 + (size_t)k * 8) + 1);
      const double vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int i = 0; i < kCtaRowsPerWarp; ++i) {
        if (i < nr) {
          const double hv = (double)__ldg(h + (size_t)(r0 + i) * d + k);
#pragma unroll
          for (int q = 0; q < 8; ++q) p[i][q] = fma(hv, vv[q], p[i][q]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kCtaRowsPerWarp; ++i)
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) p[i][q] += __shfl_xor_sync(0xFFFFFFFFu, p[i][q], o);
    // ---- pass 2: out = a h + b + eta (p U^T)
    for (int k = lane; k < d; k += 32) {
      const float4 u0 = __ldg(reinterpret_cast<const float4*>(U8 + (size_t)k * 8));
      const float4 u1 = __ldg(reinterpret_cast<const float4*>(U8 + (size_t)k * 8) + 1);
      const double uu[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      const double ak = (double)__ldg(a + k), bk = (double)__ldg(b + k);
#pragma unroll
      for (int i = 0; i < kCtaRowsPerWarp; ++i) {
        if (i < nr) {
          double lr = 0.0;
#pragma unroll
          for (int q = 0; q < 8; ++q) lr = fma(p[i][q], uu[q], lr);
          const double hv = (double)__ldg(h + (size_t)(r0 + i) * d + k);
          out[(size_t)(r0 + i) * d + k] = __double2float_rn(fma(ak, hv, bk) + e * lr);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_cta_apply(const float* h, int64_t M, int d, const float* U8, const float* V8,
                             const float* a, const float* b, float eta, float* out,
                             cudaStream_t s, bool pdl) {
  if (M == 0) return cudaSuccess;
  const int64_t warps = (M + kCtaRowsPerWarp - 1) / kCtaRowsPerWarp;
  const int64_t want = (warps * 32 + kCtaThreads - 1) / kCtaThreads;
  const int grid = (int)std::min<int64_t>(want, (int64_t)num_sms() * 8);
  return launch_kernel(k_cta_apply, dim3(grid), dim3(kCtaThreads), 0, s, pdl, h, M, d, U8, V8,
                       a, b, eta, out);
}

}  // namespace lq
