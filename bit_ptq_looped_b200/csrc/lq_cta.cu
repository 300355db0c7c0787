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
// the precision of the carried state.  Both contractions run on the FP64
// tensor-core MMA (m8n8k4): a block takes 8 rows; pass 1 forms p = h V
// (8 x 8) with each warp summing a 1/8 slice of the d columns and the slices
// added in shared memory; pass 2 forms p U^T one 8-column tile per MMA pair,
// the warps taking tiles in turn, and writes a*h + b + eta * (p U^T) from the
// accumulator fragments.  U and V are held as float64 d x 8 (rank padded with
// zero columns), so no fragment needs a conversion except the h loads.
#include <algorithm>

#include "lq_common.cuh"

namespace lq {
namespace {

constexpr int kCtaThreads = 256;
constexpr int kCtaWarps = kCtaThreads / 32;

__device__ __forceinline__ void dmma_884(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

// fragments (lane = 4 g + t): A[g][t], B[t][g], C[g][2t], C[g][2t + 1]
__global__ void __launch_bounds__(kCtaThreads) k_cta_apply(
    const float* h, int64_t M, int d, const double* __restrict__ U8,
    const double* __restrict__ V8, const float* __restrict__ a, const float* __restrict__ b,
    float eta, float* out) {
  __shared__ double pp[kCtaWarps][8][8];  // per-warp partial projections
  __shared__ double ps[8][8];             // p = h V of the block's 8 rows
  pdl_trigger();
  pdl_wait();  // h is the previous kernel's output
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const double e = (double)eta;
  const int slice = d / kCtaWarps;  // columns per warp in pass 1 (a multiple of 4)
  const int n_tiles = d >> 3;
  for (int64_t r0 = (int64_t)blockIdx.x * 8; r0 < M; r0 += (int64_t)gridDim.x * 8) {
    const int64_t row = r0 + g;
    const bool row_ok = row < M;
    const float* hrow = h + (row_ok ? row : r0) * (int64_t)d;
    // ---- pass 1: this warp's slice of p = h V
    double acc[2] = {0.0, 0.0};
    const int k0 = warp * slice;
#pragma unroll 8
    for (int k = k0; k < k0 + slice; k += 4) {
      const double av = row_ok ? (double)hrow[k + t] : 0.0;  // h may alias out: no .nc loads
      const double bv = __ldg(V8 + (size_t)(k + t) * 8 + g);
      dmma_884(acc, av, bv);
    }
    pp[warp][g][2 * t] = acc[0];
    pp[warp][g][2 * t + 1] = acc[1];
    __syncthreads();
    if (threadIdx.x < 64) {
      const int rr = threadIdx.x >> 3, cc = threadIdx.x & 7;
      double sum = 0.0;
#pragma unroll
      for (int w = 0; w < kCtaWarps; ++w) sum += pp[w][rr][cc];
      ps[rr][cc] = sum;
    }
    __syncthreads();
    // ---- pass 2: p U^T by 8-column tiles, then the affine part
    const double pa0 = ps[g][t], pa1 = ps[g][t + 4];
#pragma unroll 4
    for (int tile = warp; tile < n_tiles; tile += kCtaWarps) {
      const int j0 = tile * 8;
      double c[2] = {0.0, 0.0};
      dmma_884(c, pa0, __ldg(U8 + (size_t)(j0 + g) * 8 + t));
      dmma_884(c, pa1, __ldg(U8 + (size_t)(j0 + g) * 8 + t + 4));
      if (row_ok) {
        const int j = j0 + 2 * t;
        const float2 hv = *reinterpret_cast<const float2*>(hrow + j);
        const float2 av = __ldg(reinterpret_cast<const float2*>(a + j));
        const float2 bv = __ldg(reinterpret_cast<const float2*>(b + j));
        const float o0 = __double2float_rn(fma((double)av.x, (double)hv.x, (double)bv.x) + e * c[0]);
        const float o1 = __double2float_rn(fma((double)av.y, (double)hv.y, (double)bv.y) + e * c[1]);
        *reinterpret_cast<float2*>(out + row * (int64_t)d + j) = make_float2(o0, o1);
      }
    }
    __syncthreads();  // pp and ps are reused by the next 8 rows
  }
}

}  // namespace

cudaError_t launch_cta_apply(const float* h, int64_t M, int d, const double* U8, const double* V8,
                             const float* a, const float* b, float eta, float* out,
                             cudaStream_t s, bool pdl) {
  if (M == 0) return cudaSuccess;
  if (d % 32) return cudaErrorInvalidValue;
  const int64_t want = (M + 7) / 8;
  const int grid = (int)std::min<int64_t>(want, (int64_t)num_sms() * 8);
  return launch_kernel(k_cta_apply, dim3(grid), dim3(kCtaThreads), 0, s, pdl, h, M, d, U8, V8,
                       a, b, eta, out);
}

}  // namespace lq
