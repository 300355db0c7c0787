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
// the precision of the carried state.  A block takes 8 rows: it copies them to
// shared memory with 16-byte loads (row pitch d + 4 floats, so the MMA
// fragment reads of 8 rows fall in distinct banks), then pass 1 forms
// p = h V (8 x 8) on the FP64 tensor-core MMA (m8n8k4) with each warp summing
// a 1/8 slice of the d columns and the slices added in shared memory, and
// pass 2 forms p U^T one 8-column tile per MMA pair, the warps taking tiles in
// turn, and writes a*h + b + eta * (p U^T) from the accumulator fragments.  U
// and V are held as float64 d x 8 (rank padded with zero columns).
#include <algorithm>
#include <atomic>

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
  extern __shared__ __align__(16) float hs[];  // 8 rows, pitch d + 4
  __shared__ double pp[kCtaWarps][8][8];        // per-warp partial projections
  __shared__ double ps[8][8];                   // p = h V of the block's 8 rows
  pdl_trigger();
  pdl_wait();  // h is the previous kernel's output
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int ld = d + 4;
  const double e = (double)eta;
  const int slice = d / kCtaWarps;  // columns per warp in pass 1 (a multiple of 4)
  const int n_tiles = d >> 3;
  const int d4 = d >> 2;
  for (int64_t r0 = (int64_t)blockIdx.x * 8; r0 < M; r0 += (int64_t)gridDim.x * 8) {
    const int nr = M - r0 < 8 ? (int)(M - r0) : 8;
    // ---- the block's rows to shared memory (zeros past the last row), four
    // 16-byte loads of each thread in flight at a time
    for (int base = 0; base < 8 * d4; base += 4 * kCtaThreads) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * kCtaThreads + threadIdx.x;
        const int rr = i / d4, c4 = i - rr * d4;
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < 8 * d4 && rr < nr)
          v[u] = *reinterpret_cast<const float4*>(h + (r0 + rr) * (int64_t)d + 4 * c4);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * kCtaThreads + threadIdx.x;
        const int rr = i / d4, c4 = i - rr * d4;
        if (i < 8 * d4) *reinterpret_cast<float4*>(hs + rr * ld + 4 * c4) = v[u];
      }
    }
    __syncthreads();
    // ---- pass 1: this warp's slice of p = h V
    double acc[2] = {0.0, 0.0};
    const int k0 = warp * slice;
#pragma unroll 8
    for (int k = k0; k < k0 + slice; k += 4)
      dmma_884(acc, (double)hs[g * ld + k + t], __ldg(V8 + (size_t)(k + t) * 8 + g));
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
    const bool row_ok = g < nr;
#pragma unroll 4
    for (int tile = warp; tile < n_tiles; tile += kCtaWarps) {
      const int j0 = tile * 8;
      double c[2] = {0.0, 0.0};
      dmma_884(c, pa0, __ldg(U8 + (size_t)(j0 + g) * 8 + t));
      dmma_884(c, pa1, __ldg(U8 + (size_t)(j0 + g) * 8 + t + 4));
      if (row_ok) {
        const int j = j0 + 2 * t;
        const float2 hv = *reinterpret_cast<const float2*>(hs + g * ld + j);
        const float2 av = __ldg(reinterpret_cast<const float2*>(a + j));
        const float2 bv = __ldg(reinterpret_cast<const float2*>(b + j));
        const float o0 = __double2float_rn(fma((double)av.x, (double)hv.x, (double)bv.x) + e * c[0]);
        const float o1 = __double2float_rn(fma((double)av.y, (double)hv.y, (double)bv.y) + e * c[1]);
        *reinterpret_cast<float2*>(out + (r0 + g) * (int64_t)d + j) = make_float2(o0, o1);
      }
    }
    __syncthreads();  // hs, pp and ps are reused by the next 8 rows
  }
}

}  // namespace

size_t cta_smem_bytes(int d) { return (size_t)8 * (d + 4) * sizeof(float); }

cudaError_t launch_cta_apply(const float* h, int64_t M, int d, const double* U8, const double* V8,
                             const float* a, const float* b, float eta, float* out,
                             cudaStream_t s, bool pdl) {
  if (M == 0) return cudaSuccess;
  const size_t smem = cta_smem_bytes(d);
  if (d % 32 || smem > 200u * 1024u) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> attr_dev_mask{0};  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (!((attr_dev_mask.load() >> (dev & 63)) & 1u)) {
    cudaError_t e = cudaFuncSetAttribute(k_cta_apply, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         200 * 1024);
    if (e != cudaSuccess) return e;
    attr_dev_mask.fetch_or(1ull << (dev & 63));
  }
  const int64_t want = (M + 7) / 8;
  const int grid = (int)std::min<int64_t>(want, (int64_t)num_sms() * 8);
  return launch_kernel(k_cta_apply, dim3(grid), dim3(kCtaThreads), smem, s, pdl, h, M, d, U8, V8,
                       a, b, eta, out);
}

unsigned long long bounds_fail_cta() { return lq_take_bounds_fail(); }

}  // namespace lq
