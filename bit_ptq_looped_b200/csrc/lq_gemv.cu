// Decode-sized group-rescaled GEMV (M <= 16 tokens), weight streaming from HBM.
//
//   y[m,n] = sum_g s_a[m,g] s_w[n,g] sum_{k in g} q_a[m,k] q_w[n,k]
//
// Same arithmetic as the tensor-core GEMM, for the decode regime where each
// loop reads the packed 4-bit weights once and the activation is a handful of
// rows.  A warp walks weight rows n; lane L owns groups L, L+32, ...: one
// 16-byte load brings the 32 packed codes of a group, one 4-byte load its
// step.  The activation codes of all M rows sit in shared memory, rearranged
// so a group's even and odd elements form separate 32-bit words that match
// the low and high nibbles of the packed weights.
//
// Integer dot: weight nibble v (two's complement q_w) is read as v ^ 8 =
// q_w + 8 in [1, 15], so dp4a(unsigned weights, signed activations) gives
// sum (q_w + 8) q_a; subtracting 8 * sum q_a (precomputed per row and group)
// leaves the exact sum q_w q_a.
#include <algorithm>

#include "lq_common.cuh"

namespace lq {
namespace {

constexpr int kGemvThreads = 256;
constexpr int kRowsPerIter = 2;

__device__ __forceinline__ int dp4a_us(uint32_t a_unsigned, uint32_t b_signed, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_unsigned), "r"(b_signed), "r"(c));
  return d;
}

// shared layout: act[m][i][g] = uint2{even word, odd word} of word i (0..3) of
// group g of row m;  asum[m][g] = sum of the group's codes;  sa[m][g] steps.
template <int MB>
__global__ void __launch_bounds__(kGemvThreads) k_group_gemv(
    const int8_t* __restrict__ qa, const float* __restrict__ sa, const uint8_t* __restrict__ w4,
    const float* __restrict__ sw, float* __restrict__ y, int M, int N, int K) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int G = K / kGroup;
  uint2* act = reinterpret_cast<uint2*>(smem_raw);                        // M*4*G
  int* asum = reinterpret_cast<int*>(act + (size_t)M * 4 * G);           // M*G
  float* ssa = reinterpret_cast<float*>(asum + (size_t)M * G);           // M*G

  // ---- stage the activation: one thread per 8-code chunk, 4 chunks per group
  const int n_chunks = M * K / 8;
  for (int base = 0; base < n_chunks; base += kGemvThreads) {
    const int ch = base + threadIdx.x;
    const bool valid = ch < n_chunks;
    uint2 raw = make_uint2(0, 0);
    if (valid) raw = __ldg(reinterpret_cast<const uint2*>(qa) + ch);
    // bytes c0..c7 -> even word (c0,c2,c4,c6), odd word (c1,c3,c5,c7)
    const uint32_t ev = __byte_perm(raw.x, raw.y, 0x6420);
    const uint32_t od = __byte_perm(raw.x, raw.y, 0x7531);
    int s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      s += (int)(int8_t)((raw.x >> (8 * i)) & 0xFF) + (int)(int8_t)((raw.y >> (8 * i)) & 0xFF);
    s += __shfl_xor_sync(0xFFFFFFFFu, s, 1);
    s += __shfl_xor_sync(0xFFFFFFFFu, s, 2);
    if (valid) {
      const int m = ch / (K / 8);
      const int rem = ch - m * (K / 8);
      const int g = rem >> 2, i = rem & 3;
      act[((size_t)m * 4 + i) * G + g] = make_uint2(ev, od);
      if (i == 0) {
        asum[m * G + g] = s;
        ssa[m * G + g] = sa[(size_t)m * G + g];
      }
    }
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (kGemvThreads / 32);
  const int rowstride = K / 2;  // bytes per packed weight row
  for (int n0 = (blockIdx.x * (kGemvThreads / 32) + warp) * kRowsPerIter; n0 < N;
       n0 += warps_total * kRowsPerIter) {
    float part[kRowsPerIter][MB];
#pragma unroll
    for (int r = 0; r < kRowsPerIter; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m) part[r][m] = 0.f;
    for (int g = lane; g < G; g += 32) {
      uint4 wv[kRowsPerIter];
      float swv[kRowsPerIter];
#pragma unroll
      for (int r = 0; r < kRowsPerIter; ++r) {
        const int n = min(n0 + r, N - 1);
        wv[r] = __ldg(reinterpret_cast<const uint4*>(w4 + (size_t)n * rowstride) + g);
        swv[r] = __ldg(sw + (size_t)n * G + g);
      }
#pragma unroll
      for (int r = 0; r < kRowsPerIter; ++r) {
        const uint32_t wu[4] = {wv[r].x ^ 0x88888888u, wv[r].y ^ 0x88888888u,
                                wv[r].z ^ 0x88888888u, wv[r].w ^ 0x88888888u};
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          if (m < M) {
            int d = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint2 av = act[((size_t)m * 4 + i) * G + g];
              d = dp4a_us(wu[i] & 0x0F0F0F0Fu, av.x, d);
              d = dp4a_us((wu[i] >> 4) & 0x0F0F0F0Fu, av.y, d);
            }
            d -= 8 * asum[m * G + g];
            part[r][m] = fmaf(ssa[m * G + g] * swv[r], (float)d, part[r][m]);
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kRowsPerIter; ++r) {
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        float v = part[r][m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        part[r][m] = v;
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < kRowsPerIter; ++r) {
        const int n = n0 + r;
        if (n < N) {
#pragma unroll
          for (int m = 0; m < MB; ++m)
            if (m < M) y[(size_t)m * N + n] = part[r][m];
        }
      }
    }
  }
}

template <int MB>
cudaError_t launch_mb(const int8_t* qa, const float* sa, const uint8_t* w4, const float* sw,
                      float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s) {
  const int64_t G = K / kGroup;
  const size_t smem = (size_t)M * 4 * G * 8 + (size_t)M * G * 8;
  auto* k = k_group_gemv<MB>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t warps_needed = (N + kRowsPerIter - 1) / kRowsPerIter;
  const int64_t blocks = (warps_needed + 7) / 8;
  const int grid = (int)std::min<int64_t>(blocks, (int64_t)num_sms() * 4);
  k<<<grid, kGemvThreads, smem, s>>>(qa, sa, w4, sw, y, (int)M, (int)N, (int)K);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_group_gemv(const int8_t* qa, const float* sa, const uint8_t* w4,
                              const float* sw, float* y, int64_t M, int64_t N, int64_t K,
                              cudaStream_t s) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (M <= 1) return launch_mb<1>(qa, sa, w4, sw, y, M, N, K, s);
  if (M <= 4) return launch_mb<4>(qa, sa, w4, sw, y, M, N, K, s);
  return launch_mb<16>(qa, sa, w4, sw, y, M, N, K, s);
}

}  // namespace lq
