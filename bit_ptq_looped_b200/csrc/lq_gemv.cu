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
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvGroupsPerLane = 8;  // K <= 8192: each lane owns at most 8 groups of a row

__device__ __forceinline__ int dp4a_us(uint32_t a_unsigned, uint32_t b_signed, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_unsigned), "r"(b_signed), "r"(c));
  return d;
}

// Warp w of block x owns weight rows n0 .. n0 + RPW - 1, n0 = (x * 8 + w) * RPW;
// lane L owns groups L, L + 32, ... of each row.  Every weight load of the
// warp is issued at entry, before the activation is staged in shared memory,
// so the weight stream overlaps the staging.
// shared layout: act[m][i][g] = uint2{even word, odd word} of word i (0..3) of
// group g of row m;  asum[m][g] = sum of the group's codes;  ssa[m][g] steps.
template <int MB, int RPW>
__global__ void __launch_bounds__(kGemvThreads) k_group_gemv(
    const int8_t* __restrict__ qa, const float* __restrict__ sa, const uint8_t* __restrict__ w4,
    const float* __restrict__ sw, float* __restrict__ y, int M, int N, int K) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int G = K / kGroup;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = (blockIdx.x * kGemvWarps + warp) * RPW;
  const int rowstride = K / 2;  // bytes per packed weight row

  // ---- weight stream of this warp (registers)
  uint4 wv[RPW][kGemvGroupsPerLane];
  float swv[RPW][kGemvGroupsPerLane];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const int n = min(n0 + r, N - 1);
#pragma unroll
    for (int gi = 0; gi < kGemvGroupsPerLane; ++gi) {
      const int g = lane + 32 * gi;
      if (g < G) {
        wv[r][gi] = __ldg(reinterpret_cast<const uint4*>(w4 + (size_t)n * rowstride) + g);
        swv[r][gi] = __ldg(sw + (size_t)n * G + g);
      } else {
        wv[r][gi] = make_uint4(0, 0, 0, 0);
        swv[r][gi] = 0.f;
      }
    }
  }

  // ---- stage the activation: one thread per 8-code chunk, 4 chunks per group
  uint2* act = reinterpret_cast<uint2*>(smem_raw);                        // M*4*G
  int* asum = reinterpret_cast<int*>(act + (size_t)M * 4 * G);           // M*G
  float* ssa = reinterpret_cast<float*>(asum + (size_t)M * G);           // M*G
  const int n_chunks = M * K / 8;
  constexpr int kU = 4;  // staging loads in flight per thread
  for (int base = 0; base < n_chunks; base += kU * kGemvThreads) {
    uint2 raw[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int ch = base + u * kGemvThreads + threadIdx.x;
      raw[u] = ch < n_chunks ? __ldg(reinterpret_cast<const uint2*>(qa) + ch) : make_uint2(0, 0);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int ch = base + u * kGemvThreads + threadIdx.x;
      // n_chunks is a multiple of 4, so the 4 lanes of a group agree on validity
      const bool valid = ch < n_chunks;
      // bytes c0..c7 -> even word (c0,c2,c4,c6), odd word (c1,c3,c5,c7)
      const uint32_t ev = __byte_perm(raw[u].x, raw[u].y, 0x6420);
      const uint32_t od = __byte_perm(raw[u].x, raw[u].y, 0x7531);
      int sum = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        sum += (int)(int8_t)((raw[u].x >> (8 * i)) & 0xFF) +
               (int)(int8_t)((raw[u].y >> (8 * i)) & 0xFF);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
      if (valid) {
        const int m = ch / (K / 8);
        const int rem = ch - m * (K / 8);
        const int g = rem >> 2, i = rem & 3;
        act[((size_t)m * 4 + i) * G + g] = make_uint2(ev, od);
        if (i == 0) {
          asum[m * G + g] = sum;
          ssa[m * G + g] = sa[(size_t)m * G + g];
        }
      }
    }
  }
  __syncthreads();
  if (n0 >= N) return;

  // ---- integer dots: weight nibble v read as v ^ 8 = q_w + 8 in [1, 15]
  float part[RPW][MB];
#pragma unroll
  for (int r = 0; r < RPW; ++r)
#pragma unroll
    for (int m = 0; m < MB; ++m) part[r][m] = 0.f;
#pragma unroll
  for (int gi = 0; gi < kGemvGroupsPerLane; ++gi) {
    const int g = lane + 32 * gi;
    if (g < G) {
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        const uint4 w = wv[r][gi];
        const uint32_t wu[4] = {w.x ^ 0x88888888u, w.y ^ 0x88888888u, w.z ^ 0x88888888u,
                                w.w ^ 0x88888888u};
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
            part[r][m] = fmaf(ssa[m * G + g] * swv[r][gi], (float)d, part[r][m]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
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
    for (int r = 0; r < RPW; ++r) {
      const int n = n0 + r;
      if (n < N) {
#pragma unroll
        for (int m = 0; m < MB; ++m)
          if (m < M) y[(size_t)m * N + n] = part[r][m];
      }
    }
  }
}

template <int MB, int RPW>
cudaError_t launch_mb(const int8_t* qa, const float* sa, const uint8_t* w4, const float* sw,
                      float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s) {
  const int64_t G = K / kGroup;
  const size_t smem = (size_t)M * 4 * G * 8 + (size_t)M * G * 8;
  auto* k = k_group_gemv<MB, RPW>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t warps_needed = (N + RPW - 1) / RPW;
  const int64_t blocks = (warps_needed + kGemvWarps - 1) / kGemvWarps;
  k<<<(unsigned)blocks, kGemvThreads, smem, s>>>(qa, sa, w4, sw, y, (int)M, (int)N, (int)K);
  return cudaGetLastError();
}

template <int MB>
cudaError_t launch_rows(const int8_t* qa, const float* sa, const uint8_t* w4, const float* sw,
                        float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s) {
  // two rows per warp once there are enough rows to fill the GPU twice over
  if (N >= 4096) return launch_mb<MB, 2>(qa, sa, w4, sw, y, M, N, K, s);
  return launch_mb<MB, 1>(qa, sa, w4, sw, y, M, N, K, s);
}

}  // namespace

cudaError_t launch_group_gemv(const int8_t* qa, const float* sa, const uint8_t* w4,
                              const float* sw, float* y, int64_t M, int64_t N, int64_t K,
                              cudaStream_t s) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (K > (int64_t)kGroup * 32 * kGemvGroupsPerLane) return cudaErrorInvalidValue;
  if (M <= 1) return launch_rows<1>(qa, sa, w4, sw, y, M, N, K, s);
  if (M <= 4) return launch_rows<4>(qa, sa, w4, sw, y, M, N, K, s);
  return launch_rows<16>(qa, sa, w4, sw, y, M, N, K, s);
}

}  // namespace lq
