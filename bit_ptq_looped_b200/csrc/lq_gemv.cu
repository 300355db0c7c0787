// Decode-sized group-rescaled GEMV (M <= 16 tokens), weight streaming from HBM.
//
//   y[m,n] = sum_g s_a[m,g] s_w[n,g] sum_{k in g} q_a[m,k] q_w[n,k]
//
// Same arithmetic as the tensor-core GEMM, for the decode regime where each
// loop reads the packed 4-bit weights once and the activation is a handful of
// rows.  Up to 4 tokens use dp4a on the CUDA cores (below); 5 to 16 tokens use
// the integer tensor-core MMA (k_group_gemv_mma, further down).
// Warp w of the grid owns weight rows w, w + W, w + 2W, ... (W warps in
// the grid); lane L owns groups L, L + 32, ... of each row: one 16-byte load
// brings the 32 packed codes of a group, one 4-byte load its step.  The
// activation codes of all M rows arrive in the kOpGemvAct layout (even and odd
// codes of a group in separate 32-bit words that match the low and high
// nibbles of the packed weights) and are copied to shared memory as they are.
//
// Integer dot: weight nibble v (two's complement q_w) is read as v ^ 8 =
// q_w + 8 in [1, 15], so dp4a(unsigned weights, signed activations) gives
// sum (q_w + 8) q_a; subtracting 8 * sum q_a (the group sums the quantizer
// wrote) leaves the exact sum q_w q_a.
//
// The first batch of weight rows is loaded into registers before pdl_wait, so
// under programmatic dependent launch the weight stream of this launch
// overlaps the quantizer that produces its activation.
#include <algorithm>
#include <mutex>
#include <unordered_map>

#include "lq_common.cuh"

namespace lq {
namespace {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

__device__ __forceinline__ int dp4a_us(uint32_t a_unsigned, uint32_t b_signed, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_unsigned), "r"(b_signed), "r"(c));
  return d;
}

// MB: activation rows handled (M <= MB); GPL: group slots per lane (G <= 32 * GPL);
// RPW: weight rows per warp per batch; kDB: prefetch batch b + 1 while folding b
// (worth its registers only when a warp has more than one batch).
// shared layout: act vectors [(m * 2 + h) * G + g] (uint4), then asum[M * G], ssa[M * G].
// (launch bounds: the streaming variant states a minimum of one block per SM
// so that it keeps its prefetch registers, which measured faster than trading
// them for occupancy; the single-batch decode variant keeps the occupancy that
// lets the next kernels of a sequence start beside it)
template <int MB, int GPL, int RPW, bool kDB>
__global__ void __launch_bounds__(kGemvThreads, kDB ? 1 : 3) k_group_gemv(
    const int8_t* __restrict__ qa, const int* __restrict__ asum_g, const float* __restrict__ sa,
    const uint8_t* __restrict__ w4, const float* __restrict__ sw, float* __restrict__ y, int M,
    int N, int K) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_trigger();
  const int G = K / kGroup;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kGemvWarps + warp;       // this warp's index in the grid
  const int W = gridDim.x * kGemvWarps;                 // warps in the grid
  const size_t rowstride = (size_t)K / 2;               // bytes per packed weight row

  // register sets of weight rows: with kDB, batch b + 1 is in flight while batch b is folded
  constexpr int kSets = kDB ? 2 : 1;
  uint4 wv[kSets][RPW][GPL];
  float swv[kSets][RPW][GPL];
  auto load_batch = [&](int buf, int j0) {  // rows gw + (j0 + r) * W, r < RPW
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const int n = gw + (j0 + r) * W;
#pragma unroll
      for (int gi = 0; gi < GPL; ++gi) {
        const int g = lane + 32 * gi;
        if (n < N && g < G) {
          wv[buf][r][gi] = __ldg(reinterpret_cast<const uint4*>(w4 + (size_t)n * rowstride) + g);
          swv[buf][r][gi] = __ldg(sw + (size_t)n * G + g);
        } else {
          wv[buf][r][gi] = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
          swv[buf][r][gi] = 0.f;
        }
      }
    }
  };
  load_batch(0, 0);

  // ---- the activation: written by the previous kernel of the sequence
  pdl_wait();
  uint4* act = reinterpret_cast<uint4*>(smem_raw);                   // M * 2 * G vectors
  int* asum = reinterpret_cast<int*>(act + (size_t)M * 2 * G);       // M * G
  float* ssa = reinterpret_cast<float*>(asum + (size_t)M * G);       // M * G
  {
    const int n_vec = M * 2 * G;
    const uint4* src = reinterpret_cast<const uint4*>(qa);
    for (int i = threadIdx.x; i < n_vec; i += kGemvThreads) act[i] = __ldg(src + i);
    for (int i = threadIdx.x; i < M * G; i += kGemvThreads) {
      asum[i] = __ldg(asum_g + i);
      ssa[i] = __ldg(sa + i);
    }
  }
  __syncthreads();

  // fold batch `buf` (rows gw + (j0 + r) * W) into y
  auto fold_batch = [&](int buf, int j0) {
    float part[RPW][MB];
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m) part[r][m] = 0.f;
#pragma unroll
    for (int gi = 0; gi < GPL; ++gi) {
      const int g = lane + 32 * gi;
      if (g < G) {
        uint32_t lo[RPW][4], hi[RPW][4];
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
          const uint4 w = wv[buf][r][gi];
          const uint32_t wu[4] = {w.x ^ 0x88888888u, w.y ^ 0x88888888u, w.z ^ 0x88888888u,
                                  w.w ^ 0x88888888u};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            lo[r][i] = wu[i] & 0x0F0F0F0Fu;
            hi[r][i] = (wu[i] >> 4) & 0x0F0F0F0Fu;
          }
        }
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          if (m < M) {
            const uint4 a0 = act[gemv_act_vec_index(m, 0, g, G)];
            const uint4 a1 = act[gemv_act_vec_index(m, 1, g, G)];
            const int corr = 8 * asum[m * G + g];
            const float sam = ssa[m * G + g];
#pragma unroll
            for (int r = 0; r < RPW; ++r) {
              int d = dp4a_us(lo[r][0], a0.x, 0);
              d = dp4a_us(hi[r][0], a0.y, d);
              d = dp4a_us(lo[r][1], a0.z, d);
              d = dp4a_us(hi[r][1], a0.w, d);
              d = dp4a_us(lo[r][2], a1.x, d);
              d = dp4a_us(hi[r][2], a1.y, d);
              d = dp4a_us(lo[r][3], a1.z, d);
              d = dp4a_us(hi[r][3], a1.w, d);
              part[r][m] = fmaf(sam * swv[buf][r][gi], (float)(d - corr), part[r][m]);
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
    // lane (r * MB + m) % 32 writes y[m, n_r]
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const int n = gw + (j0 + r) * W;
#pragma unroll
      for (int m = 0; m < MB; ++m)
        if (lane == ((r * MB + m) & 31) && m < M && n < N) y[(size_t)m * N + n] = part[r][m];
    }
  };

  if (kDB) {
    // batches alternate between the two register sets (the loop is unrolled by
    // two so that every register index is static)
    for (int j0 = 0; gw + j0 * W < N; j0 += 2 * RPW) {
      const bool more1 = gw + (j0 + RPW) * W < N;
      if (more1) load_batch(kSets - 1, j0 + RPW);
      fold_batch(0, j0);
      if (!more1) break;
      if (gw + (j0 + 2 * RPW) * W < N) load_batch(0, j0 + 2 * RPW);
      fold_batch(kSets - 1, j0 + RPW);
    }
  } else {
    for (int j0 = 0; gw + j0 * W < N; j0 += RPW) {
      if (j0 > 0) load_batch(0, j0);
      fold_batch(0, j0);
    }
  }
}

// ---------------------------------------------------------------------------
// 5 to 16 tokens: the integer dots on the tensor cores (mma.sync m16n8k32,
// u8 x s8 -> s32).  A warp takes 16 weight rows at a time and walks all groups
// of K; one MMA per group and block of 8 tokens.  The group's 32 codes form
// the MMA's K dimension in the order of the packed words: thread (g, t) of the
// MMA holds k-quad t = the low nibbles of weight word t (codes 8t, 8t+2, 8t+4,
// 8t+6) and k-quad t + 4 = its high nibbles, and the activation fragments are
// the matching even and odd code words e_t, o_t of the kOpGemvAct layout.
// Weight nibbles enter as v ^ 8 = q_w + 8 (unsigned); the accumulator starts at
// -8 * sum q_a, so the MMA returns sum q_w q_a exactly.  Each output (row,
// token) belongs to one thread, which folds s_w * s_a * sum per group.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_u8s8_16832(int (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int NB>  // blocks of 8 tokens
__global__ void __launch_bounds__(kGemvThreads, 2) k_group_gemv_mma(
    const int8_t* __restrict__ qa, const int* __restrict__ asum_g, const float* __restrict__ sa,
    const uint8_t* __restrict__ w4, const float* __restrict__ sw, float* __restrict__ y, int M,
    int N, int K) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_trigger();
  const int G = K / kGroup;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int gw = blockIdx.x * kGemvWarps + warp, W = gridDim.x * kGemvWarps;
  const size_t rowstride = (size_t)K / 2;

  // first weight words of this warp's first row block, before the wait
  constexpr int kU = 4;  // groups per load batch
  uint32_t wA[kU], wB[kU];
  float swA[kU], swB[kU];
  auto load_groups = [&](int n0, int g0) {
    const int na = n0 + g, nb = n0 + g + 8;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int grp = g0 + u;
      const bool oka = na < N && grp < G, okb = nb < N && grp < G;
      wA[u] = oka ? __ldg(reinterpret_cast<const uint32_t*>(w4 + (size_t)na * rowstride) +
                          grp * 4 + t)
                  : 0x88888888u;
      wB[u] = okb ? __ldg(reinterpret_cast<const uint32_t*>(w4 + (size_t)nb * rowstride) +
                          grp * 4 + t)
                  : 0x88888888u;
      swA[u] = oka ? __ldg(sw + (size_t)na * G + grp) : 0.f;
      swB[u] = okb ? __ldg(sw + (size_t)nb * G + grp) : 0.f;
    }
  };
  if (gw * 16 < N) load_groups(gw * 16, 0);

  pdl_wait();  // the activation is the previous kernel's output
  uint4* act = reinterpret_cast<uint4*>(smem_raw);
  int* asum = reinterpret_cast<int*>(act + (size_t)M * 2 * G);
  float* ssa = reinterpret_cast<float*>(asum + (size_t)M * G);
  {
    const int n_vec = M * 2 * G;
    const uint4* src = reinterpret_cast<const uint4*>(qa);
    for (int i = threadIdx.x; i < n_vec; i += kGemvThreads) act[i] = __ldg(src + i);
    for (int i = threadIdx.x; i < M * G; i += kGemvThreads) {
      asum[i] = __ldg(asum_g + i);
      ssa[i] = __ldg(sa + i);
    }
  }
  __syncthreads();
  const uint32_t* act32 = reinterpret_cast<const uint32_t*>(act);

  for (int rb = gw; rb * 16 < N; rb += W) {
    const int n0 = rb * 16;
    float acc[NB][4];
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;
    for (int g0 = 0; g0 < G; g0 += kU) {
      if (rb != gw || g0 != 0) load_groups(n0, g0);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int grp = g0 + u;
        if (grp < G) {
          const uint32_t xa = wA[u] ^ 0x88888888u, xb = wB[u] ^ 0x88888888u;
          const uint32_t a0 = xa & 0x0F0F0F0Fu, a1 = xb & 0x0F0F0F0Fu;
          const uint32_t a2 = (xa >> 4) & 0x0F0F0F0Fu, a3 = (xb >> 4) & 0x0F0F0F0Fu;
#pragma unroll
          for (int j = 0; j < NB; ++j) {
            const int mb = j * 8 + g;          // token of the B fragment column
            const int m0 = j * 8 + 2 * t;      // tokens of this thread's C columns
            uint32_t b0 = 0, b1 = 0;
            if (mb < M) {
              const uint32_t* e = act32 + ((size_t)(mb * 2 + (t >> 1)) * G + grp) * 4 + (t & 1) * 2;
              b0 = e[0];
              b1 = e[1];
            }
            const bool v0 = m0 < M, v1 = m0 + 1 < M;
            const int c0 = v0 ? -8 * asum[m0 * G + grp] : 0;
            const int c1 = v1 ? -8 * asum[(m0 + 1) * G + grp] : 0;
            int c[4] = {c0, c1, c0, c1};
            mma_u8s8_16832(c, a0, a1, a2, a3, b0, b1);
            const float s0 = v0 ? ssa[m0 * G + grp] : 0.f;
            const float s1 = v1 ? ssa[(m0 + 1) * G + grp] : 0.f;
            acc[j][0] = fmaf(swA[u] * s0, (float)c[0], acc[j][0]);
            acc[j][1] = fmaf(swA[u] * s1, (float)c[1], acc[j][1]);
            acc[j][2] = fmaf(swB[u] * s0, (float)c[2], acc[j][2]);
            acc[j][3] = fmaf(swB[u] * s1, (float)c[3], acc[j][3]);
          }
        }
      }
    }
    const int na = n0 + g, nb = n0 + g + 8;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int m0 = j * 8 + 2 * t;
      if (na < N) {
        if (m0 < M) y[(size_t)m0 * N + na] = acc[j][0];
        if (m0 + 1 < M) y[(size_t)(m0 + 1) * N + na] = acc[j][1];
      }
      if (nb < N) {
        if (m0 < M) y[(size_t)m0 * N + nb] = acc[j][2];
        if (m0 + 1 < M) y[(size_t)(m0 + 1) * N + nb] = acc[j][3];
      }
    }
  }
}

size_t gemv_smem_bytes(int64_t M, int64_t G) { return (size_t)M * G * (32 + 8); }
constexpr size_t kGemvMaxSmem = 200u * 1024u;  // the activation bound of the GEMV path

template <int MB, int GPL, int RPW, bool kDB>
cudaError_t launch_cfg(const int8_t* qa, const int* asum, const float* sa, const uint8_t* w4,
                       const float* sw, float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                       bool pdl) {
  const size_t smem = gemv_smem_bytes(M, K / kGroup);
  auto* k = k_group_gemv<MB, GPL, RPW, kDB>;
  // resident blocks per SM for this instantiation and shared-memory size
  static std::mutex mu;
  static std::unordered_map<size_t, int> per_sm_cache;
  int per_sm = 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = per_sm_cache.find(smem);
    if (it == per_sm_cache.end()) {
      // the attribute is one per function: raise it once to the largest activation
      // any call can stage, never lower it under an earlier call's size
      if (per_sm_cache.empty()) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kGemvMaxSmem);
        if (e != cudaSuccess) return e;
      }
      cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kGemvThreads, smem);
      if (e != cudaSuccess) return e;
      if (per_sm < 1) return cudaErrorInvalidConfiguration;
      per_sm_cache.emplace(smem, per_sm);
    } else {
      per_sm = it->second;
    }
  }
  // enough warps for one batch of RPW rows each, capped at one resident wave
  const int64_t warps_needed = (N + RPW - 1) / RPW;
  const int64_t want = (warps_needed + kGemvWarps - 1) / kGemvWarps;
  const int64_t blocks = std::min<int64_t>(want, (int64_t)num_sms() * per_sm);
  return launch_kernel(k, dim3((unsigned)blocks), dim3(kGemvThreads), smem, s, pdl, qa, asum, sa,
                       w4, sw, y, (int)M, (int)N, (int)K);
}

// one batch per warp fits in a resident wave: no prefetch registers needed
template <int MB, int GPL, int RPW>
cudaError_t launch_rpw(const int8_t* qa, const int* asum, const float* sa, const uint8_t* w4,
                       const float* sw, float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                       bool pdl) {
  const int64_t one_wave_rows = (int64_t)num_sms() * 2 * kGemvWarps * RPW;
  if (N <= one_wave_rows)
    return launch_cfg<MB, GPL, RPW, false>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
  return launch_cfg<MB, GPL, RPW, true>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
}

template <int NB>
cudaError_t launch_mma(const int8_t* qa, const int* asum, const float* sa, const uint8_t* w4,
                       const float* sw, float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                       bool pdl) {
  const size_t smem = gemv_smem_bytes(M, K / kGroup);
  auto* k = k_group_gemv_mma<NB>;
  static std::mutex mu;
  static std::unordered_map<size_t, int> per_sm_cache;
  int per_sm = 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = per_sm_cache.find(smem);
    if (it == per_sm_cache.end()) {
      // the attribute is one per function: raise it once to the largest activation
      // any call can stage, never lower it under an earlier call's size
      if (per_sm_cache.empty()) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kGemvMaxSmem);
        if (e != cudaSuccess) return e;
      }
      cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kGemvThreads, smem);
      if (e != cudaSuccess) return e;
      if (per_sm < 1) return cudaErrorInvalidConfiguration;
      per_sm_cache.emplace(smem, per_sm);
    } else {
      per_sm = it->second;
    }
  }
  const int64_t warps_needed = (N + 15) / 16;
  const int64_t want = (warps_needed + kGemvWarps - 1) / kGemvWarps;
  const int64_t blocks = std::min<int64_t>(want, (int64_t)num_sms() * per_sm);
  return launch_kernel(k, dim3((unsigned)blocks), dim3(kGemvThreads), smem, s, pdl, qa, asum, sa,
                       w4, sw, y, (int)M, (int)N, (int)K);
}

template <int MB>
cudaError_t launch_mb(const int8_t* qa, const int* asum, const float* sa, const uint8_t* w4,
                      const float* sw, float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                      bool pdl) {
  const int64_t G = K / kGroup;
  if (G > 128) return launch_rpw<MB, 8, 1>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
  if (G > 64) return launch_rpw<MB, 4, 1>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
  // up to 4 tokens: when one resident wave covers N, three weight rows per warp in a single
  // batch (decode-sized launches, latency-bound); beyond that, two rows per warp
  // with the next batch in flight, the fastest streaming shape measured (a
  // 263 MB launch at M = 4: 2.98 TB/s, against 2.25 with three rows and 2.52
  // with one)
  if (N >= (int64_t)num_sms() * kGemvWarps * 3 * 3 / 2) {
    if (N <= (int64_t)num_sms() * 2 * kGemvWarps * 3)
      return launch_cfg<MB, 2, 3, false>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
    return launch_cfg<MB, 2, 2, true>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
  }
  return launch_rpw<MB, 2, 1>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
}

}  // namespace

cudaError_t launch_group_gemv(const int8_t* qa, const int* asum, const float* sa,
                              const uint8_t* w4, const float* sw, float* y, int64_t M, int64_t N,
                              int64_t K, cudaStream_t s, bool pdl) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (K > (int64_t)kGroup * 32 * 8 || M > kGemvMaxM ||
      gemv_smem_bytes(M, K / kGroup) > kGemvMaxSmem)
    return cudaErrorInvalidValue;
  if (M <= 1) return launch_mb<1>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
  if (M <= 4) return launch_mb<4>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
  // 5 to 16 tokens: integer tensor-core MMAs (8 tokens per MMA)
  if (M <= 8) return launch_mma<1>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
  return launch_mma<2>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl);
}

}  // namespace lq
