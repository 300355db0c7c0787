// Activation / weight quantizers of the looped linear (sm_100a).
//
// k_quant_only    : group-32 absmax + LAS step + RTN on an already transformed
//                   input (HBM-bound).
// k_rotate_quant  : fused x (P1 kron P2) + the same quantizer.  The rotation
//                   is two small contractions per token row, X -> P2 then
//                   P1^T, both held in shared memory and accumulated in
//                   float64, rounded once to float32 before quantizing.
//                   With kStoreF32 it writes the rotated rows instead (used
//                   for the offline weight fold W (Q1 kron Q2)).
//
// Definitions ("paper_specification.yaml" of the LoopQ reproduction):
//   step      s = fl32(fl32(c * absmax) / q_max)     (lq1 Eq. (4), las Section 4.1,
//                                                     implementation_status lq2)
//   code      q = clip(rne(fl32(x / s)), -q_max, q_max), q = 0 when s == 0
//   group     32 consecutive elements along K        (lq1 granularity, Table 6)
//   transform x (P1 kron P2) = vec(P1^T X P2), X the row-major a x b reshape
//             (shared_transformed_backbone, Eqs. (2)-(3); lq3 Kronecker)
#include <cuda_bf16.h>

#include <algorithm>

#include "lq_common.cuh"

namespace lq {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void load8(const float* __restrict__ x, int64_t chunk, float (&v)[8]) {
  const float4* p = reinterpret_cast<const float4*>(x + chunk * 8);
  float4 a = __ldg(p), b = __ldg(p + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ void load8(const __nv_bfloat16* __restrict__ x, int64_t chunk,
                                      float (&v)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(x + chunk * 8));
  uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
    v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
  }
}

// Quantize the 8 values a thread holds; the 4 consecutive lanes 4j..4j+3 of
// a warp hold one group of 32.  Every lane of the warp must call this.
__device__ __forceinline__ float quant_group8(const float (&v)[8], float c, int qmax,
                                              int (&q)[8]) {
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[i]));
  am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
  am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
  // s = fl32(fl32(c * absmax) / q_max): two IEEE round-to-nearest operations
  const float s = __fdiv_rn(__fmul_rn(c, am), (float)qmax);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int qi = 0;
    if (s != 0.f) {
      const float r = __fdiv_rn(v[i], s);  // fl32(x / s), true division
      qi = __float2int_rn(r);              // round half to even
      qi = min(max(qi, -qmax), qmax);
    }
    q[i] = qi;
  }
  return s;
}

// Write one thread's 8 codes (and its group's step from lane 4j).
__device__ __forceinline__ void store_codes(const int (&q)[8], float s, int64_t chunk,
                                            int8_t* __restrict__ codes8, int opf,
                                            uint8_t* __restrict__ codes4,
                                            float* __restrict__ scales) {
  if (codes8) {
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      w0 |= encode_code_byte(q[i], opf) << (8 * i);
      w1 |= encode_code_byte(q[i + 4], opf) << (8 * i);
    }
    reinterpret_cast<uint2*>(codes8)[chunk] = make_uint2(w0, w1);
  }
  if (codes4) {
    uint32_t p = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = (uint32_t)q[2 * j] & 0xFu, hi = (uint32_t)q[2 * j + 1] & 0xFu;
      p |= (lo | (hi << 4)) << (8 * j);
    }
    reinterpret_cast<uint32_t*>(codes4)[chunk] = p;
  }
  if ((threadIdx.x & 3) == 0) scales[chunk >> 2] = s;
}

template <typename Tin>
__global__ void __launch_bounds__(kThreads) k_quant_only(const Tin* __restrict__ x,
                                                         int64_t n_chunks, float c, int qmax,
                                                         int8_t* __restrict__ codes8, int opf,
                                                         uint8_t* __restrict__ codes4,
                                                         float* __restrict__ scales) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  // n_chunks is a multiple of 4 and the loop bound is warp-uniform, so the
  // 4 lanes of a group are all valid or all invalid
  for (int64_t base = (int64_t)blockIdx.x * kThreads; base < n_chunks; base += stride) {
    const int64_t ch = base + threadIdx.x;
    const bool valid = ch < n_chunks;
    float v[8];
    if (valid) {
      load8(x, ch, v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    int q[8];
    const float s = quant_group8(v, c, qmax, q);
    if (valid) store_codes(q, s, ch, codes8, opf, codes4, scales);
  }
}

// ---------------------------------------------------------------------------
// fused Kronecker rotation + quantization
// ---------------------------------------------------------------------------
struct RotSmem {
  double* P1;  // a x a
  double* P2;  // b x b
  double* X;   // R x K   (input rows, then the float32 result Z aliased on it)
  double* Y;   // R x K   (X P2)
};

__device__ __forceinline__ void load_row_chunk(const float* __restrict__ x, int64_t chunk,
                                               double* dst) {
  float v[8];
  load8(x, chunk, v);
  double2* d = reinterpret_cast<double2*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = make_double2((double)v[2 * i], (double)v[2 * i + 1]);
}
__device__ __forceinline__ void load_row_chunk(const __nv_bfloat16* __restrict__ x,
                                               int64_t chunk, double* dst) {
  float v[8];
  load8(x, chunk, v);
  double2* d = reinterpret_cast<double2*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = make_double2((double)v[2 * i], (double)v[2 * i + 1]);
}

template <typename Tin, bool kStoreF32>
__global__ void __launch_bounds__(kThreads) k_rotate_quant(
    const Tin* __restrict__ x, int64_t M, int K, const float* __restrict__ P1, int a,
    const float* __restrict__ P2, int b, int R, float c, int qmax, int8_t* __restrict__ codes8,
    int opf, uint8_t* __restrict__ codes4, float* __restrict__ scales,
    float* __restrict__ out_f32) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RotSmem sm;
  sm.P1 = reinterpret_cast<double*>(smem_raw);
  sm.P2 = sm.P1 + a * a;
  sm.X = sm.P2 + b * b;
  sm.Y = sm.X + (size_t)R * K;
  float* Z = reinterpret_cast<float*>(sm.X);

  const int tid = threadIdx.x;
  for (int i = tid; i < a * a; i += kThreads) sm.P1[i] = (double)P1[i];
  for (int i = tid; i < b * b; i += kThreads) sm.P2[i] = (double)P2[i];

  const int ct_n = b >> 2;           // column tiles (strided columns ct + jj*ct_n)
  const int rt_n = (R * a) >> 2;     // row tiles of 4 rows of the R*a x b stacks
  const int n_tiles = rt_n * ct_n;
  const int row_chunks = K >> 3;     // 8-element chunks per token row

  for (int64_t m0 = (int64_t)blockIdx.x * R; m0 < M; m0 += (int64_t)gridDim.x * R) {
    const int rows = (M - m0 < (int64_t)R) ? (int)(M - m0) : R;
    __syncthreads();  // the previous iteration's Z is consumed, P1/P2 are loaded
    // ---- load R token rows as float64 (rows past M are zero)
    for (int ch = tid; ch < R * row_chunks; ch += kThreads) {
      const int r = ch / row_chunks;
      double* dst = sm.X + (size_t)ch * 8;
      if (r < rows) {
        load_row_chunk(x + (size_t)m0 * K, ch, dst);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = 0.0;
      }
    }
    __syncthreads();
    // ---- stage 1: Y[(r,i), j] = sum_q X[(r,i), q] P2[q, j]
    for (int tile = tid; tile < n_tiles; tile += kThreads) {
      const int rt = tile / ct_n, ct = tile - rt * ct_n;
      const double* xr = sm.X + (size_t)(rt * 4) * b;
      double acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
      for (int q = 0; q < b; ++q) {
        double xv[4], pv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) xv[i] = xr[i * b + q];
#pragma unroll
        for (int j = 0; j < 4; ++j) pv[j] = sm.P2[q * b + ct + j * ct_n];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fma(xv[i], pv[j], acc[i][j]);
      }
      double* yr = sm.Y + (size_t)(rt * 4) * b;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) yr[i * b + ct + j * ct_n] = acc[i][j];
    }
    __syncthreads();
    // ---- stage 2: Z[r, i, j] = sum_p P1[p, i] Y[r, p, j], rounded once to float32
    for (int tile = tid; tile < n_tiles; tile += kThreads) {
      const int rt = tile / ct_n, ct = tile - rt * ct_n;
      const int ri0 = rt * 4;
      const int r = ri0 / a, i0 = ri0 - r * a;
      const double* yr = sm.Y + (size_t)r * K;
      double acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
      for (int p = 0; p < a; ++p) {
        double wv[4], yv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) wv[i] = sm.P1[p * a + i0 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) yv[j] = yr[p * b + ct + j * ct_n];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fma(wv[i], yv[j], acc[i][j]);
      }
      float* zr = Z + (size_t)ri0 * b;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) zr[i * b + ct + j * ct_n] = __double2float_rn(acc[i][j]);
    }
    __syncthreads();
    // ---- epilogue
    const int n_chunks = R * row_chunks;
    if (kStoreF32) {
      for (int ch = tid; ch < rows * row_chunks; ch += kThreads) {
        const float4* src = reinterpret_cast<const float4*>(Z + (size_t)ch * 8);
        float4* dst = reinterpret_cast<float4*>(out_f32 + (size_t)m0 * K + (size_t)ch * 8);
        dst[0] = src[0];
        dst[1] = src[1];
      }
    } else {
      for (int base = 0; base < n_chunks; base += kThreads) {
        const int ch = base + tid;
        const bool valid = ch < n_chunks && (ch / row_chunks) < rows;
        float v[8];
        if (valid) {
          const float4* src = reinterpret_cast<const float4*>(Z + (size_t)ch * 8);
          float4 u0 = src[0], u1 = src[1];
          v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
          v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = 0.f;
        }
        int q[8];
        const float s = quant_group8(v, c, qmax, q);
        if (valid) store_codes(q, s, m0 * row_chunks + ch, codes8, opf, codes4, scales);
      }
    }
  }
}

__global__ void k_codes4_to_operand(const uint8_t* __restrict__ codes4, int64_t n_words, int opf,
                                    uint8_t* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_words; i += stride) {
    const uint32_t w = reinterpret_cast<const uint32_t*>(codes4)[i];
    uint32_t o0 = 0, o1 = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      int nib = (int)((w >> (4 * j)) & 0xFu);
      nib = nib >= 8 ? nib - 16 : nib;
      const uint32_t byte = encode_code_byte(nib, opf);
      if (j < 4) o0 |= byte << (8 * j); else o1 |= byte << (8 * (j - 4));
    }
    reinterpret_cast<uint2*>(out)[i] = make_uint2(o0, o1);
  }
}

__global__ void k_transpose_f32(const float* __restrict__ in, int64_t rows, int64_t cols,
                                float* __restrict__ out) {
  __shared__ float tile[32][33];
  const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t r = r0 + i, cc = c0 + threadIdx.x;
    if (r < rows && cc < cols) tile[i][threadIdx.x] = in[r * cols + cc];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t cc = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && cc < cols) out[cc * rows + r] = tile[threadIdx.x][i];
  }
}

template <typename F>
cudaError_t set_smem(F* f, size_t bytes) {
  static_assert(sizeof(F*) > 0, "");
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

size_t rotate_smem_bytes(int a, int b, int* rows_per_block) {
  const size_t fixed = 8u * (size_t)(a * a + b * b);
  const size_t per_row = 16u * (size_t)(a * b);
  // prefer two resident blocks per SM (<= 110 KB each), else one (<= 224 KB)
  int best = 0;
  for (int R = 16; R >= 1; R >>= 1) {
    if (fixed + per_row * R <= 110u * 1024u) { best = R; break; }
  }
  if (best == 0 && fixed + per_row <= 224u * 1024u) best = 1;
  if (rows_per_block) *rows_per_block = best;
  return best ? fixed + per_row * best : 0;
}

cudaError_t launch_quantize(const void* x, int x_dtype, int64_t M, int64_t K, const float* P1,
                            int a, const float* P2, int b, float c, int bits, int8_t* codes8,
                            int opf, uint8_t* codes4, float* scales, cudaStream_t s) {
  const int qmax = bits == 8 ? 127 : 7;
  if (M == 0) return cudaSuccess;
  if (P1 == nullptr) {
    const int64_t n_chunks = M * K / 8;
    const int64_t want = (n_chunks + kThreads - 1) / kThreads;
    const int grid = (int)std::min<int64_t>(want, (int64_t)num_sms() * 8);
    if (x_dtype == LQ_BF16)
      k_quant_only<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
          (const __nv_bfloat16*)x, n_chunks, c, qmax, codes8, opf, codes4, scales);
    else
      k_quant_only<float><<<grid, kThreads, 0, s>>>((const float*)x, n_chunks, c, qmax, codes8,
                                                    opf, codes4, scales);
    return cudaGetLastError();
  }
  int R = 0;
  const size_t smem = rotate_smem_bytes(a, b, &R);
  if (smem == 0) return cudaErrorInvalidValue;
  const int per_sm = smem <= 110u * 1024u ? 2 : 1;
  const int64_t want = (M + R - 1) / R;
  const int grid = (int)std::min<int64_t>(want, (int64_t)num_sms() * per_sm);
  cudaError_t e;
  if (x_dtype == LQ_BF16) {
    auto* k = k_rotate_quant<__nv_bfloat16, false>;
    if ((e = set_smem(k, smem)) != cudaSuccess) return e;
    k<<<grid, kThreads, smem, s>>>((const __nv_bfloat16*)x, M, (int)K, P1, a, P2, b, R, c, qmax,
                                   codes8, opf, codes4, scales, nullptr);
  } else {
    auto* k = k_rotate_quant<float, false>;
    if ((e = set_smem(k, smem)) != cudaSuccess) return e;
    k<<<grid, kThreads, smem, s>>>((const float*)x, M, (int)K, P1, a, P2, b, R, c, qmax, codes8,
                                   opf, codes4, scales, nullptr);
  }
  return cudaGetLastError();
}

cudaError_t launch_rotate_store(const float* x, int64_t M, int64_t K, const float* Q1, int a,
                                const float* Q2, int b, float* out, cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  int R = 0;
  const size_t smem = rotate_smem_bytes(a, b, &R);
  if (smem == 0) return cudaErrorInvalidValue;
  const int per_sm = smem <= 110u * 1024u ? 2 : 1;
  const int grid = (int)std::min<int64_t>((M + R - 1) / R, (int64_t)num_sms() * per_sm);
  auto* k = k_rotate_quant<float, true>;
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  k<<<grid, kThreads, smem, s>>>(x, M, (int)K, Q1, a, Q2, b, R, 1.0f, 7, nullptr, kOpInt8,
                                 nullptr, nullptr, out);
  return cudaGetLastError();
}

cudaError_t launch_codes4_to_operand(const uint8_t* codes4, int64_t n_bytes, int opf,
                                     uint8_t* out, cudaStream_t s) {
  const int64_t n_words = n_bytes / 4;
  if (n_words == 0) return cudaSuccess;
  const int grid = (int)std::min<int64_t>((n_words + 255) / 256, (int64_t)num_sms() * 16);
  k_codes4_to_operand<<<grid, 256, 0, s>>>(codes4, n_words, opf, out);
  return cudaGetLastError();
}

cudaError_t launch_transpose_f32(const float* in, int64_t rows, int64_t cols, float* out,
                                 cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  dim3 grid((unsigned)((cols + 31) / 32), (unsigned)((rows + 31) / 32));
  k_transpose_f32<<<grid, dim3(32, 8), 0, s>>>(in, rows, cols, out);
  return cudaGetLastError();
}

}  // namespace lq
