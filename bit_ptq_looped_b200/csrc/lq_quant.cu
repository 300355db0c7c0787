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
#include <map>
#include <mutex>

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
//
// The code is rne(fl32(x / s)) clamped to [-q_max, q_max], decided without a
// division per element: r1 = fl32(x * fl32(1 / s)) lies within 1.5 ulp of
// fl32(x / s), so the two round to the same integer unless a half-integer
// lies within that distance of r1.  Values within 2^-14 of a half-integer
// (far more than 1.5 ulp for |r1| < 128, the range that can round inside
// [-q_max, q_max]) take the true IEEE division instead, and so does a whole
// group whose 1 / s overflows.  Clamping before rounding gives the same code
// (the bounds are integers).  Adding 1.5 * 2^23 rounds to the nearest integer
// (ties to even) and leaves the code's two's-complement byte in the low bits.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float quant_group8(const float (&v)[8], float c, int qmax,
                                              uint32_t (&qb)[8]) {
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[i]));
  am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
  am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
  // s = fl32(fl32(c * absmax) / q_max): two IEEE round-to-nearest operations
  const float s = __fdiv_rn(__fmul_rn(c, am), (float)qmax);
  const float inv = __frcp_rn(s);
  const float qm = (float)qmax;
  const bool slow_group = !(inv <= 3.0e38f);  // 1/s overflowed (or s == 0)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float r1 = fminf(fmaxf(__fmul_rn(v[i], inv), -qm), qm);
    float f = __fadd_rn(r1, kRoundMagic);
    const float rr = __fsub_rn(f, kRoundMagic);
    const float tie_dist = 0.5f - fabsf(r1 - rr);
    if (slow_group || !(tie_dist > 6.103515625e-05f)) {  // 2^-14
      const float r = s != 0.f ? fminf(fmaxf(__fdiv_rn(v[i], s), -qm), qm) : 0.f;
      f = __fadd_rn(r, kRoundMagic);  // fl32(x / s), then RNE
    }
    qb[i] = __float_as_uint(f);
  }
  return s;
}

// two's-complement code bytes (low byte of each qb) -> one 32-bit word
__device__ __forceinline__ uint32_t pack_bytes4(uint32_t b0, uint32_t b1, uint32_t b2,
                                                uint32_t b3) {
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// E4M3 byte of an integer code |q| <= 7 held as the low byte of qb
__device__ __forceinline__ uint32_t e4m3_byte(uint32_t qb) {
  const int q = (int)(int8_t)(qb & 0xFFu);
  const uint32_t mag = (uint32_t)(q < 0 ? -q : q);
  const uint32_t byte = __byte_perm((uint32_t)(kE4M3Int0to7 & 0xFFFFFFFFull),
                                    (uint32_t)(kE4M3Int0to7 >> 32), mag) & 0xFFu;
  return byte | (q < 0 ? 0x80u : 0u);
}

// Sum of the 32 codes of the group whose 8 codes this thread holds (the 4
// lanes 4j..4j+3 of the group all get it).  Every lane of the warp must call it.
__device__ __forceinline__ int group_code_sum(const uint32_t (&qb)[8]) {
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) sum += (int)(int8_t)(qb[i] & 0xFFu);
  sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
  sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
  return sum;
}

// Write one thread's 8 codes (and its group's step from lane 4j).  chunk is
// the index of the 8-code chunk in the M x K activation.  kGemvAct selects the
// decode GEMV layout (opf == kOpGemvAct): G is the number of groups per row
// and gsum the group's code sum.
template <bool kGemvAct>
__device__ __forceinline__ void store_codes(const uint32_t (&qb)[8], float s, int64_t chunk,
                                            int8_t* __restrict__ codes8, int opf,
                                            uint8_t* __restrict__ codes4,
                                            float* __restrict__ scales, int G = 0, int gsum = 0,
                                            int* __restrict__ asum = nullptr) {
  if (codes8) {
    uint2 w;
    if (opf == kOpE4M3) {
      w.x = pack_bytes4(e4m3_byte(qb[0]), e4m3_byte(qb[1]), e4m3_byte(qb[2]), e4m3_byte(qb[3]));
      w.y = pack_bytes4(e4m3_byte(qb[4]), e4m3_byte(qb[5]), e4m3_byte(qb[6]), e4m3_byte(qb[7]));
    } else {
      w.x = pack_bytes4(qb[0], qb[1], qb[2], qb[3]);
      w.y = pack_bytes4(qb[4], qb[5], qb[6], qb[7]);
    }
    if (kGemvAct) {
      // chunk = (m * G + g) * 4 + i: words e_i, o_i of group g of row m
      const int64_t grp = chunk >> 2;
      const int i = (int)(chunk & 3);
      const int64_t m = grp / G, g = grp - m * G;
      const uint32_t ev = __byte_perm(w.x, w.y, 0x6420), od = __byte_perm(w.x, w.y, 0x7531);
      uint2* dst = reinterpret_cast<uint2*>(codes8) + 2 * gemv_act_vec_index(m, i >> 1, g, G) +
                   (i & 1);
      *dst = make_uint2(ev, od);
      if (i == 0) asum[grp] = gsum;
    } else {
      reinterpret_cast<uint2*>(codes8)[chunk] = w;
    }
  }
  if (codes4) {
    uint32_t p = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) p |= (qb[j] & 0xFu) << (4 * j);
    reinterpret_cast<uint32_t*>(codes4)[chunk] = p;
  }
  if ((threadIdx.x & 3) == 0) scales[chunk >> 2] = s;
}

// floor(n / d) for n, d < 2^16 with one multiply-high (d fixed per launch)
struct FastDiv {
  uint32_t d, m;
  __device__ __forceinline__ explicit FastDiv(uint32_t dd) : d(dd), m((0xFFFFFFFFu / dd) + 1u) {}
  __device__ __forceinline__ uint32_t div(uint32_t n) const { return d == 1u ? n : __umulhi(n, m); }
};

template <typename Tin, bool kGemvAct>
__global__ void __launch_bounds__(kThreads) k_quant_only(const Tin* __restrict__ x,
                                                         int64_t n_chunks, float c, int qmax,
                                                         int8_t* __restrict__ codes8, int opf,
                                                         uint8_t* __restrict__ codes4,
                                                         float* __restrict__ scales, int G,
                                                         int* __restrict__ asum, int x_early) {
  pdl_trigger();
  if (!x_early) pdl_wait();
  // Two 8-element chunks per thread per step (blockDim apart) keep more loads
  // in flight.  n_chunks is a multiple of 4 and every bound below is
  // warp-uniform, so the 4 lanes of a group are all valid or all invalid.
  const int64_t stride = (int64_t)gridDim.x * (2 * kThreads);
  bool waited = !x_early;
  for (int64_t base = (int64_t)blockIdx.x * (2 * kThreads); base < n_chunks; base += stride) {
    const int64_t ch0 = base + threadIdx.x, ch1 = ch0 + kThreads;
    const bool v0 = ch0 < n_chunks, v1 = ch1 < n_chunks;
    float a0[8], a1[8];
    if (v0) load8(x, ch0, a0);
    if (v1) load8(x, ch1, a1);
    if (!v0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) a0[i] = 0.f;
    }
    if (!v1) {
#pragma unroll
      for (int i = 0; i < 8; ++i) a1[i] = 0.f;
    }
    uint32_t q0[8], q1[8];
    const float s0 = quant_group8(a0, c, qmax, q0);
    const float s1 = quant_group8(a1, c, qmax, q1);
    int gs0 = 0, gs1 = 0;
    if (kGemvAct) {
      gs0 = group_code_sum(q0);
      gs1 = group_code_sum(q1);
    }
    if (!waited) {  // the previous kernel may still read the output buffers
      pdl_wait();
      waited = true;
    }
    if (v0) store_codes<kGemvAct>(q0, s0, ch0, codes8, opf, codes4, scales, G, gs0, asum);
    if (v1) store_codes<kGemvAct>(q1, s1, ch1, codes8, opf, codes4, scales, G, gs1, asum);
  }
}

// ---------------------------------------------------------------------------
// fused Kronecker rotation + quantization
//
// A block takes R token rows.  Stage 1 forms Y = X P2 for the R*a rows of
// the row-major reshapes X (a x b each); stage 2 forms Z_r = P1^T Y_r per
// token.  Both stages run on the FP64 tensor-core MMA (m8n8k4, float64
// inputs, products and sums), so x~ is the float64 value rounded once to
// float32.  Shared-memory operands are stored so that every fragment load
// reads 8 rows x 4 consecutive doubles of a row-major array whose row pitch
// is the row length + 4 doubles (conflict-free):
//   P2T[j][q] = P2[q][j]   (b x (b+4))      YT[r][j][p] = Y[r][p][j]  (R*b x (a+4))
//   P1T[i][p] = P1[p][i]   (a x (a+4))
//   X[(r,i)][q] float32 (exact copies of the bf16/fp32 inputs; (R*a) x (b+4)),
//   Z[r][i][j] float32 with the same pitch, aliased on X once stage 1 is done.
// ---------------------------------------------------------------------------
struct RotLayout {
  int a, b, R, lda, ldb, ldz;
  size_t off_p1t, off_yt, off_x, bytes;  // double offsets (X: float offset base) / bytes
};

__host__ __device__ inline RotLayout rot_layout(int a, int b, int R) {
  RotLayout L;
  L.a = a;
  L.b = b;
  L.R = R;
  L.lda = a + 4;
  L.ldb = b + 4;
  L.ldz = b + 4;
  L.off_p1t = (size_t)b * L.ldb;  // after P2T (doubles)
  L.off_yt = L.off_p1t + (size_t)a * L.lda;
  L.off_x = L.off_yt + (size_t)R * b * L.lda;  // doubles before the float region
  L.bytes = 8 * L.off_x + 4 * (size_t)R * a * L.ldb;
  return L;
}

__device__ __forceinline__ void dmma_8x8x4(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

// One warp task of an (8*TM) x (8*TN) output block of C = A B, with A given
// row-major (A[row][k], pitch lda_) and B given transposed (Bt[col][k], pitch
// ldb_).  Output tiles beyond n_col_tiles are skipped.  Calls
// emit(row, col, v0, v1) for C[row][col], C[row][col + 1].
template <int TM, int TN, typename TA, typename Emit>
__device__ __forceinline__ void warp_mma_task(const TA* __restrict__ A, int lda_,
                                              const double* __restrict__ Bt, int ldb_, int kdim,
                                              int row0, int col_tile0, int n_col_tiles,
                                              Emit emit) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  double acc[TM][TN][2];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
  const TA* a_ptr = A + (size_t)(row0 + g) * lda_ + t;
  const double* b_ptr = Bt + (size_t)(col_tile0 * 8 + g) * ldb_ + t;
  for (int k = 0; k < kdim; k += 4) {
    double av[TM], bv[TN];
#pragma unroll
    for (int i = 0; i < TM; ++i) av[i] = (double)a_ptr[(size_t)(8 * i) * lda_ + k];
#pragma unroll
    for (int j = 0; j < TN; ++j)
      bv[j] = (col_tile0 + j < n_col_tiles) ? b_ptr[(size_t)(8 * j) * ldb_ + k] : 0.0;
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) dmma_8x8x4(acc[i][j], av[i], bv[j]);
  }
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j)
      if (col_tile0 + j < n_col_tiles)
        emit(row0 + 8 * i + g, (col_tile0 + j) * 8 + 2 * t, acc[i][j][0], acc[i][j][1]);
}

template <typename Tin>
__device__ __forceinline__ void load_row_chunk8(const Tin* __restrict__ x, int64_t chunk,
                                                float* dst) {
  float v[8];
  load8(x, chunk, v);
  float4* d = reinterpret_cast<float4*>(dst);
  d[0] = make_float4(v[0], v[1], v[2], v[3]);
  d[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// 8 input elements held as raw vectors, so a prefetch does not wait for its data.
// kCg: load through L2 only (data the same kernel wrote on another SM), else
// through the read-only path (data written before the kernel started).
template <typename Tin> struct RawChunk;
template <> struct RawChunk<float> {
  float4 v0, v1;
  template <bool kCg = false>
  __device__ __forceinline__ void load(const float* __restrict__ x, int64_t chunk) {
    const float4* p = reinterpret_cast<const float4*>(x + chunk * 8);
    v0 = kCg ? __ldcg(p) : __ldg(p);
    v1 = kCg ? __ldcg(p + 1) : __ldg(p + 1);
  }
  __device__ __forceinline__ void zero() { v0 = v1 = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void store(float* dst) const {
    reinterpret_cast<float4*>(dst)[0] = v0;
    reinterpret_cast<float4*>(dst)[1] = v1;
  }
};
template <> struct RawChunk<__nv_bfloat16> {
  uint4 v;
  template <bool kCg = false>
  __device__ __forceinline__ void load(const __nv_bfloat16* __restrict__ x, int64_t chunk) {
    const uint4* p = reinterpret_cast<const uint4*>(x + chunk * 8);
    v = kCg ? __ldcg(p) : __ldg(p);
  }
  __device__ __forceinline__ void zero() { v = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void store(float* dst) const {
    reinterpret_cast<float4*>(dst)[0] =
        make_float4(bf16_bits_to_f32(v.x & 0xFFFFu), bf16_bits_to_f32(v.x >> 16),
                    bf16_bits_to_f32(v.y & 0xFFFFu), bf16_bits_to_f32(v.y >> 16));
    reinterpret_cast<float4*>(dst)[1] =
        make_float4(bf16_bits_to_f32(v.z & 0xFFFFu), bf16_bits_to_f32(v.z >> 16),
                    bf16_bits_to_f32(v.w & 0xFFFFu), bf16_bits_to_f32(v.w >> 16));
  }
};

constexpr int kRotTM = 2, kRotTN = 2;  // warp task: 16 x 16 outputs (measured best of 1-4 x 2-4)

// The row tiles tile0, tile0 + tile_step, ... (R rows each) of one launch's
// rows; the caller has waited for its predecessor unless x_early.
template <typename Tin, bool kStoreF32>
__device__ __forceinline__ void rotate_quant_tiles(
    const Tin* __restrict__ x, int64_t M, int K, const float* __restrict__ P1, int a,
    const float* __restrict__ P2, int b, int R, const LoopSegs& segs, int qmax,
    int8_t* __restrict__ codes8,
    int opf, uint8_t* __restrict__ codes4, float* __restrict__ scales,
    float* __restrict__ out_f32, int* __restrict__ asum, int x_early, int64_t tile0,
    int64_t tile_step, unsigned char* smem_raw) {
  bool waited = !x_early;
  const RotLayout L = rot_layout(a, b, R);
  double* sm = reinterpret_cast<double*>(smem_raw);
  double* P2T = sm;
  double* P1T = sm + L.off_p1t;
  double* YT = sm + L.off_yt;
  float* X = reinterpret_cast<float*>(sm + L.off_x);
  float* Z = X;  // (R*a) rows of pitch ldz floats, written after stage 1
  // per row of the tile: input offset (elements; read before the stage-1
  // barrier) and the loop's clip (read in the epilogue, so kept per tile parity)
  __shared__ int64_t row_off[16];
  __shared__ float row_c[2][16];

  const int tid = threadIdx.x, warp = tid >> 5;
  constexpr int kWarps = kThreads / 32;
  const int row_chunks = K >> 3;
  const FastDiv fd_rowc((uint32_t)row_chunks), fd_b((uint32_t)b), fd_a((uint32_t)a);

  // ---- input tiles are prefetched into registers as raw vectors: the first
  // one here, together with the factors (one memory round trip, not one per
  // element: for a few rows this latency is most of the kernel's time), and
  // each next one at the start of the previous tile's MMA stages
  constexpr int kXU = 2, kFU = 24;
  // (without x_early the kernel has already waited for its predecessor above)
  const bool x_pre = R * row_chunks <= kXU * kThreads;
  RawChunk<Tin> xr[kXU];
  auto prefetch_tile = [&](int64_t m0p) {
#pragma unroll
    for (int u = 0; u < kXU; ++u) {
      const int ch = u * kThreads + tid;
      const int r = (int)fd_rowc.div((uint32_t)ch);
      if (ch < R * row_chunks && m0p + r < M) {
        const int64_t gr = m0p + r, j = gr / segs.seg_rows;
        xr[u].load(x + j * segs.x_stride + (gr - j * segs.seg_rows) * K, ch - r * row_chunks);
      } else {
        xr[u].zero();
      }
    }
  };
  if (x_pre) prefetch_tile(tile0 * R);
  {
    const int n2 = b * b, nf = n2 + a * a;
    for (int base = 0; base < nf; base += kFU * kThreads) {
      float v[kFU];
#pragma unroll
      for (int u = 0; u < kFU; ++u) {
        const int e = base + u * kThreads + tid;
        v[u] = e < n2 ? __ldg(P2 + e) : (e < nf ? __ldg(P1 + (e - n2)) : 0.f);
      }
#pragma unroll
      for (int u = 0; u < kFU; ++u) {
        const int e = base + u * kThreads + tid;
        if (e < n2) {  // P2T[j][q] = P2[q][j]
          const int q = (int)fd_b.div((uint32_t)e), j = e - q * b;
          P2T[(size_t)j * L.ldb + q] = (double)v[u];
        } else if (e < nf) {  // P1T[i][p] = P1[p][i]
          const int e1 = e - n2, p = (int)fd_a.div((uint32_t)e1), i = e1 - p * a;
          P1T[(size_t)i * L.lda + p] = (double)v[u];
        }
      }
    }
  }

  // stage 1 tasks: (R*a/16) row pairs x ceil(b/32) column quads
  const int ct = b >> 3;
  const int s1_rt = (R * a) / (8 * kRotTM);
  const int s1_ctq = (ct + kRotTN - 1) / kRotTN;
  const int s1_tasks = s1_rt * s1_ctq;
  // stage 2 tasks per token: (a/16) x ceil(b/32)
  const int s2_rt = a / (8 * kRotTM);
  const int s2_tasks = R * s2_rt * s1_ctq;
  const FastDiv fd_s1ctq((uint32_t)s1_ctq), fd_s2tok((uint32_t)(s2_rt * s1_ctq));

  int par = 0;
  for (int64_t m0 = tile0 * R; m0 < M; m0 += tile_step * R, par ^= 1) {
    const int rows = (M - m0 < (int64_t)R) ? (int)(M - m0) : R;
    if (tid < rows) {
      const int64_t r = m0 + tid, j = r / segs.seg_rows;
      row_off[tid] = j * segs.x_stride + (r - j * segs.seg_rows) * K;
      float cj = segs.c[0];  // static indices keep the parameter block out of local memory
#pragma unroll
      for (int u = 1; u < kMaxLoopsPerLaunch; ++u)
        if (j == u) cj = segs.c[u];
      row_c[par][tid] = cj;
    }
    __syncthreads();  // previous Z consumed; factors and row offsets staged
    if (x_pre) {  // the prefetched registers (zeros past the last row)
#pragma unroll
      for (int u = 0; u < kXU; ++u) {
        const int ch = u * kThreads + tid;
        if (ch < R * row_chunks) {
          const int r = (int)fd_rowc.div((uint32_t)ch), k8 = (ch - r * row_chunks) * 8;
          const int i = (int)fd_b.div((uint32_t)k8), q = k8 - i * b;
          const size_t off = (size_t)(r * a + i) * L.ldb + q;
          if (LQ_IN_RANGE(off + 7, (size_t)R * a * L.ldb)) xr[u].store(X + off);
        }
      }
    } else {
      for (int ch = tid; ch < R * row_chunks; ch += kThreads) {
        const int r = (int)fd_rowc.div((uint32_t)ch), k8 = (ch - r * row_chunks) * 8;
        const int i = (int)fd_b.div((uint32_t)k8), q = k8 - i * b;
        float* dst = X + (size_t)(r * a + i) * L.ldb + q;
        if (r < rows) {
          load_row_chunk8(x + row_off[r], ch - r * row_chunks, dst);
        } else {
          reinterpret_cast<float4*>(dst)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
          reinterpret_cast<float4*>(dst)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
    __syncthreads();
    // the next tile's input is in flight during this tile's MMA stages
    if (x_pre && m0 + tile_step * R < M) prefetch_tile(m0 + tile_step * R);
    // ---- stage 1: Y[(r,i), j] = sum_q X[(r,i), q] P2[q, j]  -> YT[r][j][i]
    for (int task = warp; task < s1_tasks; task += kWarps) {
      const int rt = (int)fd_s1ctq.div((uint32_t)task), cq = task - rt * s1_ctq;
      warp_mma_task<kRotTM, kRotTN>(X, L.ldb, P2T, L.ldb, b, rt * 8 * kRotTM, cq * kRotTN, ct,
                                    [&](int ri, int j, double v0, double v1) {
                                      const int r = (int)fd_a.div((uint32_t)ri), i = ri - r * a;
                                      double* yt = YT + ((size_t)r * b + j) * L.lda + i;
                                      if (!LQ_IN_RANGE(((size_t)r * b + j + 1) * L.lda + i,
                                                       (size_t)R * b * L.lda))
                                        return;
                                      yt[0] = v0;
                                      yt[L.lda] = v1;
                                    });
    }
    __syncthreads();
    // ---- stage 2: Z[r][i][j] = sum_p P1[p, i] Y[r][p][j], rounded once to float32
    for (int task = warp; task < s2_tasks; task += kWarps) {
      const int r = (int)fd_s2tok.div((uint32_t)task);
      const int rem = task - r * (s2_rt * s1_ctq);
      const int rt = (int)fd_s1ctq.div((uint32_t)rem), cq = rem - rt * s1_ctq;
      warp_mma_task<kRotTM, kRotTN>(P1T, L.lda, YT + (size_t)r * b * L.lda, L.lda, a,
                                    rt * 8 * kRotTM, cq * kRotTN, ct,
                                    [&](int i, int j, double v0, double v1) {
                                      float2* z = reinterpret_cast<float2*>(
                                          Z + (size_t)(r * a + i) * L.ldz + j);
                                      if (!LQ_IN_RANGE((size_t)(r * a + i) * L.ldz + j + 1,
                                                       (size_t)R * a * L.ldz))
                                        return;
                                      *z = make_float2(__double2float_rn(v0),
                                                       __double2float_rn(v1));
                                    });
    }
    __syncthreads();
    if (!waited) {  // the previous kernel may still read the output buffers
      pdl_wait();
      waited = true;
    }
    // ---- epilogue: chunk ch covers elements 8*ch .. 8*ch+7 of the R-row tile
    if (kStoreF32) {
      for (int ch = tid; ch < rows * row_chunks; ch += kThreads) {
        const int r = (int)fd_rowc.div((uint32_t)ch), k8 = (ch - r * row_chunks) * 8;
        const int i = (int)fd_b.div((uint32_t)k8), j = k8 - i * b;
        const float4* src = reinterpret_cast<const float4*>(Z + (size_t)(r * a + i) * L.ldz + j);
        float4* dst = reinterpret_cast<float4*>(out_f32 + (size_t)m0 * K + (size_t)ch * 8);
        dst[0] = src[0];
        dst[1] = src[1];
      }
    } else {
      const int n_chunks = R * row_chunks;
      for (int base = 0; base < n_chunks; base += kThreads) {
        const int ch = base + tid;
        const int r = (int)fd_rowc.div((uint32_t)ch);
        const bool valid = ch < n_chunks && r < rows;
        float v[8];
        const float c = valid ? row_c[par][r] : 1.f;
        if (valid) {
          const int k8 = (ch - r * row_chunks) * 8;
          const int i = (int)fd_b.div((uint32_t)k8), j = k8 - i * b;
          const float4* src =
              reinterpret_cast<const float4*>(Z + (size_t)(r * a + i) * L.ldz + j);
          const float4 u0 = src[0], u1 = src[1];
          v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
          v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
        uint32_t q[8];
        const float s = quant_group8(v, c, qmax, q);
        if (opf == kOpGemvAct) {
          const int gs = group_code_sum(q);
          if (valid)
            store_codes<true>(q, s, m0 * row_chunks + ch, codes8, opf, codes4, scales,
                              K / kGroup, gs, asum);
        } else if (valid) {
          if (LQ_IN_RANGE(m0 * row_chunks + ch, M * row_chunks))
            store_codes<false>(q, s, m0 * row_chunks + ch, codes8, opf, codes4, scales);
        }
      }
    }
  }
}

template <typename Tin, bool kStoreF32>
__global__ void __launch_bounds__(kThreads, 2) k_rotate_quant(
    const Tin* __restrict__ x, int64_t M, int K, const float* __restrict__ P1, int a,
    const float* __restrict__ P2, int b, int R, const LoopSegs segs, int qmax,
    int8_t* __restrict__ codes8,
    int opf, uint8_t* __restrict__ codes4, float* __restrict__ scales,
    float* __restrict__ out_f32, int* __restrict__ asum, int x_early) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_trigger();
  if (!x_early) pdl_wait();
  rotate_quant_tiles<Tin, kStoreF32>(x, M, K, P1, a, P2, b, R, segs, qmax, codes8, opf, codes4,
                                     scales, out_f32, asum, x_early, blockIdx.x, gridDim.x,
                                     smem_raw);
}

// The grouped decode quantizer: block (x, y) takes row tiles x, x + gridDim.x,
// ... (R rows each) of unit y, staging the unit's factors once; blocks past
// the unit's tiles exit.  The inputs were written before the sequence began.
template <typename Tin>
__global__ void __launch_bounds__(kThreads, 2) k_rotate_quant_units(
    const __grid_constant__ GroupLaunch P, int R) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_trigger();
  const GroupUnit& U = P.u[blockIdx.y];
  const int64_t tiles = (U.rows + R - 1) / R;
  if ((int64_t)blockIdx.x >= tiles) return;
  LoopSegs segs;
  segs.seg_rows = U.seg_rows;
  segs.x_stride = U.x_stride;
#pragma unroll
  for (int u = 0; u < kMaxLoopsPerLaunch; ++u) segs.c[u] = U.c[u];
  rotate_quant_tiles<Tin, false>(static_cast<const Tin*>(U.x), U.rows, U.K, U.P1, U.a, U.P2,
                                 U.b, R, segs, U.qmax, U.codes, kOpGemvAct, nullptr, U.scales,
                                 nullptr, U.asum, 1, blockIdx.x, gridDim.x, smem_raw);
}

// ---------------------------------------------------------------------------
// Warp-specialised fused rotation + quantization for many token rows.
//
// The same arithmetic as k_rotate_quant (X -> X P2 -> P1^T (X P2) on the
// FP64 tensor-core MMA, float64 sums rounded once to float32, then the
// group-32 quantizer), but the FP64 MMA never waits for the quantizer: one
// persistent block per SM runs
//   8 MMA warps   stage 1 into YT, stage 2 into Z (written over the tile's X),
//   4 quant warps staging the next tiles' inputs into shared memory and
//                 quantizing the finished Z tiles,
// over two X/Z tile buffers.  Per tile i (buffer s = i % 2) the quant warps
// load X(i) into buffer s and arrive on barrier XFULL[s]; the MMA warps wait
// there, rotate, write Z(i) into buffer s and arrive on ZFULL[s]; the quant
// warps wait there, quantize Z(i) and only then load X(i + 2) into the same
// buffer.  Hand-offs are named barriers (bar.arrive by the producer,
// bar.sync by the consumer), which order the shared-memory accesses of both
// sides; every barrier use alternates with the opposite one, so no
// generation is ever skipped.  The input of tile i + 2 is fetched into
// registers before the quant warps wait for Z(i), so its global-memory
// latency overlaps the MMA stages.
//
// Shared memory: P2T [b][b+4] and P1T [a][a+4] (float64), YT [R][b][a+4]
// (float64, MMA warps only), and two X/Z buffers of R*a rows x (b+4) floats.
// ---------------------------------------------------------------------------
// Two configurations (template arguments), chosen per factor shape at launch:
// 8 MMA warps with 16 x 32 warp tasks (more independent MMA chains per warp)
// when both stages split evenly over 8 warps, else 12 MMA warps with 16 x 16
// tasks (32 x 64 factors: 4 % faster with the wide tasks; 64 x 88: 4 % with
// 12 warps).
constexpr int kWsQWarps = 4;
constexpr int kWsQThreads = 32 * kWsQWarps;
template <int kMmaWarps>
__host__ __device__ constexpr int ws_threads() { return 32 * (kMmaWarps + kWsQWarps); }
constexpr int kWsLoadU = 8;  // input chunks (8 elements) per quant thread in flight
constexpr size_t kWsSmemLimit = 226u * 1024u;  // dynamic shared memory of one block
// named barrier ids (0 is __syncthreads)
constexpr int kBarWsMma = 1;    // MMA warps among themselves
constexpr int kBarWsQ = 2;      // quant warps among themselves
constexpr int kBarWsXFull = 3;  // + s: X of buffer s staged
constexpr int kBarWsZFull = 5;  // + s: Z of buffer s written

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

struct WsLayout {
  int a, b, R, lda, ldb, ldz;
  size_t off_p1t, off_yt, off_x, xz_floats, bytes;  // double offsets; floats per X/Z buffer
};

__host__ __device__ inline WsLayout ws_layout(int a, int b, int R) {
  WsLayout L;
  L.a = a;
  L.b = b;
  L.R = R;
  L.lda = a + 4;
  L.ldb = b + 4;
  L.ldz = b + 4;
  L.off_p1t = (size_t)b * L.ldb;
  L.off_yt = L.off_p1t + (size_t)a * L.lda;
  L.off_x = L.off_yt + (size_t)R * b * L.lda;
  L.xz_floats = (size_t)R * a * L.ldb;
  L.bytes = 8 * L.off_x + 4 * 2 * L.xz_floats;
  return L;
}

template <typename Tin, int kTN, int kWsMmaWarps>
__global__ void __launch_bounds__(ws_threads<kWsMmaWarps>(), 1) k_rotate_quant_ws(
    const Tin* __restrict__ x, int64_t M, int K, const float* __restrict__ P1, int a,
    const float* __restrict__ P2, int b, int R, const LoopSegs segs, int qmax,
    int8_t* __restrict__ codes8, int opf, uint8_t* __restrict__ codes4,
    float* __restrict__ scales, int x_early) {
  constexpr int kWsMmaThreads = 32 * kWsMmaWarps;
  constexpr int kWsThreads = ws_threads<kWsMmaWarps>();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_trigger();
  if (!x_early) pdl_wait();
  const WsLayout L = ws_layout(a, b, R);
  double* sm = reinterpret_cast<double*>(smem_raw);
  double* P2T = sm;
  double* P1T = sm + L.off_p1t;
  double* YT = sm + L.off_yt;
  float* XZ0 = reinterpret_cast<float*>(sm + L.off_x);
  __shared__ float row_c[2][16];  // clip of each row of each buffer

  const int tid = threadIdx.x, warp = tid >> 5;
  const int row_chunks = K >> 3;
  const FastDiv fd_rowc((uint32_t)row_chunks), fd_b((uint32_t)b), fd_a((uint32_t)a);

  // factors, all threads, float64, transposed
  {
    constexpr int kFU = 16;
    const int n2 = b * b, nf = n2 + a * a;
    for (int base = 0; base < nf; base += kFU * kWsThreads) {
      float v[kFU];
#pragma unroll
      for (int u = 0; u < kFU; ++u) {
        const int e = base + u * kWsThreads + tid;
        v[u] = e < n2 ? __ldg(P2 + e) : (e < nf ? __ldg(P1 + (e - n2)) : 0.f);
      }
#pragma unroll
      for (int u = 0; u < kFU; ++u) {
        const int e = base + u * kWsThreads + tid;
        if (e < n2) {  // P2T[j][q] = P2[q][j]
          const int q = (int)fd_b.div((uint32_t)e), j = e - q * b;
          P2T[(size_t)j * L.ldb + q] = (double)v[u];
        } else if (e < nf) {  // P1T[i][p] = P1[p][i]
          const int e1 = e - n2, p = (int)fd_a.div((uint32_t)e1), i = e1 - p * a;
          P1T[(size_t)i * L.lda + p] = (double)v[u];
        }
      }
    }
  }
  __syncthreads();

  const int64_t n_tiles = (M + R - 1) / R;
  const int64_t my_tiles =
      n_tiles > (int64_t)blockIdx.x ? (n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (warp < kWsMmaWarps) {
    // ---------------- MMA warps ----------------
    const int ct = b >> 3;
    const int s1_ctq = (ct + kTN - 1) / kTN;
    const int s1_tasks = ((R * a) / (8 * kRotTM)) * s1_ctq;
    const int s2_rt = a / (8 * kRotTM);
    const int s2_tasks = R * s2_rt * s1_ctq;
    const FastDiv fd_s1ctq((uint32_t)s1_ctq), fd_s2tok((uint32_t)(s2_rt * s1_ctq));
    for (int64_t it = 0; it < my_tiles; ++it) {
      const int sb = (int)(it & 1);
      float* XZ = XZ0 + sb * L.xz_floats;
      named_sync(kBarWsXFull + sb, kWsThreads);  // X(it) staged
      // stage 1: Y[(r,i), j] = sum_q X[(r,i), q] P2[q, j]  -> YT[r][j][i]
      for (int task = warp; task < s1_tasks; task += kWsMmaWarps) {
        const int rt = (int)fd_s1ctq.div((uint32_t)task), cq = task - rt * s1_ctq;
        warp_mma_task<kRotTM, kTN>(XZ, L.ldb, P2T, L.ldb, b, rt * 8 * kRotTM, cq * kTN, ct,
                                      [&](int ri, int j, double v0, double v1) {
                                        const int r = (int)fd_a.div((uint32_t)ri), i = ri - r * a;
                                        double* yt = YT + ((size_t)r * b + j) * L.lda + i;
                                        if (!LQ_IN_RANGE(((size_t)r * b + j + 1) * L.lda + i,
                                                         (size_t)R * b * L.lda))
                                          return;
                                        yt[0] = v0;
                                        yt[L.lda] = v1;
                                      });
      }
      named_sync(kBarWsMma, kWsMmaThreads);  // YT complete, X(it) no longer read
      // stage 2: Z[r][i][j] = sum_p P1[p, i] Y[r][p][j], rounded once to float32
      for (int task = warp; task < s2_tasks; task += kWsMmaWarps) {
        const int r = (int)fd_s2tok.div((uint32_t)task);
        const int rem = task - r * (s2_rt * s1_ctq);
        const int rt = (int)fd_s1ctq.div((uint32_t)rem), cq = rem - rt * s1_ctq;
        warp_mma_task<kRotTM, kTN>(P1T, L.lda, YT + (size_t)r * b * L.lda, L.lda, a,
                                      rt * 8 * kRotTM, cq * kTN, ct,
                                      [&](int i, int j, double v0, double v1) {
                                        float2* z = reinterpret_cast<float2*>(
                                            XZ + (size_t)(r * a + i) * L.ldz + j);
                                        if (!LQ_IN_RANGE((size_t)(r * a + i) * L.ldz + j + 1,
                                                         L.xz_floats))
                                          return;
                                        *z = make_float2(__double2float_rn(v0),
                                                         __double2float_rn(v1));
                                      });
      }
      named_arrive(kBarWsZFull + sb, kWsThreads);  // Z(it) written
      named_sync(kBarWsMma, kWsMmaThreads);        // YT free for the next tile
    }
  } else {
    // ---------------- quant warps: stage inputs, quantize outputs ----------------
    const int qt = tid - kWsMmaThreads;
    const int n_chunks = R * row_chunks;
    bool waited = !x_early;
    RawChunk<Tin> xr[kWsLoadU];
    // load the input of tile `it` into registers (first kWsLoadU chunks per thread)
    auto fetch = [&](int64_t it) {
      const int64_t m0 = ((int64_t)blockIdx.x + it * gridDim.x) * R;
#pragma unroll
      for (int u = 0; u < kWsLoadU; ++u) {
        const int ch = u * kWsQThreads + qt;
        const int r = (int)fd_rowc.div((uint32_t)ch);
        if (ch < n_chunks && m0 + r < M) {
          const int64_t gr = m0 + r, j = gr / segs.seg_rows;
          xr[u].load(x + j * segs.x_stride + (gr - j * segs.seg_rows) * K, ch - r * row_chunks);
        } else {
          xr[u].zero();
        }
      }
    };
    // store tile `it`'s input into its buffer (the registers, then any rest directly)
    auto stage = [&](int64_t it) {
      const int sb = (int)(it & 1);
      float* X = XZ0 + sb * L.xz_floats;
      const int64_t m0 = ((int64_t)blockIdx.x + it * gridDim.x) * R;
#pragma unroll
      for (int u = 0; u < kWsLoadU; ++u) {
        const int ch = u * kWsQThreads + qt;
        if (ch < n_chunks) {
          const int r = (int)fd_rowc.div((uint32_t)ch), k8 = (ch - r * row_chunks) * 8;
          const int i = (int)fd_b.div((uint32_t)k8), q = k8 - i * b;
          const size_t off = (size_t)(r * a + i) * L.ldb + q;
          if (LQ_IN_RANGE(off + 7, L.xz_floats)) xr[u].store(X + off);
        }
      }
      for (int ch = kWsLoadU * kWsQThreads + qt; ch < n_chunks; ch += kWsQThreads) {
        const int r = (int)fd_rowc.div((uint32_t)ch), k8 = (ch - r * row_chunks) * 8;
        const int i = (int)fd_b.div((uint32_t)k8), q = k8 - i * b;
        RawChunk<Tin> v;
        if (m0 + r < M) {
          const int64_t gr = m0 + r, j = gr / segs.seg_rows;
          v.load(x + j * segs.x_stride + (gr - j * segs.seg_rows) * K, ch - r * row_chunks);
        } else {
          v.zero();
        }
        const size_t off = (size_t)(r * a + i) * L.ldb + q;
        if (LQ_IN_RANGE(off + 7, L.xz_floats)) v.store(X + off);
      }
      if (qt < R) {
        const int64_t gr = m0 + qt, j = gr / segs.seg_rows;
        float cj = segs.c[0];  // static indices keep the parameter block out of local memory
#pragma unroll
        for (int u = 1; u < kMaxLoopsPerLaunch; ++u)
          if (j == u) cj = segs.c[u];
        row_c[sb][qt] = cj;
      }
    };
    for (int64_t it = 0; it < my_tiles + 2; ++it) {
      const int sb = (int)(it & 1);
      if (it < my_tiles) fetch(it);
      if (it >= 2) {
        // quantize Z(it - 2) from buffer sb
        named_sync(kBarWsZFull + sb, kWsThreads);
        if (!waited) {  // the previous kernel may still read the output buffers
          pdl_wait();
          waited = true;
        }
        const float* Z = XZ0 + sb * L.xz_floats;
        const int64_t m0 = ((int64_t)blockIdx.x + (it - 2) * gridDim.x) * R;
        const int rows = (M - m0 < (int64_t)R) ? (int)(M - m0) : R;
        for (int base = 0; base < n_chunks; base += kWsQThreads) {
          const int ch = base + qt;
          const int r = (int)fd_rowc.div((uint32_t)ch);
          const bool valid = ch < n_chunks && r < rows;
          float v[8];
          const float c = valid ? row_c[sb][r] : 1.f;
          if (valid) {
            const int k8 = (ch - r * row_chunks) * 8;
            const int i = (int)fd_b.div((uint32_t)k8), j = k8 - i * b;
            const float4* src =
                reinterpret_cast<const float4*>(Z + (size_t)(r * a + i) * L.ldz + j);
            const float4 u0 = src[0], u1 = src[1];
            v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
            v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
          }
          uint32_t q[8];
          const float sc = quant_group8(v, c, qmax, q);
          if (valid && LQ_IN_RANGE(m0 * row_chunks + ch, M * row_chunks))
            store_codes<false>(q, sc, m0 * row_chunks + ch, codes8, opf, codes4, scales);
        }
        named_sync(kBarWsQ, kWsQThreads);  // Z(it - 2) and its clips fully read
      }
      if (it < my_tiles) {
        stage(it);
        named_arrive(kBarWsXFull + sb, kWsThreads);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// fused rotation + quantization for a few token rows (decode)
//
// With only a handful of rows the row-tile kernel above leaves most SMs idle
// and each block's time is mostly load and MMA latency.  Here block (row m,
// slice s) computes the 32 columns J = [32s, 32s + 32) of Z = P1^T X P2 for
// one row: Y_J = X P2[:, J] (a x 32, b-long dots), then Z_J = P1^T Y_J (a-long
// dots), both on the FP64 tensor-core MMA like the row-tile kernel, rounded
// once to float32.  When b is a multiple of 32, row i of Z_J is exactly
// quantization group i * b/32 + s, so each block quantizes whole groups.
// Shared-memory operands, row pitches padded by 4 elements:
//   X[i][q] f32 (a x b), P2T[j][q] = P2[q][32s + j] (32 x b), P1T[i][p] = P1[p][i]
//   (a x a), YT[j][p] = Y_J[p][j] (32 x a), Z[i][j] f32 (a x 32).
// ---------------------------------------------------------------------------
constexpr int kSmallMaxA = 64, kSmallMaxB = 128;
constexpr int64_t kSmallRotMaxRows = 16;  // up to the decode GEMV's row limit

struct SmallRotLayout {
  int ldx, ldp2, ldp1, ldy, ldz;
  size_t off_p2t, off_p1t, off_yt, off_x, off_z, bytes;  // byte offsets
};

__host__ __device__ inline SmallRotLayout small_rot_layout(int a, int b) {
  SmallRotLayout L;
  L.ldx = b + 4;
  L.ldp2 = b + 4;
  L.ldp1 = a + 4;
  L.ldy = a + 4;
  L.ldz = 32 + 4;
  L.off_p2t = 0;
  L.off_p1t = L.off_p2t + 8 * (size_t)32 * L.ldp2;
  L.off_yt = L.off_p1t + 8 * (size_t)a * L.ldp1;
  L.off_x = L.off_yt + 8 * (size_t)32 * L.ldy;
  L.off_z = L.off_x + 4 * (size_t)a * L.ldx;
  L.bytes = L.off_z + 4 * (size_t)a * L.ldz;
  return L;
}

// One block's work: row m of the launch (input row xrow, clip c), column
// slice sl.  With x_early the input is read before pdl_wait, which then comes
// before the first store (a previous kernel may still read the output
// buffers); without it the caller has waited already.  kCg: the input was
// written by the same kernel (read through L2, not the read-only path).
template <typename Tin, bool kCg = false>
__device__ __forceinline__ void rotate_quant_small_block(
    const Tin* __restrict__ xrow, int K, const float* __restrict__ P1, int a,
    const float* __restrict__ P2, int b, float c, int qmax, int8_t* __restrict__ codes8, int opf,
    uint8_t* __restrict__ codes4, float* __restrict__ scales, int* __restrict__ asum,
    int x_early, int m, int sl, unsigned char* smem_raw, bool factors_ready = false) {
  const int tid = threadIdx.x, warp = tid >> 5;
  constexpr int kWarps = kThreads / 32;
  const SmallRotLayout L = small_rot_layout(a, b);
  double* P2T = reinterpret_cast<double*>(smem_raw + L.off_p2t);
  double* P1T = reinterpret_cast<double*>(smem_raw + L.off_p1t);
  double* YT = reinterpret_cast<double*>(smem_raw + L.off_yt);
  float* Xs = reinterpret_cast<float*>(smem_raw + L.off_x);
  float* Zs = reinterpret_cast<float*>(smem_raw + L.off_z);
  const FastDiv fd_b((uint32_t)b), fd_a((uint32_t)a);

  // ---- loads, all of a thread's in flight together
  {
    constexpr int kP2U = kSmallMaxB * 32 / kThreads, kP1U = kSmallMaxA * kSmallMaxA / kThreads;
    constexpr int kXU = kSmallMaxA * kSmallMaxB / 8 / kThreads;
    const int n2 = b * 32, n1 = a * a, nx = K >> 3;  // P2 slice, P1, input chunks of 8
    float p2v[kP2U], p1v[kP1U];
    RawChunk<Tin> xv[kXU];
#pragma unroll
    for (int u = 0; u < kXU; ++u)
      if (u * kThreads + tid < nx) xv[u].template load<kCg>(xrow, u * kThreads + tid);
#pragma unroll
    for (int u = 0; u < kP2U; ++u) {  // element (q, j) = (e / 32, e % 32) of the slice
      const int e = u * kThreads + tid;
      p2v[u] = e < n2 && !factors_ready ? __ldg(P2 + (size_t)(e >> 5) * b + 32 * sl + (e & 31))
                                        : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kP1U; ++u) {
      const int e = u * kThreads + tid;
      p1v[u] = e < n1 && !factors_ready ? __ldg(P1 + e) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kXU; ++u) {
      const int ch = u * kThreads + tid;
      if (ch < nx) {
        const int k8 = ch * 8, i = (int)fd_b.div((uint32_t)k8), q = k8 - i * b;
        xv[u].store(Xs + (size_t)i * L.ldx + q);
      }
    }
    if (!factors_ready) {
#pragma unroll
      for (int u = 0; u < kP2U; ++u) {
        const int e = u * kThreads + tid;
        if (e < n2) P2T[(size_t)(e & 31) * L.ldp2 + (e >> 5)] = (double)p2v[u];
      }
#pragma unroll
      for (int u = 0; u < kP1U; ++u) {
        const int e = u * kThreads + tid;
        if (e < n1) {
          const int pp = (int)fd_a.div((uint32_t)e), i = e - pp * a;
          P1T[(size_t)i * L.ldp1 + pp] = (double)p1v[u];
        }
      }
    }
  }
  __syncthreads();

  // warp tasks of 8 x 16 outputs: (a / 8) row tiles x 2 column pairs
  const int n_tasks = (a >> 3) * 2;
  // ---- Y_J[p][j] = sum_q X[p][q] P2[q][32 s + j]  -> YT[j][p]
  for (int task = warp; task < n_tasks; task += kWarps) {
    warp_mma_task<1, 2>(Xs, L.ldx, P2T, L.ldp2, b, (task >> 1) * 8, (task & 1) * 2, 4,
                        [&](int pp, int j, double v0, double v1) {
                          YT[(size_t)j * L.ldy + pp] = v0;
                          YT[(size_t)(j + 1) * L.ldy + pp] = v1;
                        });
  }
  __syncthreads();
  // ---- Z_J[i][j] = sum_p P1[p][i] Y_J[p][j], rounded once to float32
  for (int task = warp; task < n_tasks; task += kWarps) {
    warp_mma_task<1, 2>(P1T, L.ldp1, YT, L.ldy, a, (task >> 1) * 8, (task & 1) * 2, 4,
                        [&](int i, int j, double v0, double v1) {
                          *reinterpret_cast<float2*>(Zs + (size_t)i * L.ldz + j) =
                              make_float2(__double2float_rn(v0), __double2float_rn(v1));
                        });
  }
  __syncthreads();
  if (x_early) pdl_wait();  // the previous kernel may still read the output buffers

  // ---- quantize: thread t takes chunk t % 4 (8 values) of group row t / 4
  const int G = K / kGroup;
  for (int base = 0; base < a * 4; base += kThreads) {
    if (base + (tid & ~31) >= a * 4) break;  // whole warp past the last group
    const int t = base + tid;
    const bool valid = t < a * 4;
    const int i = t >> 2, cq = t & 3;
    float v[8];
    if (valid) {
      const float4* src = reinterpret_cast<const float4*>(Zs + (size_t)i * L.ldz + 8 * cq);
      const float4 u0 = src[0], u1 = src[1];
      v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
      v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
    }
    uint32_t q[8];
    const float st = quant_group8(v, c, qmax, q);
    // chunk of element i * b + 32 s + 8 cq of row m
    const int64_t chunk = ((int64_t)m * K + (int64_t)i * b + 32 * sl + 8 * cq) >> 3;
    if (opf == kOpGemvAct) {
      const int gs = group_code_sum(q);
      if (valid) store_codes<true>(q, st, chunk, codes8, opf, codes4, scales, G, gs, asum);
    } else if (valid) {
      store_codes<false>(q, st, chunk, codes8, opf, codes4, scales);
    }
  }
}

template <typename Tin>
__global__ void __launch_bounds__(kThreads) k_rotate_quant_small(
    const Tin* __restrict__ x, int K, const float* __restrict__ P1, int a,
    const float* __restrict__ P2, int b, const LoopSegs segs, int qmax,
    int8_t* __restrict__ codes8, int opf, uint8_t* __restrict__ codes4,
    float* __restrict__ scales, int* __restrict__ asum, int x_early) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_trigger();
  if (!x_early) pdl_wait();
  const int S = b >> 5;
  const int m = blockIdx.x / S, sl = blockIdx.x - m * S;
  const int64_t jseg = (int64_t)m / segs.seg_rows;
  const Tin* xrow = x + jseg * segs.x_stride + ((int64_t)m - jseg * segs.seg_rows) * K;
  float c = segs.c[0];  // static indices keep the parameter block out of local memory
#pragma unroll
  for (int u = 1; u < kMaxLoopsPerLaunch; ++u)
    if (jseg == u) c = segs.c[u];
  rotate_quant_small_block<Tin>(xrow, K, P1, a, P2, b, c, qmax, codes8, opf, codes4, scales,
                                asum, x_early, m, sl, smem_raw);
}

// ---------------------------------------------------------------------------
// Chain-mode decode: one persistent kernel over the steps of a stack.
//
// One block per SM (a cooperative launch, so every block is resident and a
// wait never depends on a block that has not started).  Per step:
//  1. every block starts copying its slice of the step's weights (rows
//     [n0, n1) of N: packed codes and steps, both contiguous in memory) into
//     shared memory with cp.async, not waited for yet;
//  2. blocks 0 .. M * b/32 - 1 widen their factors (copied raw during the
//     previous step) into float64 operands, wait until every block has
//     written the previous step's output (a counter of blocks), then rotate
//     and quantize one (row, 32-column slice) of the step's input each (the
//     few-row block above), write the activation codes (kOpGemvAct layout),
//     steps and group sums, count themselves done, and start copying the
//     next step's factors;
//  3. every block waits for the step's quantize blocks (a second counter),
//     copies the activation into shared memory, waits for its weight rows
//     and forms y[m][n] for them: two weight rows per warp, lane per group,
//     dp4a on the offset-binary nibbles minus 8 * sum q_a, the fold with both
//     steps in float32, a butterfly sum over the lanes per token (the same
//     arithmetic, in the same order, as the dp4a GEMV kernel), and counts
//     itself done.
// Only the blocks that need a result wait for it; the counters only grow
// within a launch (zeroed before it), so no reset races a waiter.  A wait
// gives up after limit_ns: the block records LQ_ERR_DEVICE_TIMEOUT, drains
// its copies and returns, and every other waiter then gives up at once.
// ---------------------------------------------------------------------------
__device__ int g_chain_status = 0;
constexpr int kChainMaxM = 4;

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Step counters in global memory (zeroed before the launch): a block signals
// after its stores (block barrier, then one thread's fence and atomic add),
// and a block waits until a counter reaches a target (one thread's acquire
// loads, then a block barrier).  A wait gives up after limit_ns, or at once
// when another block already has; false then.
// (the block barrier orders the block's stores before thread 0's release add,
// and thread 0's acquire load before the block's loads after the barrier)
__device__ __forceinline__ void chain_signal(unsigned* cnt) {
  __syncthreads();
  if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(cnt) : "memory");
}

__device__ bool chain_wait(const unsigned* cnt, unsigned target, uint64_t limit_ns) {
  __shared__ int ok;
  if (threadIdx.x == 0) {
    ok = 1;
    if ((int)(ld_acquire_u32(cnt) - target) < 0) {
      const uint64_t t0 = global_timer_ns();
      while ((int)(ld_acquire_u32(cnt) - target) < 0) {
        if (*(volatile int*)&g_chain_status != 0 || global_timer_ns() - t0 > limit_ns) {
          atomicExch(&g_chain_status, (int)LQ_ERR_DEVICE_TIMEOUT);
          ok = 0;
          break;
        }
      }
    }
  }
  __syncthreads();
  return ok != 0;
}

// The few-row block's factors: P2's 32-column slice sl (b rows of 32 floats)
// and P1 (a x a), copied raw into `fsm` by cp.async ahead of their step (one
// commit group, possibly empty, per call), then widened into the block's
// float64 operands in shared memory.
__host__ __device__ inline size_t chain_fac_bytes(int a, int b) {
  return ((size_t)b * 32 + (size_t)a * a) * sizeof(float);
}
__device__ __forceinline__ void chain_issue_factors(const ChainStep& S, int sl, bool mine,
                                                    unsigned char* fsm) {
  if (mine) {
    const int n2 = S.b * 8, n1 = S.a * S.a / 4;  // 16-byte chunks
    for (int i = threadIdx.x; i < n2; i += kThreads) {
      const int q = i >> 3, c = i & 7;
      cp_async16(smem_u32(fsm + 16 * (size_t)i), S.P2 + (size_t)q * S.b + 32 * sl + 4 * c);
    }
    for (int i = threadIdx.x; i < n1; i += kThreads)
      cp_async16(smem_u32(fsm + (size_t)S.b * 128 + 16 * (size_t)i), S.P1 + 4 * (size_t)i);
  }
  cp_async_commit();
}
__device__ __forceinline__ void chain_widen_factors(int a, int b, const unsigned char* fsm,
                                                    unsigned char* smem_raw) {
  const SmallRotLayout L = small_rot_layout(a, b);
  double* P2T = reinterpret_cast<double*>(smem_raw + L.off_p2t);
  double* P1T = reinterpret_cast<double*>(smem_raw + L.off_p1t);
  const float* p2 = reinterpret_cast<const float*>(fsm);
  const float* p1 = p2 + (size_t)b * 32;
  const FastDiv fd_a((uint32_t)a);
  for (int e = threadIdx.x; e < b * 32; e += kThreads)
    P2T[(size_t)(e & 31) * L.ldp2 + (e >> 5)] = (double)p2[e];
  for (int e = threadIdx.x; e < a * a; e += kThreads) {
    const int pp = (int)fd_a.div((uint32_t)e), i = e - pp * a;
    P1T[(size_t)i * L.ldp1 + pp] = (double)p1[e];
  }
}

__host__ __device__ inline size_t chain_act_bytes(int M, int K, int a, int b) {
  const size_t act = (size_t)M * K + 2 * (size_t)M * (K / kGroup) * 4;
  const size_t rot = small_rot_layout(a, b).bytes;
  return ((act > rot ? act : rot) + 15) & ~(size_t)15;
}

__global__ void __launch_bounds__(kThreads, 1) k_chain_decode(const __grid_constant__ ChainLaunch P,
                                                                uint64_t limit_ns) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kWarps = kThreads / 32;
  const int M = P.M;
  // shared memory: rotation scratch, later the activation | raw factors | weights, their steps
  unsigned char* fsm = smem_raw + P.act_bytes;
  unsigned char* wsm = fsm + P.fac_bytes;
  auto q_slice = [&](int st) {  // this block's slice in step st's quantize, or -1
    const int Sl = P.s[st].b >> 5;
    return (int)blockIdx.x < M * Sl ? (int)blockIdx.x % Sl : -1;
  };
  chain_issue_factors(P.s[0], q_slice(0), q_slice(0) >= 0, fsm);
  unsigned q_target = 0;  // quantize blocks of the steps so far
  for (int s = 0; s < P.n_steps; ++s) {
    const ChainStep& S = P.s[s];
    const int K = S.K, N = S.N, G = K / kGroup;
    const int n0 = (int)((int64_t)N * blockIdx.x / gridDim.x);
    const int n1 = (int)((int64_t)N * (blockIdx.x + 1) / gridDim.x);
    const int rows = n1 - n0;
    float* swsm = reinterpret_cast<float*>(wsm + (size_t)rows * (K / 2));
    {  // this block's weight rows of the step (pending groups: factors, weights)
      const int n_w = rows * (K / 32), n_s = rows * G / 4;  // 16-byte chunks
      const uint8_t* wsrc = S.w4 + (size_t)n0 * (K / 2);
      const float* ssrc = S.sw + (size_t)n0 * G;
      for (int i = tid; i < n_w; i += kThreads) cp_async16(smem_u32(wsm + 16 * (size_t)i), wsrc + 16 * (size_t)i);
      for (int i = tid; i < n_s; i += kThreads) cp_async16(smem_u32(swsm + 4 * (size_t)i), ssrc + 4 * (size_t)i);
      cp_async_commit();
    }
    // ---- quantize the step's input: its factors (copied during the previous
    // step) widened first, then, once every block has written the previous
    // step's output, the input rows
    const int Sl = S.b >> 5;
    q_target += (unsigned)(M * Sl);
    const int sl = q_slice(s);
    if (sl >= 0) {
      const int m = (int)blockIdx.x / Sl;
      cp_async_wait<1>();  // the factors (the weights may still be in flight)
      __syncthreads();
      chain_widen_factors(S.a, S.b, fsm, smem_raw);
      if (s > 0 && !chain_wait(P.bar + 1, (unsigned)s * gridDim.x, limit_ns)) {
        cp_async_wait<0>();
        return;
      }
      if (S.x_bf16)
        rotate_quant_small_block<__nv_bfloat16, true>(
            static_cast<const __nv_bfloat16*>(S.x) + (size_t)m * K, K, S.P1, S.a, S.P2, S.b, S.c,
            S.qmax, P.codes, kOpGemvAct, nullptr, P.scales, P.asum, 0, m, sl, smem_raw, true);
      else
        rotate_quant_small_block<float, true>(static_cast<const float*>(S.x) + (size_t)m * K, K,
                                              S.P1, S.a, S.P2, S.b, S.c, S.qmax, P.codes,
                                              kOpGemvAct, nullptr, P.scales, P.asum, 0, m, sl,
                                              smem_raw, true);
      chain_signal(P.bar);
    }
    // the next step's factors (pending groups: weights, next factors); the
    // rotation above has finished reading this step's
    if (s + 1 < P.n_steps) chain_issue_factors(P.s[s + 1], q_slice(s + 1), q_slice(s + 1) >= 0, fsm);
    // ---- every quantize block of this step has written its codes
    if (!chain_wait(P.bar, q_target, limit_ns)) {
      cp_async_wait<0>();
      return;
    }
    // ---- the GEMV of this block's weight rows
    uint4* act = reinterpret_cast<uint4*>(smem_raw);              // M * 2 * G vectors
    int* asum = reinterpret_cast<int*>(act + (size_t)M * 2 * G);  // M * G
    float* ssa = reinterpret_cast<float*>(asum + (size_t)M * G);  // M * G
    {
      // written by other blocks of this kernel: loads through L2
      const uint4* src = reinterpret_cast<const uint4*>(P.codes);
      for (int i = tid; i < M * 2 * G; i += kThreads) act[i] = __ldcg(src + i);
      for (int i = tid; i < M * G; i += kThreads) {
        asum[i] = __ldcg(P.asum + i);
        ssa[i] = __ldcg(P.scales + i);
      }
    }
    if (s + 1 < P.n_steps)
      cp_async_wait<1>();  // the weights (the next factors may still be in flight)
    else
      cp_async_wait<0>();
    __syncthreads();
    // two weight rows per warp at a time: r0 = 2 * warp, + 2 * kWarps, ...
    for (int r0 = 2 * warp; r0 < rows; r0 += 2 * kWarps) {
      const bool two = r0 + 1 < rows;
      float part[2][kChainMaxM];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int m = 0; m < kChainMaxM; ++m) part[h][m] = 0.f;
      for (int g = lane; g < G; g += 32) {
        uint32_t lo[2][4], hi[2][4];
        float swg[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = two ? r0 + h : r0;
          const uint4 w = reinterpret_cast<const uint4*>(wsm + (size_t)r * (K / 2))[g];
          const uint32_t wu[4] = {w.x ^ 0x88888888u, w.y ^ 0x88888888u, w.z ^ 0x88888888u,
                                  w.w ^ 0x88888888u};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            lo[h][i] = wu[i] & 0x0F0F0F0Fu;
            hi[h][i] = (wu[i] >> 4) & 0x0F0F0F0Fu;
          }
          swg[h] = swsm[(size_t)r * G + g];
        }
#pragma unroll
        for (int m = 0; m < kChainMaxM; ++m) {
          if (m < M) {
            const uint4 a0 = act[gemv_act_vec_index(m, 0, g, G)];
            const uint4 a1 = act[gemv_act_vec_index(m, 1, g, G)];
            const int corr = 8 * asum[m * G + g];
            const float sam = ssa[m * G + g];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              int d = dp4a_us(lo[h][0], a0.x, 0);
              d = dp4a_us(hi[h][0], a0.y, d);
              d = dp4a_us(lo[h][1], a0.z, d);
              d = dp4a_us(hi[h][1], a0.w, d);
              d = dp4a_us(lo[h][2], a1.x, d);
              d = dp4a_us(hi[h][2], a1.y, d);
              d = dp4a_us(lo[h][3], a1.z, d);
              d = dp4a_us(hi[h][3], a1.w, d);
              part[h][m] = fmaf(sam * swg[h], (float)(d - corr), part[h][m]);
            }
          }
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int m = 0; m < kChainMaxM; ++m) {
          float v = part[h][m];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
          part[h][m] = v;
        }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = n0 + r0 + h;
        if (h == 0 || two) {
#pragma unroll
          for (int m = 0; m < kChainMaxM; ++m)
            if (lane == m && m < M && LQ_IN_RANGE((size_t)m * N + n, (size_t)M * N))
              S.y[(size_t)m * N + n] = part[h][m];
        }
      }
    }
    chain_signal(P.bar + 1);  // this block's rows of the step's output are written
  }
  cp_async_wait<0>();
}

// a step-counter wait that nothing satisfies
__global__ void k_grid_wait_selftest(unsigned* bar, uint64_t limit_ns) {
  if (threadIdx.x == 0) {
    bar[0] = 0u;
    bar[1] = 0u;
  }
  __syncthreads();
  chain_wait(bar, 1u, limit_ns);
}

// The tensor-core GEMM's weight operand, expanded from the resident packed
// codes for one launch: blocks [0, n_conv) turn packed words (8 codes) into
// 8 code bytes (E4M3 or int8, as the GEMM's kind reads them); blocks from
// n_conv on transpose the N x G steps into G x N in 32 x 32 tiles.  Under
// programmatic dependent launch it waits for its predecessor before writing
// (the previous GEMM of the sequence may still read the same workspace).
__global__ void __launch_bounds__(256) k_weight_operand(
    const uint8_t* __restrict__ codes4, int64_t n_words, int opf, uint8_t* __restrict__ op,
    const float* __restrict__ sw, int64_t N, int64_t G, float* __restrict__ sw_t, int n_conv) {
  pdl_trigger();
  if ((int)blockIdx.x < n_conv) {
    const int64_t stride = (int64_t)n_conv * blockDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t w = i0 < n_words ? __ldg(reinterpret_cast<const uint32_t*>(codes4) + i0) : 0u;
    pdl_wait();
    for (int64_t i = i0; i < n_words; i += stride) {
      if (i != i0) w = __ldg(reinterpret_cast<const uint32_t*>(codes4) + i);
      uint32_t o0 = 0, o1 = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        int nib = (int)((w >> (4 * j)) & 0xFu);
        nib = nib >= 8 ? nib - 16 : nib;
        const uint32_t byte = encode_code_byte(nib, opf);
        if (j < 4) o0 |= byte << (8 * j); else o1 |= byte << (8 * (j - 4));
      }
      reinterpret_cast<uint2*>(op)[i] = make_uint2(o0, o1);
    }
    return;
  }
  // steps: tile t of the (N / 32 rounded up) x (G / 32 rounded up) tiles
  __shared__ float tile[32][33];
  const int64_t t = (int64_t)blockIdx.x - n_conv;
  const int64_t tiles_g = (G + 31) / 32;
  const int64_t r0 = (t / tiles_g) * 32, c0 = (t % tiles_g) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const int64_t r = r0 + i, cc = c0 + tx;
    if (r < N && cc < G) tile[i][tx] = __ldg(sw + r * G + cc);
  }
  __syncthreads();
  pdl_wait();
  for (int i = ty; i < 32; i += 8) {
    const int64_t cc = c0 + i, r = r0 + tx;
    if (r < N && cc < G) sw_t[cc * N + r] = tile[tx][i];
  }
}


template <typename F>
cudaError_t set_smem(F* f, size_t bytes) {
  // The limit is one per function and recorded schedules (CUDA graphs) launch
  // with whatever it is at replay: only ever raise it, so that a smaller call
  // never lowers it under a larger one recorded earlier.
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, size_t> raised;  // per device and function
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  size_t& cur = raised[{dev, (const void*)f}];
  if (bytes <= cur) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) cur = bytes;
  return e;
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
  // prefer two resident blocks per SM (<= 112 KB each, leaving room for the
  // static row arrays), else one (<= 226 KB)
  int best = 0;
  for (int R = 16; R >= 1; R >>= 1) {
    if (rot_layout(a, b, R).bytes <= 112u * 1024u) { best = R; break; }
  }
  if (best == 0 && rot_layout(a, b, 1).bytes <= 226u * 1024u) best = 1;
  if (rows_per_block) *rows_per_block = best;
  return best ? rot_layout(a, b, best).bytes : 0;
}

cudaError_t launch_quantize(const void* x, int x_dtype, int64_t M, int64_t K, const float* P1,
                            int a, const float* P2, int b, const LoopSegs& segs, int bits,
                            int8_t* codes8, int opf, uint8_t* codes4, float* scales,
                            cudaStream_t s, bool pdl, bool x_early, int* asum) {
  const int qmax = bits == 8 ? 127 : 7;
  if (M == 0) return cudaSuccess;
  const float c = segs.c[0];
  if (P1 == nullptr && segs.seg_rows < M) return cudaErrorInvalidValue;
  if (opf == kOpGemvAct && (codes8 == nullptr || asum == nullptr)) return cudaErrorInvalidValue;
  const int G = (int)(K / kGroup);
  const int xe = x_early ? 1 : 0;
  if (P1 == nullptr) {
    const int64_t n_chunks = M * K / 8;
    const int64_t want = (n_chunks + 2 * kThreads - 1) / (2 * kThreads);
    const int grid = (int)std::min<int64_t>(want, (int64_t)num_sms() * 8);
    const bool gv = opf == kOpGemvAct;
    if (x_dtype == LQ_BF16)
      return launch_kernel(gv ? k_quant_only<__nv_bfloat16, true> : k_quant_only<__nv_bfloat16, false>,
                           dim3(grid), dim3(kThreads), 0, s, pdl, (const __nv_bfloat16*)x,
                           n_chunks, c, qmax, codes8, opf, codes4, scales, G, asum, xe);
    return launch_kernel(gv ? k_quant_only<float, true> : k_quant_only<float, false>, dim3(grid),
                         dim3(kThreads), 0, s, pdl, (const float*)x, n_chunks, c, qmax, codes8,
                         opf, codes4, scales, G, asum, xe);
  }
  if (M <= kSmallRotMaxRows && b % 32 == 0 && a <= kSmallMaxA && b <= kSmallMaxB) {
    // a few rows: one block per (row, 32-column slice) on the FP64 FMA units
    const size_t ssm = small_rot_layout(a, b).bytes;
    const int grid = (int)(M * (b / 32));
    cudaError_t e;
    if (x_dtype == LQ_BF16) {
      auto* k = k_rotate_quant_small<__nv_bfloat16>;
      if ((e = set_smem(k, ssm)) != cudaSuccess) return e;
      return launch_kernel(k, dim3(grid), dim3(kThreads), ssm, s, pdl, (const __nv_bfloat16*)x,
                           (int)K, P1, a, P2, b, segs, qmax, codes8, opf, codes4, scales, asum,
                           xe);
    }
    auto* k = k_rotate_quant_small<float>;
    if ((e = set_smem(k, ssm)) != cudaSuccess) return e;
    return launch_kernel(k, dim3(grid), dim3(kThreads), ssm, s, pdl, (const float*)x, (int)K,
                         P1, a, P2, b, segs, qmax, codes8, opf, codes4, scales, asum, xe);
  }
  {  // many rows: the warp-specialised kernel, one persistent block per SM
    int Rw = 0;
    for (int r = 16; r >= 1; r >>= 1)
      if (ws_layout(a, b, r).bytes <= kWsSmemLimit) {
        Rw = r;
        break;
      }
    if (Rw > 0 && opf != kOpGemvAct && M >= (int64_t)Rw * num_sms() * 4) {
      const size_t wsm = ws_layout(a, b, Rw).bytes;
      const int64_t tiles = (M + Rw - 1) / Rw;
      const int grid = (int)std::min<int64_t>(tiles, (int64_t)num_sms());
      // wide warp tasks on 8 MMA warps when both stages split evenly, else 12 warps
      const int ctq4 = ((b >> 3) + 3) / 4;
      const bool wide = (b >> 3) % 4 == 0 && ((Rw * a) / 16 * ctq4) % 8 == 0 &&
                        (Rw * (a / 16) * ctq4) % 8 == 0;
      auto go = [&](auto* k, int threads, const auto* xin) -> cudaError_t {
        cudaError_t e = set_smem(k, wsm);
        if (e != cudaSuccess) return e;
        return launch_kernel(k, dim3(grid), dim3(threads), wsm, s, pdl, xin, M, (int)K, P1, a,
                             P2, b, Rw, segs, qmax, codes8, opf, codes4, scales, xe);
      };
      if (x_dtype == LQ_BF16) {
        const auto* xb = (const __nv_bfloat16*)x;
        return wide ? go(k_rotate_quant_ws<__nv_bfloat16, 4, 8>, ws_threads<8>(), xb)
                    : go(k_rotate_quant_ws<__nv_bfloat16, 2, 12>, ws_threads<12>(), xb);
      }
      const auto* xf = (const float*)x;
      return wide ? go(k_rotate_quant_ws<float, 4, 8>, ws_threads<8>(), xf)
                  : go(k_rotate_quant_ws<float, 2, 12>, ws_threads<12>(), xf);
    }
  }
  int R = 0;
  size_t smem = rotate_smem_bytes(a, b, &R);
  if (smem == 0) return cudaErrorInvalidValue;
  if (M < (int64_t)R * num_sms()) {  // too few rows to fill the GPU: one row per block
    R = 1;
    smem = rot_layout(a, b, 1).bytes;
  }
  const int per_sm = smem <= 112u * 1024u ? 2 : 1;
  const int64_t want = (M + R - 1) / R;
  const int grid = (int)std::min<int64_t>(want, (int64_t)num_sms() * per_sm);
  cudaError_t e;
  if (x_dtype == LQ_BF16) {
    auto* k = k_rotate_quant<__nv_bfloat16, false>;
    if ((e = set_smem(k, smem)) != cudaSuccess) return e;
    return launch_kernel(k, dim3(grid), dim3(kThreads), smem, s, pdl, (const __nv_bfloat16*)x, M,
                         (int)K, P1, a, P2, b, R, segs, qmax, codes8, opf, codes4, scales,
                         (float*)nullptr, asum, xe);
  }
  auto* k = k_rotate_quant<float, false>;
  if ((e = set_smem(k, smem)) != cudaSuccess) return e;
  return launch_kernel(k, dim3(grid), dim3(kThreads), smem, s, pdl, (const float*)x, M, (int)K,
                       P1, a, P2, b, R, segs, qmax, codes8, opf, codes4, scales, (float*)nullptr,
                       asum, xe);
}

cudaError_t launch_rotate_store(const float* x, int64_t M, int64_t K, const float* Q1, int a,
                                const float* Q2, int b, float* out, cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  int R = 0;
  size_t smem = rotate_smem_bytes(a, b, &R);
  if (smem == 0) return cudaErrorInvalidValue;
  if (M < (int64_t)R * num_sms()) {  // too few rows to fill the GPU: one row per block
    R = 1;
    smem = rot_layout(a, b, 1).bytes;
  }
  const int per_sm = smem <= 112u * 1024u ? 2 : 1;
  const int grid = (int)std::min<int64_t>((M + R - 1) / R, (int64_t)num_sms() * per_sm);
  auto* k = k_rotate_quant<float, true>;
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  k<<<grid, kThreads, smem, s>>>(x, M, (int)K, Q1, a, Q2, b, R, one_loop(1.0f), 7, nullptr,
                                 kOpInt8, nullptr, nullptr, out, nullptr, 1);
  return cudaGetLastError();
}


cudaError_t launch_weight_operand(const uint8_t* codes4, const float* sw, int64_t N, int64_t K,
                                  int opf, uint8_t* op, float* sw_t, cudaStream_t s, bool pdl) {
  const int64_t n_words = N * K / 8, G = K / kGroup;
  if (n_words == 0) return cudaSuccess;
  const int n_conv = (int)std::min<int64_t>((n_words + 255) / 256, (int64_t)num_sms() * 8);
  const int64_t n_tr = ((N + 31) / 32) * ((G + 31) / 32);
  if (n_conv + n_tr > INT32_MAX) return cudaErrorInvalidValue;
  return launch_kernel(k_weight_operand, dim3((unsigned)(n_conv + n_tr)), dim3(256), 0, s, pdl,
                       codes4, n_words, opf, op, sw, N, G, sw_t, n_conv);
}


bool group_unit_ok(int64_t rows, int64_t K, int a, int b) {
  int R = 0;
  return rows >= 1 && rows <= kGemvMaxM && K <= 8192 && (int64_t)a * b == K &&
         rotate_smem_bytes(a, b, &R) > 0;
}

cudaError_t launch_quantize_units(const GroupLaunch& P, int x_dtype, cudaStream_t s, bool pdl) {
  if (P.n_units <= 0) return cudaSuccess;
  if (P.n_units > kGroupMaxUnits) return cudaErrorInvalidValue;
  // one row-tile height for the launch: the smallest any unit's factors need
  int R = 16, max_tiles = 0;
  for (int i = 0; i < P.n_units; ++i) {
    const GroupUnit& U = P.u[i];
    int Ru = 0;
    if (!group_unit_ok(U.rows, U.K, U.a, U.b) || U.seg_rows < 1 ||
        (U.rows + U.seg_rows - 1) / U.seg_rows > kMaxLoopsPerLaunch)
      return cudaErrorInvalidValue;
    rotate_smem_bytes(U.a, U.b, &Ru);
    R = std::min(R, Ru);
  }
  size_t smem = 0;
  for (int i = 0; i < P.n_units; ++i) {
    smem = std::max(smem, rot_layout(P.u[i].a, P.u[i].b, R).bytes);
    max_tiles = std::max(max_tiles, (P.u[i].rows + R - 1) / R);
  }
  // about one resident wave (two blocks per SM) over all units: each block
  // stages its unit's factors once and takes several of its tiles
  const int per_unit = std::max(1, std::min(max_tiles, (2 * num_sms() + P.n_units - 1) / P.n_units));
  const dim3 grid((unsigned)per_unit, (unsigned)P.n_units);
  cudaError_t e;
  if (x_dtype == LQ_BF16) {
    auto* k = k_rotate_quant_units<__nv_bfloat16>;
    if ((e = set_smem(k, smem)) != cudaSuccess) return e;
    return launch_kernel(k, grid, dim3(kThreads), smem, s, pdl, P, R);
  }
  auto* k = k_rotate_quant_units<float>;
  if ((e = set_smem(k, smem)) != cudaSuccess) return e;
  return launch_kernel(k, grid, dim3(kThreads), smem, s, pdl, P, R);
}

bool chain_decode_ok(int M, int K, int N, int a, int b, size_t* act, size_t* fac, size_t* wts) {
  if (M < 1 || M > kChainMaxM || K % 128 || K > 8192 || N < 1 || (int64_t)a * b != K ||
      b % 32 || a % 4 || a > kSmallMaxA || b > kSmallMaxB || M * (b / 32) > num_sms())
    return false;
  const int G = K / kGroup;
  const size_t rows_max = (size_t)(N + num_sms() - 1) / num_sms();
  *act = chain_act_bytes(M, K, a, b);
  *fac = chain_fac_bytes(a, b);
  *wts = rows_max * (K / 2 + (size_t)G * 4);
  return *act + *fac + *wts <= 220u * 1024u;
}

cudaError_t launch_chain_decode(const ChainLaunch& P, size_t smem, cudaStream_t s) {
  if (P.n_steps <= 0) return cudaSuccess;
  if (P.n_steps > kChainMaxSteps || P.M < 1 || P.M > kChainMaxM || P.act_bytes % 16 ||
      P.fac_bytes % 16 || smem > 220u * 1024u)
    return cudaErrorInvalidValue;
  cudaError_t e = set_smem(k_chain_decode, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_chain_decode, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  e = cudaMemsetAsync(P.bar, 0, 2 * sizeof(unsigned), s);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)num_sms());
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint64_t limit_ns = 200ull * 1000 * 1000;  // 200 ms per barrier
  return cudaLaunchKernelEx(&cfg, k_chain_decode, P, limit_ns);
}

int take_chain_status() {
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_chain_status, sizeof(int)) != cudaSuccess) return (int)LQ_ERR_CUDA;
  if (v != 0) cudaMemcpyToSymbol(g_chain_status, &zero, sizeof(int));
  return v;
}

cudaError_t launch_grid_wait_selftest(uint64_t limit_ns, cudaStream_t s, unsigned* bar) {
  k_grid_wait_selftest<<<1, 32, 0, s>>>(bar, limit_ns);
  return cudaGetLastError();
}

unsigned long long bounds_fail_quant() { return lq_take_bounds_fail(); }

}  // namespace lq
