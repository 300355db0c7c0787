// Decode-sized group-rescaled GEMV (M <= 16 tokens), weight streaming from HBM.
//
//   y[m,n] = sum_g s_a[m,g] s_w[n,g] sum_{k in g} q_a[m,k] q_w[n,k]
//
// Same arithmetic as the tensor-core GEMM, for the decode regime where each
// loop reads the packed 4-bit weights once and the activation is a handful of
// rows.  One token, and 2 to 4 tokens on launches of less than about one
// resident wave of rows, use dp4a on the CUDA cores (below); 5 to 16 tokens,
// and 2 to 4 on streaming launches, use the integer tensor-core MMA
// (k_group_gemv_mma, further down).
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
#include <map>
#include <mutex>
#include <set>
#include <tuple>
#include <type_traits>

#include "lq_common.cuh"

namespace lq {
namespace {

// output offset of activation row m (rows in segments of seg_rows, segment
// starts y_stride floats apart) and the extent of the rows' outputs
__device__ __forceinline__ size_t gemv_y_offset(int m, int seg_rows, long long y_stride, int N) {
  const int j = m / seg_rows;
  return (size_t)j * (size_t)y_stride + (size_t)(m - j * seg_rows) * N;
}
__device__ __forceinline__ size_t gemv_y_extent(int M, int seg_rows, long long y_stride, int N) {
  return gemv_y_offset(M - 1, seg_rows, y_stride, N) + N;
}

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;


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
    int N, int K, int seg_rows, long long y_stride) {
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
        if (lane == ((r * MB + m) & 31) && m < M && n < N) {
          const size_t yi = gemv_y_offset(m, seg_rows, y_stride, N) + n;
          if (LQ_IN_RANGE(yi, gemv_y_extent(M, seg_rows, y_stride, N))) y[yi] = part[r][m];
        }
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
// 2 to 16 tokens on a streaming launch, and 5 to 16 tokens always: the integer
// dots on the tensor cores (mma.sync m16n8k32, u8 x s8 -> s32), one MMA per
// group, 16 weight rows and block of 8 tokens.
//
// Fragments.  The group's 32 codes form the MMA's K dimension in the order of
// the packed words: thread (g, t) of the MMA holds k-quad t = the low nibbles
// of weight word t (codes 8t, 8t+2, 8t+4, 8t+6) and k-quad t + 4 = its high
// nibbles; the activation fragments are the matching even and odd code words
// e_t, o_t of the kOpGemvAct layout.  Weight nibbles enter as v ^ 8 = q_w + 8
// (unsigned), and the MMA adds sum (q_w + 8) q_a to a constant accumulator
// input of 1.5 * 2^23 (as an integer): its result is the float bit pattern of
// 1.5 * 2^23 + sum (q_w + 8) q_a (|sum| < 2^22), and one float add of
// -(1.5 * 2^23 + 8 sum q_a) (exact: integers below 2^24) leaves the exact
// dot sum q_w q_a, with no int-to-float conversion.  Each output (row, token)
// belongs to one thread, which folds s_w * s_a * dot per group in float32
// (packed f32x2 arithmetic).
//
// Weight stream.  Each warp owns a ring of kS shared-memory stages; a stage is
// 16 rows x kU groups of packed codes (16 bytes per row and group) plus their
// steps, brought in by cp.async (kU lanes copy a row's kU * 16 contiguous
// bytes) and read back with ldmatrix, which hands thread (g, t) word t of row
// g: the A fragment, transposed in the load.  Chunks are stored XOR-swizzled
// by row so that the 8 row addresses of an ldmatrix hit distinct banks.  The
// warp walks its row blocks (rb = warp, + all warps, ...) stage by stage with
// kS - 1 stages in flight; cp.async.wait_group is the only wait.
// The activation (codes of all tokens) is staged once per block in shared
// memory in MMA-fragment order (lane-contiguous, conflict-free), with the
// float offsets -(1.5 * 2^23 + 8 sum q_a) and s_a of each (group, token block,
// thread) in one 16-byte record.
// ---------------------------------------------------------------------------
// d = A B + c (every accumulator input c)
__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1, int c) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%11,%12,%13};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c), "r"(c), "r"(c), "r"(c));
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

constexpr int kMmaWarps = 8;
constexpr int kFloatBias = 0x4B400000;  // bit pattern of 1.5 * 2^23 = 12582912

// shared memory of one block: activation fragments, then kMmaWarps rings
__host__ __device__ constexpr size_t mma_act_bytes(int NB, int64_t G) {
  return (size_t)G * NB * (32 * 8 + 4 * 16);  // uint2 [G][NB][32], float4 [G][NB][4]
}
__host__ __device__ constexpr size_t mma_stage_bytes(int kU) { return (size_t)16 * kU * (16 + 4); }

// One block's work: warp w walks the row blocks rb_first(w), + rb_step, ...
// (my_rb of them); all warps of the block stage the same activation.
template <int NB, int kS, int kU>
__device__ __forceinline__ void gemv_mma_block(
    const int8_t* __restrict__ qa, const int* __restrict__ asum_g, const float* __restrict__ sa,
    const uint8_t* __restrict__ w4, const float* __restrict__ sw, float* __restrict__ y, int M,
    int N, int K, int seg_rows, long long y_stride, int rb_first, int rb_step, int my_rb,
    unsigned char* smem_raw) {
  static_assert(kU % 8 == 0 && kS >= 2, "stages of whole 8-chunk swizzle blocks, double buffered");
  constexpr int kStageW = 16 * kU * 16;  // packed codes of a stage
  constexpr int kStage = (int)mma_stage_bytes(kU);
  const int G = K / kGroup;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const size_t rowstride = (size_t)K / 2;
  unsigned char* ring = smem_raw + mma_act_bytes(NB, G) + (size_t)warp * kS * kStage;
  const uint32_t ring_s = smem_u32(ring);
  const int stages_per_rb = (G + kU - 1) / kU;
  const int n_stages = my_rb * stages_per_rb;
  const bool vec_steps = (G & 3) == 0;  // 16-byte step chunks are aligned
  const size_t y_ext = gemv_y_extent(M, seg_rows, y_stride, N);
  (void)y_ext;

  // copy stage b of this warp (row block rb_first + (b / stages_per_rb) * rb_step, groups
  // (b % stages_per_rb) * kU ..) into slot b % kS; one commit group per stage
  // the stage issued next: its row block and first group (calls come in stage
  // order, so they advance by one stage each, without a division)
  int is_rb = rb_first, is_g0 = 0;
  auto issue = [&](int b) {
    if (b < n_stages) {
      const int rb = is_rb, g0 = is_g0;
      if (g0 + kU >= G) {
        is_g0 = 0;
        is_rb += rb_step;
      } else {
        is_g0 += kU;
      }
      const uint32_t st = ring_s + (uint32_t)((b % kS) * kStage);
      const bool full = rb * 16 + 16 <= N && g0 + kU <= G;  // no row or group outside
      const uint8_t* wb = w4 + (size_t)rb * 16 * rowstride + (size_t)g0 * 16;
      const float* sb = sw + (size_t)rb * 16 * G + g0;
#pragma unroll
      for (int i = 0; i < kU / 2; ++i) {
        const int c = lane + 32 * i, r = c / kU, u = c % kU;
        if (full || (rb * 16 + r < N && g0 + u < G))
          cp_async16(st + (uint32_t)((r * kU + (u ^ (r & 7))) * 16),
                     wb + (uint32_t)(r * (int)rowstride + u * 16));
      }
#pragma unroll
      for (int i = 0; i < kU / 8; ++i) {
        const int c = lane + 32 * i, r = c / (kU / 4), h = c % (kU / 4), n = rb * 16 + r;
        const int grp = g0 + 4 * h;
        const uint32_t dst = st + kStageW + (uint32_t)(r * kU * 4 + h * 16);
        const float* src = sb + (uint32_t)(r * G + 4 * h);
        if (vec_steps) {
          if (n < N && grp < G) cp_async16(dst, src);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (n < N && grp + e < G) cp_async4(dst + 4 * e, src + e);
        }
      }
    }
    cp_async_commit();
  };
  // the weight stream does not depend on the previous kernel: start it first
#pragma unroll
  for (int b = 0; b < kS - 1; ++b) issue(b);

  pdl_wait();  // the activation is the previous kernel's output
  uint2* bfrag = reinterpret_cast<uint2*>(smem_raw);
  float4* offs_sa = reinterpret_cast<float4*>(bfrag + (size_t)G * NB * 32);
  {
    // activation words in source order: uint2 ((m * 2 + h) * G + grp) * 2 + c2 is
    // the fragment of lane (m % 8) * 4 + 2h + c2 in token block m / 8
    const uint2* src = reinterpret_cast<const uint2*>(qa);
    const int n_src = M * 2 * G * 2;
    for (int i = threadIdx.x; i < n_src; i += kMmaWarps * 32) {
      const int c2 = i & 1, grp = (i >> 1) % G, mh = (i >> 1) / G, h = mh & 1, m = mh >> 1;
      bfrag[((size_t)grp * NB + (m >> 3)) * 32 + (m & 7) * 4 + 2 * h + c2] = __ldg(src + i);
    }
    const int n_pad = (NB * 8 - M) * 2 * G * 2;  // empty token slots: zero codes
    for (int i = threadIdx.x; i < n_pad; i += kMmaWarps * 32) {
      const int c2 = i & 1, grp = (i >> 1) % G, mh = (i >> 1) / G, h = mh & 1, m = M + (mh >> 1);
      bfrag[((size_t)grp * NB + (m >> 3)) * 32 + (m & 7) * 4 + 2 * h + c2] = make_uint2(0u, 0u);
    }
    for (int i = threadIdx.x; i < G * NB * 4; i += kMmaWarps * 32) {
      const int tt = i & 3, j = (i >> 2) % NB, grp = (i >> 2) / NB;
      const int m0 = j * 8 + 2 * tt;
      const float o0 = m0 < M ? 8.f * (float)__ldg(asum_g + (size_t)m0 * G + grp) : 0.f;
      const float o1 = m0 + 1 < M ? 8.f * (float)__ldg(asum_g + (size_t)(m0 + 1) * G + grp) : 0.f;
      offs_sa[i] = make_float4(-12582912.0f - o0, -12582912.0f - o1,
                               m0 < M ? __ldg(sa + (size_t)m0 * G + grp) : 0.f,
                               m0 + 1 < M ? __ldg(sa + (size_t)(m0 + 1) * G + grp) : 0.f);
    }
  }
  __syncthreads();

  float2 acc[NB][2];  // [token block][row g, row g + 8] x (token m0, m0 + 1)
#pragma unroll
  for (int j = 0; j < NB; ++j) acc[j][0] = acc[j][1] = make_float2(0.f, 0.f);
  // group pair (u, u + 1) of a stage: ldmatrix matrices 0-3 = rows 0-7 / 8-15 of
  // group u, then of u + 1; lane L addresses row L % 8 of matrix L / 8
  const int lm_row = (lane & 7) + 8 * ((lane >> 3) & 1), lm_du = lane >> 4;
  auto fold_group = [&](int grp, uint32_t wa, uint32_t wb, float swa, float swb) {
    const uint32_t xa = wa ^ 0x88888888u, xb = wb ^ 0x88888888u;
    const uint32_t a0 = xa & 0x0F0F0F0Fu, a1 = xb & 0x0F0F0F0Fu;
    const uint32_t a2 = (xa >> 4) & 0x0F0F0F0Fu, a3 = (xb >> 4) & 0x0F0F0F0Fu;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const size_t f = (size_t)grp * NB + j;
      const uint2 b = bfrag[f * 32 + lane];
      const float4 os = offs_sa[f * 4 + t];
      const float2 off = make_float2(os.x, os.y), s01 = make_float2(os.z, os.w);
      int d[4];
      mma_u8s8_16832(d, a0, a1, a2, a3, b.x, b.y, kFloatBias);
      const float2 da = fadd2(make_float2(__int_as_float(d[0]), __int_as_float(d[1])), off);
      const float2 db = fadd2(make_float2(__int_as_float(d[2]), __int_as_float(d[3])), off);
      acc[j][0] = ffma2(fmul2(make_float2(swa, swa), s01), da, acc[j][0]);
      acc[j][1] = ffma2(fmul2(make_float2(swb, swb), s01), db, acc[j][1]);
    }
  };
  // the groups of one stage; kFull: all kU groups exist (no per-group branches,
  // so that the loads and MMAs of the whole stage can be scheduled together)
  auto fold_stage = [&](auto full_tag, uint32_t st, const float* ssw, int g0) {
    constexpr bool kFull = decltype(full_tag)::value;
#pragma unroll
    for (int q = 0; q < kU / 4; ++q) {
      if (kFull || g0 + 4 * q < G) {
        const float4 fa = *reinterpret_cast<const float4*>(ssw + g * kU + 4 * q);
        const float4 fb = *reinterpret_cast<const float4*>(ssw + (g + 8) * kU + 4 * q);
        const float fa4[4] = {fa.x, fa.y, fa.z, fa.w}, fb4[4] = {fb.x, fb.y, fb.z, fb.w};
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const int u = 4 * q + 2 * p;
          if (kFull || g0 + u < G) {
            uint32_t w[4];
            const int uu = u + lm_du;
            ldmatrix_x4(st + (uint32_t)((lm_row * kU + (uu ^ (lm_row & 7))) * 16), w);
            fold_group(g0 + u, w[0], w[1], fa4[2 * p], fb4[2 * p]);
            if (kFull || g0 + u + 1 < G) fold_group(g0 + u + 1, w[2], w[3], fa4[2 * p + 1], fb4[2 * p + 1]);
          }
        }
      }
    }
  };

  int rb = rb_first, g0 = 0;
  for (int b = 0; b < n_stages; ++b) {
    issue(b + kS - 1);
    cp_async_wait<kS - 1>();  // this thread's copies of stage b have landed
    __syncwarp();             // ... and every other lane's
    const uint32_t st = ring_s + (uint32_t)((b % kS) * kStage);
    const float* ssw = reinterpret_cast<const float*>(ring + (b % kS) * kStage + kStageW);
    if (g0 + kU <= G)
      fold_stage(std::true_type{}, st, ssw, g0);
    else
      fold_stage(std::false_type{}, st, ssw, g0);
    __syncwarp();  // every lane is done with this slot before it is refilled
    if (g0 + kU >= G) {  // last stage of the row block: write its outputs
      const int na = rb * 16 + g, nb = na + 8;
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        const int m0 = j * 8 + 2 * t;
        const size_t o0 = gemv_y_offset(m0, seg_rows, y_stride, N);
        const size_t o1 = gemv_y_offset(m0 + 1, seg_rows, y_stride, N);
        if (na < N) {
          if (m0 < M && LQ_IN_RANGE(o0 + na, y_ext)) y[o0 + na] = acc[j][0].x;
          if (m0 + 1 < M && LQ_IN_RANGE(o1 + na, y_ext)) y[o1 + na] = acc[j][0].y;
        }
        if (nb < N) {
          if (m0 < M && LQ_IN_RANGE(o0 + nb, y_ext)) y[o0 + nb] = acc[j][1].x;
          if (m0 + 1 < M && LQ_IN_RANGE(o1 + nb, y_ext)) y[o1 + nb] = acc[j][1].y;
        }
        acc[j][0] = acc[j][1] = make_float2(0.f, 0.f);
      }
      g0 = 0;
      rb += rb_step;
    } else {
      g0 += kU;
    }
  }
  cp_async_wait<0>();  // no copy outlives the block
}

template <int NB, int kS, int kU, int kMinBlocks>
__global__ void __launch_bounds__(kMmaWarps * 32, kMinBlocks) k_group_gemv_mma(
    const int8_t* __restrict__ qa, const int* __restrict__ asum_g, const float* __restrict__ sa,
    const uint8_t* __restrict__ w4, const float* __restrict__ sw, float* __restrict__ y, int M,
    int N, int K, int seg_rows, long long y_stride) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_trigger();
  const int warp = threadIdx.x >> 5;
  const int gw = blockIdx.x * kMmaWarps + warp, W = gridDim.x * kMmaWarps;
  const int n_rb = (N + 15) / 16;
  const int my_rb = gw < n_rb ? (n_rb - gw + W - 1) / W : 0;
  gemv_mma_block<NB, kS, kU>(qa, asum_g, sa, w4, sw, y, M, N, K, seg_rows, y_stride, gw, W, my_rb,
                             smem_raw);
}

// The grouped decode GEMV: unit u owns blocks [blk0_u, blk0_{u+1}), which split
// its row blocks into equal contiguous ranges; the warps of a block take the
// range's row blocks in turn.
template <int NB, int kS, int kU, int kMinBlocks>
__global__ void __launch_bounds__(kMmaWarps * 32, kMinBlocks) k_group_gemv_mma_units(
    const __grid_constant__ GroupLaunch P) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_trigger();
  int lo = 0, hi = P.n_units - 1;  // the last unit whose first block is at or before this one
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (P.u[mid].blk0 <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
  }
  const GroupUnit& U = P.u[lo];
  const int nblk = (lo + 1 < P.n_units ? P.u[lo + 1].blk0 : P.total_blocks) - U.blk0;
  const int j = (int)blockIdx.x - U.blk0;
  const int n_rb = (U.N + 15) / 16;
  const int rb0 = (int)((int64_t)n_rb * j / nblk), rb1 = (int)((int64_t)n_rb * (j + 1) / nblk);
  const int first = rb0 + (int)(threadIdx.x >> 5);
  const int my_rb = first < rb1 ? (rb1 - first + kMmaWarps - 1) / kMmaWarps : 0;
  gemv_mma_block<NB, kS, kU>(U.codes, U.asum, U.scales, U.w4, U.sw, U.y, U.rows, U.N, U.K,
                             U.seg_rows, U.y_stride, first, kMmaWarps, my_rb, smem_raw);
}

size_t gemv_smem_bytes(int64_t M, int64_t G) { return (size_t)M * G * (32 + 8); }
constexpr size_t kGemvMaxSmem = 200u * 1024u;  // the activation bound of the GEMV path
constexpr size_t kMmaMaxSmem = 227u * 1024u;   // opt-in shared memory of one block

// Resident blocks per SM of kernel k with `smem` bytes of dynamic shared memory
// on the current device.  The first query for a (device, kernel) raises the
// kernel's limit there to max_smem, the largest size any call uses, so that it
// is never lowered under a launch recorded earlier; results are cached.
template <typename F>
cudaError_t blocks_per_sm(F* k, int threads, size_t smem, size_t max_smem, int* per_sm) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, size_t>, int> cache;
  static std::set<std::pair<int, const void*>> raised;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_tuple(dev, (const void*)k, smem);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *per_sm = it->second;
    return cudaSuccess;
  }
  if (!raised.count({dev, (const void*)k})) {
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_smem);
    if (e != cudaSuccess) return e;
    raised.insert({dev, (const void*)k});
  }
  int n = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, smem);
  if (e != cudaSuccess) return e;
  if (n < 1) return cudaErrorInvalidConfiguration;
  cache.emplace(key, n);
  *per_sm = n;
  return cudaSuccess;
}

template <int MB, int GPL, int RPW, bool kDB>
cudaError_t launch_cfg(const int8_t* qa, const int* asum, const float* sa, const uint8_t* w4,
                       const float* sw, float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                       bool pdl, int seg, long long ys) {
  const size_t smem = gemv_smem_bytes(M, K / kGroup);
  auto* k = k_group_gemv<MB, GPL, RPW, kDB>;
  int per_sm = 0;
  cudaError_t e = blocks_per_sm(k, kGemvThreads, smem, kGemvMaxSmem, &per_sm);
  if (e != cudaSuccess) return e;
  // enough warps for one batch of RPW rows each, capped at one resident wave
  const int64_t warps_needed = (N + RPW - 1) / RPW;
  const int64_t want = (warps_needed + kGemvWarps - 1) / kGemvWarps;
  const int64_t blocks = std::min<int64_t>(want, (int64_t)num_sms() * per_sm);
  return launch_kernel(k, dim3((unsigned)blocks), dim3(kGemvThreads), smem, s, pdl, qa, asum, sa,
                       w4, sw, y, (int)M, (int)N, (int)K, seg, ys);
}

// one batch per warp fits in a resident wave: no prefetch registers needed
template <int MB, int GPL, int RPW>
cudaError_t launch_rpw(const int8_t* qa, const int* asum, const float* sa, const uint8_t* w4,
                       const float* sw, float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                       bool pdl, int seg, long long ys) {
  const int64_t one_wave_rows = (int64_t)num_sms() * 2 * kGemvWarps * RPW;
  if (N <= one_wave_rows)
    return launch_cfg<MB, GPL, RPW, false>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
  return launch_cfg<MB, GPL, RPW, true>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
}

template <int NB, int kS, int kU>
cudaError_t launch_mma(const int8_t* qa, const int* asum, const float* sa, const uint8_t* w4,
                       const float* sw, float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                       bool pdl, int seg, long long ys) {
  const int64_t G = K / kGroup;
  const size_t smem = mma_act_bytes(NB, G) + (size_t)kMmaWarps * kS * mma_stage_bytes(kU);
  if (smem > kMmaMaxSmem) return cudaErrorInvalidValue;
  auto* k = k_group_gemv_mma<NB, kS, kU, 2>;
  int per_sm = 0;
  cudaError_t e = blocks_per_sm(k, kMmaWarps * 32, smem, kMmaMaxSmem, &per_sm);
  if (e != cudaSuccess) return e;
  const int64_t row_blocks = (N + 15) / 16;
  const int64_t want = (row_blocks + kMmaWarps - 1) / kMmaWarps;
  const int64_t blocks = std::min<int64_t>(want, (int64_t)num_sms() * per_sm);
  return launch_kernel(k, dim3((unsigned)blocks), dim3(kMmaWarps * 32), smem, s, pdl, qa, asum,
                       sa, w4, sw, y, (int)M, (int)N, (int)K, seg, ys);
}

// the tensor-core GEMV for M tokens: one block of 8 tokens with 16-group
// stages (2 in flight per warp), or two blocks with 8-group stages (3 in
// flight); the activation and the rings fit a block's shared memory up to
// K = 8544 at 16 tokens, above the K <= 8192 of the GEMV path
cudaError_t launch_tc(const int8_t* qa, const int* asum, const float* sa, const uint8_t* w4,
                      const float* sw, float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                      bool pdl, int seg, long long ys) {
  if (M <= 8) return launch_mma<1, 2, 16>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
  return launch_mma<2, 3, 8>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
}

template <int MB>
cudaError_t launch_mb(const int8_t* qa, const int* asum, const float* sa, const uint8_t* w4,
                      const float* sw, float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                      bool pdl, int seg, long long ys) {
  const int64_t G = K / kGroup;
  if (G > 128) return launch_rpw<MB, 8, 1>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
  if (G > 64) return launch_rpw<MB, 4, 1>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
  // up to 4 tokens: when one resident wave covers N, three weight rows per warp in a single
  // batch (decode-sized launches, latency-bound); beyond that, two rows per warp
  // with the next batch in flight, the fastest streaming shape measured (a
  // 263 MB launch at M = 4: 2.98 TB/s, against 2.25 with three rows and 2.52
  // with one)
  if (N >= (int64_t)num_sms() * kGemvWarps * 3 * 3 / 2) {
    if (N <= (int64_t)num_sms() * 2 * kGemvWarps * 3)
      return launch_cfg<MB, 2, 3, false>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
    return launch_cfg<MB, 2, 2, true>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
  }
  return launch_rpw<MB, 2, 1>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
}

// grouped decode GEMV: units get blocks in proportion to their row blocks, one
// resident wave over all units (at least one block per unit, at most one per
// row block)
template <int NB, int kS, int kU>
cudaError_t launch_units_cfg(GroupLaunch& P, int64_t G, int64_t total_rb, cudaStream_t s,
                             bool pdl) {
  const size_t smem = mma_act_bytes(NB, G) + (size_t)kMmaWarps * kS * mma_stage_bytes(kU);
  if (smem > kMmaMaxSmem) return cudaErrorInvalidValue;
  auto* k = k_group_gemv_mma_units<NB, kS, kU, 2>;
  int per_sm = 0;
  cudaError_t e = blocks_per_sm(k, kMmaWarps * 32, smem, kMmaMaxSmem, &per_sm);
  if (e != cudaSuccess) return e;
  const int64_t slots = (int64_t)num_sms() * per_sm;
  int64_t blk = 0;
  for (int i = 0; i < P.n_units; ++i) {
    const int64_t n_rb = (P.u[i].N + 15) / 16;
    const int64_t nb = std::max<int64_t>(1, std::min(n_rb, (n_rb * slots + total_rb - 1) / total_rb));
    P.u[i].blk0 = (int)blk;
    blk += nb;
  }
  if (blk > INT32_MAX) return cudaErrorInvalidValue;
  P.total_blocks = (int)blk;
  return launch_kernel(k, dim3((unsigned)blk), dim3(kMmaWarps * 32), smem, s, pdl, P);
}

}  // namespace

cudaError_t launch_group_gemv(const int8_t* qa, const int* asum, const float* sa,
                              const uint8_t* w4, const float* sw, float* y, int64_t M, int64_t N,
                              int64_t K, cudaStream_t s, bool pdl, int64_t seg_rows,
                              int64_t y_stride) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (K > (int64_t)kGroup * 32 * 8 || M > kGemvMaxM ||
      gemv_smem_bytes(M, K / kGroup) > kGemvMaxSmem || seg_rows < 1 || y_stride < 0)
    return cudaErrorInvalidValue;
  const int seg = (int)std::min<int64_t>(seg_rows, M);
  const long long ys = seg >= M ? 0 : (long long)y_stride;
  if (seg < M && ys < (long long)seg * N) return cudaErrorInvalidValue;  // segments overlap
  // one token: dp4a (a 263 MB launch timed alone: 5.47 TB/s, against 5.25
  // on the tensor-core path, whose block prologue shows when launches are
  // isolated)
  if (M <= 1) return launch_mb<1>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
  // 2 to 4 tokens: dp4a while the rows fit in about one resident wave of
  // warps (one memory latency per warp, the decode-sized launches); once the
  // launch streams at least a wave of 16-row blocks, the tensor-core path
  // with its deeper weight pipeline (a 263 MB launch at M = 4: 5.5 TB/s
  // against 2.9 with dp4a)
  if (M <= 4 && N < (int64_t)num_sms() * 2 * kMmaWarps * 16)
    return launch_mb<4>(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
  return launch_tc(qa, asum, sa, w4, sw, y, M, N, K, s, pdl, seg, ys);
}

cudaError_t launch_gemv_units(GroupLaunch& P, cudaStream_t s, bool pdl) {
  if (P.n_units <= 0) return cudaSuccess;
  if (P.n_units > kGroupMaxUnits) return cudaErrorInvalidValue;
  int max_rows = 0;
  int64_t max_G = 0, total_rb = 0;
  for (int i = 0; i < P.n_units; ++i) {
    const GroupUnit& U = P.u[i];
    if (U.rows < 1 || U.rows > kGemvMaxM || U.K % kGroup || U.K > kGroup * 32 * 8 || U.N < 1 ||
        U.seg_rows < 1 || (U.rows > U.seg_rows && U.y_stride < (long long)U.seg_rows * U.N))
      return cudaErrorInvalidValue;
    max_rows = std::max(max_rows, U.rows);
    max_G = std::max<int64_t>(max_G, U.K / kGroup);
    total_rb += (U.N + 15) / 16;
  }
  if (max_rows <= 8) return launch_units_cfg<1, 2, 16>(P, max_G, total_rb, s, pdl);
  return launch_units_cfg<2, 3, 8>(P, max_G, total_rb, s, pdl);
}

unsigned long long bounds_fail_gemv() { return lq_take_bounds_fail(); }

}  // namespace lq
