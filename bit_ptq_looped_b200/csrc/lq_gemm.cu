// Group-rescaled integer GEMM on the 5th-generation tensor cores (sm_100a).
//
//   y[m,n] = sum_g s_a[m,g] s_w[n,g] sum_{k in g} q_a[m,k] q_w[n,k],  g = 32-wide K groups
//
// ("paper_specification.yaml" of the LoopQ reproduction: lq1_quantization,
// weights and activations group-wise with group size 32, W4 with A4/A8.)
//
// The kernel is persistent: one CTA per SM walks the 128 x 128 tiles of y
// (t = blockIdx.x, + gridDim.x, ...; m-block-major order so concurrently
// processed tiles share A rows and all of B in L2).  Barriers, TMEM and the
// operand ring are set up once per CTA, and the pipeline runs straight across
// tile boundaries: the tensor core starts a tile's first groups while the
// epilogue still folds and stores the previous tile.  Each 32-wide K group is exactly one
// tcgen05.mma instruction (K = 32 bytes for 8-bit operands), written to its
// own TMEM accumulator, because the next group carries different scales and
// cannot be summed into it.  Four 128-column accumulators rotate through the
// 512 TMEM columns, so the tensor core runs up to three groups ahead of the
// epilogue, which folds every group into float32 registers:
//   y += (s_a[m,g] * s_w[n,g]) * acc_g[m,n].
//
// Operands:
//   W4A4: codes stored as FP8 E4M3 bytes (|q| <= 7 is exact in E4M3) and
//         multiplied with kind::f8f6f4, whose float32 accumulator holds the
//         integer group sum (|acc| <= 32*49) exactly;
//   W4A8: codes stored as int8 and multiplied with kind::i8 (int32 sums).
//
// Warp roles (576 threads): warps 0-15 epilogue, warp 16 TMA producer, warp
// 17 MMA issuer.  Epilogue warp w reads TMEM lane quadrant w % 4 (its 32 rows)
// and the 32-column block w / 4 of the accumulators, two groups at a time (one
// barrier wait per pair), releases the buffers, and folds the columns with
// packed f32x2 arithmetic.
// (Variants that pipelined the TMEM loads across pieces or groups, split the
// groups between two warp sets, or ran two CTAs per SM measured no faster.)
// Every mbarrier wait is bounded; on expiry the kernel records
// LQ_ERR_DEVICE_TIMEOUT in a device status word, stops all roles, frees its
// TMEM and returns.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "lq_common.cuh"

namespace lq {
namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int BK = 128;                 // K elements (bytes) per pipeline stage
constexpr int GPS = BK / kGroup;        // groups per stage = 4
constexpr int STAGES = 5;
constexpr int ACC_BUFS = 4;             // 4 x 128 TMEM columns
constexpr int TMEM_COLS = 512;
constexpr int EPI_WARPS = 16;          // 4 lane quadrants x 4 column blocks
constexpr int WARP_TMA = EPI_WARPS;
constexpr int WARP_MMA = EPI_WARPS + 1;
constexpr int THREADS = 32 * (EPI_WARPS + 2);
constexpr int EPI_COLS = BN * 4 / EPI_WARPS;  // 32 columns per epilogue warp

constexpr uint32_t A_BYTES = BM * BK;          // 16 KB
constexpr uint32_t B_BYTES = BN * BK;          // 16 KB
constexpr uint32_t SA_BYTES = BM * GPS * 4;    // 2 KB  [BM][4] float
constexpr uint32_t SW_BYTES = GPS * BN * 4;    // 2 KB  [4][BN] float
constexpr uint32_t STAGE_TX = A_BYTES + B_BYTES + SA_BYTES + SW_BYTES;

constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_B = OFF_A + STAGES * A_BYTES;
constexpr uint32_t OFF_SA = OFF_B + STAGES * B_BYTES;
constexpr uint32_t OFF_SW = OFF_SA + STAGES * SA_BYTES;
constexpr uint32_t OFF_BAR = OFF_SW + STAGES * SW_BYTES;
constexpr uint32_t N_BARS = 2 * STAGES + 2 * ACC_BUFS + 1;
constexpr uint32_t OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack to align the base to 1024

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

__device__ int g_gemm_status = 0;

// Bounded wait that ignores the abort flag: used at teardown so that no bulk
// copy or MMA of this CTA is still in flight when it exits.
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicExch(&g_gemm_status, (int)LQ_ERR_DEVICE_TIMEOUT);
      return;
    }
  }
}

// K-major operand tile, 128-byte rows, 128-byte swizzle, 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);  // start address (16-byte units)
  d |= (uint64_t)1u << 16;                  // leading byte offset (unused for this layout)
  d |= (uint64_t)(1024u >> 4) << 32;        // stride byte offset: 8 rows x 128 B
  d |= (uint64_t)1u << 46;                  // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                  // layout: 128-byte swizzle
  return d;
}

template <int kKindI8>
__host__ __device__ constexpr uint32_t instr_desc() {
  // bits: [4,6) D format, [7,10) A format, [10,13) B format, 15/16 A/B major
  // (0 = K-major), [17,23) N >> 3, [24,29) M >> 4
  return (kKindI8 ? (2u << 4) | (1u << 7) | (1u << 10)   // S32 <- s8 x s8
                  : (1u << 4) | (0u << 7) | (0u << 10))  // F32 <- e4m3 x e4m3
         | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// two accumulator columns as float32: E4M3 path reads float32 sums directly;
// int8 path converts exactly (|acc| < 2^22) through the mantissa of 1.5 * 2^23
template <int kKindI8>
__device__ __forceinline__ float2 acc_pair(uint32_t r0, uint32_t r1) {
  if (kKindI8) {
    const float2 biased = make_float2(__int_as_float((int)r0 + 0x4B400000),
                                      __int_as_float((int)r1 + 0x4B400000));
    return fadd2(biased, make_float2(-12582912.0f, -12582912.0f));
  }
  return make_float2(__uint_as_float(r0), __uint_as_float(r1));
}

template <int kKindI8>
__global__ void __launch_bounds__(THREADS, 1)
    k_group_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSW,
                 float* __restrict__ y, int M, int N, int G, int64_t y_seg_rows,
                 int64_t y_stride) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_kb = G / GPS;
  const int tiles_n = (N + BN - 1) / BN;
  const int n_tiles = tiles_n * ((M + BM - 1) / BM);

  const uint32_t bar_full = base + OFF_BAR;
  const uint32_t bar_empty = bar_full + STAGES * 8;
  const uint32_t bar_accf = bar_empty + STAGES * 8;
  const uint32_t bar_acce = bar_accf + ACC_BUFS * 8;
  const uint32_t bar_drain = bar_acce + ACC_BUFS * 8;  // all MMAs of this CTA retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_MISC + 4);

  pdl_trigger();  // the next kernel of the sequence may start its own prologue
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1 + EPI_WARPS);
    }
    for (int b = 0; b < ACC_BUFS; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, EPI_WARPS);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_TMA && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSA);
    prefetch_tmap(&tmSW);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == WARP_TMA) {
    if (lane == 0) {
      pdl_wait();  // A and its steps come from the previous kernel
      int kbg = 0;  // k-blocks issued by this CTA over all its tiles
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const int m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
        for (int kb = 0; kb < n_kb; ++kb, ++kbg) {
          const int st = kbg % STAGES;
          const uint32_t ph = (uint32_t)(kbg / STAGES) & 1u;
          if (!mbar_wait_bounded(bar_empty + 8 * st, ph ^ 1u, abort_flag, &g_gemm_status,
                                 kWaitLimitNs)) {
            ok = false;
            break;
          }
          const uint32_t full = bar_full + 8 * st;
          mbar_arrive_expect_tx(full, STAGE_TX);
          tma_load_2d(base + OFF_A + st * A_BYTES, &tmA, full, kb * BK, m0);
          tma_load_2d(base + OFF_B + st * B_BYTES, &tmB, full, kb * BK, n0);
          tma_load_2d(base + OFF_SA + st * SA_BYTES, &tmSA, full, kb * GPS, m0);
          tma_load_2d(base + OFF_SW + st * SW_BYTES, &tmSW, full, n0, kb * GPS);
        }
      }
      // never leave the CTA with bulk copies in flight: wait (bounded, even
      // after an abort) for the last STAGES loads to land
      for (int kb = max(0, kbg - STAGES); kb < kbg; ++kb)
        mbar_wait_drain(bar_full + 8 * (kb % STAGES), (uint32_t)(kb / STAGES) & 1u);
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc<kKindI8>();
      int kbg = 0, gi = 0;  // running k-block and group counters over all tiles
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        for (int kb = 0; kb < n_kb && ok; ++kb, ++kbg) {
          const int st = kbg % STAGES;
          const uint32_t ph = (uint32_t)(kbg / STAGES) & 1u;
          if (!mbar_wait_bounded(bar_full + 8 * st, ph, abort_flag, &g_gemm_status,
                                 kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_st = base + OFF_A + st * A_BYTES;
          const uint32_t b_st = base + OFF_B + st * B_BYTES;
          for (int j = 0; j < GPS; ++j, ++gi) {
            const int buf = gi % ACC_BUFS;
            const uint32_t aph = (uint32_t)(gi / ACC_BUFS) & 1u;
            if (!mbar_wait_bounded(bar_acce + 8 * buf, aph ^ 1u, abort_flag, &g_gemm_status,
                                   kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // one MMA per 32-wide group: advance 32 bytes inside the swizzled 128-byte rows
            umma_ss<kKindI8>(tmem_base + (uint32_t)(buf * BN), sw128_kmajor_desc(a_st + 32u * j),
                             sw128_kmajor_desc(b_st + 32u * j), idesc, 0u);
            umma_commit(bar_accf + 8 * buf);
          }
          if (ok) umma_commit(bar_empty + 8 * st);
        }
      }
      // retire every MMA of this CTA before TMEM is released
      umma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0u);
    }
  } else {
    // ---------------- epilogue: warps 0..EPI_WARPS-1 ----------------
    // Groups are folded in pairs (gi, gi + 1) of the same stage.  The MMAs of a
    // CTA retire in issue order, so the barrier of group gi + 1 covers both.
    static_assert(EPI_COLS == 32 && GPS % 2 == 0, "pairs of groups, two 16-column halves");
    const int quad = warp & 3;
    const int col0 = (warp >> 2) * EPI_COLS;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)col0;
    pdl_wait();  // y may be read by a kernel before the previous one
    bool ok = true;
    int kbg0 = 0, gi0 = 0;  // this tile's first k-block and group in the CTA's sequence
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, kbg0 += n_kb, gi0 += G) {
      const int m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
      float2 acc[EPI_COLS / 2];
#pragma unroll
      for (int i = 0; i < EPI_COLS / 2; ++i) acc[i] = make_float2(0.f, 0.f);
      for (int g = 0; g < G && ok; g += 2) {
        const int kbg = kbg0 + g / GPS, j = g % GPS, st = kbg % STAGES;
        const int gi = gi0 + g;  // G is a multiple of 4, so gi % 4 == g % 4
        if (j == 0)  // the pair's steps arrive with its stage
          ok = mbar_wait_bounded(bar_full + 8 * st, (uint32_t)(kbg / STAGES) & 1u, abort_flag,
                                 &g_gemm_status, kWaitLimitNs);
        const int b0 = gi % ACC_BUFS, b1 = (gi + 1) % ACC_BUFS;
        ok = ok && mbar_wait_bounded(bar_accf + 8 * b1, (uint32_t)((gi + 1) / ACC_BUFS) & 1u,
                                     abort_flag, &g_gemm_status, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after();
        const float* sa_row =
            reinterpret_cast<const float*>(gbase + OFF_SA + st * SA_BYTES) + row * 4;
        const float sa0 = sa_row[j], sa1 = sa_row[j + 1];
        const float2 s20 = make_float2(sa0, sa0), s21 = make_float2(sa1, sa1);
        const float4* sw0 =
            reinterpret_cast<const float4*>(gbase + OFF_SW + st * SW_BYTES) + (j * BN + col0) / 4;
        const float4* sw1 = sw0 + BN / 4;
        uint32_t rA[16], rB[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // column halves 0-15, 16-31
          tmem_ld_32x32b_x16(lane_base + (uint32_t)(b0 * BN + 16 * h), rA);
          tmem_ld_32x32b_x16(lane_base + (uint32_t)(b1 * BN + 16 * h), rB);
          tmem_wait_ld();
          if (h == 1) {  // both accumulators fully read: hand the buffers back
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(bar_acce + 8 * b0);
              mbar_arrive(bar_acce + 8 * b1);
            }
          }
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const float4 w0 = sw0[4 * h + c4], w1 = sw1[4 * h + c4];
            float2& a0 = acc[8 * h + 2 * c4];
            float2& a1 = acc[8 * h + 2 * c4 + 1];
            a0 = ffma2(fmul2(s20, make_float2(w0.x, w0.y)),
                       acc_pair<kKindI8>(rA[4 * c4 + 0], rA[4 * c4 + 1]), a0);
            a1 = ffma2(fmul2(s20, make_float2(w0.z, w0.w)),
                       acc_pair<kKindI8>(rA[4 * c4 + 2], rA[4 * c4 + 3]), a1);
            a0 = ffma2(fmul2(s21, make_float2(w1.x, w1.y)),
                       acc_pair<kKindI8>(rB[4 * c4 + 0], rB[4 * c4 + 1]), a0);
            a1 = ffma2(fmul2(s21, make_float2(w1.z, w1.w)),
                       acc_pair<kKindI8>(rB[4 * c4 + 2], rB[4 * c4 + 3]), a1);
          }
        }
        if (j + 2 == GPS) {  // this stage's shared-memory steps are no longer needed
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_empty + 8 * st);
        }
      }
      const int gm = m0 + row;
      if (ok && gm < M) {
        const int64_t jseg = gm / y_seg_rows;  // loop segment of this row
        float* yr = y + jseg * y_stride + (gm - jseg * y_seg_rows) * (int64_t)N + n0 + col0;
#pragma unroll
        for (int c4 = 0; c4 < EPI_COLS / 4; ++c4) {
          if (n0 + col0 + 4 * c4 < N && LQ_IN_RANGE(n0 + col0 + 4 * c4 + 3, N))
            *reinterpret_cast<float4*>(yr + 4 * c4) =
                make_float4(acc[2 * c4].x, acc[2 * c4].y, acc[2 * c4 + 1].x, acc[2 * c4 + 1].y);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_map_2d(CUtensorMap* map, const void* ptr, CUtensorMapDataType dt, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle sw) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int kKindI8>
cudaError_t launch_impl(const uint8_t* A, const float* sa, const uint8_t* B, const float* sw_t,
                        float* y, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                        const char** why, bool pdl, int64_t y_seg_rows, int64_t y_stride) {
  const int64_t G = K / kGroup;
  CUtensorMap mA, mB, mSA, mSW;
  if (!make_map_2d(&mA, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, BK, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mB, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, N, K, BK, BN,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mSA, sa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, G, M, G * 4, GPS, BM,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&mSW, sw_t, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, N, G, N * 4, BN, GPS,
                   CU_TENSOR_MAP_SWIZZLE_NONE)) {
    if (why) *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  static uint64_t attr_set_mask = 0;  // one bit per device
  auto* k = k_group_gemm<kKindI8>;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!((attr_set_mask >> (dev & 63)) & 1u)) {
    cudaError_t e =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set_mask |= 1ull << (dev & 63);
  }
  // persistent: one CTA per SM (1 CTA fits per SM), at most one per tile
  const int64_t n_tiles = ((N + BN - 1) / BN) * ((M + BM - 1) / BM);
  if (n_tiles > INT32_MAX) {
    if (why) *why = "too many output tiles";
    return cudaErrorInvalidValue;
  }
  dim3 grid((unsigned)std::min<int64_t>(n_tiles, num_sms()));
  return launch_kernel(k, grid, dim3(THREADS), SMEM_BYTES, s, pdl, mA, mB, mSA, mSW, y, (int)M,
                       (int)N, (int)G, y_seg_rows, y_stride);
}

}  // namespace

cudaError_t launch_group_gemm(const uint8_t* A, const float* sa, const uint8_t* B,
                              const float* sw_t, float* y, int64_t M, int64_t N, int64_t K,
                              int opf, cudaStream_t s, const char** why, bool pdl,
                              int64_t y_seg_rows, int64_t y_stride) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (y_seg_rows <= 0) return cudaErrorInvalidValue;
  if (opf == kOpE4M3)
    return launch_impl<0>(A, sa, B, sw_t, y, M, N, K, s, why, pdl, y_seg_rows, y_stride);
  return launch_impl<1>(A, sa, B, sw_t, y, M, N, K, s, why, pdl, y_seg_rows, y_stride);
}

namespace {
// One thread waits on an mbarrier phase that nothing completes, through the
// same bounded wait the GEMM roles use; it gives up after limit_ns.
__global__ void k_wait_selftest(uint64_t limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  abort_flag = 0;
  fence_mbar_init();
  mbar_wait_bounded(b, 0u, &abort_flag, &g_gemm_status, limit_ns);
}
}  // namespace

// ---------------------------------------------------------------------------
// Trajectory Hessian H (+)= sum_t X_t^T X_t ("Quantizing Looped Transformers:
// Feedback Exposure and Calibration Blindness", Appendix Table 19, H_t =
// X_t^T X_t; accumulating the GPTQ Hessian across recurrence steps).
//
// The T loop inputs (bf16, R = T*M rows of K) are first transposed to Xt
// (K x R_pad, R_pad = R rounded up to 64, zero padded), so that the reduction
// index is contiguous.  Then H = Xt Xt^T on the tensor cores: one CTA per
// 128 x 128 tile of the upper triangle (the lower one is its mirror), a TMA
// warp streaming 128 x 64 bf16 tiles of both row blocks through a 6-stage
// ring, an MMA warp issuing four kind::f16 MMAs (K = 16 each) per stage, and
// four epilogue warps.  bf16 products are exact in float32; what rounds is
// the summation.  The tensor core's float32 accumulation loses up to about
// one unit in the last place per MMA (it does not round to nearest), which
// over a reduction of thousands of rows grows into a relative error of some
// 1e-5.  So the reduction is cut into slices of 256 rows (16 MMAs): each slice
// is summed by the tensor core into its own TMEM accumulator (four rotate
// through the 512 columns, so the tensor core runs up to three slices ahead),
// and the epilogue adds the finished slices, in order, into float32 registers
// (round to nearest), then writes the tile and, off the diagonal, its
// transpose.
// ---------------------------------------------------------------------------
namespace {

constexpr int HT = 128;               // tile rows / columns of H
constexpr int HK = 64;                // reduction elements per stage (128-byte bf16 rows)
constexpr int H_STAGES = 6;
constexpr int H_SLICE_STAGES = 4;     // stages per accumulator slice: 256 rows, 16 MMAs
constexpr int H_ACC_BUFS = 4;         // 4 x 128 TMEM columns
constexpr int H_TMEM_COLS = HT * H_ACC_BUFS;
constexpr uint32_t H_TILE_BYTES = HT * HK * 2;  // 16 KB
constexpr uint32_t H_STAGE_TX = 2 * H_TILE_BYTES;
constexpr int H_EPI_WARPS = 4;
constexpr int H_WARP_TMA = H_EPI_WARPS, H_WARP_MMA = H_EPI_WARPS + 1;
constexpr int H_THREADS = 32 * (H_EPI_WARPS + 2);
constexpr uint32_t H_OFF_A = 0;
constexpr uint32_t H_OFF_B = H_OFF_A + H_STAGES * H_TILE_BYTES;
constexpr uint32_t H_OFF_BAR = H_OFF_B + H_STAGES * H_TILE_BYTES;
// full, empty per stage; accumulator full, empty per slice buffer; drain
constexpr uint32_t H_N_BARS = 2 * H_STAGES + 2 * H_ACC_BUFS + 1;
constexpr uint32_t H_OFF_MISC = H_OFF_BAR + H_N_BARS * 8;
constexpr uint32_t H_SMEM_BYTES = H_OFF_MISC + 16 + 1024;

__host__ __device__ constexpr uint32_t instr_desc_bf16() {
  // F32 accumulator, A and B bf16, both K-major, N = M = 128
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(HT >> 3) << 17) |
         ((uint32_t)(HT >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}

// tile index of the upper triangle (row-major over mb <= nb) -> (mb, nb)
__device__ __forceinline__ void upper_tile(int t, int nt, int& mb, int& nb) {
  mb = 0;
  while (t >= nt - mb) {
    t -= nt - mb;
    ++mb;
  }
  nb = mb + t;
}

__global__ void __launch_bounds__(H_THREADS, 1)
    k_hessian(const __grid_constant__ CUtensorMap tmX, float* __restrict__ H, int K, int n_kb,
              int accumulate) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_full = base + H_OFF_BAR;
  const uint32_t bar_empty = bar_full + H_STAGES * 8;
  const uint32_t bar_accf = bar_empty + H_STAGES * 8;
  const uint32_t bar_acce = bar_accf + H_ACC_BUFS * 8;
  const uint32_t bar_drain = bar_acce + H_ACC_BUFS * 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + H_OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + H_OFF_MISC + 4);
  const int nt = K / HT;
  const int n_slices = (n_kb + H_SLICE_STAGES - 1) / H_SLICE_STAGES;
  int mb, nb;
  upper_tile(blockIdx.x, nt, mb, nb);
  const int m0 = mb * HT, n0 = nb * HT;

  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < H_STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < H_ACC_BUFS; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, H_EPI_WARPS);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == H_WARP_TMA && lane == 0) prefetch_tmap(&tmX);
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), H_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == H_WARP_TMA) {
    if (lane == 0) {
      pdl_wait();  // Xt comes from the transpose kernel
      int issued = 0;
      for (int kb = 0; kb < n_kb; ++kb) {
        const int st = kb % H_STAGES;
        const uint32_t ph = (uint32_t)(kb / H_STAGES) & 1u;
        if (!mbar_wait_bounded(bar_empty + 8 * st, ph ^ 1u, abort_flag, &g_gemm_status,
                               kWaitLimitNs))
          break;
        const uint32_t full = bar_full + 8 * st;
        mbar_arrive_expect_tx(full, H_STAGE_TX);
        tma_load_2d(base + H_OFF_A + st * H_TILE_BYTES, &tmX, full, kb * HK, m0);
        tma_load_2d(base + H_OFF_B + st * H_TILE_BYTES, &tmX, full, kb * HK, n0);
        issued = kb + 1;
      }
      for (int kb = max(0, issued - H_STAGES); kb < issued; ++kb)
        mbar_wait_drain(bar_full + 8 * (kb % H_STAGES), (uint32_t)(kb / H_STAGES) & 1u);
    }
  } else if (warp == H_WARP_MMA) {
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc_bf16();
      bool ok = true;
      for (int j = 0; j < n_slices && ok; ++j) {
        const int buf = j % H_ACC_BUFS;
        // the epilogue has read this buffer's previous slice
        if (!mbar_wait_bounded(bar_acce + 8 * buf, ((uint32_t)(j / H_ACC_BUFS) & 1u) ^ 1u,
                               abort_flag, &g_gemm_status, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * HT);
        const int kb_end = min(n_kb, (j + 1) * H_SLICE_STAGES);
        for (int kb = j * H_SLICE_STAGES; kb < kb_end; ++kb) {
          const int st = kb % H_STAGES;
          if (!mbar_wait_bounded(bar_full + 8 * st, (uint32_t)(kb / H_STAGES) & 1u, abort_flag,
                                 &g_gemm_status, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_st = base + H_OFF_A + st * H_TILE_BYTES;
          const uint32_t b_st = base + H_OFF_B + st * H_TILE_BYTES;
#pragma unroll
          for (int i = 0; i < HK / 16; ++i)  // K = 16 bf16 = 32 bytes per MMA
            umma_bf16(d, sw128_kmajor_desc(a_st + 32u * i), sw128_kmajor_desc(b_st + 32u * i),
                      idesc, (kb > j * H_SLICE_STAGES || i != 0) ? 1u : 0u);
          umma_commit(bar_empty + 8 * st);
        }
        if (ok) umma_commit(bar_accf + 8 * buf);
      }
      umma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0u);
    }
  } else {
    // ---- epilogue: warp q reads TMEM lanes 32q..32q+31 = rows m0 + 32q + lane
    const int q = warp;
    const int row = q * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
    float h[HT];
#pragma unroll
    for (int i = 0; i < HT; ++i) h[i] = 0.f;
    bool ok = true;
    for (int j = 0; j < n_slices && ok; ++j) {
      const int buf = j % H_ACC_BUFS;
      ok = mbar_wait_bounded(bar_accf + 8 * buf, (uint32_t)(j / H_ACC_BUFS) & 1u, abort_flag,
                             &g_gemm_status, kWaitLimitNs);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < HT / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(lane_base + (uint32_t)(buf * HT + 32 * c), r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) h[32 * c + i] += __uint_as_float(r[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acce + 8 * buf);
    }
    pdl_wait();  // H may be read by an earlier kernel of the stream
    if (ok) {
      // tile (m0 + row, n0 + i): each thread writes the 128 consecutive floats of its row
      float* dst = H + (size_t)(m0 + row) * K + n0;
#pragma unroll
      for (int i = 0; i < HT; i += 4) {
        float4 v = make_float4(h[i], h[i + 1], h[i + 2], h[i + 3]);
        if (accumulate) {
          const float4 o = *reinterpret_cast<const float4*>(dst + i);
          v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
        }
        *reinterpret_cast<float4*>(dst + i) = v;
      }
      if (nb != mb) {
        // mirrored tile (n0 + i, m0 + row): for each i the 32 lanes write 32
        // consecutive floats
#pragma unroll
        for (int i = 0; i < HT; ++i) {
          float* md = H + (size_t)(n0 + i) * K + m0 + row;
          float v = h[i];
          if (accumulate) v += *md;
          *md = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, H_TMEM_COLS);
  }
}

// X (R x K bf16, row-major) -> Xt (K x Rp, zero columns past R).  A block
// moves a 64 x 64 tile with 16-byte loads and stores on both sides.
__global__ void __launch_bounds__(256) k_transpose_bf16(const uint16_t* __restrict__ X,
                                                        int64_t R, int64_t K, int64_t Rp,
                                                        uint16_t* __restrict__ Xt) {
  __shared__ uint16_t tile[64][64 + 2];
  pdl_trigger();
  const int64_t r0 = (int64_t)blockIdx.x * 64, k0 = (int64_t)blockIdx.y * 64;
#pragma unroll
  for (int u = 0; u < 2; ++u) {  // 64 rows x 8 chunks of 8 elements
    const int i = u * 256 + threadIdx.x, row = i >> 3, c8 = (i & 7) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r0 + row < R) v = __ldg(reinterpret_cast<const uint4*>(X + (r0 + row) * K + k0 + c8));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      tile[row][c8 + 2 * e] = (uint16_t)(w[e] & 0xFFFFu);
      tile[row][c8 + 2 * e + 1] = (uint16_t)(w[e] >> 16);
    }
  }
  __syncthreads();
  pdl_wait();  // the previous kernel may still read Xt
#pragma unroll
  for (int u = 0; u < 2; ++u) {  // 64 output rows (k) x 8 chunks of 8 (r)
    const int i = u * 256 + threadIdx.x, kk = i >> 3, r8 = (i & 7) * 8;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w[e] = (uint32_t)tile[r8 + 2 * e][kk] | ((uint32_t)tile[r8 + 2 * e + 1][kk] << 16);
    if (r0 + r8 < Rp)
      *reinterpret_cast<uint4*>(Xt + (k0 + kk) * Rp + r0 + r8) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

int64_t hessian_rows_padded(int64_t R) { return (R + HK - 1) / HK * HK; }

cudaError_t launch_trajectory_hessian(const uint16_t* X, int64_t R, int64_t K, uint16_t* Xt,
                                      float* H, int accumulate, cudaStream_t s,
                                      const char** why) {
  const int64_t Rp = hessian_rows_padded(R);
  dim3 tg((unsigned)(Rp / 64), (unsigned)(K / 64));  // Rp and K are multiples of 64
  cudaError_t e = launch_kernel(k_transpose_bf16, tg, dim3(256), 0, s, false, X, R, K, Rp, Xt);
  if (e != cudaSuccess) return e;
  CUtensorMap mX;
  if (!make_map_2d(&mX, Xt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Rp, K, Rp * 2, HK, HT,
                   CU_TENSOR_MAP_SWIZZLE_128B)) {
    if (why) *why = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  static uint64_t attr_set_mask = 0;  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (!((attr_set_mask >> (dev & 63)) & 1u)) {
    e = cudaFuncSetAttribute(k_hessian, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)H_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set_mask |= 1ull << (dev & 63);
  }
  const int nt = (int)(K / HT);
  return launch_kernel(k_hessian, dim3((unsigned)(nt * (nt + 1) / 2)), dim3(H_THREADS),
                       H_SMEM_BYTES, s, true, mX, H, (int)K, (int)(Rp / HK), accumulate);
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t s) {
  k_wait_selftest<<<1, 32, 0, s>>>(limit_ns);
  return cudaGetLastError();
}

lq_status read_and_clear_device_status(cudaStream_t s) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_error(e, "stream synchronize");
  int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_gemm_status, sizeof(int));
  if (e != cudaSuccess) return cuda_error(e, "read device status");
  if (v != 0) {
    e = cudaMemcpyToSymbol(g_gemm_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_error(e, "clear device status");
    take_chain_status();  // one report covers both status words
    set_error("a bounded device-side wait expired in the GEMM kernel (status %d)", v);
    return (lq_status)v;
  }
  v = take_chain_status();
  if (v != 0) {
    set_error("a grid barrier of the persistent decode kernel gave up (status %d)", v);
    return (lq_status)v;
  }
  return LQ_OK;
}

unsigned long long bounds_fail_gemm() { return lq_take_bounds_fail(); }

}  // namespace lq
