// Shared device/host helpers of the lq library (sm_100a only).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lq.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "lq is written for sm_100a (B200) only"
#endif

namespace lq {

constexpr int kGroup = 32;

// Operand byte format of the codes a consumer kernel reads.
enum OperandFormat : int {
  kOpInt8 = 0,  // two's-complement int8 codes (tcgen05 kind::i8, GEMV)
  kOpE4M3 = 1,  // the same integer codes (|q| <= 7) encoded as FP8 E4M3 (kind::f8f6f4)
  kOpGemvAct = 2,  // int8 codes in the decode GEMV's word order, plus per-group code sums
};

// Decode GEMV activation layout (written by the quantizer with kOpGemvAct,
// read by k_group_gemv).  For row m and group g the 32 int8 codes c0..c31
// become eight 32-bit words: e_i = (c_{8i}, c_{8i+2}, c_{8i+4}, c_{8i+6}) and
// o_i = (c_{8i+1}, c_{8i+3}, c_{8i+5}, c_{8i+7}), low byte first, which line
// up with the low and high nibbles of packed weight word i.  Half h of the
// group holds {e_2h, o_2h, e_2h+1, o_2h+1} as one 16-byte vector at vector
// index (m * 2 + h) * G + g, so the lanes of a warp that own consecutive
// groups read consecutive vectors.  The group's code sum goes to
// asum[m * G + g].
__host__ __device__ inline int64_t gemv_act_vec_index(int64_t m, int64_t h, int64_t g, int64_t G) {
  return (m * 2 + h) * G + g;
}

// ---------------------------------------------------------------------------
// host-side error text (thread-local), defined in lq_api.cu
// ---------------------------------------------------------------------------
void set_error(const char* fmt, ...);
lq_status cuda_error(cudaError_t e, const char* what);

// ---------------------------------------------------------------------------
// code encoders shared by the quantize kernels
// ---------------------------------------------------------------------------
// E4M3 bytes of the integers 0..7: 0, 1.0x2^0, 1.0x2^1, 1.5x2^1, 1.0x2^2,
// 1.25x2^2, 1.5x2^2, 1.75x2^2 (bias 7, 3 mantissa bits), one byte each.
constexpr unsigned long long kE4M3Int0to7 = 0x4E4C4A4844403800ull;

__device__ __forceinline__ uint32_t encode_e4m3_int(int q) {
  uint32_t mag = (uint32_t)(q < 0 ? -q : q);
  uint32_t byte = (uint32_t)(kE4M3Int0to7 >> (8u * mag)) & 0xFFu;
  return byte | (q < 0 ? 0x80u : 0u);
}

__device__ __forceinline__ uint32_t encode_code_byte(int q, int opf) {
  return opf == kOpE4M3 ? encode_e4m3_int(q) : ((uint32_t)q & 0xFFu);
}

// Several loops of one layer in one quantize launch (open mode): launch row r
// belongs to loop segment j = r / seg_rows, reads its input row from
// x + j * x_stride + (r - j * seg_rows) * K (elements) and uses clip c[j].
// A single loop is seg_rows >= M, c[0] its clip.
constexpr int kMaxLoopsPerLaunch = 8;
struct LoopSegs {
  int64_t seg_rows;
  int64_t x_stride;
  float c[kMaxLoopsPerLaunch];
};
inline LoopSegs one_loop(float c) {
  LoopSegs s{};
  s.seg_rows = INT64_MAX;
  s.x_stride = 0;
  s.c[0] = c;
  return s;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch (PTX griddepcontrol).  A kernel launched with
// programmatic stream serialization may start while the previous kernel of
// the stream is still running, as soon as every block of that kernel has
// executed pdl_trigger (or exited).  pdl_wait blocks the calling thread until
// the previous kernel has completed and its memory writes are visible; in a
// kernel launched without the attribute it returns at once.  Every kernel of
// the library calls pdl_wait before its first global write and before reading
// anything an earlier kernel of the same sequence wrote, so completion is
// ordered along the stream exactly as without the attribute.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch `kernel` on stream s, with programmatic stream serialization when
// `pdl` is set (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---------------------------------------------------------------------------
// Index checks of the bounds-check build (-DLQ_BOUNDS_CHECK).  At the checked
// stores a kernel tests the index against the extent it writes; an index out
// of range is recorded (source line and index of the first one, in a status
// word of the kernel's own source file) and the store is skipped, so the
// check never writes out of bounds itself.  lq_check_device reports a
// recorded violation.  In the normal build LQ_IN_RANGE is `true` and costs
// nothing.
// ---------------------------------------------------------------------------
#ifdef LQ_BOUNDS_CHECK
static __device__ unsigned long long g_lq_bounds_fail = 0ull;
__device__ __forceinline__ bool lq_in_range(long long idx, long long extent, int line) {
  if (idx >= 0 && idx < extent) return true;
  atomicCAS(&g_lq_bounds_fail, 0ull,
            ((unsigned long long)line << 40) | ((unsigned long long)idx & 0xFFFFFFFFFFull));
  return false;
}
#define LQ_IN_RANGE(idx, extent) lq_in_range((long long)(idx), (long long)(extent), __LINE__)
// first violation recorded by this source file's kernels (0: none), cleared
static inline unsigned long long lq_take_bounds_fail() {
  unsigned long long v = 0ull, z = 0ull;
  if (cudaMemcpyFromSymbol(&v, g_lq_bounds_fail, sizeof(v)) != cudaSuccess) return ~0ull;
  if (v) cudaMemcpyToSymbol(g_lq_bounds_fail, &z, sizeof(z));
  return v;
}
#else
#define LQ_IN_RANGE(idx, extent) true
static inline unsigned long long lq_take_bounds_fail() { return 0ull; }
#endif
// per source file: the first recorded violation of its kernels (0: none)
unsigned long long bounds_fail_quant();
unsigned long long bounds_fail_gemm();
unsigned long long bounds_fail_gemv();
unsigned long long bounds_fail_cta();

// ---------------------------------------------------------------------------
// PTX wrappers: mbarrier, TMA, tcgen05
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// non-blocking probe of an mbarrier phase
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// cp.async copies into shared memory (one commit group per call of commit)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}

// sum of four products of unsigned bytes (a) and signed bytes (b), plus c
__device__ __forceinline__ int dp4a_us(uint32_t a_unsigned, uint32_t b_signed, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_unsigned), "r"(b_signed), "r"(c));
  return d;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase.  Gives up after `limit_ns` of wall time
// or as soon as *abort becomes non-zero; returns false in both cases (and
// raises *abort on a timeout so the other roles of the CTA stop too).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int* abort, int* dev_status,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort = 1;
      atomicExch(dev_status, (int)LQ_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"((uint64_t)map), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem] = A[smem desc] * B[smem desc]^T (accumulate when acc != 0)
template <int kKindI8>
__device__ __forceinline__ void umma_ss(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t acc) {
  if (kKindI8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
  }
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// TMEM lane (quadrant base + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// 32 lanes x 16 consecutive 32-bit columns
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// packed two-lane float32 arithmetic (sm_100a)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(*reinterpret_cast<unsigned long long*>(&d))
      : "l"(*reinterpret_cast<const unsigned long long*>(&a)),
        "l"(*reinterpret_cast<const unsigned long long*>(&b)),
        "l"(*reinterpret_cast<const unsigned long long*>(&c)));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(*reinterpret_cast<unsigned long long*>(&d))
      : "l"(*reinterpret_cast<const unsigned long long*>(&a)),
        "l"(*reinterpret_cast<const unsigned long long*>(&b)));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(*reinterpret_cast<unsigned long long*>(&d))
      : "l"(*reinterpret_cast<const unsigned long long*>(&a)),
        "l"(*reinterpret_cast<const unsigned long long*>(&b)));
  return d;
}

// ---------------------------------------------------------------------------
// launch entry points implemented by the kernel files (host side)
// ---------------------------------------------------------------------------
int num_sms();

// quantize / rotate (lq_quant.cu)
// pdl: launch with programmatic stream serialization; x_early: x was written
// before the sequence started, so it may be read before pdl_wait.  asum: the
// per-group code sums of the kOpGemvAct layout (else unused).
// segs: the clip (and, for the rotating path, the loop segments) of the rows;
// without P1 the launch must be a single loop.
cudaError_t launch_quantize(const void* x, int x_dtype, int64_t M, int64_t K, const float* P1,
                            int a, const float* P2, int b, const LoopSegs& segs, int bits,
                            int8_t* codes8, int opf, uint8_t* codes4, float* scales,
                            cudaStream_t s, bool pdl = false, bool x_early = true,
                            int* asum = nullptr);
cudaError_t launch_rotate_store(const float* x, int64_t M, int64_t K, const float* Q1, int a,
                                const float* Q2, int b, float* out, cudaStream_t s);
// The GEMM weight operand of one launch from the resident codes and steps:
// N x K code bytes (E4M3 or int8 per opf) and the steps transposed to G x N.
cudaError_t launch_weight_operand(const uint8_t* codes4, const float* sw, int64_t N, int64_t K,
                                  int opf, uint8_t* op, float* sw_t, cudaStream_t s, bool pdl);
size_t rotate_smem_bytes(int a, int b, int* rows_per_block);

// GEMM (lq_gemm.cu).  Output row r goes to y + j * y_stride + (r - j * y_seg_rows) * N,
// j = r / y_seg_rows (one segment when y_seg_rows >= M).
cudaError_t launch_group_gemm(const uint8_t* A, const float* sa, const uint8_t* B,
                              const float* sw_t, float* y, int64_t M, int64_t N, int64_t K,
                              int opf, cudaStream_t s, const char** why, bool pdl = false,
                              int64_t y_seg_rows = INT64_MAX, int64_t y_stride = 0);
lq_status read_and_clear_device_status(cudaStream_t s);
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t s);

// CTA (lq_cta.cu): U8, V8 are float64 d x 8 (rank padded with zero columns), d % 32 == 0
cudaError_t launch_cta_apply(const float* h, int64_t M, int d, const double* U8, const double* V8,
                             const float* a, const float* b, float eta, float* out,
                             cudaStream_t s, bool pdl);

// trajectory Hessian (lq_gemm.cu): X is R x K bf16; Xt scratch of K x
// hessian_rows_padded(R) bf16; K a multiple of 128; H K x K float32
int64_t hessian_rows_padded(int64_t R);
cudaError_t launch_trajectory_hessian(const uint16_t* X, int64_t R, int64_t K, uint16_t* Xt,
                                      float* H, int accumulate, cudaStream_t s,
                                      const char** why);

// GEMV (lq_gemv.cu)
// qa: activation codes in the kOpGemvAct layout, asum their group sums.
// Rows come in segments of seg_rows (the loops of one launch): row m is written
// at y + (m / seg_rows) * y_stride + (m % seg_rows) * N (one segment: seg_rows = M).
cudaError_t launch_group_gemv(const int8_t* qa, const int* asum, const float* sa,
                              const uint8_t* w4, const float* sw, float* y, int64_t M, int64_t N,
                              int64_t K, cudaStream_t s, bool pdl = false,
                              int64_t seg_rows = INT64_MAX, int64_t y_stride = 0);
constexpr int kGemvMaxM = 16;

// ---------------------------------------------------------------------------
// Grouped decode: the independent (layer, loop batch) units of a decode-sized
// open-mode stack in one quantize launch and one GEMV launch.  A unit holds
// rows = seg_rows * (loops) activation rows: row m is row m % seg_rows of loop
// m / seg_rows, read at x + (m / seg_rows) * x_stride + (m % seg_rows) * K
// elements and written at y + (m / seg_rows) * y_stride + (m % seg_rows) * N;
// its activation codes (kOpGemvAct layout), steps and group sums live in its
// own workspace region.  The table is a kernel parameter (__grid_constant__).
// ---------------------------------------------------------------------------
struct GroupUnit {
  const void* x;
  const float* P1;
  const float* P2;
  const uint8_t* w4;  // resident packed codes, N x K/2
  const float* sw;    // resident steps, N x K/32
  float* y;
  int8_t* codes;
  float* scales;
  int* asum;
  long long x_stride;  // elements between the loops' inputs
  long long y_stride;  // floats between the loops' outputs
  float c[kMaxLoopsPerLaunch];  // LAS clip of each loop of the unit
  int K, N, a, b, seg_rows, rows, qmax;
  int blk0;  // GEMV: first block of the unit (set by launch_gemv_units)
};
constexpr int kGroupMaxUnits = 96;  // 96 x 152 B of parameters (the limit is 32764 B)
struct GroupLaunch {
  GroupUnit u[kGroupMaxUnits];
  int n_units;
  int total_blocks;  // GEMV blocks over all units
};
// ---------------------------------------------------------------------------
// Chain-mode decode in one persistent kernel: the steps of a chain-mode stack
// (each step's input the previous step's output) with grid barriers between
// the few-row quantize and the GEMV of each step.  The table is a kernel
// parameter; `work` is the step's activation region (codes in the kOpGemvAct
// layout, steps, group sums) followed by the barrier's two words.
// ---------------------------------------------------------------------------
struct ChainStep {
  const void* x;   // M x K input rows (the stack's input, else the previous output)
  const float* P1;
  const float* P2;
  const uint8_t* w4;  // resident packed codes, N x K/2
  const float* sw;    // resident steps, N x K/32
  float* y;           // M x N output
  float c;            // LAS clip of the step's loop
  int K, N, a, b, qmax, x_bf16;
};
constexpr int kChainMaxSteps = 128;  // 128 x 80 B of parameters
struct ChainLaunch {
  ChainStep s[kChainMaxSteps];
  int n_steps, M;
  int act_bytes, fac_bytes;  // shared-memory regions: rotation / activation, raw factors
  int8_t* codes;
  float* scales;
  int* asum;
  unsigned* bar;  // two words, zeroed before the launch
};
// whether a step's shapes fit the persistent kernel (its shared memory and the
// few-row rotation), and the step's shared-memory regions: rotation scratch /
// activation, raw factors, weight rows (the launch takes the maximum of each)
bool chain_decode_ok(int M, int K, int N, int a, int b, size_t* act, size_t* fac, size_t* wts);
cudaError_t launch_chain_decode(const ChainLaunch& P, size_t smem, cudaStream_t s);
// the persistent kernel's status word (LQ_ERR_DEVICE_TIMEOUT after a grid
// barrier gave up), read and cleared
int take_chain_status();
// diagnostic: a grid barrier that one block never reaches, bounded by limit_ns
cudaError_t launch_grid_wait_selftest(uint64_t limit_ns, cudaStream_t s, unsigned* bar);

// whether a unit's shapes fit the grouped kernels (few-row rotation, GEMV rows)
bool group_unit_ok(int64_t rows, int64_t K, int a, int b);
cudaError_t launch_quantize_units(const GroupLaunch& P, int x_dtype, cudaStream_t s, bool pdl);
cudaError_t launch_gemv_units(GroupLaunch& P, cudaStream_t s, bool pdl);

}  // namespace lq
