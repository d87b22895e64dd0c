// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA tile loads, tcgen05
// (TMEM allocation, MMA, commit, loads) and a few warp utilities.
//
// Every wait here is bounded: a wait that does not complete within
// kWaitTimeoutNs sets the CTA's abort flag and the launch's error word, then
// returns false so that the caller can unwind instead of hanging the GPU.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace dsa {

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s: far above any legitimate wait

// Error bits written to the per-launch device error word.
enum : uint32_t {
  kErrTimeout = 1u << 0,   // a bounded wait gave up
  kErrOverflow = 1u << 1,  // a fixed-capacity buffer would have overflowed
  kErrSeed = 1u << 2,      // the seed list failed validation
  kErrNonFinite = 1u << 3, // a causally visible pair scored inf or NaN (non-finite input)
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
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

// Bounded wait for the phase with the given parity to complete.
// abort_flag is a CTA-shared flag; err is the launch's device error word;
// limit_ns bounds the wait (kWaitTimeoutNs unless a caller passes less).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int* abort_flag, uint32_t* err,
                                          uint64_t limit_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 2-D tiled bulk tensor load global -> shared, completion on an mbarrier.
// c0 is the inner (column) coordinate, c1 the row coordinate.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int32_t c0,
                                            int32_t c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a
// multiple of 16), completion on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// 16-byte asynchronous global -> shared copy (L1 bypass) and its groups.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Prefetch a 2-D tile of a tensor map into L2 (no shared-memory destination).
__device__ __forceinline__ void tma_prefetch_l2_2d(const void* tmap, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(c0), "r"(c1)
               : "memory");
}

// ---------------------------------------------------------------- tcgen05
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
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate, one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, FP8 (E4M3) inputs, fp32 accumulate, one thread.
__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane
// (base lane + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Shared-memory matrix descriptor for a K-major bf16 operand stored as
// 128-byte rows with the 128B swizzle (8-row atoms of 1024 bytes).
// byte_addr: shared address of the first row, plus the K offset inside the
// 128-byte row (a multiple of 32 bytes for one K=16 step).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t byte_addr) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((byte_addr >> 4) & 0x3FFFu);  // start address
  desc |= static_cast<uint64_t>(1u) << 16;                     // leading byte offset (unused)
  desc |= static_cast<uint64_t>(1024u >> 4) << 32;             // stride byte offset: 8 rows
  desc |= static_cast<uint64_t>(1u) << 46;                     // descriptor version (sm_100)
  desc |= static_cast<uint64_t>(2u) << 61;                     // 128-byte swizzle
  return desc;
}

// Instruction descriptor: kind::f16, A = B = bf16, D = fp32, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                   // D format fp32
         | (1u << 7)                                 // A format bf16
         | (1u << 10)                                // B format bf16
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Instruction descriptor: kind::f8f6f4, A = B = E4M3 (format code 0), D = fp32,
// both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4)                                   // D format fp32
         | (0u << 7)                                 // A format E4M3
         | (0u << 10)                                // B format E4M3
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Warpgroup-wide register reallocation (all 128 threads of the warpgroup).
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------- misc
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Index score of one (query, key) from its H head dot products and the
// query's head weights:
//     I = sum_j w_j * max(dot_j, 0)
// in a fixed fp32 order shared by every scoring kernel of this library:
// eight partial sums a_c (c = j mod 8), each an fp32 FMA chain over its heads
// in ascending j starting from +0, combined as
// ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7)).
// The eight chains give the epilogue enough independent work to issue every
// cycle (one chain of H FMAs would stall on FMA latency).
//
// Each step is computed as fma(w_j / 2, dot_j + |dot_j|, a_c), which equals
// fma(w_j, max(dot_j, 0), a_c) bit for bit: dot + |dot| is exactly 2 dot or
// +0, and w / 2 is exact for normal weights, so the product is the same real
// number and the FMA rounds once either way.  The add (with an absolute-value
// operand) and the FMA run on the FMA pipe, where a max would take the ALU,
// and heads j and j+1 (chains c and c+1) advance together in one paired add
// and one paired FMA (__fadd2_rn, __ffma2_rn: per component the same
// operations as + and fmaf).  head_acc16 adds 16 consecutive
// heads (j0 .. j0+15, j0 a multiple of 16) to the chains, held as pairs
// a[c/2] = (a_c, a_c+1); wh holds the HALVED weights of those heads.
__device__ __forceinline__ void head_acc16(float2 (&a)[4], const uint32_t (&x)[16], const float* wh) {
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    const float x0 = __uint_as_float(x[j]), x1 = __uint_as_float(x[j + 1]);
    a[(j & 7) >> 1] = __ffma2_rn(make_float2(wh[j], wh[j + 1]),
                                 __fadd2_rn(make_float2(x0, x1), make_float2(fabsf(x0), fabsf(x1))),
                                 a[(j & 7) >> 1]);
  }
}
// The same 16 heads with the halved weights read from shared memory (16-byte
// broadcast loads; identical arithmetic).
__device__ __forceinline__ void head_acc16_smem(float2 (&a)[4], const uint32_t (&x)[16], const float* wh) {
  float wv[16];
#pragma unroll
  for (int j4 = 0; j4 < 4; ++j4) {
    const float4 v = reinterpret_cast<const float4*>(wh)[j4];
    wv[4 * j4 + 0] = v.x;
    wv[4 * j4 + 1] = v.y;
    wv[4 * j4 + 2] = v.z;
    wv[4 * j4 + 3] = v.w;
  }
  head_acc16(a, x, wv);
}
__device__ __forceinline__ float head_finish(const float2 (&a)[4]) {
  return ((a[0].x + a[0].y) + (a[1].x + a[1].y)) + ((a[2].x + a[2].y) + (a[3].x + a[3].y));
}
// Halved head weight as head_acc16 takes it (exact for normal weights).
__device__ __forceinline__ float half_weight(float w) { return 0.5f * w; }

// Monotone 32-bit code of an fp32 score: larger score <=> larger code.
// -0 is folded onto +0 first.
__device__ __forceinline__ uint32_t score_code(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__host__ __device__ __forceinline__ float code_score(uint32_t c) {
  uint32_t u = (c & 0x80000000u) ? (c & 0x7FFFFFFFu) : ~c;
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float f;
  __builtin_memcpy(&f, &u, 4);
  return f;
#endif
}

// The lowest fp32 score whose record can reach the threshold record thr:
// the value of thr's score code (-inf for codes at or below the code of
// -inf).  A finite score below it has a smaller code and so a smaller record;
// for codes above that of +inf the result is NaN and no score passes.
__device__ __forceinline__ float threshold_floor(uint64_t thr) {
  const uint32_t c = static_cast<uint32_t>(thr >> 32);
  return c <= 0x007FFFFFu ? -INFINITY : code_score(c);
}

// Record = (score code << 32) | (0xFFFFFFFF - key).  Ordering records as
// unsigned 64-bit integers is the selection order: score descending, then
// key ascending.  Keys are < 2^31, so a record is never 0.
__device__ __forceinline__ uint64_t make_record(float s, uint32_t key) {
  return (static_cast<uint64_t>(score_code(s)) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - key);
}
__host__ __device__ __forceinline__ uint32_t record_key(uint64_t r) {
  return 0xFFFFFFFFu - static_cast<uint32_t>(r);
}
__host__ __device__ __forceinline__ float record_score(uint64_t r) {
  return code_score(static_cast<uint32_t>(r >> 32));
}

}  // namespace dsa
