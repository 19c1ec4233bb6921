// Device helpers shared by the sm_100a kernels: bounded mbarrier waits, TMA
// tile loads, tcgen05 (UMMA) issue / commit / TMEM loads, shared-memory matrix
// descriptors, and the per-device error word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "infv2.h"

namespace infv2 {

// Kernels record a failure (first one wins) in a per-device error word whose
// address the host passes in, instead of trapping; the host reads and clears
// it through infv2_device_status().
__device__ __forceinline__ void report_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// The debug build (INFV2_CHECKS=1) adds device-side checks of data-dependent
// indices and invariants.  A failed check records INFV2_ERR_CHECK and the
// kernel carries on exactly as the default build would: a check never traps
// and never changes a result.
#ifndef INFV2_CHECKS
#define INFV2_CHECKS 0
#endif
__device__ __forceinline__ void check(bool ok, int* err) {
  if (INFV2_CHECKS && !ok) report_error(err, INFV2_ERR_CHECK);
}

// Entry e of a block list row as the attention kernels use it: entries < 0
// and blocks past the query's own (no key t <= pos) are skipped (-1).  The
// debug build checks that non-negative neighbours ascend (no repeats).
__device__ __forceinline__ int list_block(const int* row, int e, int pos, int* err) {
  const int x = __ldg(row + e);
  if (INFV2_CHECKS && e > 0 && x >= 0) {
    const int prev = __ldg(row + e - 1);
    check(prev < x, err);
  }
  return x > (pos >> 6) ? -1 : x;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lane_id() {
  uint32_t l;
  asm volatile("mov.u32 %0, %%laneid;" : "=r"(l));
  return l;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Gives up after
// timeout_ns of wall time, records INFV2_ERR_TIMEOUT and returns false, so
// that no kernel of this library can spin forever.
struct WaitCtx {
  int* err;            // device error word
  uint64_t timeout_ns; // wall-time limit of one wait
};

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtx& w) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try(bar, parity)) return true;
    if ((n & 1023u) == 0 && globaltimer_ns() - t0 > w.timeout_ns) {
      report_error(w.err, INFV2_ERR_TIMEOUT);
      return false;
    }
  }
}

// Wait for two phases at once: both first tests are in flight together, so a
// pair of already-completed phases costs one test latency, not two.
__device__ __forceinline__ bool mbar_wait2(uint32_t bar0, uint32_t parity0, uint32_t bar1,
                                           uint32_t parity1, const WaitCtx& w) {
  const bool ok0 = mbar_try(bar0, parity0);
  const bool ok1 = mbar_try(bar1, parity1);
  if (ok0 && ok1) return true;
  return (ok0 || mbar_wait(bar0, parity0, w)) && (ok1 || mbar_wait(bar1, parity1, w));
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 3-D tiled bulk-tensor load into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
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

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 inputs, fp32 accumulate.  A (M rows =
// TMEM lanes) holds two bf16 per 32-bit column, lower K index in the low half;
// one K = 16 step is 8 columns.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once all tcgen05.mma issued so far by this thread complete.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// Each thread of the warp reads 32 consecutive fp32 columns of its TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// tcgen05.wait::ld that also names the loaded registers, so that no use of
// them can be scheduled before the load has completed.
__device__ __forceinline__ void tmem_ld_wait_regs(float (&v)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]),
        "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]),
        "+f"(v[14]), "+f"(v[15]), "+f"(v[16]), "+f"(v[17]), "+f"(v[18]), "+f"(v[19]),
        "+f"(v[20]), "+f"(v[21]), "+f"(v[22]), "+f"(v[23]), "+f"(v[24]), "+f"(v[25]),
        "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]), "+f"(v[30]), "+f"(v[31])
      :
      : "memory");
}

// Each thread of the warp writes 32 consecutive 32-bit columns of its TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// Each thread of the warp writes 16 consecutive 32-bit columns of its TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
// 16-lane TMEM access (shapes 16x256b / 16x128b): the warp covers 16 lanes
// (TMEM rows) starting at the address's lane; thread t holds rows t/4 and
// t/4 + 8.  16x256b.x8: per 8-column repetition j, registers 4j .. 4j+3 are
// (row t/4, columns 8j + 2(t%4) + {0, 1}) then (row t/4 + 8, the same columns).
// The load and its tcgen05.wait::ld are one asm statement: the registers an
// asynchronous TMEM load writes exist for the compiler only once it has
// completed, so no copy of them can be scheduled in between.
__device__ __forceinline__ void tmem_ld16x256_x8(uint32_t taddr, float (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]), "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15]), "=f"(v[16]), "=f"(v[17]), "=f"(v[18]), "=f"(v[19]), "=f"(v[20]), "=f"(v[21]), "=f"(v[22]), "=f"(v[23]), "=f"(v[24]), "=f"(v[25]), "=f"(v[26]), "=f"(v[27]), "=f"(v[28]), "=f"(v[29]), "=f"(v[30]), "=f"(v[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st16x256_x8(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// 16x128b.x16: per 4-column repetition j, registers 2j, 2j+1 are (row t/4,
// column 4j + t%4) and (row t/4 + 8, the same column).
__device__ __forceinline__ void tmem_st16x128_x16(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored as TMA writes it
// with 128-byte swizzling: rows of 128 bytes (64 bf16), 8-row groups 1024 bytes
// apart.  `addr` may be offset by k*32 bytes to select the k-th 16-element
// slice inside the 128-byte swizzle atom.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);   // start address
  d |= (uint64_t)1u << 16;                   // leading byte offset (unused when swizzled)
  d |= (uint64_t)(1024u >> 4) << 32;         // stride byte offset: 8 rows * 128 B
  d |= (uint64_t)1u << 46;                   // descriptor version for sm_100
  d |= (uint64_t)2u << 61;                   // layout: 128-byte swizzle
  return d;
}

// Shared-memory matrix descriptor for an MN-major operand in the same TMA
// layout (rows of 64 MN-contiguous bf16 = one K index per 128-byte row):
// 8 K-rows form a 1024-byte swizzle atom (stride byte offset), and the next 64
// MN elements start `mn_chunk_bytes` further on (leading byte offset).
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(uint32_t addr, uint32_t mn_chunk_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((mn_chunk_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major,
                                                       bool b_mn_major) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17)     // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// ---------------------------------------------------------------- misc

// Maximum of three floats in one instruction (the three-operand max.f32 of
// sm_100); like fmaxf, a NaN operand is ignored in favour of the others.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x evaluated on the FMA pipe (to take load off the MUFU unit), for
// x <= ~127; inputs below -127 (and -inf) give 0.  Cody-Waite style split
// x = n + r with n the nearest integer (the 1.5*2^23 shifter leaves n in the
// low mantissa bits) and r in [-0.5, 0.5]; 2^r is a degree-5 polynomial whose
// coefficients were fitted for this library by iteratively reweighted least
// squares on Chebyshev nodes of [-0.5, 0.5] (max relative error 2.3e-7 with
// fp32 Horner evaluation); 2^n is added to the exponent field.
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -127.0f);
  const float shifter = 12582912.0f;  // 1.5 * 2^23
  const float t = x + shifter;
  const float n = t - shifter;
  const float r = x - n;
  float p = 1.32764666e-3f;
  p = fmaf(p, r, 9.67554096e-3f);
  p = fmaf(p, r, 5.55071346e-2f);
  p = fmaf(p, r, 2.40221202e-1f);
  p = fmaf(p, r, 6.93146944e-1f);
  p = fmaf(p, r, 1.00000012f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Packed fp32 pairs (sm_100 f32x2 instructions): one instruction per two
// lanes' worth of FMA / ADD, each half rounded exactly like its scalar form.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// exp2_fma on a pair, with the packed instructions (same split and polynomial).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -127.0f);
  x.y = fmaxf(x.y, -127.0f);
  const float2 sh = make_float2(12582912.0f, 12582912.0f);
  const float2 t = fadd2(x, sh);
  const float2 nn = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 r = ffma2(nn, make_float2(-1.0f, -1.0f), x);
  float2 p = make_float2(1.32764666e-3f, 1.32764666e-3f);
  p = ffma2(p, r, make_float2(9.67554096e-3f, 9.67554096e-3f));
  p = ffma2(p, r, make_float2(5.55071346e-2f, 5.55071346e-2f));
  p = ffma2(p, r, make_float2(2.40221202e-1f, 2.40221202e-1f));
  p = ffma2(p, r, make_float2(6.93146944e-1f, 6.93146944e-1f));
  p = ffma2(p, r, make_float2(1.00000012f, 1.00000012f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// 2^x on a pair with a cheaper polynomial, for probabilities that are rounded
// to bf16 afterwards: x is clamped to [-127, 64], split as n + r with n the
// nearest integer, and 2^r (r in [-0.5, 0.5]) is 1 + c1 r + c2 r^2 + c3 r^3
// with c1..c3 fitted for this library by iteratively reweighted least squares
// on Chebyshev nodes (max relative error 1.0e-4 with fp32 Horner evaluation,
// 19x below bf16's rounding step).  The constant term is exactly 1: then the
// clamped bottom, n = -127 with r = 0, lands on exponent field 0 and gives
// exactly +0 (x <= -127 and -inf give 0), and no x in range can borrow from
// the sign bit when n is added to the exponent.
__device__ __forceinline__ float2 exp2_cubic2(float2 x) {
  x.x = fminf(fmaxf(x.x, -127.0f), 64.0f);
  x.y = fminf(fmaxf(x.y, -127.0f), 64.0f);
  const float2 sh = make_float2(12582912.0f, 12582912.0f);
  const float2 t = fadd2(x, sh);
  const float2 nn = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 r = ffma2(nn, make_float2(-1.0f, -1.0f), x);
  float2 p = ffma2(make_float2(5.50089143e-2f, 5.50089143e-2f), r,
                   make_float2(2.42210969e-1f, 2.42210969e-1f));
  p = ffma2(p, r, make_float2(6.93282902e-1f, 6.93282902e-1f));
  p = ffma2(p, r, make_float2(1.0f, 1.0f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Number of stage-1 kernels whose whole window lies at or before query i.
__host__ __device__ __forceinline__ int visible_kernels(int i, int l_c1, int s_c1) {
  return i >= l_c1 - 1 ? (i - l_c1 + 1) / s_c1 + 1 : 0;
}

}  // namespace infv2

// ------------------------------------------------------------------ host side
namespace infv2 {

// Build a 3-D bf16 tensor map (dims innermost first) with 128-byte swizzle.
// Returns false if the driver rejects it.
bool make_tmap_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                  uint32_t box2);

// Status of the last launch / runtime call as an infv2_status.
int launch_status(cudaError_t e);

// Identity of the calling thread's current CUDA context (0 if none or unknown).
uintptr_t current_context();

// Device address of this device's kernel error word (looked up once per device
// and context).
int* error_word();

// Wall-time limit of every bounded wait inside a kernel (default 2 s).
uint64_t wait_timeout_ns();

inline WaitCtx wait_ctx() { return WaitCtx{error_word(), wait_timeout_ns()}; }

// Multiprocessor count of the current device (cached).
int sm_count();

// Allow `bytes` of dynamic shared memory for `kernel` (once per kernel).
template <class K>
inline bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
         cudaSuccess;
}

}  // namespace infv2
