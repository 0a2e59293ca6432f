// Thin inline-PTX layer for sm_100a: mbarriers with bounded waits, TMA tile
// and row-gather loads, tcgen05 (TMEM allocation, UMMA issue/commit, TMEM
// loads/stores) and the shared-memory / instruction descriptors UMMA reads.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace hsa {
namespace tc {

HSA_DEV uint32_t smem_u32(const void* p) { return uint32_t(__cvta_generic_to_shared(p)); }

// ----------------------------------------------------------------- mbarrier
HSA_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
HSA_DEV void fence_barrier_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
HSA_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
HSA_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
HSA_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: while the phase is incomplete the
// thread may sleep for up to `ns` nanoseconds, waking when the phase
// completes, instead of coming straight back to probe again.
HSA_DEV bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Bounded wait on a phase. The first probe is a plain try_wait (a phase that
// is already complete answers at once); later probes sleep, so waiting warps
// do not take issue slots from the warps doing the work. Gives up after
// kWaitCycles SM cycles (about two seconds), setting *err, or as soon as
// another thread has set *err; returns whether the phase completed. Callers
// then skip the dependent work and run to completion, so a lost arrival can
// never hang the GPU.
constexpr long long kWaitCycles = 1ll << 32;
constexpr uint32_t kSuspendNs = 100000;
// The same with an explicit limit in SM cycles (a test can shorten it) and a
// suspend hint scaled to it.
HSA_DEV bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* err, long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint32_t ns = limit < kWaitCycles ? 1000u : kSuspendNs;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_sleep(bar, parity, ns)) return true;
    if ((it & 15u) == 0 && *(volatile int*)err) return false;
    if (clock64() - t0 > limit) break;
  }
  atomicExch(err, 1);
  return false;
}
HSA_DEV bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* err) {
  return mbar_wait_bounded(bar, parity, err, kWaitCycles);
}

// Named barrier `id` over `count` threads (a multiple of 32) that also ORs a
// predicate across them: every participant gets the same answer.
HSA_DEV bool bar_or(int id, int count, bool v) {
  uint32_t out;
  asm volatile(
      "{\n .reg .pred a, b;\n setp.ne.u32 a, %3, 0;\n bar.red.or.pred b, %1, %2, a;\n selp.u32 %0, 1, 0, b;\n}"
      : "=r"(out)
      : "r"(id), "r"(count), "r"(uint32_t(v))
      : "memory");
  return out != 0;
}
HSA_DEV void bar_sync(int id, int count) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory"); }

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32: relative error
// about 2^-22, subnormal results flushed to zero, 2^-inf = 0).
HSA_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

HSA_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ----------------------------------------------------------------- TMA
HSA_DEV void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
// 16-byte global -> shared copy through the async-copy path (bypasses L1).
HSA_DEV void cp_async16(uint32_t dst_smem, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst_smem), "l"(src) : "memory");
}
// The same copy when `valid`, else 16 zero bytes written without reading `src`.
HSA_DEV void cp_async16_zfill(uint32_t dst_smem, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst_smem), "l"(src), "r"(valid ? 16u : 0u)
               : "memory");
}
// Arrive on `bar` once all of this thread's earlier cp.async copies land
// (the arrival is one of the barrier's expected arrivals).
HSA_DEV void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
HSA_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
HSA_DEV void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ----------------------------------------------------------------- tcgen05
HSA_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
HSA_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
HSA_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
HSA_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
HSA_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem], bf16 inputs, fp32 accumulate.
HSA_DEV void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The same MMA with each descriptor passed as its two 32-bit halves. Offsets
// within a tile change only the start-address field in the low half (an
// in-bounds shared-memory address never carries out of it), so a caller can
// step the low words with 32-bit adds and reuse the high words.
HSA_DEV void mma_bf16_split(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo, uint32_t b_hi,
                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n .reg .b64 a, b;\n setp.ne.b32 p, %6, 0;\n mov.b64 a, {%1, %2};\n mov.b64 b, {%3, %4};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p;\n}"
      ::"r"(d_tmem), "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every previously issued tcgen05.mma of this thread completes.
HSA_DEV void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp gets lane
// (quadrant base + i), columns [col, col+16).
HSA_DEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
HSA_DEV void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}
HSA_DEV void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
HSA_DEV void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
HSA_DEV void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
HSA_DEV void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
HSA_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
HSA_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 32 lanes x N consecutive 32-bit columns as floats (N a multiple of 8), one wait.
template <int N>
HSA_DEV void tmem_load_f32(uint32_t taddr, float (&v)[N]) {
  static_assert(N % 8 == 0, "whole 8-column groups");
  uint32_t r[N];
  if constexpr (N % 16 == 0) {
#pragma unroll
    for (int c = 0; c < N / 16; ++c) tmem_ld16(taddr + 16 * c, *reinterpret_cast<uint32_t(*)[16]>(r + 16 * c));
  } else {
#pragma unroll
    for (int c = 0; c < N / 8; ++c) tmem_ld8(taddr + 8 * c, *reinterpret_cast<uint32_t(*)[8]>(r + 8 * c));
  }
  tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < N; ++e) v[e] = __uint_as_float(r[e]);
}
template <int N>
HSA_DEV void tmem_store_f32(uint32_t taddr, const float (&v)[N]) {
  static_assert(N % 8 == 0, "whole 8-column groups");
  uint32_t r[N];
#pragma unroll
  for (int e = 0; e < N; ++e) r[e] = __float_as_uint(v[e]);
  if constexpr (N % 16 == 0) {
#pragma unroll
    for (int c = 0; c < N / 16; ++c) tmem_st16(taddr + 16 * c, *reinterpret_cast<const uint32_t(*)[16]>(r + 16 * c));
  } else {
#pragma unroll
    for (int c = 0; c < N / 8; ++c) tmem_st8(taddr + 8 * c, *reinterpret_cast<const uint32_t(*)[8]>(r + 8 * c));
  }
  tmem_wait_st();
}

// ----------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor (sm_100 UMMA): start address, leading and
// stride byte offsets (16-byte units), version 1, swizzle layout code
// (0 none, 2 = 128B, 4 = 64B, 6 = 32B).
enum Swizzle : uint32_t { kSwNone = 0, kSw128 = 2, kSw64 = 4, kSw32 = 6 };
HSA_DEV uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes, uint32_t swz) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3fffu);
  d |= uint64_t((lbo_bytes >> 4) & 0x3fffu) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3fffu) << 32;
  d |= uint64_t(1) << 46;  // descriptor version for sm_100
  d |= uint64_t(swz & 7u) << 61;
  return d;
}

// Instruction descriptor of kind::f16 with bf16 A/B, fp32 D, M x N tile;
// a_mn / b_mn select MN-major (transposed) operands.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                 // D format fp32
         | (1u << 7)               // A format bf16
         | (1u << 10)              // B format bf16
         | (uint32_t(a_mn) << 15)  // A major
         | (uint32_t(b_mn) << 16)  // B major
         | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Byte offset of a 16-byte chunk inside a swizzled tile whose rows are
// `row_bytes` long (32, 64 or 128) and whose base is 1024-byte aligned:
// the chunk index is XORed with the row's position in the swizzle period.
HSA_DEV uint32_t swz_offset(uint32_t row, uint32_t chunk, uint32_t row_bytes) {
  const uint32_t lin = row * row_bytes + chunk * 16u;
  const uint32_t mask = row_bytes == 128 ? 7u : row_bytes == 64 ? 3u : 1u;
  return lin ^ (((lin >> 7) & mask) << 4);
}

}  // namespace tc
}  // namespace hsa
