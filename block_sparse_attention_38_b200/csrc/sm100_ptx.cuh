// sm100_ptx.cuh -- thin inline-PTX wrappers for the sm_100a features the
// forward kernel uses: mbarriers, TMA tiled loads, the tensor memory (TMEM)
// allocator, tcgen05.mma with TMEM accumulators, tcgen05.ld/st and the
// shared-memory matrix descriptors.  Written from the PTX ISA (tcgen05,
// cp.async.bulk.tensor and mbarrier chapters); no multicast form is used.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace bsa {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}


// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Non-blocking: true when the phase of parity `parity` has completed.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Suspends the thread until the phase of parity `parity` has completed or
// about `hint_ns` nanoseconds have passed; true when the phase completed.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// --------------------------------------------------------------------- TMA
// 3-D tiled load global -> shared, completion counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 3-D tiled prefetch of a box into L2 (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------- TMEM
// Whole-warp operations.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
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
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
               :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
               :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
               : "memory");
}


// The helpers below issue TMEM loads or stores together with their
// tcgen05.wait in one asm statement.  The registers of a tcgen05.ld are
// written, and those of a tcgen05.st read, asynchronously until the wait; in
// one statement the compiler cannot place a spill or another value in them
// in between.


// Loads the 64 columns at `taddr` into r as fp32 and waits for them.  The
// outputs are early-clobber, so none shares a register with the address.
__device__ __forceinline__ void tmem_ld64_wait(uint32_t taddr, float (&r)[64]) {
  asm volatile(
      "{\n\ttcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=&f"(r[0]), "=&f"(r[1]), "=&f"(r[2]), "=&f"(r[3]), "=&f"(r[4]), "=&f"(r[5]), "=&f"(r[6]), "=&f"(r[7]), "=&f"(r[8]), "=&f"(r[9]), "=&f"(r[10]), "=&f"(r[11]), "=&f"(r[12]), "=&f"(r[13]), "=&f"(r[14]), "=&f"(r[15]), "=&f"(r[16]), "=&f"(r[17]), "=&f"(r[18]), "=&f"(r[19]), "=&f"(r[20]), "=&f"(r[21]), "=&f"(r[22]), "=&f"(r[23]), "=&f"(r[24]), "=&f"(r[25]), "=&f"(r[26]), "=&f"(r[27]), "=&f"(r[28]), "=&f"(r[29]), "=&f"(r[30]), "=&f"(r[31]), "=&f"(r[32]), "=&f"(r[33]), "=&f"(r[34]), "=&f"(r[35]), "=&f"(r[36]), "=&f"(r[37]), "=&f"(r[38]), "=&f"(r[39]), "=&f"(r[40]), "=&f"(r[41]), "=&f"(r[42]), "=&f"(r[43]), "=&f"(r[44]), "=&f"(r[45]), "=&f"(r[46]), "=&f"(r[47]), "=&f"(r[48]), "=&f"(r[49]), "=&f"(r[50]), "=&f"(r[51]), "=&f"(r[52]), "=&f"(r[53]), "=&f"(r[54]), "=&f"(r[55]), "=&f"(r[56]), "=&f"(r[57]), "=&f"(r[58]), "=&f"(r[59]), "=&f"(r[60]), "=&f"(r[61]), "=&f"(r[62]), "=&f"(r[63])
      : "r"(taddr)
      : "memory");
}

// Loads the 32 columns at `taddr` into r[0..31] (lo) or r[32..63] (hi) as
// fp32 and waits for them; the other half of r is left undefined.
__device__ __forceinline__ void tmem_ld32lo_wait(uint32_t taddr, float (&r)[64]) {
  asm volatile(
      "{\n\ttcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=&f"(r[0]), "=&f"(r[1]), "=&f"(r[2]), "=&f"(r[3]), "=&f"(r[4]), "=&f"(r[5]), "=&f"(r[6]), "=&f"(r[7]), "=&f"(r[8]), "=&f"(r[9]), "=&f"(r[10]), "=&f"(r[11]), "=&f"(r[12]), "=&f"(r[13]), "=&f"(r[14]), "=&f"(r[15]), "=&f"(r[16]), "=&f"(r[17]), "=&f"(r[18]), "=&f"(r[19]), "=&f"(r[20]), "=&f"(r[21]), "=&f"(r[22]), "=&f"(r[23]), "=&f"(r[24]), "=&f"(r[25]), "=&f"(r[26]), "=&f"(r[27]), "=&f"(r[28]), "=&f"(r[29]), "=&f"(r[30]), "=&f"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32hi_wait(uint32_t taddr, float (&r)[64]) {
  asm volatile(
      "{\n\ttcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=&f"(r[32]), "=&f"(r[33]), "=&f"(r[34]), "=&f"(r[35]), "=&f"(r[36]), "=&f"(r[37]), "=&f"(r[38]), "=&f"(r[39]), "=&f"(r[40]), "=&f"(r[41]), "=&f"(r[42]), "=&f"(r[43]), "=&f"(r[44]), "=&f"(r[45]), "=&f"(r[46]), "=&f"(r[47]), "=&f"(r[48]), "=&f"(r[49]), "=&f"(r[50]), "=&f"(r[51]), "=&f"(r[52]), "=&f"(r[53]), "=&f"(r[54]), "=&f"(r[55]), "=&f"(r[56]), "=&f"(r[57]), "=&f"(r[58]), "=&f"(r[59]), "=&f"(r[60]), "=&f"(r[61]), "=&f"(r[62]), "=&f"(r[63])
      : "r"(taddr)
      : "memory");
}

// Stores r[0..63] to the 64 columns at `taddr` and waits for the store.
__device__ __forceinline__ void tmem_st64_wait(uint32_t taddr, const uint32_t (&r)[64]) {
  asm volatile(
      "{\n\ttcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};\n\t"
      "tcgen05.wait::st.sync.aligned;\n\t}"
      :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]), "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]), "r"(r[41]), "r"(r[42]), "r"(r[43]), "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]), "r"(r[49]), "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]), "r"(r[56]), "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63])
      : "memory");
}

// Loads the 32 columns at `taddr` into r and waits for them.
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "{\n\ttcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=&r"(r[0]), "=&r"(r[1]), "=&r"(r[2]), "=&r"(r[3]), "=&r"(r[4]), "=&r"(r[5]), "=&r"(r[6]), "=&r"(r[7]), "=&r"(r[8]), "=&r"(r[9]), "=&r"(r[10]), "=&r"(r[11]), "=&r"(r[12]), "=&r"(r[13]), "=&r"(r[14]), "=&r"(r[15]), "=&r"(r[16]), "=&r"(r[17]), "=&r"(r[18]), "=&r"(r[19]), "=&r"(r[20]), "=&r"(r[21]), "=&r"(r[22]), "=&r"(r[23]), "=&r"(r[24]), "=&r"(r[25]), "=&r"(r[26]), "=&r"(r[27]), "=&r"(r[28]), "=&r"(r[29]), "=&r"(r[30]), "=&r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Stores r to the 32 columns at `taddr` and waits for the store.
__device__ __forceinline__ void tmem_st32_wait(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "{\n\ttcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;\n\t}"
      :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// ---------------------------------------------------------------- tcgen05.mma
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, fp32 accumulate.
// Issued by a single thread.
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T: A (M x K, bf16, two K-consecutive
// elements per 32-bit column, lower index in the low half) read from tensor
// memory, B from shared memory.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One step's chain of K=16 MMAs in a single asm statement, so the issuing
// thread runs nothing but 32-bit descriptor adds between them (the tensor
// core idles while the issuer computes).  The start-address field of a
// shared-memory descriptor is its low 14 bits (address >> 4); shared
// addresses stay below 2^18 bytes, so the adds never carry out of the low word.

// S (fp32, TMEM) = A B^T over K = 16*NK: A and B K-major SW128 tiles of 128
// rows, 64-column atoms 128*128 bytes apart (descriptor lo/hi words given for
// the first slice).  The first MMA overwrites S.
template <int NK>
__device__ __forceinline__ void umma_qk_chain(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi,
                                              uint32_t b_lo, uint32_t b_hi, uint32_t idesc);
template <>
__device__ __forceinline__ void umma_qk_chain<4>(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi,
                                                 uint32_t b_lo, uint32_t b_hi, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t.reg .b32 al, bl, one;\n\t.reg .b64 ad, bd;\n\t"
      "mov.b32 one, 1;\n\tsetp.eq.b32 pt, one, 1;\n\tsetp.eq.b32 pf, one, 0;\n\t"
      "add.s32 al, %1, 0;\n\tadd.s32 bl, %3, 0;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pf;\n\t"
      "add.s32 al, %1, 2;\n\tadd.s32 bl, %3, 2;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.s32 al, %1, 4;\n\tadd.s32 bl, %3, 4;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.s32 al, %1, 6;\n\tadd.s32 bl, %3, 6;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "}"
      :: "r"(d_tmem), "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc)
      : "memory");
}
template <>
__device__ __forceinline__ void umma_qk_chain<8>(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi,
                                                 uint32_t b_lo, uint32_t b_hi, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t.reg .b32 al, bl, one;\n\t.reg .b64 ad, bd;\n\t"
      "mov.b32 one, 1;\n\tsetp.eq.b32 pt, one, 1;\n\tsetp.eq.b32 pf, one, 0;\n\t"
      "add.s32 al, %1, 0;\n\tadd.s32 bl, %3, 0;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pf;\n\t"
      "add.s32 al, %1, 2;\n\tadd.s32 bl, %3, 2;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.s32 al, %1, 4;\n\tadd.s32 bl, %3, 4;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.s32 al, %1, 6;\n\tadd.s32 bl, %3, 6;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.s32 al, %1, 1024;\n\tadd.s32 bl, %3, 1024;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.s32 al, %1, 1026;\n\tadd.s32 bl, %3, 1026;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.s32 al, %1, 1028;\n\tadd.s32 bl, %3, 1028;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.s32 al, %1, 1030;\n\tadd.s32 bl, %3, 1030;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "}"
      :: "r"(d_tmem), "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc)
      : "memory");
}

// O (fp32, TMEM) (+)= P V over 128 keys: P (bf16 pairs) in TMEM, 8 columns per
// K=16 slice from a_tmem; V an MN-major SW128 tile, 16 key rows = 2048 bytes
// per slice.  The first MMA accumulates only if `accumulate` is non-zero.
__device__ __forceinline__ void umma_pv_chain8(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                               uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p0, pt;\n\t.reg .b32 bl, at, one;\n\t.reg .b64 bd;\n\t"
      "mov.b32 one, 1;\n\tsetp.eq.b32 pt, one, 1;\n\tsetp.ne.b32 p0, %5, 0;\n\t"
      "add.s32 at, %1, 0;\n\tadd.s32 bl, %2, 0;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %4, p0;\n\t"
      "add.s32 at, %1, 8;\n\tadd.s32 bl, %2, 128;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %4, pt;\n\t"
      "add.s32 at, %1, 16;\n\tadd.s32 bl, %2, 256;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %4, pt;\n\t"
      "add.s32 at, %1, 24;\n\tadd.s32 bl, %2, 384;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %4, pt;\n\t"
      "add.s32 at, %1, 32;\n\tadd.s32 bl, %2, 512;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %4, pt;\n\t"
      "add.s32 at, %1, 40;\n\tadd.s32 bl, %2, 640;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %4, pt;\n\t"
      "add.s32 at, %1, 48;\n\tadd.s32 bl, %2, 768;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %4, pt;\n\t"
      "add.s32 at, %1, 56;\n\tadd.s32 bl, %2, 896;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [at], bd, %4, pt;\n\t"
      "}"
      :: "r"(d_tmem), "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D (PTX ISA,
// "Instruction descriptor"): bits 4-5 D format (1 = f32), 7-9 A format
// (1 = bf16), 10-12 B format, 15/16 A/B major (0 = K-major, 1 = MN-major),
// 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major,
                                                      bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor (PTX ISA, "Shared memory descriptor"):
// bits 0-13 start address >> 4, 16-29 leading-dimension byte offset >> 4,
// 32-45 stride-dimension byte offset >> 4, 46-47 version (1 on sm_100),
// 61-63 layout (kLayoutSW128 = 2: 128-byte swizzle, atom 8 rows x 128 B on a
// 1024-byte boundary; kLayoutSW64 = 4: 64-byte swizzle, atom 8 rows x 64 B on
// a 512-byte boundary).
// K-major swizzled operands: SBO = byte distance between 8-row groups; LBO unused.
// MN-major swizzled operands: LBO = byte distance between swizzle-atom columns
// along M/N, SBO = byte distance between 8-row groups along K.
constexpr uint32_t kLayoutSW128 = 2;
constexpr uint32_t kLayoutSW64 = 4;

__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                          uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}

__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                uint32_t sbo_bytes) {
  return sdesc(saddr, lbo_bytes, sbo_bytes, kLayoutSW128);
}

// Makes the 32 registers look rewritten at this point of the program, so that
// no use of a tcgen05.ld destination is scheduled above the tcgen05.wait::ld
// that precedes this call.
__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
  asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// ------------------------------------------------------------------- math
// Packed pairs of fp32 (one instruction for two lanes of arithmetic).
__device__ __forceinline__ void mul2(float& a, float& b, float s) {
  asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %2};\n\t"
      "mul.rn.ftz.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(s));
}
__device__ __forceinline__ void add2(float& a, float& b, float s) {
  asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %2};\n\t"
      "add.rn.ftz.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(s));
}
// (a, b) += (c, d)
__device__ __forceinline__ void acc2(float& a, float& b, float c, float d) {
  asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "add.rn.ftz.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(c), "f"(d));
}
// (a, b) = (a, b) * s + c, one rounding per lane
__device__ __forceinline__ void fma2(float& a, float& b, float s, float c) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %2};\n\t"
      "mov.b64 z, {%3, %3};\n\tfma.rn.ftz.f32x2 x, x, y, z;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(s), "f"(c));
}
// (a, b) = (a, b) * (xa, xb) + c
__device__ __forceinline__ void fma2v(float& a, float& b, float xa, float xb, float c) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "mov.b64 z, {%4, %4};\n\tfma.rn.ftz.f32x2 x, x, y, z;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(xa), "f"(xb), "f"(c));
}
// (a, b) -= (c, d)
__device__ __forceinline__ void sub2v(float& a, float& b, float c, float d) {
  asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "sub.rn.ftz.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(c), "f"(d));
}

// 2^a, 2^b on the FMA pipe, for inputs up to 127.  Cody and Waite's range
// reduction x = n + f, n = rint(x), f in [-1/2, 1/2]; 2^f by the degree-3
// minimax polynomial of exp2_poly.py (relative error below 7.5e-5); 2^n
// added to the exponent field.  The rint is the fp32 addition of 1.5 * 2^23,
// which leaves n in the low mantissa bits of t, so (bits(t) << 23) is n << 23
// modulo 2^32.  Inputs are clamped at -126.5 so that n >= -126 and the
// exponent field cannot wrap: anything below comes out as a denormal under
// 2^-126 (flushed to zero by the ftz arithmetic that follows).
__device__ __forceinline__ void exp2_poly2(float& a, float& b) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  a = fmaxf(a, -126.5f);
  b = fmaxf(b, -126.5f);
  float ta = a, tb = b;
  add2(ta, tb, kRound);
  float na = ta, nb = tb;
  add2(na, nb, -kRound);
  float fa = a, fb = b;
  sub2v(fa, fb, na, nb);
  float pa = 0.0551716685f, pb = 0.0551716685f;
  fma2v(pa, pb, fa, fb, 0.242611125f);
  fma2v(pa, pb, fa, fb, 0.693260968f);
  fma2v(pa, pb, fa, fb, 0.999928057f);
  a = __uint_as_float(__float_as_uint(pa) + (__float_as_uint(ta) << 23));
  b = __uint_as_float(__float_as_uint(pb) + (__float_as_uint(tb) << 23));
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}


}  // namespace bsa
