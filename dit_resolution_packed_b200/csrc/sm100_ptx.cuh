// sm100_ptx.cuh -- thin inline-PTX wrappers for the sm_100a features the
// attention kernel uses: mbarriers with bounded waits, TMA tensor copies,
// tensor-map updates, and the 5th-generation tensor core (tcgen05 MMA with
// accumulators in tensor memory).
//
// Encodings follow the PTX ISA (tcgen05 instruction descriptor, shared-memory
// matrix descriptor).  Only the forms used by this library are wrapped.
#pragma once
#include <cstdint>

#include "exp2_poly.cuh"

namespace pa {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
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
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Shared state of the bounded waits of one CTA: an abort flag in shared
// memory, the kernel's status word in global memory, and the wait limit.
struct WaitCtl {
  volatile int* abort_flag;  // shared memory; nonzero once any wait of the CTA gave up
  int* status;               // global status word (first error wins)
  uint64_t limit_ns;
  int timeout_code;
};

__device__ __forceinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, const WaitCtl& w) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*w.abort_flag) return false;
      if (global_timer_ns() - t0 > w.limit_ns) {
        *w.abort_flag = 1;
        atomicCAS(w.status, 0, w.timeout_code);
        __threadfence();
        return false;
      }
    }
  }
}

// Waits for the phase of `bar` with the given parity to complete.  Returns
// false (after recording a timeout) if it does not complete within the limit
// or if another wait of the CTA has already given up.  Never traps or spins
// without bound.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  return mbar_wait_slow(a, parity, w);
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int32_t x, int32_t y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const void* tmap, int32_t x, int32_t y, const void* src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(x), "r"(y), "r"(smem_u32(src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Orders this thread's generic-proxy shared-memory writes before later async-proxy (TMA) reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Tensor maps living in global memory, rewritten on the device.
__device__ __forceinline__ void tmap_replace_address(void* gmap, const void* addr) {
  asm volatile("tensormap.replace.tile.global_address.global.b1024.b64 [%0], %1;" ::"l"(
                   reinterpret_cast<uint64_t>(gmap)),
               "l"(reinterpret_cast<uint64_t>(addr))
               : "memory");
}
__device__ __forceinline__ void tmap_replace_dim1(void* gmap, uint32_t extent) {
  asm volatile("tensormap.replace.tile.global_dim.global.b1024.b32 [%0], 1, %1;" ::"l"(
                   reinterpret_cast<uint64_t>(gmap)),
               "r"(extent)
               : "memory");
}
__device__ __forceinline__ void tmap_replace_dim0(void* gmap, uint32_t extent) {
  asm volatile("tensormap.replace.tile.global_dim.global.b1024.b32 [%0], 0, %1;" ::"l"(
                   reinterpret_cast<uint64_t>(gmap)),
               "r"(extent)
               : "memory");
}
__device__ __forceinline__ void fence_tmap_release() {
  asm volatile("fence.proxy.tensormap::generic.release.gpu;" ::: "memory");
}
__device__ __forceinline__ void fence_tmap_acquire(const void* gmap) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(reinterpret_cast<uint64_t>(gmap))
               : "memory");
}

// ---------------------------------------------------------------- register split
// Executed by every warp of a warpgroup.  The block's register pool is fixed at
// launch (threads x registers per thread); .inc waits until .dec calls of other
// warpgroups have returned enough registers, so the split must add up.
template <uint32_t N>
__device__ __forceinline__ void regs_increase() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_decrease() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------- programmatic dependent launch
// Lets the next kernel of the stream (launched with programmatic serialization)
// start its prologue before this grid finishes.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Waits until the preceding grid of the stream has completed and its memory is
// visible; returns at once when the launch had no programmatic dependency.
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- named barriers
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- tcgen05
// Tensor-memory allocation: executed by one whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Same MMAs with the two shared-memory descriptors given as their low 32 bits
// (start address and leading byte offset) and one shared high word (stride
// byte offset, version, swizzle): unrolled issue loops then keep only 32-bit
// values live.
__device__ __forceinline__ void mma_bf16_ss_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 da, {%1, %3};\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_ts_lo(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Predicated forms for an issuer loop run by a whole warp: every lane computes
// the (warp-uniform) operands, only the lane with `issue` != 0 issues.  Keeping
// the operand arithmetic out of single-lane code lets it stay warp-uniform.
__device__ __forceinline__ void mma_bf16_ss_lo_if(uint32_t issue, uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                                  uint32_t hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "setp.ne.b32 q, %6, 0;\n\t"
      "mov.b64 da, {%1, %3};\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate), "r"(issue)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_ts_lo_if(uint32_t issue, uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                                  uint32_t hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b64 db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "setp.ne.b32 q, %6, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate), "r"(issue)
      : "memory");
}
__device__ __forceinline__ void mma_commit_if(uint32_t issue, uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %1, 0;\n\t"
      "@q tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(smem_u32(bar)),
      "r"(issue)
      : "memory");
}

// One lane of a converged warp, chosen by the hardware: returns 1 there, 0 elsewhere.
__device__ __forceinline__ uint32_t elect_one_sync() {
  uint32_t r;
  asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\tselp.b32 %0, 1, 0, e;\n\t}\n" : "=r"(r));
  return r;
}

// Arrives once on `bar` when every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, dense.
//   bits 4-5 D format (1 = f32); 7-9 A format (1 = bf16); 10-12 B format (1 = bf16);
//   bit 15 A major (0 = K); bit 16 B major (0 = K, 1 = MN); 17-22 N/8; 24-28 M/16.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t M, uint32_t N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((N >> 3) << 17) |
         ((M >> 4) << 24);
}
// The same with the major-ness of A chosen too (bit 15: 1 = A is MN-major in shared memory).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_ab(uint32_t M, uint32_t N, bool a_mn_major, bool b_mn_major) {
  return idesc_bf16_f32(M, N, b_mn_major) | ((a_mn_major ? 1u : 0u) << 15);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand:
//   bits 0-13 start address >> 4; 16-29 leading byte offset >> 4; 32-45 stride
//   byte offset >> 4; 46-47 version (1); 49-51 base offset (0: atoms 1024-byte
//   aligned); 61-63 layout (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Split form of sdesc_sw128: low word (start address, leading byte offset) and
// high word (stride byte offset, version 1, 128-byte swizzle).
__host__ __device__ constexpr uint32_t sdesc_sw128_lo(uint32_t saddr, uint32_t lbo_bytes) {
  return ((saddr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}
__host__ __device__ constexpr uint32_t sdesc_sw128_hi(uint32_t sbo_bytes) {
  return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
}

// Tensor memory <-> registers, 32 data-path lanes x 32-bit, one lane per thread.
#define PA_TMEM_LD32(taddr, r)                                                                                   \
  asm volatile(                                                                                                  \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18," \
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                                             \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),          \
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),    \
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),  \
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])   \
      : "r"(taddr))

#define PA_TMEM_LD16(taddr, r)                                                                                 \
  asm volatile(                                                                                                \
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"   \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),        \
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])   \
      : "r"(taddr))

#define PA_TMEM_ST16(taddr, r)                                                                                 \
  asm volatile(                                                                                                \
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" \
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),      \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])               \
      : "memory")

#define PA_TMEM_ST32(taddr, r)                                                                                   \
  asm volatile(                                                                                                  \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17," \
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),                               \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),         \
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), \
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]),            \
      "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])                                     \
      : "memory")

// Loads 128 consecutive 32-bit columns of this thread's tensor-memory lane into
// 64 register pairs (column 2i in the low half of pair i), waiting once for all.
__device__ __forceinline__ void tmem_ld128_pairs(uint32_t taddr, uint64_t (&v)[64]) {
  asm volatile(
      "{\n\t.reg .b32 t<128>;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {t0, t1, t2, t3, t4, t5, t6, t7, t8, t9, t10, t11, t12, t13, t14, t15, t16, t17, t18, t19, t20, t21, t22, t23, t24, t25, t26, t27, t28, t29, t30, t31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {t32, t33, t34, t35, t36, t37, t38, t39, t40, t41, t42, t43, t44, t45, t46, t47, t48, t49, t50, t51, t52, t53, t54, t55, t56, t57, t58, t59, t60, t61, t62, t63}, [%65];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {t64, t65, t66, t67, t68, t69, t70, t71, t72, t73, t74, t75, t76, t77, t78, t79, t80, t81, t82, t83, t84, t85, t86, t87, t88, t89, t90, t91, t92, t93, t94, t95}, [%66];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {t96, t97, t98, t99, t100, t101, t102, t103, t104, t105, t106, t107, t108, t109, t110, t111, t112, t113, t114, t115, t116, t117, t118, t119, t120, t121, t122, t123, t124, t125, t126, t127}, [%67];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t"
      "mov.b64 %0, {t0, t1};\n\t"
      "mov.b64 %1, {t2, t3};\n\t"
      "mov.b64 %2, {t4, t5};\n\t"
      "mov.b64 %3, {t6, t7};\n\t"
      "mov.b64 %4, {t8, t9};\n\t"
      "mov.b64 %5, {t10, t11};\n\t"
      "mov.b64 %6, {t12, t13};\n\t"
      "mov.b64 %7, {t14, t15};\n\t"
      "mov.b64 %8, {t16, t17};\n\t"
      "mov.b64 %9, {t18, t19};\n\t"
      "mov.b64 %10, {t20, t21};\n\t"
      "mov.b64 %11, {t22, t23};\n\t"
      "mov.b64 %12, {t24, t25};\n\t"
      "mov.b64 %13, {t26, t27};\n\t"
      "mov.b64 %14, {t28, t29};\n\t"
      "mov.b64 %15, {t30, t31};\n\t"
      "mov.b64 %16, {t32, t33};\n\t"
      "mov.b64 %17, {t34, t35};\n\t"
      "mov.b64 %18, {t36, t37};\n\t"
      "mov.b64 %19, {t38, t39};\n\t"
      "mov.b64 %20, {t40, t41};\n\t"
      "mov.b64 %21, {t42, t43};\n\t"
      "mov.b64 %22, {t44, t45};\n\t"
      "mov.b64 %23, {t46, t47};\n\t"
      "mov.b64 %24, {t48, t49};\n\t"
      "mov.b64 %25, {t50, t51};\n\t"
      "mov.b64 %26, {t52, t53};\n\t"
      "mov.b64 %27, {t54, t55};\n\t"
      "mov.b64 %28, {t56, t57};\n\t"
      "mov.b64 %29, {t58, t59};\n\t"
      "mov.b64 %30, {t60, t61};\n\t"
      "mov.b64 %31, {t62, t63};\n\t"
      "mov.b64 %32, {t64, t65};\n\t"
      "mov.b64 %33, {t66, t67};\n\t"
      "mov.b64 %34, {t68, t69};\n\t"
      "mov.b64 %35, {t70, t71};\n\t"
      "mov.b64 %36, {t72, t73};\n\t"
      "mov.b64 %37, {t74, t75};\n\t"
      "mov.b64 %38, {t76, t77};\n\t"
      "mov.b64 %39, {t78, t79};\n\t"
      "mov.b64 %40, {t80, t81};\n\t"
      "mov.b64 %41, {t82, t83};\n\t"
      "mov.b64 %42, {t84, t85};\n\t"
      "mov.b64 %43, {t86, t87};\n\t"
      "mov.b64 %44, {t88, t89};\n\t"
      "mov.b64 %45, {t90, t91};\n\t"
      "mov.b64 %46, {t92, t93};\n\t"
      "mov.b64 %47, {t94, t95};\n\t"
      "mov.b64 %48, {t96, t97};\n\t"
      "mov.b64 %49, {t98, t99};\n\t"
      "mov.b64 %50, {t100, t101};\n\t"
      "mov.b64 %51, {t102, t103};\n\t"
      "mov.b64 %52, {t104, t105};\n\t"
      "mov.b64 %53, {t106, t107};\n\t"
      "mov.b64 %54, {t108, t109};\n\t"
      "mov.b64 %55, {t110, t111};\n\t"
      "mov.b64 %56, {t112, t113};\n\t"
      "mov.b64 %57, {t114, t115};\n\t"
      "mov.b64 %58, {t116, t117};\n\t"
      "mov.b64 %59, {t118, t119};\n\t"
      "mov.b64 %60, {t120, t121};\n\t"
      "mov.b64 %61, {t122, t123};\n\t"
      "mov.b64 %62, {t124, t125};\n\t"
      "mov.b64 %63, {t126, t127};\n\t"
      "}\n"
      : "=l"(v[0]), "=l"(v[1]), "=l"(v[2]), "=l"(v[3]), "=l"(v[4]), "=l"(v[5]), "=l"(v[6]), "=l"(v[7]), "=l"(v[8]), "=l"(v[9]), "=l"(v[10]), "=l"(v[11]), "=l"(v[12]), "=l"(v[13]), "=l"(v[14]), "=l"(v[15]), "=l"(v[16]), "=l"(v[17]), "=l"(v[18]), "=l"(v[19]), "=l"(v[20]), "=l"(v[21]), "=l"(v[22]), "=l"(v[23]), "=l"(v[24]), "=l"(v[25]), "=l"(v[26]), "=l"(v[27]), "=l"(v[28]), "=l"(v[29]), "=l"(v[30]), "=l"(v[31]), "=l"(v[32]), "=l"(v[33]), "=l"(v[34]), "=l"(v[35]), "=l"(v[36]), "=l"(v[37]), "=l"(v[38]), "=l"(v[39]), "=l"(v[40]), "=l"(v[41]), "=l"(v[42]), "=l"(v[43]), "=l"(v[44]), "=l"(v[45]), "=l"(v[46]), "=l"(v[47]), "=l"(v[48]), "=l"(v[49]), "=l"(v[50]), "=l"(v[51]), "=l"(v[52]), "=l"(v[53]), "=l"(v[54]), "=l"(v[55]), "=l"(v[56]), "=l"(v[57]), "=l"(v[58]), "=l"(v[59]), "=l"(v[60]), "=l"(v[61]), "=l"(v[62]), "=l"(v[63])
      : "r"(taddr), "r"(taddr + 32), "r"(taddr + 64), "r"(taddr + 96)
      : "memory");
}

// *addr += {a, b, c, d} (four fp32 reductions in one request, in L2; relaxed).
__device__ __forceinline__ void red_add_v4_f32(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- math
// Packed fp32 pairs (sm_100): two lanes per 64-bit register, each rounded to nearest.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float f2_lo(uint64_t a) { return __uint_as_float(static_cast<uint32_t>(a)); }
__device__ __forceinline__ float f2_hi(uint64_t a) { return __uint_as_float(static_cast<uint32_t>(a >> 32)); }
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// Three-input max / min (sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// exp2 of both lanes of a pair (MUFU), result as a pair.
__device__ __forceinline__ uint64_t ex2x2(uint64_t x) {
  uint64_t y;
  asm("{\n\t.reg .f32 a, b, c, d;\n\t"
      "mov.b64 {a, b}, %1;\n\t"
      "ex2.approx.ftz.f32 c, a;\n\t"
      "ex2.approx.ftz.f32 d, b;\n\t"
      "mov.b64 %0, {c, d};\n\t}"
      : "=l"(y)
      : "l"(x));
  return y;
}
// exp2 of both lanes of a pair on the FMA pipe (no MUFU): Cody-Waite style
// reduction x = n + f, n = round(x) by the 1.5*2^23 addition trick, |f| <= 1/2,
// then 2^f by the degree-3 minimax polynomial of exp2_poly.cuh (Horner, packed
// fma) and 2^n by adding n to the exponent field.  Inputs are clamped to
// >= -125 so that 2^n stays a normal number; the result is then < 2^-124,
// negligible against the row sum (>= 1).  Max relative error ~7.5e-5.
// `k` holds the pair constants: {magic, magic}, {-magic, -magic}, C0..C3 pairs.
struct Exp2PolyConsts {
  uint64_t magic, neg_magic, c0, c1, c2, c3;
};
__device__ __forceinline__ uint64_t ex2x2_poly(uint64_t x, const Exp2PolyConsts& k) {
  uint64_t y;
  asm("{\n\t.reg .f32 a, b;\n\t.reg .b64 xc, t, n, f, p;\n\t.reg .b32 tl, th, pl, ph, rl, rh;\n\t"
      "mov.b64 {a, b}, %1;\n\t"
      "max.f32 a, a, 0fC2FA0000;\n\t"  // -125
      "max.f32 b, b, 0fC2FA0000;\n\t"
      "mov.b64 xc, {a, b};\n\t"
      "add.rn.f32x2 t, xc, %2;\n\t"      // t = x + magic: round(x) in the low mantissa bits
      "add.rn.f32x2 n, t, %3;\n\t"       // n = round(x) as a float
      "sub.rn.f32x2 f, xc, n;\n\t"       // f = x - n, |f| <= 1/2
      "fma.rn.f32x2 p, %7, f, %6;\n\t"   // C3 f + C2
      "fma.rn.f32x2 p, p, f, %5;\n\t"    // (..) f + C1
      "fma.rn.f32x2 p, p, f, %4;\n\t"    // (..) f + C0
      "mov.b64 {tl, th}, t;\n\t"
      "mov.b64 {pl, ph}, p;\n\t"
      "mad.lo.u32 rl, tl, 8388608, pl;\n\t"  // exponent += n (bits of t hold n mod 2^9)
      "mad.lo.u32 rh, th, 8388608, ph;\n\t"
      "mov.b64 %0, {rl, rh};\n\t}"
      : "=l"(y)
      : "l"(x), "l"(k.magic), "l"(k.neg_magic), "l"(k.c0), "l"(k.c1), "l"(k.c2), "l"(k.c3));
  return y;
}

// bf16x2 of a pair (low lane -> low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2_pair(uint64_t x) {
  uint32_t r;
  asm("{\n\t.reg .f32 a, b;\n\t"
      "mov.b64 {a, b}, %1;\n\t"
      "cvt.rn.bf16x2.f32 %0, b, a;\n\t}"
      : "=r"(r)
      : "l"(x));
  return r;
}
// acc += (fp32 value of the low bf16 of p, fp32 value of the high bf16 of p), lane-wise.
__device__ __forceinline__ uint64_t add_bf16x2_as_f32x2(uint64_t acc, uint32_t p) {
  uint64_t d;
  asm("{\n\t.reg .b32 lo, hi;\n\t.reg .b64 w;\n\t"
      "shl.b32 lo, %2, 16;\n\t"
      "and.b32 hi, %2, 0xffff0000;\n\t"
      "mov.b64 w, {lo, hi};\n\t"
      "add.rn.f32x2 %0, %1, w;\n\t}"
      : "=l"(d)
      : "l"(acc), "r"(p));
  return d;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  // cvt packs its first source into the upper half.
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace pa
