// Fifth-generation tensor-core primitives for sm_100a: tensor-memory (TMEM) allocation, the
// single-thread tcgen05.mma with shared-memory operand descriptors, its completion on an mbarrier,
// and TMEM -> register loads, plus the TMA tensor copies that stage the operands.
//
// Conventions used by the kernels here (cta_group::1, kind::f16, bf16 operands, fp32 accumulator):
//  * An operand tile in shared memory is written by a TMA tensor copy with the 128-byte swizzle:
//    rows of 128 bytes, the 16-byte chunk c of row r stored at chunk c ^ (r mod 8), the pattern
//    repeating every 8 rows (1 KB).  Tiles start on a 1 KB boundary.
//  * K-major operand (rows contiguous along the contraction): 8-row groups 1 KB apart; one MMA
//    takes K = 16 (32 bytes of each row), so step k within a 64-wide row starts 32 k bytes in.
//  * MN-major operand (rows contiguous along M): each row of the staged box holds 64 consecutive
//    M elements for one k; boxes of 64 M-elements sit `mn_stride` bytes apart, groups of 8 k rows
//    1 KB apart; step k (16 rows) starts 2 KB k in.
//  * The accumulator of an M = 128 MMA occupies TMEM lanes 0..127 (row i of D in lane i) and N
//    consecutive 32-bit columns; warp w of the CTA may read lanes 32 (w mod 4) .. 32 (w mod 4) + 31.
#pragma once

#include <cuda.h>  // CUtensorMap

#include "common.cuh"
#include "tma.cuh"

namespace csffn {

// cuTensorMapEncodeTiled, looked up once from the driver through the runtime (dense_mma.cu).
typedef CUresult (*TensorMapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                      const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
TensorMapEncodeFn tensor_map_encoder();

// ---------------------------------------------------------------------------------------------
// Descriptors
// ---------------------------------------------------------------------------------------------

// Shared-memory matrix descriptor (64 bits): start address >> 4 in bits 0-13, leading byte offset
// >> 4 in bits 16-29, stride byte offset >> 4 in bits 32-45, descriptor version 1 in bits 46-47,
// base offset 0 (tiles are 1 KB aligned), layout type in bits 61-63 (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t umma_desc(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major, 128-byte swizzle: the leading offset is unused (encoded as 16 bytes), 8-row groups 1 KB apart.
__device__ __forceinline__ uint64_t umma_desc_k(uint32_t smem_addr) { return umma_desc(smem_addr, 16u, 1024u); }
// MN-major, 128-byte swizzle: 64-element M groups `mn_stride` bytes apart, 8-row k groups 1 KB apart.
__device__ __forceinline__ uint64_t umma_desc_mn(uint32_t smem_addr, uint32_t mn_stride) {
  return umma_desc(smem_addr, mn_stride, 1024u);
}

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), bf16 A and B (bits 7-9 and
// 10-12 = 1), A major-ness in bit 15 (0 = K-major, 1 = MN-major), B K-major, N >> 3 in bits 17-22,
// M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool a_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------------------------
// TMEM allocation (one full warp executes each of these)
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Order tcgen05 operations against thread synchronisation (barriers, mbarrier waits).
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---------------------------------------------------------------------------------------------
// MMA (issued by one thread)
// ---------------------------------------------------------------------------------------------

// D[tmem] (+)= A[smem desc] * B[smem desc]^T; accumulate == 0 overwrites D.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every MMA this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------------------------------------
// TMEM -> registers (warp-collective): 16 consecutive 32-bit columns of this thread's lane.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------------------------
// TMA tensor copies global -> shared (no multicast), completing on an mbarrier, with an L2 policy.
// The innermost coordinate x must be a multiple of 16 bytes' worth of elements.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar,
                                                 uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
      "%3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_plain(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_plain(void* dst, const CUtensorMap* tm, int x, int y, int z,
                                                  uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Bounded wait that ignores the CTA's abort flag: for draining copies or MMAs still in flight before
// the CTA's shared memory or TMEM is released.  Gives up after a second and records the timeout.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitNs) {
      atomicOr(err, kDevErrTimeout);
      return;
    }
  }
}

// AND of `pred` over the `threads` threads that meet at named barrier `bar` (a barrier among them).
__device__ __forceinline__ bool named_all(int bar, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(bar), "r"(threads)
      : "memory");
  return r != 0;
}

// Programmatic dependent launch: let the next kernel in the stream start scheduling, and wait for
// the previous kernel's completion (and its memory) before touching what it wrote.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_prior() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace csffn
