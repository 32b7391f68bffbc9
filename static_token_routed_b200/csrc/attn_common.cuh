// Device helpers shared by the tensor-core attention kernels (attn_dense.cu,
// attn_skinny.cu, bwd_scores_tc.cu): shared-memory alignment, cp.async row
// copies, a barrier of a warp subset that ANDs a flag, a bounded spin, the
// MN-major-A instruction descriptor and the warp transpose-reduction.
#pragma once
#include <cstdint>

#include "sm100.cuh"

namespace l3 {
namespace attn {

using namespace sm100;

// the next 1024-byte boundary (128-byte-swizzled operands need it)
__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// 16 bytes global -> shared; src_bytes = 0 writes zeros (nothing is read)
__device__ __forceinline__ void cp_async16_zfill(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// until at most N of this thread's committed groups are still in flight
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// barrier `ID` of the N threads that pass it, every thread getting the AND of
// their flags (so that they leave a loop together)
template <int ID, int N>
__device__ __forceinline__ bool sync_and(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "n"(ID), "n"(N)
      : "memory");
  return r != 0;
}

// wait for a phase of `bar`, giving up after WAIT_LIMIT_NS (drain paths)
__device__ __forceinline__ void spin_bounded(uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity) && globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
  }
}

// kind::f16 instruction descriptor with an MN-major A operand: the K-major
// form's bits plus the A-major bit
__host__ __device__ constexpr uint32_t idesc_f16_amn(uint32_t ab_format, uint32_t M, uint32_t N) {
  return idesc_f16(ab_format, 0, M, N) | (1u << 15);
}

// Butterfly over the warp: v[t] holds this lane's value for token t (32 of
// them); the return value is the max (SUM = false) or sum over the 32 lanes
// for token t = lane. Each step trades half of the values a lane still holds
// with the partner lane and combines the other half (31 shuffles in all).
template <bool SUM>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      // keep tokens i + (upper ? w : 0) of this block, send the others
      const float keep = upper ? v[i + w] : v[i];
      const float send = upper ? v[i] : v[i + w];
      const float got = __shfl_xor_sync(0xffffffffu, send, w);
      v[i] = SUM ? keep + got : fmaxf(keep, got);
    }
  }
  return v[0];
}

}  // namespace attn
}  // namespace l3
