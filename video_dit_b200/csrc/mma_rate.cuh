// mma_rate.cuh -- cycles per tcgen05.mma for the operand kinds the attention
// kernels could use, measured on the device the library runs on.
//
// The INT4 kernel's Q K^T is an exact integer product.  Two tensor-core kinds
// can form it: kind::i8 (s8 operands, s32 accumulators) and kind::f8f6f4 with
// the codes as e4m3 subnormals (fp32 accumulators holding the same integers,
// scaled by 2^-18).  This kernel times a chain of MMAs of one kind and shape
// issued back to back into one accumulator (the pattern of the K steps of a
// score tile), so both kinds are measured on identical shapes, operands in
// shared memory.  kind::f16 is timed the same way for reference.
#pragma once
#include <cstdint>

#include "sm100.cuh"

namespace rota {

constexpr int kRateThreads = 128;
constexpr int kRateSmem = 16384 + 32768 + 64 + 1024;   // A 128 x 128 B, B 256 x 128 B, barrier, TMEM slot, alignment

__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(id), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(id), "r"(acc)
      : "memory");
}

// kind: 0 = f8f6f4 (e4m3 x e4m3 -> f32), 1 = i8 (s8 x s8 -> s32), 2 = f16 (f16 x f16 -> f32).
// One CTA: warp 0 issues `iters` x 4 MMAs of M = 128, N = n, 128 bytes of K
// per row per 4 MMAs (K = 32 for the 8-bit kinds, 16 for f16), all into TMEM
// column 0; out[0] = clock64 cycles from the first issue to the commit's
// completion.  The operand bytes are small values that are valid in every
// kind (0x00-0x07: e4m3 subnormals, small s8 integers, small fp16 halves).
__global__ void __launch_bounds__(kRateThreads, 1) mma_rate_kernel(int kind, int n, int iters, uint64_t limit_ns,
                                                                     unsigned long long* out) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  uint8_t* A = sm;              // 128 rows x 128 bytes
  uint8_t* B = sm + 16384;      // 256 rows x 128 bytes
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 16384 + 32768);
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + 16384 + 32768 + 8);
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < (16384 + 32768) / 4; i += kRateThreads)
    reinterpret_cast<uint32_t*>(sm)[i] = (static_cast<uint32_t>(i) * 2654435761u) & 0x07070707u;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (warp == 0) {
    const uint32_t id = kind == 1 ? idesc(2, 1, 1, 128, n) : idesc(1, 0, 0, 128, n);
    const uint32_t hi = sdesc_hi(1024, 2);   // 128-byte rows, 128B swizzle
    const uint32_t la = sdesc_lo(smem_u32(A)), lb = sdesc_lo(smem_u32(B));
    const unsigned long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = (static_cast<uint64_t>(hi) << 32) | (la + 2 * k);
          const uint64_t bd = (static_cast<uint64_t>(hi) << 32) | (lb + 2 * k);
          const uint32_t acc = (it | k) ? 1u : 0u;
          if (kind == 0)
            mma_f8_ss(tmem, ad, bd, id, acc);
          else if (kind == 1)
            mma_i8_ss(tmem, ad, bd, id, acc);
          else
            mma_f16(tmem, ad, bd, id, acc);
        }
      }
      __syncwarp();
    }
    if (elect_one()) mma_commit(bar);
    __syncwarp();
    const bool ok = warp_wait(bar, 0, limit_ns);
    const unsigned long long t1 = clock64();
    if (tid == 0) out[0] = ok ? t1 - t0 : 0ull;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace rota
