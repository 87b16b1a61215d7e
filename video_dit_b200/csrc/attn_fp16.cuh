// attn_fp16.cuh -- FP16 FlashAttention forward for the flagged heads.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: "selective FP16
// fallback for accuracy-sensitive attention blocks and denoising steps".
//
// Per CTA: 128 query rows of one flagged head, thread i owns row i.
// Per 64-key block: fp16 K (K-major) and V^T tiles staged in shared memory,
// S = Q K^T on the tensor core (tcgen05.mma kind::f16, fp32 in TMEM), an fp32
// online softmax in base 2, P rounded to fp16 into shared memory, acc = P V
// (kind::f16, fp32 in TMEM), O = O * alpha + acc in registers; out = O / l.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "sm100.cuh"

namespace rota {

struct Fp16Params {
  const __half* q_rope;
  const __half* k_rope;
  const __half* v;
  float* out;
  int H, N;
  float scale_log2;     // RN(sm_scale * log2 e)
  uint64_t timeout_ns;
  int nheads;
  int16_t heads[256];
};

constexpr int kF16Threads = 128;

template <int D>
struct F16Smem {
  static constexpr int KATOMS = D * 2 / 128;      // 128-byte K atoms per Q/K row
  static constexpr int Q_BYTES = kBM * D * 2;
  static constexpr int K_BYTES = kBN * D * 2;
  static constexpr int V_BYTES = D * kBN * 2;     // V^T: D rows of 64 keys (128 B)
  static constexpr int P_BYTES = kBM * kBN * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + K_BYTES;
  static constexpr int OFF_P = OFF_V + V_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int OFF_TMEM = OFF_BAR + 8;
  static constexpr int OFF_FLAG = OFF_TMEM + 4;
  static constexpr int BYTES = OFF_FLAG + 4;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr int TMEM_COLS = (kBN + D) <= 128 ? 128 : 256;
};

// Byte offset of (row, byte k) in a K-major fp16 tile of `rows` rows stored as
// consecutive [rows x 128 B] atoms along K, 128-byte swizzle.
__device__ __forceinline__ uint32_t swz_atoms(uint32_t row, uint32_t kbyte, uint32_t rows) {
  return (kbyte >> 7) * rows * 128 + swz<128>(row, kbyte & 127);
}

template <int D>
__global__ void __launch_bounds__(kF16Threads, 1) attn_fp16_kernel(const __grid_constant__ Fp16Params p) {
  using L = F16Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint8_t* sP = smem + L::OFF_P;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  int* sAbort = reinterpret_cast<int*>(smem + L::OFF_FLAG);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int qt = blockIdx.x;
  const int h = p.heads[blockIdx.y];
  const int b = blockIdx.z;
  const size_t head = (size_t)b * p.H + h;
  const int row = qt * kBM + tid;
  const int nkb = (p.N + kBN - 1) / kBN;

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    *sAbort = 0;
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(sTmem, L::TMEM_COLS);
    tmem_relinquish();
  }
  {
    const __half* qsrc = p.q_rope + head * p.N * D;
    for (int i = tid; i < kBM * D / 8; i += kF16Threads) {
      const int r = i / (D / 8), c = i % (D / 8);
      const int n = qt * kBM + r;
      uint4 w = make_uint4(0, 0, 0, 0);
      if (n < p.N) w = __ldg(reinterpret_cast<const uint4*>(qsrc + (size_t)n * D + c * 8));
      *reinterpret_cast<uint4*>(sQ + swz_atoms(r, c * 16, kBM)) = w;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t t_lane = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem, tO = tmem + kBN;
  constexpr uint32_t ID_S = idesc(1, 0, 0, kBM, kBN);   // f16 x f16 -> f32
  constexpr uint32_t ID_PV = idesc(1, 0, 0, kBM, D);

  float O[D];
#pragma unroll
  for (int c = 0; c < D; ++c) O[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  uint32_t phase = 0;
  bool aborted = false;

#pragma unroll 1
  for (int kb = 0; kb < nkb; ++kb) {
    const __half* ksrc = p.k_rope + (head * p.N + (size_t)kb * kBN) * D;
    const __half* vsrc = p.v + (head * p.N + (size_t)kb * kBN) * D;
    const int nvalid = min(kBN, p.N - kb * kBN);
    for (int i = tid; i < kBN * D / 8; i += kF16Threads) {
      const int r = i / (D / 8), c = i % (D / 8);
      uint4 kw = make_uint4(0, 0, 0, 0), vw = make_uint4(0, 0, 0, 0);
      if (r < nvalid) {
        kw = __ldg(reinterpret_cast<const uint4*>(ksrc + (size_t)r * D + c * 8));
        vw = __ldg(reinterpret_cast<const uint4*>(vsrc + (size_t)r * D + c * 8));
      }
      *reinterpret_cast<uint4*>(sK + swz_atoms(r, c * 16, kBN)) = kw;
      // V^T: channel rows of 64 keys; key r -> byte 2r of rows 8c .. 8c+7
      const uint16_t* vh = reinterpret_cast<const uint16_t*>(&vw);
#pragma unroll
      for (int j = 0; j < 8; ++j) *reinterpret_cast<uint16_t*>(sV + swz<128>(c * 8 + j, 2 * r)) = vh[j];
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    if (tid == 0) {
      tc_fence_after();
      const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t atom = (k * 32) >> 7, within = (k * 32) & 127;
        mma_f16(tS, sdesc(qa + atom * kBM * 128 + within, 1024, 2), sdesc(ka + atom * kBN * 128 + within, 1024, 2),
                ID_S, k > 0);
      }
      mma_commit(bar);
    }
    if (!mbar_wait(bar, phase, p.timeout_ns)) *sAbort = 1;
    phase ^= 1;
    __syncthreads();
    if (*sAbort) { aborted = true; break; }
    tc_fence_after();

    float s[kBN];
    {
      uint32_t r0[32], r1[32];
      tmem_ld32(tS + t_lane, r0);
      tmem_ld32(tS + t_lane + 32, r1);
      tmem_wait_dep2(r0, r1);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        s[j] = __uint_as_float(r0[j]) * p.scale_log2;
        s[32 + j] = __uint_as_float(r1[j]) * p.scale_log2;
      }
    }
    float bmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < kBN; ++j)
      if (j < nvalid) bmax = fmaxf(bmax, s[j]);
    const float m_new = fmaxf(m, bmax);
    const float alpha = ex2_approx(m - m_new);
    m = m_new;
    float psum = 0.f;
    uint32_t pw[kBN / 2];
#pragma unroll
    for (int j2 = 0; j2 < kBN / 2; ++j2) {
      float p0 = (2 * j2 < nvalid) ? ex2_approx(s[2 * j2] - m) : 0.f;
      float p1 = (2 * j2 + 1 < nvalid) ? ex2_approx(s[2 * j2 + 1] - m) : 0.f;
      const __half2 hp = __floats2half2_rn(p0, p1);
      const float2 back = __half22float2(hp);
      psum += back.x + back.y;
      pw[j2] = *reinterpret_cast<const uint32_t*>(&hp);
    }
    l = l * alpha + psum;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint4*>(sP + swz<128>(tid, 16 * j)) = make_uint4(pw[4 * j], pw[4 * j + 1], pw[4 * j + 2], pw[4 * j + 3]);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    if (tid == 0) {
      tc_fence_after();
      const uint32_t pa = smem_u32(sP), va = smem_u32(sV);
#pragma unroll
      for (int k = 0; k < kBN / 16; ++k)
        mma_f16(tO, sdesc(pa + 32 * k, 1024, 2), sdesc(va + 32 * k, 1024, 2), ID_PV, k > 0);
      mma_commit(bar);
    }
    if (!mbar_wait(bar, phase, p.timeout_ns)) *sAbort = 1;
    phase ^= 1;
    __syncthreads();
    if (*sAbort) { aborted = true; break; }
    tc_fence_after();
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {
      uint32_t a[32];
      tmem_ld32(tO + t_lane + 32 * j, a);
      tmem_wait_dep(a);
#pragma unroll
      for (int t = 0; t < 32; ++t) O[32 * j + t] = __fmaf_rn(O[32 * j + t], alpha, __uint_as_float(a[t]));
    }
    tc_fence_before();
    __syncthreads();
  }

  if (!aborted && row < p.N) {
    const float inv_l = 1.f / l;
    float4* dst = reinterpret_cast<float4*>(p.out + (head * p.N + row) * D);
#pragma unroll
    for (int c4 = 0; c4 < D / 4; ++c4)
      dst[c4] = make_float4(O[4 * c4] * inv_l, O[4 * c4 + 1] * inv_l, O[4 * c4 + 2] * inv_l, O[4 * c4 + 3] * inv_l);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace rota
