// attn_int4.cuh -- INT4 FlashAttention forward with range-optimised P codes.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: a mixed-precision INT4
// FlashAttention in which P = exp(QK - max(QK)) >= 0 is quantised with a
// fixed scale and zero-point so that all 16 unsigned 4-bit levels are used
// ("Range-optimized P Quantization").
//
// Per CTA: 128 query rows of one head; thread i owns row i (TMEM lane i).
// Per 64-key block:
//   1. packed s4 K / V codes -> s8 in shared memory (128-bit loads, swizzled
//      K-major layouts the tensor core reads directly);
//   2. S = Qc Kc^T on the tensor core (tcgen05.mma kind::i8, s32 in TMEM);
//   3. per row: c = RN(RN(sq sk) kappa), running max m over the block,
//      d = fma(S, c, -m), u = rne(15 * 2^d) (exact: estimate + threshold fix),
//      row sum l and the u8 codes written to shared memory;
//   4. acc = P V_c on the tensor core (kind::i8, u8 x s8 -> s32 in TMEM);
//   5. O = O * 2^(m_old - m) + v_scale * acc in fp32 registers.
// The epilogue writes O / l.
#pragma once
#include <climits>
#include <cstdint>

#include "sm100.cuh"

namespace rota {

struct Int4Params {
  const uint8_t* q_codes;
  const uint8_t* k_codes;
  const float* q_scale;
  const float* k_scale;
  const uint8_t* v_codes;
  const float* v_scale;
  float* out;
  int H, N, nblk;
  float kappa;          // RN(sm_scale * log2 e)
  float tau[16];        // tau[k]: smallest fp32 d with rne(15 * 2^d) >= k (k = 1..15)
  uint64_t timeout_ns;  // bound of every mbarrier wait
  int inject_skip;      // fault injection: skip the first score MMA
  int nheads;
  int16_t heads[256];   // the INT4 heads to process (blockIdx.y indexes this list)
  // debug dump (DUMP kernels only)
  int32_t* s_dump;
  uint8_t* p_dump;
  int dbg_r0, dbg_nr;
};

constexpr int kInt4Threads = 128;

template <int D>
struct Int4Smem {
  static constexpr int QROW = D;          // bytes per s8 row of Q / K
  static constexpr int Q_BYTES = kBM * D;
  static constexpr int K_BYTES = kBN * D;
  static constexpr int V_BYTES = D * kBN;  // V^T: D rows of 64 keys
  static constexpr int P_BYTES = kBM * kBN;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + K_BYTES;
  static constexpr int OFF_P = OFF_V + V_BYTES;
  static constexpr int OFF_VS = OFF_P + P_BYTES;       // D floats
  static constexpr int OFF_TAU = OFF_VS + D * 4;       // 16 floats
  static constexpr int OFF_BAR = OFF_TAU + 64;         // 8-byte aligned
  static constexpr int OFF_TMEM = OFF_BAR + 8;
  static constexpr int OFF_FLAG = OFF_TMEM + 4;
  static constexpr int BYTES = OFF_FLAG + 4;
  static constexpr int ALLOC = BYTES + 1024;           // + alignment slack
  static constexpr int TMEM_COLS = (kBN + D) <= 128 ? 128 : 256;
  static constexpr uint32_t LAYOUT_QK = D == 128 ? 2u : 4u;  // 128B / 64B swizzle
  static constexpr uint32_t SBO_QK = 8 * D;
};

// Range-optimised P code u = rne(15 * 2^d) in exact arithmetic, d <= ~0.
// The MUFU estimate is within ~4e-6 of 15 * 2^d; only when it falls within
// 1e-4 of a half-integer is the decision taken by the exact threshold table.
__device__ __forceinline__ uint32_t pcode(float d, const float* tau) {
  const float e = 15.f * ex2_approx(d);
  const float r = __fsub_rn(__fadd_rn(e, 12582912.f), 12582912.f);  // rne to integer
  const float fr = e - r;
  uint32_t u = static_cast<uint32_t>(r);
  if (fabsf(fr) > 0.5f - 1e-4f) {
    int j = fr > 0.f ? static_cast<int>(r) + 1 : static_cast<int>(r);
    j = max(1, min(15, j));
    u = d >= tau[j] ? j : j - 1;
  }
  return u;
}

template <int D, bool DUMP>
__global__ void __launch_bounds__(kInt4Threads, 1) attn_int4_kernel(const __grid_constant__ Int4Params p) {
  using L = Int4Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint8_t* sP = smem + L::OFF_P;
  float* sVs = reinterpret_cast<float*>(smem + L::OFF_VS);
  float* sTau = reinterpret_cast<float*>(smem + L::OFF_TAU);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  int* sAbort = reinterpret_cast<int*>(smem + L::OFF_FLAG);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int qt = blockIdx.x;
  const int h = p.heads[blockIdx.y];
  const int b = blockIdx.z;
  const size_t head = (size_t)b * p.H + h;
  const int npad = p.nblk * kBN;
  const int row = qt * kBM + tid;

  if (tid < 16) sTau[tid] = p.tau[tid];
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

  // Q tile: packed s4 rows -> s8, swizzled K-major.
  {
    const uint8_t* qsrc = p.q_codes + (head * npad + (size_t)qt * kBM) * (D / 2);
    for (int i = tid; i < kBM * D / 32; i += kInt4Threads) {
      const int r = i / (D / 32), c = i % (D / 32);
      uint4 w = make_uint4(0, 0, 0, 0);
      if (qt * kBM + r < npad) w = __ldg(reinterpret_cast<const uint4*>(qsrc + (size_t)r * (D / 2) + c * 16));
      uint32_t o[8];
      s4x8_to_s8(w.x, o[0], o[1]);
      s4x8_to_s8(w.y, o[2], o[3]);
      s4x8_to_s8(w.z, o[4], o[5]);
      s4x8_to_s8(w.w, o[6], o[7]);
      *reinterpret_cast<uint4*>(sQ + swz<L::QROW>(r, c * 32)) = make_uint4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<uint4*>(sQ + swz<L::QROW>(r, c * 32 + 16)) = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
  const float sq = row < npad ? __ldg(p.q_scale + head * p.nblk + row / kBN) : 0.f;

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t t_lane = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem;        // columns [0, 64): S (s32)
  const uint32_t tO = tmem + kBN;  // columns [64, 64 + D): P V accumulator (s32)

  constexpr uint32_t ID_S = idesc(2, 1, 1, kBM, kBN);   // s8 x s8 -> s32, 128 x 64
  constexpr uint32_t ID_PV = idesc(2, 0, 1, kBM, D);    // u8 x s8 -> s32, 128 x D

  float O[D];
#pragma unroll
  for (int c = 0; c < D; ++c) O[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  uint32_t phase = 0;
  bool aborted = false;

#pragma unroll 1
  for (int kb = 0; kb < p.nblk; ++kb) {
    // ---- stage K and V codes of this block ----
    const uint8_t* ksrc = p.k_codes + (head * npad + (size_t)kb * kBN) * (D / 2);
    for (int i = tid; i < kBN * D / 32; i += kInt4Threads) {
      const int r = i / (D / 32), c = i % (D / 32);
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(ksrc + (size_t)r * (D / 2) + c * 16));
      uint32_t o[8];
      s4x8_to_s8(w.x, o[0], o[1]);
      s4x8_to_s8(w.y, o[2], o[3]);
      s4x8_to_s8(w.z, o[4], o[5]);
      s4x8_to_s8(w.w, o[6], o[7]);
      *reinterpret_cast<uint4*>(sK + swz<L::QROW>(r, c * 32)) = make_uint4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<uint4*>(sK + swz<L::QROW>(r, c * 32 + 16)) = make_uint4(o[4], o[5], o[6], o[7]);
    }
    const uint8_t* vsrc = p.v_codes + (head * p.nblk + kb) * (size_t)D * 32;
    for (int i = tid; i < D * 2; i += kInt4Threads) {
      const int c = i >> 1, hlf = i & 1;
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(vsrc + (size_t)c * 32 + hlf * 16));
      uint32_t o[8];
      s4x8_to_s8(w.x, o[0], o[1]);
      s4x8_to_s8(w.y, o[2], o[3]);
      s4x8_to_s8(w.z, o[4], o[5]);
      s4x8_to_s8(w.w, o[6], o[7]);
      *reinterpret_cast<uint4*>(sV + swz<64>(c, hlf * 32)) = make_uint4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<uint4*>(sV + swz<64>(c, hlf * 32 + 16)) = make_uint4(o[4], o[5], o[6], o[7]);
    }
    if (tid < D) sVs[tid] = __ldg(p.v_scale + (head * p.nblk + kb) * D + tid);
    const float sk = __ldg(p.k_scale + head * p.nblk + kb);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- S = Qc Kc^T ----
    if (tid == 0) {
      tc_fence_after();
      if (!(p.inject_skip && kb == 0)) {
        const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK);
#pragma unroll
        for (int k = 0; k < D / 32; ++k)
          mma_i8(tS, sdesc(qa + 32 * k, L::SBO_QK, L::LAYOUT_QK), sdesc(ka + 32 * k, L::SBO_QK, L::LAYOUT_QK),
                 ID_S, k > 0);
        mma_commit(bar);
      }
    }
    if (!mbar_wait(bar, phase, p.timeout_ns)) *sAbort = 1;
    phase ^= 1;
    __syncthreads();
    if (*sAbort) { aborted = true; break; }
    tc_fence_after();

    int32_t S[kBN];
    {
      uint32_t r0[32], r1[32];
      tmem_ld32(tS + t_lane, r0);
      tmem_ld32(tS + t_lane + 32, r1);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        S[j] = static_cast<int32_t>(r0[j]);
        S[32 + j] = static_cast<int32_t>(r1[j]);
      }
    }

    // ---- running max, P codes, row sum ----
    const int nvalid = min(kBN, p.N - kb * kBN);
    const float c = __fmul_rn(__fmul_rn(sq, sk), p.kappa);
    int smax = INT_MIN;
#pragma unroll
    for (int j = 0; j < kBN; ++j)
      if (j < nvalid) smax = max(smax, S[j]);
    const float m_new = fmaxf(m, __fmul_rn(static_cast<float>(smax), c));
    const float alpha = ex2_approx(m - m_new);  // m = -inf on the first block: alpha = 0
    m = m_new;
    uint32_t usum = 0;
    uint32_t pw[kBN / 4];
#pragma unroll
    for (int j4 = 0; j4 < kBN / 4; ++j4) {
      uint32_t w = 0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int j = 4 * j4 + t;
        const float dd = __fmaf_rn(static_cast<float>(S[j]), c, -m);
        uint32_t u = pcode(dd, sTau);
        if (j >= nvalid) u = 0;
        usum += u;
        w |= u << (8 * t);
      }
      pw[j4] = w;
    }
    l = __fmaf_rn(l, alpha, static_cast<float>(usum));
#pragma unroll
    for (int j = 0; j < kBN / 16; ++j)
      *reinterpret_cast<uint4*>(sP + swz<64>(tid, 16 * j)) = make_uint4(pw[4 * j], pw[4 * j + 1], pw[4 * j + 2], pw[4 * j + 3]);
    if (DUMP && row >= p.dbg_r0 && row < p.dbg_r0 + p.dbg_nr) {
      const size_t base = (size_t)(row - p.dbg_r0) * p.N + (size_t)kb * kBN;
      for (int j = 0; j < nvalid; ++j) {
        p.s_dump[base + j] = S[j];
        p.p_dump[base + j] = static_cast<uint8_t>((pw[j >> 2] >> (8 * (j & 3))) & 0xFF);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- acc = P Vc ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t pa = smem_u32(sP), va = smem_u32(sV);
#pragma unroll
      for (int k = 0; k < kBN / 32; ++k)
        mma_i8(tO, sdesc(pa + 32 * k, 512, 4), sdesc(va + 32 * k, 512, 4), ID_PV, k > 0);
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
      tmem_ld_wait();
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const float sv = sVs[32 * j + t];
        O[32 * j + t] = __fmaf_rn(O[32 * j + t], alpha, sv * static_cast<float>(static_cast<int32_t>(a[t])));
      }
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

// Exhaustive-check hook: the kernel's P-code function on an array.
__global__ void pcode_kernel(const float* d, uint8_t* u, int64_t n, Int4Params p) {
  __shared__ float tau[16];
  if (threadIdx.x < 16) tau[threadIdx.x] = p.tau[threadIdx.x];
  __syncthreads();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    u[i] = static_cast<uint8_t>(pcode(d[i], tau));
}

}  // namespace rota
