// attn_fp16.cuh -- FP16 FlashAttention forward for the flagged heads.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: selective FP16 fallback
// for accuracy-sensitive attention blocks and denoising steps.  A flagged
// head is plain softmax attention over the RoPE'd fp16 Q, K and the fp16 V:
// fp32 scores, fp32 exponentials, P rounded to fp16 for the P V product, fp32
// accumulation.
//
// One CTA = two 128-row query tiles of one flagged head, 384 threads:
//   warp 0      TMA producer: the two Q tiles once, then the K and V tiles of
//               each 64-key block (tensor-map loads straight from q_rope,
//               k_rope and v, 128-byte swizzle) into a 4-stage ring;
//   warps 1, 2  MMA issuers of tile 0 and tile 1 (warp-uniform loops, one
//               elected lane issues); warp 1 also owns the TMEM allocation;
//   warp 3      idle;
//   warps 4-7   tile 0, warps 8-11 tile 1 (thread = row = TMEM lane).
// S_t(j) = Q_t K_j^T (kind::f16, fp32 in TMEM; the softmax warps release it
// as soon as it is in registers).  P_t(j) goes to TMEM (tcgen05.st) and O_t
// accumulates in TMEM across blocks: the MMA adds P_t(j) V_j to it, with P
// read from TMEM and V_j as it sits in memory (channels contiguous: an
// MN-major B operand).
// The exponentials use a reference max m_ref per row that is raised only when
// a block's max exceeds it by more than 8 (log2 units): P stays <= 2^8, which
// fp16 holds, and O and l are rescaled in place only then (a warp rescales
// its TMEM rows after the previous P V has landed).  The raise is voted per
// warp and every row of the warp follows it; rows past N (whatever follows the
// head in the Q view) take zero scores, so the vote depends on valid rows
// only and the result does not depend on neighbouring memory.  out = O / l.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "sm100.cuh"

namespace rota {

struct Fp16Params {
  CUtensorMap tm_q;   // q_rope as [B*H*N rows, D] fp16, box 64 x 128 rows
  CUtensorMap tm_k;   // k_rope, box 64 x 64 rows
  CUtensorMap tm_v;   // v,      box 64 x 64 rows
  float* out;
  int H, N;
  float scale_log2;     // RN(sm_scale * log2 e)
  uint64_t timeout_ns;
  int nheads;
  int16_t heads[256];
};

constexpr int kF16Threads = 384;
constexpr int kF16Stages = 4;
constexpr float kRescaleLog2 = 8.f;   // raise the reference max only past this margin

template <int D>
struct F16Smem {
  static constexpr int ATOMS = D / 64;                 // 128-byte (64-channel) column atoms
  static constexpr int Q_BYTES = kBM * D * 2;          // one tile: ATOMS x [128 rows x 128 B]
  static constexpr int K_BYTES = kBN * D * 2;          // ATOMS x [64 keys x 128 B], K-major
  static constexpr int V_BYTES = kBN * D * 2;          // ATOMS x [64 keys x 128 B], channels contiguous
  static constexpr int STAGE_BYTES = K_BYTES + V_BYTES;
  static constexpr int OFF_Q = 0;                                // 2 tiles
  static constexpr int OFF_KV = OFF_Q + 2 * Q_BYTES;             // kF16Stages stages
  static constexpr int OFF_BAR = OFF_KV + kF16Stages * STAGE_BYTES;
  // barriers: kv_full[4] kv_empty[4] s_full[2 tiles] s_empty[2] p_full[2]
  //           p_empty[2] q_full mma_done[2]
  static constexpr int NBAR = 4 + 4 + 2 + 2 + 2 + 2 + 1 + 2;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;
  static constexpr int BYTES = OFF_ABORT + 4;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  // S of tile t at column t * 64; the fp16 P of tile t (A operand of P V,
  // 64 keys = 32 columns) at 128 + 32 t; O of tile t at 256 + t * D
  static constexpr uint32_t T_S = 0, T_P = 2 * kBN, T_O = 4 * kBN;
  static_assert(T_P + 2 * (kBN / 2) <= T_O && T_O + 2 * D <= TMEM_COLS, "TMEM budget");
  static_assert(ALLOC <= 232448, "shared memory budget");
  static_assert(Q_BYTES % 1024 == 0 && K_BYTES % 1024 == 0, "swizzle atom alignment");
};

template <int D>
__global__ void __launch_bounds__(kF16Threads, 1) attn_fp16_kernel(const __grid_constant__ Fp16Params p) {
  using L = F16Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 4;
  // per tile, once per block (phase j & 1)
  uint64_t* s_full = bars + 8;
  uint64_t* s_empty = bars + 10;
  uint64_t* p_full = bars + 12;
  // p_empty[t]: tile t's P V of the block has completed -- the P columns may
  // be rewritten, and O holds every block up to that one
  uint64_t* p_empty = bars + 14;
  uint64_t* q_full = bars + 16;
  uint64_t* mma_done = bars + 17;   // [2], one per MMA warp
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + L::OFF_ABORT);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = p.heads[blockIdx.y];
  const int b = blockIdx.z;
  const size_t head = (size_t)b * p.H + h;
  const int row_base = (int)(head * p.N);           // first row of this head in the [B*H*N, D] views
  const int q0 = blockIdx.x * (2 * kBM);
  const int nkb = (p.N + kBN - 1) / kBN;
  const uint64_t lim = p.timeout_ns;

  if (tid == 0) {
    for (int i = 0; i < kF16Stages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 2);   // the last P V of the block, one commit per tile
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_empty[t], 4);
      mbar_init(&p_full[t], 4);
      mbar_init(&p_empty[t], 1);
      mbar_init(&mma_done[t], 1);
    }
    mbar_init(q_full, 1);
    *sAbort = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 1) {
    tmem_alloc(sTmem, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;

  if (warp == 0) {
    // ---- TMA producer (warp-uniform loop, one elected lane issues) ----
    if (elect_one()) {
      mbar_arrive_expect_tx(q_full, 2 * L::Q_BYTES);
      for (int t = 0; t < 2; ++t)
        for (int a = 0; a < L::ATOMS; ++a)
          tma_load_2d(smem + L::OFF_Q + t * L::Q_BYTES + a * (kBM * 128), &p.tm_q, 64 * a, row_base + q0 + t * kBM,
                      q_full);
    }
    __syncwarp();
    int issued = 0;
    for (int j = 0; j < nkb; ++j) {
      const int st = j % kF16Stages;
      if (!warp_wait(&kv_empty[st], ((j / kF16Stages) & 1) ^ 1, lim)) {
        if (lane == 0) *sAbort = 1;
        break;
      }
      if (warp_flag(sAbort)) break;
      uint8_t* kt = smem + L::OFF_KV + st * L::STAGE_BYTES;
      if (elect_one()) {
        mbar_arrive_expect_tx(&kv_full[st], L::STAGE_BYTES);
        for (int a = 0; a < L::ATOMS; ++a) {
          tma_load_2d(kt + a * (kBN * 128), &p.tm_k, 64 * a, row_base + j * kBN, &kv_full[st]);
          tma_load_2d(kt + L::K_BYTES + a * (kBN * 128), &p.tm_v, 64 * a, row_base + j * kBN, &kv_full[st]);
        }
      }
      __syncwarp();
      issued = j + 1;
    }
    // drain: every issued copy has landed before the CTA may exit
    warp_wait(q_full, 0, lim);
    for (int j = (issued > kF16Stages ? issued - kF16Stages : 0); j < issued; ++j)
      warp_wait(&kv_full[j % kF16Stages], (j / kF16Stages) & 1, lim);
  } else if (warp <= 2) {
    // ---- MMA issuers: warp 1 + t issues tile t's MMAs (warp-uniform loop,
    // one elected lane issues) ----
    const int t = warp - 1;
    constexpr uint32_t ID_S = idesc(1, 0, 0, kBM, kBN);     // f16 x f16 -> f32, 128 x 64
    constexpr uint32_t ID_PV = idesc(1, 0, 0, kBM, D, 1);   // B (V) channels-contiguous
    const uint32_t qa = smem_u32(smem + L::OFF_Q) + t * L::Q_BYTES, kv_addr = smem_u32(smem + L::OFF_KV);
    const uint32_t d_s = tmem + L::T_S + t * kBN, d_o = tmem + L::T_O + t * D;
    const uint32_t ap = tmem + L::T_P + t * (kBN / 2);   // P of tile t: 16 keys = 8 columns per K step
    bool ok = warp_wait(q_full, 0, lim);
    auto issue_s = [&](int j) -> bool {
      if (!warp_wait(&s_empty[t], (j & 1) ^ 1, lim)) return false;
      tc_fence_after();
      const uint32_t ka = kv_addr + (j % kF16Stages) * L::STAGE_BYTES;
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t atom = k >> 2, within = (k & 3) * 32;
          mma_f16(d_s, sdesc(qa + atom * (kBM * 128) + within, 1024, 2),
                  sdesc(ka + atom * (kBN * 128) + within, 1024, 2), ID_S, k > 0);
        }
        mma_commit(&s_full[t]);
      }
      __syncwarp();
      return true;
    };
    auto issue_pv = [&](int j) -> bool {
      const uint32_t va = kv_addr + (j % kF16Stages) * L::STAGE_BYTES + L::K_BYTES;
      if (!warp_wait(&p_full[t], j & 1, lim)) return false;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < kBN / 16; ++k) {
          const uint64_t bd = sdesc_lbo(va + 2048 * k, kBN * 128, 1024, 2);
          const uint32_t blo = static_cast<uint32_t>(bd), bhi = static_cast<uint32_t>(bd >> 32);
          if (j == 0 && k == 0) mma_f16_ts<0>(d_o, ap + 8 * k, blo, bhi, ID_PV);
          else mma_f16_ts<1>(d_o, ap + 8 * k, blo, bhi, ID_PV);
        }
        mma_commit(&p_empty[t]);
        mma_commit(&kv_empty[j % kF16Stages]);
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; ok && j < nkb; ++j) {
      if (!warp_wait(&kv_full[j % kF16Stages], (j / kF16Stages) & 1, lim)) { ok = false; break; }
      tc_fence_after();
      if (!issue_s(j)) { ok = false; break; }
      if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
      if (warp_flag(sAbort)) { ok = false; break; }
    }
    if (ok) ok = issue_pv(nkb - 1);
    if (!ok && lane == 0) *sAbort = 1;
    // every MMA this warp issued completes before TMEM is released
    if (elect_one()) mma_commit(&mma_done[t]);
    __syncwarp();
    warp_wait(&mma_done[t], 0, lim);
  } else if (warp >= 4) {
    // ===================================================== query-tile warps
    const int t = (warp - 4) >> 2;       // tile 0 or 1
    const int r = tid & 127;             // row within the tile = TMEM lane
    const int row = q0 + t * kBM + r;
    const uint32_t t_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + L::T_S + t * kBN + t_lane;
    const uint32_t tP = tmem + L::T_P + t * (kBN / 2) + t_lane;
    const uint32_t tO = tmem + L::T_O + t * D + t_lane;
    const float c = p.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool aborted = false;

    for (int j = 0; j < nkb; ++j) {
      const int nvalid = min(kBN, p.N - j * kBN);
      if (!warp_wait(&s_full[t], j & 1, lim)) { aborted = true; break; }
      tc_fence_after();
      uint32_t sr[kBN];
      {
        uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        tmem_ld32(tS, s0);
        tmem_ld32(tS + 32, s1);
        tmem_wait_dep2(s0, s1);
      }
      // S is in registers: the MMA may compute S(j+1) into this buffer now
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[t]);
      // Rows past N hold whatever follows the head in the Q view; their scores
      // are taken as 0, so that the warp's vote on raising the reference max
      // (which every row of the warp follows) depends on valid rows only.
      if (row >= p.N) {
#pragma unroll
        for (int k = 0; k < kBN; ++k) sr[k] = 0u;
      }
      if (nvalid < kBN) {
#pragma unroll
        for (int k = 0; k < kBN; ++k)
          if (k >= nvalid) sr[k] = __float_as_uint(-INFINITY);
      }
      float x0 = -INFINITY, x1 = -INFINITY, x2 = -INFINITY, x3 = -INFINITY;
#pragma unroll
      for (int k = 0; k < kBN; k += 8) {
        x0 = max3(x0, __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]));
        x1 = max3(x1, __uint_as_float(sr[k + 2]), __uint_as_float(sr[k + 3]));
        x2 = max3(x2, __uint_as_float(sr[k + 4]), __uint_as_float(sr[k + 5]));
        x3 = max3(x3, __uint_as_float(sr[k + 6]), __uint_as_float(sr[k + 7]));
      }
      const float m_blk = __fmul_rn(fmaxf(fmaxf(x0, x1), fmaxf(x2, x3)), c);

      // ---- raise the reference max (rare); O is rescaled below ----
      const bool raise = __any_sync(0xffffffffu, m_blk > m_ref + kRescaleLog2);
      float alpha = 1.f;
      if (raise) {
        const float m_new = fmaxf(m_ref, m_blk);
        alpha = ex2_approx(m_ref - m_new);   // 0 while O is empty (m_ref = -inf)
        m_ref = m_new;
        l *= alpha;
      }

      // ---- P = 2^(S c - m_ref) in fp16, row sum of the fp16 values in fp32 ----
      uint32_t pw[kBN / 2];
      float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
      for (int k = 0; k < kBN; k += 2) {
        float d0, d1;
        fma2(d0, d1, __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]), c, c, -m_ref, -m_ref);
        const __half2 hp = __floats2half2_rn(ex2_approx(d0), ex2_approx(d1));
        // l sums the fp16 values the P V product uses, so out = O / l is exact
        // for a row whose weight sits on one key
        const float2 back = __half22float2(hp);
        add2(ls0, ls1, ls0, ls1, back.x, back.y);
        pw[k / 2] = *reinterpret_cast<const uint32_t*>(&hp);
      }
      l += ls0 + ls1;
      // the previous block's P V has completed: the P columns are free and O
      // holds every block before this one
      if (j > 0) {
        if (!warp_wait(&p_empty[t], (j - 1) & 1, lim)) { aborted = true; break; }
        tc_fence_after();
        if (raise) {
#pragma unroll 1
          for (int cb = 0; cb < D / 32; ++cb) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * cb, o);
            tmem_wait_dep(o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(tO + 32 * cb, o);
          }
        }
      }
      tmem_st32(tP, pw);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
      if (warp_flag(sAbort)) { aborted = true; break; }
    }
    // ---- epilogue: out = O / l once the last P V has landed ----
    if (!aborted && !warp_wait(&p_empty[t], (nkb - 1) & 1, lim)) aborted = true;
    if (aborted) {
      *sAbort = 1;
    } else {
      tc_fence_after();
      const float inv_l = 1.f / l;
      float* dst = p.out + ((size_t)row_base + row) * D;
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * cb, o);
        tmem_wait_dep(o);
        if (row < p.N) {
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(dst + 32 * cb + k) =
                make_float4(__uint_as_float(o[k]) * inv_l, __uint_as_float(o[k + 1]) * inv_l,
                            __uint_as_float(o[k + 2]) * inv_l, __uint_as_float(o[k + 3]) * inv_l);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace rota
