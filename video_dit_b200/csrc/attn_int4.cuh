// attn_int4.cuh -- INT4 FlashAttention forward with range-optimised P codes.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: a mixed-precision INT4
// FlashAttention in which P = exp(QK - max(QK)) >= 0 is quantised with a
// fixed scale and zero-point so that all 16 unsigned 4-bit levels are used
// ("Range-optimized P Quantization").
//
// Exact contractions on the tensor core.  S = Q K^T on the 8-bit path: a code
// v in [-7, 7] is widened to the e4m3 subnormal v * 2^-9 (exact) and
// tcgen05.mma kind::f8f6f4 sums the products in fp32; every partial sum is an
// integer multiple of 2^-18 far below 2^24 units, so S = S_int * 2^-18 holds
// exactly -- the integers an s32 accumulation gives, already in fp32 for the
// softmax.
//
// P V with the V dequantisation folded in: O += sum_k u_k * (v_k,c * s_c)
// for the block's per-channel V scale s_c.  The fp32 scale is split into two
// parts of 8 significant bits each, s_hi = s with its low 16 mantissa bits
// cleared and s_lo = (s - s_hi) likewise (s - s_hi - s_lo < 2^-14 s); a code
// (3 bits of magnitude) times either part has at most 11 significant bits, so
// the V' tiles v * s_hi and v * s_lo are exact fp16 values while they are
// normal fp16 numbers (|v * s_hi| <= 7 s <= the block's max |V|, so never
// above the fp16 range; a very small scale makes v * s_lo subnormal, rounded
// to within 2^-25 absolute), and the P codes u in 0..15 are exact fp16 too.  tcgen05.mma
// kind::f16 then forms s_hi * sum_k u v and s_lo * sum_k u v exactly (each
// block sum is an integer below 2^13 times one part: at most 21 significant
// bits) and adds them to O in TMEM.  So O accumulates on the tensor core
// across blocks, and the CUDA cores only rescale it (in TMEM) when a row's
// running max moves.
//
// The packed K / V nibbles are widened once per call by widen_kv_kernel into
// the exact shared-memory images of the operand tiles (K: e4m3, K-major,
// swizzled; V'_hi, V'_lo: fp16, channel rows of 64 keys, 128-byte swizzle), so
// the main loop moves them with plain TMA bulk copies.
//
// One CTA = two 128-row query tiles of one head (256 rows), 384 threads:
//   warp 0      TMA producer: the K, V'_hi and V'_lo tiles of each 64-key
//               block -> a 4-stage shared-memory ring (cp.async.bulk);
//   warps 1, 2  MMA issuers of tile 0 and tile 1 (warp-uniform loops, one
//               elected lane issues); warp 1 also owns the TMEM allocation;
//   warp 3      idle;
//   warps 4-7   query tile 0, warps 8-11 query tile 1 (thread = row = TMEM lane):
//               running max, P codes (fp16) and their row sum, O rescale,
//               epilogue out = O / l.
// Per 64-key block j and tile t the MMA warp issues S_t(j) = Q_t K_j^T
// (128 x 64 into the tile's one S buffer in TMEM, which the softmax warps
// release as soon as S is in their registers, so S_t(j+1) is computed while
// they work on block j) and, once tile t has written its P codes into TMEM,
// O_t += P_t V'_hi + P_t V'_lo (128 x D, O accumulated in TMEM).
#pragma once
#include <climits>
#include <cstdint>
#include <cuda_fp16.h>

#include "sm100.cuh"

namespace rota {

struct Int4Params {
  const uint8_t* q_codes;
  const uint8_t* k_codes;
  const float* q_scale;
  const float* k_scale;
  const uint8_t* v_codes;
  const float* v_scale;
  const uint8_t* work;  // widened K / V^T tiles + 512 * v_scale per (head, block)
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

constexpr int kInt4Threads = 384;
constexpr int kRowsPerCta = 2 * kBM;
constexpr int kOps = 4;   // operand stages
constexpr int kProducerRegs = 40;
constexpr int kConsumerRegs = 232;
// Register split: kProducerRegs * 128 + kConsumerRegs * 256 equals the launch
// allocation 384 * kLaunchRegs; the host refuses to launch a build whose
// register count differs (setmaxnreg.inc would otherwise wait forever).
constexpr int kLaunchRegs = (kProducerRegs * 128 + kConsumerRegs * 256) / 384;
static_assert(kLaunchRegs * 384 == kProducerRegs * 128 + kConsumerRegs * 256, "register split");

template <int D>
struct Int4Smem {
  static constexpr int ROWB = D;              // bytes per e4m3 Q / K row
  static constexpr uint32_t LAYOUT_QK = D == 128 ? 2u : 4u;  // 128B / 64B swizzle
  static constexpr uint32_t SBO_QK = 8 * D;
  static constexpr int K_BYTES = kBN * D;
  static constexpr int VP_BYTES = D * kBN * 2;                    // one V' part: D rows x 64 keys fp16
  static constexpr int OP_BYTES = K_BYTES + 2 * VP_BYTES;
  static constexpr int IMG_BYTES = OP_BYTES;                      // one block in int4_work
  static constexpr int OFF_OP = 0;                                // kOps stages
  static constexpr int OFF_TAU = OFF_OP + kOps * OP_BYTES;
  static constexpr int OFF_BAR = OFF_TAU + 64;
  // barriers: op_full[kOps] op_empty[kOps] s_full[2 tiles] s_empty[2] p_full[2]
  //           p_empty[2] q_full mma_done[2]
  static constexpr int NBAR = 2 * kOps + 2 + 2 + 2 + 2 + 1 + 2;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;
  static constexpr int BYTES = OFF_ABORT + 4;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  // S of tile t at column t * 64; the e4m3 Q rows of tile t (A operand of the
  // score MMA) at 128 + t * D / 4; the fp16 P codes of tile t (A operand of
  // P V, 64 keys = 32 columns) at 192 + 32 t; O of tile t at 256 + t * D
  static constexpr uint32_t T_S = 0, T_Q = 2 * kBN, T_P = 192, T_O = 4 * kBN;
  static_assert(T_Q + 2 * (D / 4) <= T_P && T_P + 2 * (kBN / 2) <= T_O && T_O + 2 * D <= TMEM_COLS,
                "TMEM budget");
  static_assert(IMG_BYTES % 16 == 0 && K_BYTES % 16 == 0 && VP_BYTES % 16 == 0, "bulk copy sizes");
  static_assert(OFF_OP % 1024 == 0 && OP_BYTES % 1024 == 0 && K_BYTES % 1024 == 0 && VP_BYTES % 1024 == 0,
                "swizzle atom alignment");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

// Range-optimised P code u = rne(15 * 2^d) in exact arithmetic (d <= ~0).
// The estimate rne(15 e), e = ex2.approx(d), is within ~4e-6 of the exact
// 15 * 2^d before rounding (ex2.approx: ~2 ulp); only when 15 e lies within
// 1e-5 of a half-integer is the decision taken by the exact threshold table
// tau.  (The band is validated exhaustively near every threshold by the tests.)  The main loop runs
// the same arithmetic (fast estimate for every key, this function for the keys
// it flags), so this is also the function the exhaustive test checks.
constexpr float kMagic = 12582912.f;   // 1.5 * 2^23: x + kMagic rounds x to an integer
constexpr float kNear = 0.5f - 1e-5f;  // |15 e - rne(15 e)| above this: decide exactly
__device__ __forceinline__ float pcode_f(float d, const float* tau) {
  const float e = ex2_approx(d);
  float r = __fadd_rn(__fmaf_rn(e, 15.f, kMagic), -kMagic);  // rne(15 e)
  const float fr = __fmaf_rn(e, 15.f, -r);
  if (fabsf(fr) > kNear) {
    int j = fr > 0.f ? static_cast<int>(r) + 1 : static_cast<int>(r);
    j = max(1, min(15, j));
    r = static_cast<float>(d >= tau[j] ? j : j - 1);
  }
  return r;
}

__device__ __forceinline__ uint32_t pcode(float d, const float* tau) {
  return static_cast<uint32_t>(pcode_f(d, tau));
}

// Four P codes (exact integers 0..15 in fp32) -> two words of fp16, u0 lowest.
__device__ __forceinline__ uint2 pack_f16x4(float u0, float u1, float u2, float u3) {
  const __half2 a = __floats2half2_rn(u0, u1), b = __floats2half2_rn(u2, u3);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
}

__device__ __forceinline__ void setmaxnreg_producer() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 40;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_consumer() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 232;" ::: "memory");
}
static_assert(kProducerRegs == 40 && kConsumerRegs == 232, "setmaxnreg immediates");

template <int D, bool DUMP>
__global__ void __launch_bounds__(kInt4Threads, 1) attn_int4_kernel(const __grid_constant__ Int4Params p) {
  using L = Int4Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* op_full = bars;
  uint64_t* op_empty = bars + kOps;
  // per tile, once per block (phase j & 1)
  uint64_t* s_full = bars + 2 * kOps;
  uint64_t* s_empty = bars + 2 * kOps + 2;
  uint64_t* p_full = bars + 2 * kOps + 4;
  // p_empty[t]: tile t's P V of the block has completed -- the P columns may
  // be rewritten, and O holds every block up to that one
  uint64_t* p_empty = bars + 2 * kOps + 6;
  uint64_t* q_full = bars + 2 * kOps + 8;
  uint64_t* mma_done = bars + 2 * kOps + 9;   // [2], one per MMA warp
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + L::OFF_ABORT);
  float* sTau = reinterpret_cast<float*>(smem + L::OFF_TAU);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = p.heads[blockIdx.y];
  const int b = blockIdx.z;
  const size_t head = (size_t)b * p.H + h;
  const int npad = p.nblk * kBN;
  const int nkb = p.nblk;
  const uint64_t lim = p.timeout_ns;

  if (tid < 16) sTau[tid] = p.tau[tid];
  if (tid == 0) {
    for (int i = 0; i < kOps; ++i) {
      mbar_init(&op_full[i], 1);
      mbar_init(&op_empty[i], 2);   // the last P V of the block, one commit per tile
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_empty[t], 4);
      mbar_init(&p_full[t], 4);
      mbar_init(&p_empty[t], 1);
    }
    mbar_init(q_full, 8);
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
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

  if (warp < 4) {
    // ===================================================== producer warpgroup
    setmaxnreg_producer();
    if (warp == 0) {
      // ---- TMA producer: widened tiles of block j -> operand stage j % kOps
      // (warp-uniform loop, one elected lane issues the copies) ----
      int issued = 0;
      for (int j = 0; j < nkb; ++j) {
        const int op = j % kOps;
        if (!warp_wait(&op_empty[op], ((j / kOps) & 1) ^ 1, lim)) {
          if (lane == 0) *sAbort = 1;
          break;
        }
        if (warp_flag(sAbort)) break;
        uint8_t* dst = smem + L::OFF_OP + op * L::OP_BYTES;
        const uint8_t* src = p.work + (head * p.nblk + j) * (size_t)L::IMG_BYTES;
        if (elect_one()) {
          mbar_arrive_expect_tx(&op_full[op], L::OP_BYTES);
          bulk_g2s(dst, src, L::K_BYTES, &op_full[op]);
          bulk_g2s(dst + L::K_BYTES, src + L::K_BYTES, L::VP_BYTES, &op_full[op]);
          bulk_g2s(dst + L::K_BYTES + L::VP_BYTES, src + L::K_BYTES + L::VP_BYTES, L::VP_BYTES, &op_full[op]);
        }
        __syncwarp();
        issued = j + 1;
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int j = (issued > kOps ? issued - kOps : 0); j < issued; ++j)
        warp_wait(&op_full[j % kOps], (j / kOps) & 1, lim);
    } else if (warp <= 2) {
      // ---- MMA issuers: warp 1 + t issues tile t's MMAs, so the two tiles'
      // S -> softmax -> P V chains do not wait on each other.  The whole warp
      // runs the loop (addresses and waits warp-uniform); one elected lane
      // issues each MMA and commit ----
      const int t = warp - 1;
      constexpr uint32_t ID_S = idesc(1, 0, 0, kBM, kBN);   // e4m3 x e4m3 -> f32, 128 x 64
      constexpr uint32_t ID_PV = idesc(1, 0, 0, kBM, D);    // f16 x f16 -> f32, 128 x D
      // descriptors: constant high words, low words stepped by 32 bytes (2 units) per K step
      const uint32_t hi_qk = sdesc_hi(L::SBO_QK, L::LAYOUT_QK), hi_128 = sdesc_hi(1024, 2);
      const uint32_t lo_op = sdesc_lo(smem_u32(smem + L::OFF_OP));  // + op * OP_BYTES / 16
      const uint32_t aq = tmem + L::T_Q + t * (D / 4);   // Q of tile t: 32 e4m3 elements = 8 columns per K step
      const uint32_t d_s = tmem + L::T_S + t * kBN, d_o = tmem + L::T_O + t * D;
      bool ok = warp_wait(q_full, 0, lim);
      auto issue_s = [&](int j) -> bool {
        const int op = j % kOps;
        if (!warp_wait(&s_empty[t], (j & 1) ^ 1, lim)) return false;
        tc_fence_after();
        if (p.inject_skip && j == 0 && t == 0) return true;  // fault injection: never committed
        const uint32_t lk = lo_op + op * (L::OP_BYTES >> 4);
        if (elect_one()) {
          mma_f8f6f4_ts<0>(d_s, aq, lk, hi_qk, ID_S);
#pragma unroll
          for (int k = 1; k < D / 32; ++k) mma_f8f6f4_ts<1>(d_s, aq + 8 * k, lk + 2 * k, hi_qk, ID_S);
          mma_commit(&s_full[t]);
        }
        __syncwarp();
        return true;
      };
      const uint32_t ap = tmem + L::T_P + t * (kBN / 2);   // P of tile t: 16 keys = 8 columns per K step
      auto issue_pv = [&](int j) -> bool {
        const int op = j % kOps;
        const uint32_t lvh = lo_op + op * (L::OP_BYTES >> 4) + (L::K_BYTES >> 4);
        const uint32_t lvl = lvh + (L::VP_BYTES >> 4);
        if (!warp_wait(&p_full[t], j & 1, lim)) return false;
        tc_fence_after();
        if (elect_one()) {
          if (j == 0) mma_f16_ts<0>(d_o, ap, lvh, hi_128, ID_PV);
          else mma_f16_ts<1>(d_o, ap, lvh, hi_128, ID_PV);
          mma_f16_ts<1>(d_o, ap, lvl, hi_128, ID_PV);
#pragma unroll
          for (int k = 1; k < kBN / 16; ++k) {
            mma_f16_ts<1>(d_o, ap + 8 * k, lvh + 2 * k, hi_128, ID_PV);
            mma_f16_ts<1>(d_o, ap + 8 * k, lvl + 2 * k, hi_128, ID_PV);
          }
          mma_commit(&p_empty[t]);
          mma_commit(&op_empty[op]);   // one of the stage's two arrivals (one per tile)
        }
        __syncwarp();
        return true;
      };
      for (int j = 0; ok && j < nkb; ++j) {
        if (!warp_wait(&op_full[j % kOps], (j / kOps) & 1, lim)) { ok = false; break; }
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
    }
  } else {
    // ===================================================== query-tile warpgroups
    setmaxnreg_consumer();
    const int t = (warp - 4) >> 2;            // tile 0 or 1
    const int r = tid & 127;                  // row within the tile = TMEM lane
    const int row = blockIdx.x * kRowsPerCta + t * kBM + r;
    const uint32_t t_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + L::T_S + t * kBN + t_lane;
    const uint32_t tO = tmem + L::T_O + t * D + t_lane;
    const uint32_t tP = tmem + L::T_P + t * (kBN / 2) + t_lane;

    // own Q row: packed codes -> e4m3 subnormals, K-contiguous in this lane's
    // TMEM columns (the A operand of the score MMA)
    {
      const uint8_t* qsrc = p.q_codes + (head * npad + (size_t)row) * (D / 2);
      uint32_t qw[D / 4];
#pragma unroll
      for (int cg = 0; cg < D / 32; ++cg) {
        uint4 w = make_uint4(0, 0, 0, 0);
        if (row < npad) w = __ldg(reinterpret_cast<const uint4*>(qsrc + cg * 16));
        codes8_to_e4m3(w.x, qw[8 * cg + 0], qw[8 * cg + 1]);
        codes8_to_e4m3(w.y, qw[8 * cg + 2], qw[8 * cg + 3]);
        codes8_to_e4m3(w.z, qw[8 * cg + 4], qw[8 * cg + 5]);
        codes8_to_e4m3(w.w, qw[8 * cg + 6], qw[8 * cg + 7]);
      }
      tmem_st_n<D / 4>(tmem + L::T_Q + t * (D / 4) + t_lane, qw);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    }
    const float sq = row < npad ? __ldg(p.q_scale + head * p.nblk + row / kBN) : 0.f;
    const float* ksc = p.k_scale + head * p.nblk;

    float m = -INFINITY, l = 0.f;
    bool aborted = false;
    float sk_next = __ldg(ksc);
    for (int j = 0; j < nkb; ++j) {
      const float sk = sk_next;
      if (j + 1 < nkb) sk_next = __ldg(ksc + j + 1);
      if (!warp_wait(&s_full[t], j & 1, lim)) { aborted = true; break; }
      tc_fence_after();

      const int nvalid = min(kBN, p.N - j * kBN);
      const float c = __fmul_rn(__fmul_rn(sq, sk), p.kappa);
      const float c18 = c * 262144.f;  // S here is S_int * 2^-18; c * 2^18 is exact
      float alpha, lsum, near;
      uint2 pw[kBN / 4];
      uint32_t sr[kBN];
      {
        uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        tmem_ld32(tS, s0);
        tmem_ld32(tS + 32, s1);
        tmem_wait_dep2(s0, s1);
        // S is in registers: the MMA may compute S(j+1) into this buffer now
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[t]);
        // ---- running max over the block's valid keys ----
        float smax;
        if (nvalid == kBN) {
          float x0 = -INFINITY, x1 = -INFINITY, x2 = -INFINITY, x3 = -INFINITY;
#pragma unroll
          for (int k = 0; k < kBN; k += 8) {
            x0 = max3(x0, __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]));
            x1 = max3(x1, __uint_as_float(sr[k + 2]), __uint_as_float(sr[k + 3]));
            x2 = max3(x2, __uint_as_float(sr[k + 4]), __uint_as_float(sr[k + 5]));
            x3 = max3(x3, __uint_as_float(sr[k + 6]), __uint_as_float(sr[k + 7]));
          }
          smax = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        } else {
          smax = -INFINITY;
#pragma unroll
          for (int k = 0; k < kBN; ++k)
            if (k < nvalid) smax = fmaxf(smax, __uint_as_float(sr[k]));
        }
        const float m_new = fmaxf(m, __fmul_rn(smax, c18));
        alpha = ex2_approx(m - m_new);  // 0 on the first block (m = -inf)
        m = m_new;

        // ---- P codes u = rne(15 * 2^(S c - m)): branch-free estimate for all 64 keys ----
        float n0 = 0.f, n1 = 0.f, ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int k = 0; k < kBN; k += 4) {
          float d0, d1, d2, d3, r0, r1, r2, r3, f0, f1, f2, f3;
          fma2(d0, d1, __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]), c18, c18, -m, -m);
          fma2(d2, d3, __uint_as_float(sr[k + 2]), __uint_as_float(sr[k + 3]), c18, c18, -m, -m);
          const float e0 = ex2_approx(d0), e1 = ex2_approx(d1), e2 = ex2_approx(d2), e3 = ex2_approx(d3);
          fma2(f0, f1, e0, e1, 15.f, 15.f, kMagic, kMagic);     // kMagic + rne(15 e)
          fma2(f2, f3, e2, e3, 15.f, 15.f, kMagic, kMagic);
          add2(r0, r1, f0, f1, -kMagic, -kMagic);                // rne(15 e), exact
          add2(r2, r3, f2, f3, -kMagic, -kMagic);
          fma2(f0, f1, e0, e1, 15.f, 15.f, -r0, -r1);            // 15 e - rne(15 e)
          fma2(f2, f3, e2, e3, 15.f, 15.f, -r2, -r3);
          n0 = max3(n0, fabsf(f0), fabsf(f1));
          n1 = max3(n1, fabsf(f2), fabsf(f3));
          add2(ls0, ls1, ls0, ls1, r0, r1);                      // row sum of the codes (exact integers)
          add2(ls0, ls1, ls0, ls1, r2, r3);
          pw[k / 4] = pack_f16x4(r0, r1, r2, r3);
        }
        near = fmaxf(n0, n1);
        lsum = ls0 + ls1;
      }
      // keys past N in the last block take code 0; the row sum is taken again
      if (nvalid < kBN) {
        lsum = 0.f;
#pragma unroll
        for (int w = 0; w < kBN / 4; ++w) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int sh = 16 * (e & 1);
            uint32_t word = (e & 2) ? pw[w].y : pw[w].x;
            if (4 * w + e >= nvalid) word &= ~(0xFFFFu << sh);
            lsum += __half2float(__ushort_as_half(static_cast<unsigned short>((word >> sh) & 0xFFFFu)));
            if (e & 2) pw[w].y = word;
            else pw[w].x = word;
          }
        }
      }
      if (DUMP) {
#pragma unroll
        for (int k = 0; k < kBN; ++k)
          if (k < nvalid && row >= p.dbg_r0 && row < p.dbg_r0 + p.dbg_nr)
            p.s_dump[(size_t)(row - p.dbg_r0) * p.N + (size_t)j * kBN + k] =
                static_cast<int32_t>(__uint_as_float(sr[k]) * 262144.f);
      }

      // the previous block's P V has completed: its P columns are free and O
      // holds every block before this one
      if (j > 0) {
        if (!warp_wait(&p_empty[t], (j - 1) & 1, lim)) { aborted = true; break; }
        tc_fence_after();
      }
      // ---- the running max moved on some row of the warp: rescale O ----
      if (j > 0 && !__all_sync(0xffffffffu, alpha == 1.f)) {
#pragma unroll 1
        for (int cb = 0; cb < D / 32; ++cb) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * cb, o);
          tmem_wait_dep(o);
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__fmul_rn(__uint_as_float(o[k]), alpha));
          tmem_st32(tO + 32 * cb, o);
        }
      }
      // P codes -> this lane's TMEM columns (keys 2c, 2c + 1 in column c)
      {
        uint32_t pr[kBN / 2];
#pragma unroll
        for (int w = 0; w < kBN / 4; ++w) {
          pr[2 * w] = pw[w].x;
          pr[2 * w + 1] = pw[w].y;
        }
        tmem_st32(tP, pr);
      }
      // ---- exact decisions (rare): estimates within 1e-5 of a half-integer ----
      // Recompute which keys were near a tie (same arithmetic as above), then
      // visit only the columns some lane flagged: each is read back from TMEM,
      // the flagged lanes put in the exact code, and it is stored again.
      if (__any_sync(0xffffffffu, near > kNear)) {
        tmem_st_wait();
        uint32_t mlo = 0, mhi = 0;
#pragma unroll
        for (int k = 0; k < kBN; ++k) {
          const float d = __fmaf_rn(__uint_as_float(sr[k]), c18, -m);
          const float e = ex2_approx(d);
          const float rr = __fadd_rn(__fmaf_rn(e, 15.f, kMagic), -kMagic);
          const bool hit = fabsf(__fmaf_rn(e, 15.f, -rr)) > kNear && k < nvalid;
          if (k < 32) mlo |= static_cast<uint32_t>(hit) << k;
          else mhi |= static_cast<uint32_t>(hit) << (k - 32);
        }
        uint32_t wlo = __reduce_or_sync(0xffffffffu, mlo), whi = __reduce_or_sync(0xffffffffu, mhi);
        while (wlo | whi) {
          const int k = wlo ? __ffs(wlo) - 1 : 32 + __ffs(whi) - 1;
          if (k < 32) wlo &= wlo - 1; else whi &= whi - 1;
          uint32_t sbits = 0;
#pragma unroll
          for (int kk = 0; kk < kBN; ++kk) sbits = kk == k ? sr[kk] : sbits;
          uint32_t word = tmem_ld1(tP + (k >> 1));
          tmem_wait_dep1(word);
          const bool mine = (k < 32 ? (mlo >> k) : (mhi >> (k - 32))) & 1u;
          if (mine) {
            const float d = __fmaf_rn(__uint_as_float(sbits), c18, -m);
            const float e = ex2_approx(d);
            const float rr = __fadd_rn(__fmaf_rn(e, 15.f, kMagic), -kMagic);
            const float u = pcode_f(d, sTau);
            lsum += u - rr;
            const int sh = 16 * (k & 1);
            word = (word & ~(0xFFFFu << sh)) | (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(u))) << sh);
          }
          tmem_st1(tP + (k >> 1), word);
          tmem_st_wait();
        }
      }
      l = __fmaf_rn(l, alpha, lsum);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
      if (DUMP) {
        // P codes as the MMA will read them, from the fp16 values in TMEM
        const size_t base = (size_t)(row - p.dbg_r0) * p.N + (size_t)j * kBN;
        for (int c2 = 0; c2 < kBN / 2; ++c2) {
          uint32_t word = tmem_ld1(tP + c2);
          tmem_wait_dep1(word);
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (2 * c2 + e < nvalid && row >= p.dbg_r0 && row < p.dbg_r0 + p.dbg_nr)
              p.p_dump[base + 2 * c2 + e] = static_cast<uint8_t>(
                  __half2float(__ushort_as_half(static_cast<unsigned short>((word >> (16 * e)) & 0xFFFFu))));
        }
      }
      if (warp_flag(sAbort)) { aborted = true; break; }
    }
    // ---- epilogue: out = O / l once the last P V has landed ----
    if (!aborted && !warp_wait(&p_empty[t], (nkb - 1) & 1, lim)) aborted = true;
    if (aborted) {
      *sAbort = 1;
    } else {
      tc_fence_after();
      const float inv_l = 1.f / l;
      float* dst = p.out + (head * p.N + (size_t)row) * D;
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

// Widens the packed K / V codes of one (head, 64-key block) into the exact
// shared-memory images of the attention kernel's operand tiles: K as 64 rows
// x D e4m3 subnormals (K-major, 128B / 64B swizzle); V'_hi and V'_lo as D
// channel rows x 64 keys of fp16 v * s_hi and v * s_lo (128B swizzle), with
// s_hi, s_lo the two 8-significant-bit parts of the block's channel scale.
template <int D>
__global__ void __launch_bounds__(256) widen_kv_kernel(const __grid_constant__ Int4Params p, uint8_t* work) {
  using L = Int4Smem<D>;
  const int j = blockIdx.x, h = p.heads[blockIdx.y], b = blockIdx.z;
  const size_t head = (size_t)b * p.H + h;
  const int npad = p.nblk * kBN;
  uint8_t* img = work + (head * p.nblk + j) * (size_t)L::IMG_BYTES;
  const uint8_t* kp = p.k_codes + (head * npad + (size_t)j * kBN) * (D / 2);
  for (int i = threadIdx.x; i < kBN * D / 32; i += blockDim.x) {
    const int rr = i / (D / 32), cg = i % (D / 32);
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(kp + 16 * i));
    uint32_t o[8];
    codes8_to_e4m3(w.x, o[0], o[1]);
    codes8_to_e4m3(w.y, o[2], o[3]);
    codes8_to_e4m3(w.z, o[4], o[5]);
    codes8_to_e4m3(w.w, o[6], o[7]);
    *reinterpret_cast<uint4*>(img + swz<L::ROWB>(rr, cg * 32)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(img + swz<L::ROWB>(rr, cg * 32 + 16)) = make_uint4(o[4], o[5], o[6], o[7]);
  }
  // V: channel c, keys 8q..8q+7 (one packed word) -> 16 bytes of each part
  const uint32_t* vp = reinterpret_cast<const uint32_t*>(p.v_codes + (head * p.nblk + j) * (size_t)D * 32);
  const float* vs = p.v_scale + (head * p.nblk + j) * D;
  uint8_t* vhi = img + L::K_BYTES;
  uint8_t* vlo = vhi + L::VP_BYTES;
  for (int i = threadIdx.x; i < D * 8; i += blockDim.x) {
    const int c = i >> 3, q = i & 7;
    const float sc = __ldg(vs + c);
    const float s_hi = __uint_as_float(__float_as_uint(sc) & 0xFFFF0000u);
    const float s_lo = __uint_as_float(__float_as_uint(__fsub_rn(sc, s_hi)) & 0xFFFF0000u);
    const uint32_t w = __ldg(vp + c * 8 + q);   // keys 8q .. 8q+7: byte e = key e (low) | key e+4 (high)
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      // keys 8q + e and 8q + e + 1
      float v[2];
#pragma unroll
      for (int z = 0; z < 2; ++z) {
        const int key = e + z;  // 0..7 within the word
        const uint32_t nib = (key < 4 ? (w >> (8 * key)) : (w >> (8 * (key - 4) + 4))) & 15u;
        const float mag = static_cast<float>(nib & 7u);
        v[z] = (nib & 8u) ? -mag : mag;
      }
      const __half2 a = __floats2half2_rn(v[0] * s_hi, v[1] * s_hi);
      const __half2 bb = __floats2half2_rn(v[0] * s_lo, v[1] * s_lo);
      hw[e / 2] = *reinterpret_cast<const uint32_t*>(&a);
      lw[e / 2] = *reinterpret_cast<const uint32_t*>(&bb);
    }
    *reinterpret_cast<uint4*>(vhi + swz<128>(c, 16 * q)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(vlo + swz<128>(c, 16 * q)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
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
