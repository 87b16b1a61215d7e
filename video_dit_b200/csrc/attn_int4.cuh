// attn_int4.cuh -- INT4 FlashAttention forward with range-optimised P codes.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: a mixed-precision INT4
// FlashAttention in which P = exp(QK - max(QK)) >= 0 is quantised with a
// fixed scale and zero-point so that all 16 unsigned 4-bit levels are used
// ("Range-optimized P Quantization").
//
// Exact integer contractions on the 8-bit tensor-core path.  A code v in
// [-7, 7] is widened to the e4m3 subnormal v * 2^-9 (exact), a P code u in
// 0..15 to the e4m3 normal u (exact), and tcgen05.mma kind::f8f6f4 sums the
// products in fp32: every partial sum is an integer multiple of 2^-18 (S) or
// 2^-9 (P V) far below 2^24 units, so S = S_int * 2^-18 and acc = acc_int *
// 2^-9 hold exactly -- the same integers an s32 accumulation gives, already
// in fp32 for the softmax and the V scales.
//
// The packed K / V nibbles are widened once per call by widen_kv_kernel into
// the exact shared-memory images of the operand tiles (swizzled K-major e4m3),
// so the main loop moves them with plain TMA bulk copies; widening inside the
// main loop would repeat the same work in every CTA of a head.
//
// One CTA = two 128-row query tiles of one head (256 rows), 384 threads:
//   warp 0      TMA producer: widened K / V^T tiles and V scales of each 64-key
//               block -> a 4-stage shared-memory ring (cp.async.bulk);
//   warp 1      TMEM owner and MMA issuer (one thread);
//   warps 2-3   fill the constant rows once, then idle;
//   warps 4-7   query tile 0, warps 8-11 query tile 1 (thread = row = TMEM lane):
//               running max, P codes, O update, epilogue.
// Per 64-key block j and tile t the MMA warp issues S_t = Q_t K_j^T (128 x 64)
// and, once tile t has written its P codes, PV_t = P_t [V_j^T; 1] (128 x (D+16));
// the 16 extra columns of ones return the row sum of the P codes.  The two
// tiles alternate, so the tensor core works on one while the other's CUDA
// cores run the softmax; each tile's S buffer is released as soon as its
// warps have loaded it, so S_t(j+1) overlaps the softmax of block j.
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
  static constexpr int NPV = D + 16;          // P V columns: D channels + 16 ones (row sum)
  static constexpr int ROWB = D;              // bytes per e4m3 Q / K row
  static constexpr uint32_t LAYOUT_QK = D == 128 ? 2u : 4u;  // 128B / 64B swizzle
  static constexpr uint32_t SBO_QK = 8 * D;
  static constexpr int Q_BYTES = kBM * D;
  static constexpr int K_BYTES = kBN * D;
  static constexpr int VIMG_BYTES = D * kBN;                      // widened V^T rows 0..D-1
  static constexpr int V_BYTES = ((NPV * kBN + 1023) / 1024) * 1024;
  static constexpr int OP_BYTES = K_BYTES + V_BYTES;
  static constexpr int IMG_BYTES = K_BYTES + VIMG_BYTES + D * 4;  // one block in int4_work
  static constexpr int P_BYTES = kBM * kBN;
  static constexpr int OFF_Q = 0;                              // 2 tiles
  static constexpr int OFF_OP = OFF_Q + 2 * Q_BYTES;           // kOps stages
  static constexpr int OFF_P = OFF_OP + kOps * OP_BYTES;       // 2 tiles x 2 buffers
  static constexpr int OFF_SV = OFF_P + 4 * P_BYTES;           // kOps x D floats: 512 * v_scale
  static constexpr int OFF_TAU = OFF_SV + kOps * D * 4;
  static constexpr int OFF_BAR = OFF_TAU + 64;
  // barriers: op_full[4] op_empty[4] s_full[2] s_empty[2] pv_full[2] pv_empty[2]
  //           q_full mma_done p_full[2 tiles][2 buffers]
  static constexpr int NBAR = 4 + 4 + 2 + 2 + 2 + 2 + 1 + 1 + 4;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;
  static constexpr int BYTES = OFF_ABORT + 4;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S0 = 0, T_S1 = kBN, T_PV0 = 2 * kBN, T_PV1 = 2 * kBN + NPV;
  static_assert(T_PV1 + NPV <= TMEM_COLS, "TMEM budget");
  static_assert(IMG_BYTES % 16 == 0 && K_BYTES % 16 == 0 && VIMG_BYTES % 16 == 0, "bulk copy sizes");
  static_assert(OFF_OP % 1024 == 0 && OP_BYTES % 1024 == 0 && K_BYTES % 1024 == 0 && OFF_P % 1024 == 0,
                "swizzle atom alignment");
  static_assert(OFF_SV % 16 == 0 && OFF_BAR % 8 == 0, "alignment");
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

// Four P codes (exact integers 0..15 in fp32) -> four e4m3 bytes, u0 lowest.
__device__ __forceinline__ uint32_t pack_e4m3x4(float u0, float u1, float u2, float u3) {
  uint32_t w;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(w)
      : "f"(u0), "f"(u1), "f"(u2), "f"(u3));
  return w;
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
  uint64_t* op_empty = bars + 4;
  uint64_t* s_full = bars + 8;
  uint64_t* s_empty = bars + 10;
  uint64_t* pv_full = bars + 12;
  uint64_t* pv_empty = bars + 14;
  uint64_t* q_full = bars + 16;
  uint64_t* mma_done = bars + 17;
  // One barrier per P buffer (tile t, block parity): tile t may write P(j+1)
  // before the MMA warp has waited for P(j), so a single barrier per tile
  // could complete two phases ahead of its waiter.
  uint64_t* p_full = bars + 18;  // p_full[2 * t + (j & 1)], phase (j >> 1) & 1
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + L::OFF_ABORT);
  float* sTau = reinterpret_cast<float*>(smem + L::OFF_TAU);
  float* sSv = reinterpret_cast<float*>(smem + L::OFF_SV);

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
      mbar_init(&op_empty[i], 1 + 8);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_empty[t], 4);
      mbar_init(&p_full[2 * t], 4);
      mbar_init(&p_full[2 * t + 1], 4);
      mbar_init(&pv_full[t], 1);
      mbar_init(&pv_empty[t], 4);
    }
    mbar_init(q_full, 8 + 2);
    mbar_init(mma_done, 1);
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
      if (lane == 0) {
        // ---- TMA producer: widened tiles of block j -> operand stage j % kOps ----
        int issued = 0;
        for (int j = 0; j < nkb; ++j) {
          const int op = j % kOps;
          if (!mbar_wait(&op_empty[op], ((j / kOps) & 1) ^ 1, lim)) { *sAbort = 1; break; }
          if (*sAbort) break;
          uint8_t* kt = smem + L::OFF_OP + op * L::OP_BYTES;
          const uint8_t* src = p.work + (head * p.nblk + j) * (size_t)L::IMG_BYTES;
          mbar_arrive_expect_tx(&op_full[op], L::K_BYTES + L::VIMG_BYTES + D * 4);
          bulk_g2s(kt, src, L::K_BYTES, &op_full[op]);
          bulk_g2s(kt + L::K_BYTES, src + L::K_BYTES, L::VIMG_BYTES, &op_full[op]);
          bulk_g2s(sSv + op * D, src + L::K_BYTES + L::VIMG_BYTES, D * 4, &op_full[op]);
          issued = j + 1;
        }
        // drain: every issued copy has landed before the CTA may exit
        for (int j = (issued > kOps ? issued - kOps : 0); j < issued; ++j)
          mbar_wait(&op_full[j % kOps], (j / kOps) & 1, lim);
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---- MMA issuer ----
        constexpr uint32_t ID_S = idesc(1, 0, 0, kBM, kBN);      // e4m3 x e4m3 -> f32, 128 x 64
        constexpr uint32_t ID_PV = idesc(1, 0, 0, kBM, L::NPV);  // 128 x (D + 16)
        // descriptors: constant high words, low words stepped by 32 bytes (2 units) per K step
        const uint32_t hi_qk = sdesc_hi(L::SBO_QK, L::LAYOUT_QK), hi_64 = sdesc_hi(512, 4);
        const uint32_t lo_q0 = sdesc_lo(smem_u32(smem + L::OFF_Q)), lo_q1 = lo_q0 + (L::Q_BYTES >> 4);
        const uint32_t lo_p = sdesc_lo(smem_u32(smem + L::OFF_P));   // + (2t + (j & 1)) * P_BYTES / 16
        const uint32_t lo_op = sdesc_lo(smem_u32(smem + L::OFF_OP));  // + op * OP_BYTES / 16
        bool ok = mbar_wait(q_full, 0, lim);
        auto issue_s = [&](int j, int t) -> bool {
          const int op = j % kOps;
          if (!mbar_wait(&s_empty[t], (j & 1) ^ 1, lim)) return false;
          tc_fence_after();
          if (p.inject_skip && j == 0 && t == 0) return true;  // fault injection: never committed
          const uint32_t lk = lo_op + op * (L::OP_BYTES >> 4);
          const uint32_t lq = t ? lo_q1 : lo_q0;
          const uint32_t d = tmem + (t ? L::T_S1 : L::T_S0);
          mma_f8f6f4_lh<0>(d, lq, hi_qk, lk, hi_qk, ID_S);
#pragma unroll
          for (int k = 1; k < D / 32; ++k) mma_f8f6f4_lh<1>(d, lq + 2 * k, hi_qk, lk + 2 * k, hi_qk, ID_S);
          mma_commit(&s_full[t]);
          return true;
        };
        auto issue_pv = [&](int j) -> bool {
          const int op = j % kOps;
          const uint32_t lv = lo_op + op * (L::OP_BYTES >> 4) + (L::K_BYTES >> 4);
          for (int t = 0; t < 2; ++t) {
            if (!mbar_wait(&p_full[2 * t + (j & 1)], (j >> 1) & 1, lim)) return false;
            if (!mbar_wait(&pv_empty[t], (j & 1) ^ 1, lim)) return false;
            tc_fence_after();
            const uint32_t lp = lo_p + (2 * t + (j & 1)) * (L::P_BYTES >> 4);
            const uint32_t d = tmem + (t ? L::T_PV1 : L::T_PV0);
            mma_f8f6f4_lh<0>(d, lp, hi_64, lv, hi_64, ID_PV);
#pragma unroll
            for (int k = 1; k < kBN / 32; ++k) mma_f8f6f4_lh<1>(d, lp + 2 * k, hi_64, lv + 2 * k, hi_64, ID_PV);
            mma_commit(&pv_full[t]);
          }
          mma_commit(&op_empty[op]);
          return true;
        };
        for (int j = 0; ok && j < nkb; ++j) {
          if (!mbar_wait(&op_full[j % kOps], (j / kOps) & 1, lim)) { ok = false; break; }
          tc_fence_after();
          if (!issue_s(j, 0) || !issue_s(j, 1)) { ok = false; break; }
          if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
          if (*sAbort) { ok = false; break; }
        }
        if (ok) ok = issue_pv(nkb - 1);
        if (!ok) *sAbort = 1;
        // every issued MMA completes before TMEM is released
        mma_commit(mma_done);
        mbar_wait(mma_done, 0, lim);
      }
    } else {
      // ---- warps 2, 3: the constant ones rows D..D+15 of every V^T stage (e4m3 1.0 = 0x38) ----
      const int wt = tid - 64;  // 0..63
      for (int op = 0; op < kOps; ++op) {
        uint8_t* vt = smem + L::OFF_OP + op * L::OP_BYTES + L::K_BYTES;
        for (int i = wt; i < 16 * kBN / 16; i += 64)
          *reinterpret_cast<uint4*>(vt + D * kBN + 16 * i) =
              make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    }
  } else {
    // ===================================================== query-tile warpgroups
    setmaxnreg_consumer();
    const int t = (warp - 4) >> 2;            // tile 0 or 1
    const int r = tid & 127;                  // row within the tile = TMEM lane
    const int row = blockIdx.x * kRowsPerCta + t * kBM + r;
    const uint32_t t_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + (t ? L::T_S1 : L::T_S0) + t_lane;
    const uint32_t tPV = tmem + (t ? L::T_PV1 : L::T_PV0) + t_lane;
    uint8_t* sQ = smem + L::OFF_Q + t * L::Q_BYTES;
    uint8_t* sP0 = smem + L::OFF_P + 2 * t * L::P_BYTES;   // P buffers of this tile (block parity)

    // own Q row: packed codes -> e4m3 subnormals in the swizzled Q tile
    {
      const uint8_t* qsrc = p.q_codes + (head * npad + (size_t)row) * (D / 2);
#pragma unroll
      for (int cg = 0; cg < D / 32; ++cg) {
        uint4 w = make_uint4(0, 0, 0, 0);
        if (row < npad) w = __ldg(reinterpret_cast<const uint4*>(qsrc + cg * 16));
        uint32_t o[8];
        codes8_to_e4m3(w.x, o[0], o[1]);
        codes8_to_e4m3(w.y, o[2], o[3]);
        codes8_to_e4m3(w.z, o[4], o[5]);
        codes8_to_e4m3(w.w, o[6], o[7]);
        *reinterpret_cast<uint4*>(sQ + swz<L::ROWB>(r, cg * 32)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(sQ + swz<L::ROWB>(r, cg * 32 + 16)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    }
    const float sq = row < npad ? __ldg(p.q_scale + head * p.nblk + row / kBN) : 0.f;
    const float* ksc = p.k_scale + head * p.nblk;

    float O[D];
#pragma unroll
    for (int c = 0; c < D; ++c) O[c] = 0.f;
    float m = -INFINITY, l = 0.f, alpha_prev = 0.f;
    bool aborted = false;

    // O update of block i: O = O * alpha_i + (512 v_scale_i) * acc_i; the ones
    // columns carry the sum of the block's P codes for l.
    auto o_update = [&](int i, float alpha) -> bool {
      if (!warp_wait(&pv_full[t], i & 1, lim)) return false;
      // the V scales of block i land with the operand stage (op_full)
      if (!warp_wait(&op_full[i % kOps], (i / kOps) & 1, lim)) return false;
      tc_fence_after();
      const float* sv = sSv + (i % kOps) * D;
      // alpha == 1 on every row of the warp (the running max did not move): no rescale
      const bool unit = __all_sync(0xffffffffu, alpha == 1.f);
#pragma unroll
      for (int cb = 0; cb < D / 64; ++cb) {
        uint32_t a[64];
        uint32_t(&a0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&a[0]);
        uint32_t(&a1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&a[32]);
        tmem_ld32(tPV + 64 * cb, a0);
        tmem_ld32(tPV + 64 * cb + 32, a1);
        tmem_wait_dep2(a0, a1);
        if (unit) {
#pragma unroll
          for (int k4 = 0; k4 < 16; ++k4) {
            const float4 s4 = *reinterpret_cast<const float4*>(sv + 64 * cb + 4 * k4);
            const int c = 64 * cb + 4 * k4;
            fma2(O[c], O[c + 1], s4.x, s4.y, __uint_as_float(a[4 * k4]), __uint_as_float(a[4 * k4 + 1]), O[c], O[c + 1]);
            fma2(O[c + 2], O[c + 3], s4.z, s4.w, __uint_as_float(a[4 * k4 + 2]), __uint_as_float(a[4 * k4 + 3]),
                 O[c + 2], O[c + 3]);
          }
        } else {
#pragma unroll
          for (int k4 = 0; k4 < 16; ++k4) {
            const float4 s4 = *reinterpret_cast<const float4*>(sv + 64 * cb + 4 * k4);
            const int c = 64 * cb + 4 * k4;
            float x0, x1, x2, x3;
            mul2(x0, x1, s4.x, s4.y, __uint_as_float(a[4 * k4]), __uint_as_float(a[4 * k4 + 1]));
            mul2(x2, x3, s4.z, s4.w, __uint_as_float(a[4 * k4 + 2]), __uint_as_float(a[4 * k4 + 3]));
            fma2(O[c], O[c + 1], O[c], O[c + 1], alpha, alpha, x0, x1);
            fma2(O[c + 2], O[c + 3], O[c + 2], O[c + 3], alpha, alpha, x2, x3);
          }
        }
      }
      uint32_t lsum = tmem_ld1(tPV + D);
      tmem_wait_dep1(lsum);
      l = __fmaf_rn(l, alpha, __uint_as_float(lsum));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&pv_empty[t]);
        mbar_arrive(&op_empty[i % kOps]);
      }
      return true;
    };

    float sk_next = __ldg(ksc);
    for (int j = 0; j < nkb; ++j) {
      const float sk = sk_next;
      if (j + 1 < nkb) sk_next = __ldg(ksc + j + 1);
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

      // ---- running max over the block's valid keys ----
      const int nvalid = min(kBN, p.N - j * kBN);
      const float c = __fmul_rn(__fmul_rn(sq, sk), p.kappa);
      const float c18 = c * 262144.f;  // S here is S_int * 2^-18; c * 2^18 is exact
      float smax = -INFINITY;
      if (nvalid == kBN) {
#pragma unroll
        for (int k = 0; k < kBN; k += 2) smax = max3(smax, __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]));
      } else {
#pragma unroll
        for (int k = 0; k < kBN; ++k)
          if (k < nvalid) smax = fmaxf(smax, __uint_as_float(sr[k]));
      }
      const float m_new = fmaxf(m, __fmul_rn(smax, c18));
      const float alpha = ex2_approx(m - m_new);  // 0 on the first block (m = -inf)
      m = m_new;

      // ---- P codes u = rne(15 * 2^(S c - m)): branch-free estimate for all 64 keys ----
      uint32_t pw[kBN / 4];
      float near = 0.f;
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
        near = max3(near, fabsf(f0), fabsf(f1));
        near = max3(near, fabsf(f2), fabsf(f3));
        pw[k / 4] = pack_e4m3x4(r0, r1, r2, r3);
      }
      uint8_t* sP = sP0 + (j & 1) * L::P_BYTES;
#pragma unroll
      for (int k = 0; k < kBN / 16; ++k)
        *reinterpret_cast<uint4*>(sP + swz<64>(r, 16 * k)) =
            make_uint4(pw[4 * k], pw[4 * k + 1], pw[4 * k + 2], pw[4 * k + 3]);

      // ---- exact decisions (rare): estimates within 1e-5 of a half-integer ----
      // Recompute which keys were near a tie (same arithmetic as above), then
      // visit only the columns some lane flagged; S is still in TMEM.
      if (__any_sync(0xffffffffu, near > kNear)) {
        // S is still in TMEM (s_empty is released below): reload it here so the
        // fast path above does not have to keep 64 registers alive.
        uint32_t s2[kBN];
        {
          uint32_t(&t0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s2[0]);
          uint32_t(&t1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s2[32]);
          tmem_ld32(tS, t0);
          tmem_ld32(tS + 32, t1);
          tmem_wait_dep2(t0, t1);
        }
        uint32_t mlo = 0, mhi = 0;
#pragma unroll
        for (int k = 0; k < kBN; ++k) {
          const float d = __fmaf_rn(__uint_as_float(s2[k]), c18, -m);
          const float e = ex2_approx(d);
          const float rr = __fadd_rn(__fmaf_rn(e, 15.f, kMagic), -kMagic);
          const bool hit = fabsf(__fmaf_rn(e, 15.f, -rr)) > kNear;
          if (k < 32) mlo |= static_cast<uint32_t>(hit) << k;
          else mhi |= static_cast<uint32_t>(hit) << (k - 32);
        }
        uint32_t wlo = __reduce_or_sync(0xffffffffu, mlo), whi = __reduce_or_sync(0xffffffffu, mhi);
        while (wlo | whi) {
          const int k = wlo ? __ffs(wlo) - 1 : 32 + __ffs(whi) - 1;
          if (k < 32) wlo &= wlo - 1; else whi &= whi - 1;
          uint32_t sbits = tmem_ld1(tS + k);
          tmem_wait_dep1(sbits);
          const bool mine = (k < 32 ? (mlo >> k) : (mhi >> (k - 32))) & 1u;
          if (mine) {
            const float u = pcode_f(__fmaf_rn(__uint_as_float(sbits), c18, -m), sTau);
            sP[swz<64>(r, k)] = static_cast<uint8_t>(pack_e4m3x4(u, 0.f, 0.f, 0.f) & 0xFFu);
          }
        }
      }
      // keys past N in the last block take code 0
      for (int k = nvalid; k < kBN; ++k) sP[swz<64>(r, k)] = 0;
      if (DUMP) {
        for (int k = 0; k < kBN; ++k) {
          uint32_t sbits = tmem_ld1(tS + k);
          tmem_wait_dep1(sbits);
          if (k < nvalid && row >= p.dbg_r0 && row < p.dbg_r0 + p.dbg_nr)
            p.s_dump[(size_t)(row - p.dbg_r0) * p.N + (size_t)j * kBN + k] =
                static_cast<int32_t>(__uint_as_float(sbits) * 262144.f);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[t]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[2 * t + (j & 1)]);
      if (DUMP && row >= p.dbg_r0 && row < p.dbg_r0 + p.dbg_nr) {
        // P codes as the MMA will read them, decoded from the e4m3 bytes
        const size_t base = (size_t)(row - p.dbg_r0) * p.N + (size_t)j * kBN;
        for (int k = 0; k < nvalid; ++k) {
          const uint32_t b = sP[swz<64>(r, k)];
          const uint32_t e = (b >> 3) & 15u, mt = b & 7u;
          p.p_dump[base + k] = static_cast<uint8_t>(b == 0 ? 0 : ((8u + mt) << e) >> 10);
        }
      }

      // ---- O update of the previous block (its P V is done by now) ----
      if (j > 0 && !o_update(j - 1, alpha_prev)) { aborted = true; break; }
      alpha_prev = alpha;
      if (warp_flag(sAbort)) { aborted = true; break; }
    }
    if (!aborted && !o_update(nkb - 1, alpha_prev)) aborted = true;
    if (aborted) *sAbort = 1;

    if (!aborted && row < p.N) {
      const float inv_l = 1.f / l;
      float4* dst = reinterpret_cast<float4*>(p.out + (head * p.N + row) * D);
#pragma unroll
      for (int c4 = 0; c4 < D / 4; ++c4)
        dst[c4] = make_float4(O[4 * c4] * inv_l, O[4 * c4 + 1] * inv_l, O[4 * c4 + 2] * inv_l, O[4 * c4 + 3] * inv_l);
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
// x D e4m3 subnormals (K-major, 128B / 64B swizzle), V^T as D rows x 64 keys
// (64B swizzle), followed by the block's V scales times 2^9.  HBM-bound.
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
  const uint8_t* vp = p.v_codes + (head * p.nblk + j) * (size_t)D * 32;
  uint8_t* vimg = img + L::K_BYTES;
  for (int i = threadIdx.x; i < D * 2; i += blockDim.x) {
    const int c = i >> 1, hl = i & 1;
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(vp + 16 * i));
    uint32_t o[8];
    codes8_to_e4m3(w.x, o[0], o[1]);
    codes8_to_e4m3(w.y, o[2], o[3]);
    codes8_to_e4m3(w.z, o[4], o[5]);
    codes8_to_e4m3(w.w, o[6], o[7]);
    *reinterpret_cast<uint4*>(vimg + swz<64>(c, hl * 32)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(vimg + swz<64>(c, hl * 32 + 16)) = make_uint4(o[4], o[5], o[6], o[7]);
  }
  float* sv = reinterpret_cast<float*>(img + L::K_BYTES + L::VIMG_BYTES);
  const float* vs = p.v_scale + (head * p.nblk + j) * D;
  for (int c = threadIdx.x; c < D; c += blockDim.x) sv[c] = __ldg(vs + c) * 512.f;
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
