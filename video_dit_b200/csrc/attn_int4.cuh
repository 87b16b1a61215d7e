// attn_int4.cuh -- INT4 FlashAttention forward with range-optimised P codes.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: a mixed-precision INT4
// FlashAttention in which P = exp(QK - max(QK)) >= 0 is quantised with a
// fixed scale and zero-point so that all 16 unsigned 4-bit levels are used
// ("Range-optimized P Quantization").
//
// Both contractions are exact integer products on the 8-bit tensor path.
//   * S = Q K^T: a code v in [-7, 7] is the e4m3 subnormal v * 2^-9, so
//     tcgen05.mma kind::f8f6f4 accumulates S_int * 2^-18 exactly in fp32
//     (every partial sum is an integer multiple of 2^-18 far below 2^24
//     units) -- the integers an s32 accumulation gives, already in fp32.
//   * P V, per 64-key block: a P code u in 0..15 stored as the byte u is the
//     e4m3 value u * 2^-9 (subnormal below 8, exponent field 1 from 8 to 15),
//     so the block's sum_k u_k v_k,c * 2^-18 is exact in fp32 as well
//     (|sum| <= 64 * 15 * 7 units).  It is computed transposed,
//     ACC^T = V^T P^T with M = the head's channels and N = the tile's 128
//     query rows, so a channel is a TMEM lane.
// The per-(block, channel) V scale s_c is then applied on the CUDA cores by
// correction warps in which a thread owns one channel: s_c is a register,
// and O^T (fp32, in TMEM) is updated as O <- alpha_q O + (s_c 2^18) ACC, with
// alpha_q = 2^(m_old - m_new) for the query columns whose running max moved
// (read from shared memory only in tile-blocks where one did).
//
// The packed K / V nibbles are widened once per call by widen_kv_kernel into
// the exact shared-memory images of the operand tiles (K: 64 x D e4m3,
// K-major, 128B / 64B swizzle; V^T: 128 channel rows x 64 keys e4m3, 64B
// swizzle, rows >= D zero), so the main loop moves them with plain bulk
// copies.
//
// One CTA = two 128-row query tiles of one head (256 rows), 512 threads:
//   warp 0      TMA producer: the K and V^T images of each 64-key block
//               -> a kOps-stage shared-memory ring;
//   warps 1, 3  issue S_t(j) = Q_t K_j^T (128 x 64), warp 1 for tile 0 and
//               warp 3 (which also owns the TMEM allocation) for tile 1;
//   warp 2      issues ACC^T = V_j^T P_t(j)^T for tile 0 then tile 1 into the
//               one ACC^T buffer (128 channels x 128 queries); its commit
//               also frees the P slot the MMA read;
//   warps 4-7   softmax of tile 0, warps 8-11 of tile 1 (thread = query row
//               = TMEM lane): running max, P codes into shared memory (the
//               B operand of P V), the row sum of the codes, alpha (into a
//               ring of its own, freed by the correction);
//   warps 12-15 correction (thread = channel): O^T update per block, and the
//               epilogue out = O / l.
// TMEM (512 columns): S of tile t at 64 t, ACC^T at 128, O^T of tile t at
// 256 + 128 t.
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
  const uint8_t* work;  // per (head, block): the widened K image and V^T image (IMG_BYTES)
  float* out;
  int H, N, nblk;
  float kappa;          // RN(sm_scale * log2 e)
  float tau[16];        // tau[k]: smallest fp32 d with rne(15 * 2^d) >= k (k = 1..15)
  uint64_t timeout_ns;  // bound of every mbarrier wait
  int inject_skip;      // fault injection: skip the first score MMA
  int nheads;
  int16_t heads[256];   // the INT4 heads to process (blockIdx.y indexes this list)
  // optional dumps of rows [dbg_r0, dbg_r0 + dbg_nr) (NULL: off; warp-uniform test)
  int32_t* s_dump;
  uint8_t* p_dump;
  int dbg_r0, dbg_nr;
};

constexpr int kInt4Threads = 512;
constexpr int kRowsPerCta = 2 * kBM;
constexpr int kOps = 6;   // operand stages
// The softmax may run kPSlots blocks ahead of the P V that reads its codes
// and kAlphaRing blocks ahead of the correction that reads its alpha.
// Measured at 480p: alpha entries 2 / 3 / 4 / 5 / 6 take 32.6 / 32.0 / 32.7 /
// 32.0 / 31.9 ms, and a third P slot adds 0.7 ms.  128-key groups emit block
// 2g + 1 before block 2g, so both need at least two entries.
constexpr int kPSlots = 2;
constexpr int kAlphaRing = 3;
static_assert(kPSlots >= 2 && kAlphaRing >= 2, "a 128-key group emits its two blocks out of order");
constexpr int kIssueRegs = 32;    // warps 0-3
constexpr int kSoftmaxRegs = 128; // warps 4-11
constexpr int kCorrRegs = 224;    // warps 12-15
// Register split: the warpgroups' shares add up to the launch allocation
// 512 * kLaunchRegs; the host refuses to launch a build whose register count
// differs (setmaxnreg.inc would otherwise wait forever).
constexpr int kLaunchRegs = (128 * kIssueRegs + 256 * kSoftmaxRegs + 128 * kCorrRegs) / 512;
static_assert(kLaunchRegs * 512 == 128 * kIssueRegs + 256 * kSoftmaxRegs + 128 * kCorrRegs, "register split");
static_assert(kLaunchRegs == 128, "launch allocation");

template <int D, int G = 64>
struct Int4Smem {
  // 128-key groups keep a block's scores in shared memory until the next
  // block's are in (the spill area), paid for with two fewer operand stages
  static constexpr int OPS = G == 128 ? kOps - 2 : kOps;
  static constexpr uint32_t LAYOUT_QK = D == 128 ? 2u : 4u;  // 128B / 64B swizzle of the Q and K rows
  static constexpr uint32_t SBO_QK = 8 * D;
  static constexpr int Q_BYTES = kBM * D;         // one tile, e4m3
  static constexpr int K_BYTES = kBN * D;         // one block, e4m3
  static constexpr int VT_BYTES = 128 * kBN;      // 128 channel rows x 64 keys, e4m3
  static constexpr int P_BYTES = kBM * kBN;       // one tile's codes, 128 rows x 64 keys
  static constexpr int OP_BYTES = K_BYTES + VT_BYTES;
  static constexpr int IMG_BYTES = OP_BYTES;      // one block in int4_work
  static constexpr int OFF_Q = 0;                                 // [tile]
  static constexpr int OFF_P = OFF_Q + 2 * Q_BYTES;               // [tile][slot]
  static constexpr int OFF_OP = OFF_P + 2 * kPSlots * P_BYTES;    // [stage]
  static constexpr int OFF_ALPHA = OFF_OP + OPS * OP_BYTES;       // float [tile][entry][128]
  static constexpr int OFF_FLAG = OFF_ALPHA + 2 * kAlphaRing * kBM * 4;   // int [tile][entry][4 warps]
  static constexpr int OFF_L = OFF_FLAG + 2 * kAlphaRing * 4 * 4;         // float [tile][128]
  static constexpr int OFF_TAU = OFF_L + 2 * kBM * 4;
  static constexpr int OFF_SPILL = OFF_TAU + 64;                  // float4 [tile][16][128] (G = 128)
  static constexpr int SPILL_BYTES = G == 128 ? 2 * kBM * kBN * 4 : 0;
  static constexpr int OFF_BAR = OFF_SPILL + SPILL_BYTES;
  // barriers: op_full[OPS] op_empty[OPS] q_full s_full[2] s_empty[2]
  //           p_full[2][kPSlots] p_empty[2][kPSlots] acc_full acc_empty l_full
  //           mma_done[3] a_full[2][kAlphaRing] a_empty[2][kAlphaRing]
  static constexpr int NBAR = 2 * OPS + 1 + 2 + 2 + 4 * kPSlots + 1 + 1 + 1 + 3 + 4 * kAlphaRing;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;
  static constexpr int BYTES = OFF_ABORT + 4;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0, T_ACC = 2 * kBN, T_O = 256;
  static_assert(T_ACC + kBM <= T_O && T_O + 2 * kBM <= TMEM_COLS, "TMEM budget");
  static_assert(D <= 128, "one TMEM lane per channel");
  static_assert(IMG_BYTES % 16 == 0 && K_BYTES % 16 == 0 && VT_BYTES % 16 == 0, "bulk copy sizes");
  static_assert(G == 64 || G == 128, "max group");
  static_assert(OFF_SPILL % 16 == 0, "spill alignment");
  static_assert(OFF_P % 1024 == 0 && OFF_OP % 1024 == 0 && OP_BYTES % 1024 == 0 && K_BYTES % 1024 == 0 &&
                    P_BYTES % 1024 == 0,
                "swizzle atom alignment");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

// Range-optimised P code u = min(15, rne(15 * 2^d)) in exact arithmetic.
// e = ex2.approx(d) is within 2^-22 (relative) of 2^d, so the exact
// 15 * 2^d lies in [e * kLo, e * kHi], kLo/Hi = 15 (1 -/+ 2^-20).  Adding
// kMag = 2^23 to each bound rounds it to an integer (RNE); when the two
// integers agree, so does rne(15 * 2^d), and only otherwise is the code
// decided by the exact threshold table tau.  The main loop takes the same
// two roundings for every key and compares their sums over a row's block, so
// this is also the function the exhaustive test checks.
constexpr float kMag = 8388608.f;                    // 2^23
constexpr uint32_t kMagBits = 0x4B000000u;
constexpr float kLo = 15.f - 15.f / 1048576.f;       // 15 (1 - 2^-20), exact in fp32
constexpr float kHi = 15.f + 15.f / 1048576.f;       // 15 (1 + 2^-20), exact in fp32
constexpr float kLogitBound = 1048576.f;             // |m| < 2^20: the block's max key keeps d <= 2^-5
__device__ __forceinline__ uint32_t pcode(float d, const float* tau) {
  const float e = ex2_approx(d);
  const uint32_t lo = __float_as_uint(__fmaf_rn(e, kLo, kMag)) - kMagBits;
  const uint32_t hi = __float_as_uint(__fmaf_rn(e, kHi, kMag)) - kMagBits;
  uint32_t u = lo;
  if (lo != hi && hi <= 15u && d >= tau[hi]) u = hi;
  return u < 15u ? u : 15u;
}

// 2^d on the FMA pipe (d <= 0), for a share of the keys: a Cody-Waite split
// d = n + f with n = rne(d) (the 1.5 * 2^23 addition; f = d - n in [-1/2, 1/2]
// exactly) and a degree-6 polynomial for 2^f whose coefficients were fitted
// for this kernel to the relative error of 2^f on [-1/2, 1/2] (weighted least
// squares at Chebyshev nodes, reweighted toward equal ripple, rounded to
// fp32): with one rounding per Horner step its relative error is below
// 8.5e-8 (2^-23.5), inside the 2^-22 the code decision assumes of
// ex2.approx, so the same two-rounding test and the same exact fallback
// apply.  2^n enters through the exponent field; d is clamped at -100 (the
// code is 0 there and 2^-100 is still a normal number).
constexpr float kP0 = 1.0f, kP1 = 0.6931471824645996f, kP2 = 0.24022646248340607f, kP3 = 0.05550328642129898f,
                kP4 = 0.009618489071726799f, kP5 = 0.0013399930903688073f, kP6 = 0.0001534580806037411f;
__device__ __forceinline__ void ex2_fma2(float d0, float d1, float& e0, float& e1) {
  d0 = fmaxf(d0, -100.f);
  d1 = fmaxf(d1, -100.f);
  float t0, t1, n0, n1, f0, f1;
  add2(t0, t1, d0, d1, 12582912.f, 12582912.f);      // 1.5 * 2^23 + rne(d)
  add2(n0, n1, t0, t1, -12582912.f, -12582912.f);    // rne(d), exact
  add2(f0, f1, d0, d1, -n0, -n1);                    // d - n, exact
  float p0 = kP6, p1 = kP6;
  fma2(p0, p1, p0, p1, f0, f1, kP5, kP5);
  fma2(p0, p1, p0, p1, f0, f1, kP4, kP4);
  fma2(p0, p1, p0, p1, f0, f1, kP3, kP3);
  fma2(p0, p1, p0, p1, f0, f1, kP2, kP2);
  fma2(p0, p1, p0, p1, f0, f1, kP1, kP1);
  fma2(p0, p1, p0, p1, f0, f1, kP0, kP0);
  e0 = __int_as_float(__float_as_int(p0) + ((__float_as_int(t0) - 0x4B400000) << 23));
  e1 = __int_as_float(__float_as_int(p1) + ((__float_as_int(t1) - 0x4B400000) << 23));
}

// The P code of d with the exponential taken on the FMA pipe (the function
// the main loop applies to the keys routed there; pcode() above for the rest).
__device__ __forceinline__ uint32_t pcode_fma(float d, const float* tau) {
  float e, e_unused;
  ex2_fma2(d, d, e, e_unused);
  const uint32_t lo = __float_as_uint(__fmaf_rn(e, kLo, kMag)) - kMagBits;
  const uint32_t hi = __float_as_uint(__fmaf_rn(e, kHi, kMag)) - kMagBits;
  uint32_t u = lo;
  if (lo != hi && hi <= 15u && d >= tau[hi]) u = hi;
  return u < 15u ? u : 15u;
}

// Of every four 4-key groups of a block, the first kExpFmaGroups take their
// exponentials on the FMA pipe, the rest on MUFU (measured: a share of the
// exponentials moved to the FMA pipe does not shorten this kernel, whose
// exponential unit is a quarter busy -- see the design notes; 0 keeps all on
// MUFU).
constexpr int kExpFmaGroups = 0;

__device__ __forceinline__ void setmaxnreg_issue() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 32;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_softmax() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 128;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_corr() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
}
static_assert(kIssueRegs == 32 && kSoftmaxRegs == 128 && kCorrRegs == 224, "setmaxnreg immediates");

// The max of one 64-key block's scores S = S_int * 2^-18 over the valid keys;
// keys >= nvalid (MASK) are set to -inf in sr, so they never enter a max.
template <bool MASK>
__device__ __forceinline__ float block_max(uint32_t (&sr)[kBN], int nvalid) {
  if (MASK) {
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
  return fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
}

// Every code of one block by the exact function (the rare slow path of
// block_codes); returns their sum.
__device__ __noinline__ uint32_t block_codes_exact(const uint32_t* sr, int nvalid, float c18, float m, uint32_t* pw,
                                                   const float* tau) {
  uint32_t usum = 0;
  for (int w = 0; w < kBN / 4; ++w) {
    uint32_t word = 0;
    for (int i = 0; i < 4; ++i) {
      const int k = 4 * w + i;
      const float d = k < nvalid ? __fmaf_rn(__uint_as_float(sr[k]), c18, -m) : -INFINITY;
      const uint32_t u = pcode(d, tau);
      word |= u << (8 * i);
      usum += u;
    }
    pw[w] = word;
  }
  return usum;
}

// The P codes of one 64-key block of one softmax thread against the group
// max m: bytes, 4 per word (key 4w + i in byte i of word w), keys >= nvalid
// (MASK) code 0.  Returns the sum of the codes; with R1, lsum also receives
// the row-sum term 15 * sum_k 2^d_k (the unquantised values the codes are
// rounded from, from the same exponentials).
template <bool MASK, bool R1>
__device__ __forceinline__ uint32_t block_codes(const uint32_t (&sr)[kBN], int nvalid, float c18, float m,
                                                uint32_t (&pw)[kBN / 4], const float* tau, float& lsum) {
  uint32_t usum = 0, sum_hi = 0;
  float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
  for (int k = 0; k < kBN; k += 4) {
    float d0, d1, d2, d3;
    fma2(d0, d1, __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]), c18, c18, -m, -m);
    fma2(d2, d3, __uint_as_float(sr[k + 2]), __uint_as_float(sr[k + 3]), c18, c18, -m, -m);
    if (MASK) {
      if (k + 0 >= nvalid) d0 = -INFINITY;
      if (k + 1 >= nvalid) d1 = -INFINITY;
      if (k + 2 >= nvalid) d2 = -INFINITY;
      if (k + 3 >= nvalid) d3 = -INFINITY;
    }
    float e0, e1, e2, e3;
    if ((k / 4) % 4 < kExpFmaGroups) {   // compile-time per group: the loop is unrolled
      ex2_fma2(d0, d1, e0, e1);
      ex2_fma2(d2, d3, e2, e3);
    } else {
      e0 = ex2_approx(d0);
      e1 = ex2_approx(d1);
      e2 = ex2_approx(d2);
      e3 = ex2_approx(d3);
    }
    float l0, l1, l2, l3, h0, h1, h2, h3;
    fma2(l0, l1, e0, e1, kLo, kLo, kMag, kMag);
    fma2(l2, l3, e2, e3, kLo, kLo, kMag, kMag);
    fma2(h0, h1, e0, e1, kHi, kHi, kMag, kMag);
    fma2(h2, h3, e2, e3, kHi, kHi, kMag, kMag);
    sum_hi += __float_as_uint(h0) + __float_as_uint(h1) + __float_as_uint(h2) + __float_as_uint(h3);
    pw[k / 4] = prmt(prmt(__float_as_uint(l0), __float_as_uint(l1), 0x0040u),
                     prmt(__float_as_uint(l2), __float_as_uint(l3), 0x0040u), 0x5410u);
    usum = __dp4a(pw[k / 4], 0x01010101u, usum);   // the four codes' sum, from the packed word
    if (R1) {
      add2(ls0, ls1, ls0, ls1, e0, e1);
      add2(ls0, ls1, ls0, ls1, e2, e3);
    }
  }
  if (R1) lsum = __fmul_rn(15.f, __fadd_rn(ls0, ls1));
  // Exact decisions (rare): some key of the warp's rows lies in the band
  // where the two roundings differ, or a row's max is so large that its max
  // key could round past code 15.  Out of line, so that its registers do not
  // weigh on the main path.
  // Each upper rounding is at least the lower one and 64 kMag bit patterns
  // sum to 0xC0000000 (mod 2^32): the two agree on every key exactly when
  // sum_hi - 0xC0000000 is the sum of the packed (lower) codes.
  const bool bad = (sum_hi - 0xC0000000u != usum) || !(fabsf(m) < kLogitBound);
  if (__any_sync(0xffffffffu, bad)) {
    // copies made only here, so the scores stay in registers on the main path
    uint32_t s_copy[kBN], p_copy[kBN / 4];
#pragma unroll
    for (int k = 0; k < kBN; ++k) s_copy[k] = sr[k];
    usum = block_codes_exact(s_copy, MASK ? nvalid : kBN, c18, m, p_copy, tau);
#pragma unroll
    for (int w = 0; w < kBN / 4; ++w) pw[w] = p_copy[w];
  }
  return usum;
}

// The codes of one block; returns the block's contribution to l (the code
// sum, or with R1 15 sum 2^d).
template <bool MASK, bool R1>
__device__ __forceinline__ float block_codes_l(const uint32_t (&sr)[kBN], int nvalid, float c18, float m,
                                               uint32_t (&pw)[kBN / 4], const float* tau) {
  float lsum = 0.f;
  const uint32_t usum = block_codes<MASK, R1>(sr, nvalid, c18, m, pw, tau, lsum);
  return R1 ? lsum : static_cast<float>(usum);
}

template <int D, int G, bool R1>
__global__ void __launch_bounds__(kInt4Threads, 1) attn_int4_kernel(const __grid_constant__ Int4Params p) {
  using L = Int4Smem<D, G>;
  constexpr int kOps = L::OPS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* op_full = bars;
  uint64_t* op_empty = bars + kOps;             // 3 arrivals: the two S issuers' and the P V issuer's commits
  uint64_t* q_full = bars + 2 * kOps;           // 8 softmax warps staged their Q rows
  uint64_t* s_full = q_full + 1;                // [tile], commit
  uint64_t* s_empty = s_full + 2;               // [tile], 4 softmax warps hold S in registers
  uint64_t* p_full = s_empty + 2;               // [tile][slot], 4 softmax warps wrote the codes
  uint64_t* p_empty = p_full + 2 * kPSlots;     // [tile][slot], commit of the P V that read them
  uint64_t* acc_full = p_empty + 2 * kPSlots;   // commit of a P V
  uint64_t* acc_empty = acc_full + 1;           // 4 correction warps hold ACC in registers
  uint64_t* l_full = acc_empty + 1;             // 8 softmax warps wrote their rows' l
  uint64_t* mma_done = l_full + 1;              // [3], one per MMA-issuing warp (S tile 0, P V, S tile 1)
  uint64_t* a_full = mma_done + 3;              // [tile][entry], 4 softmax warps wrote alpha and flags
  uint64_t* a_empty = a_full + 2 * kAlphaRing;  // [tile][entry], 4 correction warps are done with them
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + L::OFF_ABORT);
  float* sTau = reinterpret_cast<float*>(smem + L::OFF_TAU);
  float* sAlpha = reinterpret_cast<float*>(smem + L::OFF_ALPHA);
  int* sFlag = reinterpret_cast<int*>(smem + L::OFF_FLAG);
  float* sL = reinterpret_cast<float*>(smem + L::OFF_L);

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
      mbar_init(&op_empty[i], 3);
    }
    mbar_init(q_full, 8);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_empty[t], 4);
    }
    for (int i = 0; i < 2 * kPSlots; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_init(l_full, 8);
    for (int i = 0; i < 3; ++i) mbar_init(&mma_done[i], 1);
    for (int i = 0; i < 2 * kAlphaRing; ++i) {
      mbar_init(&a_full[i], 4);
      mbar_init(&a_empty[i], 4);
    }
    *sAbort = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 3) {
    tmem_alloc(sTmem, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;

  if (warp < 4) {
    // ======================================================== issuing warps
    setmaxnreg_issue();
    if (warp == 0) {
      // ---- TMA producer: the images of block j -> stage j % kOps ----
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
          bulk_g2s(dst + L::K_BYTES, src + L::K_BYTES, L::VT_BYTES, &op_full[op]);
        }
        __syncwarp();
        issued = j + 1;
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int j = (issued > kOps ? issued - kOps : 0); j < issued; ++j)
        warp_wait(&op_full[j % kOps], (j / kOps) & 1, lim);
    } else if (warp == 1 || warp == 3) {
      // ---- S issuers: S_t(j) = Q_t K_j^T, warp 1 for tile 0 and warp 3 (after
      // the TMEM allocation) for tile 1, so neither tile's next scores wait
      // behind the other's (warp-uniform loop, one elected lane issues) ----
      const int t = warp == 1 ? 0 : 1;
      uint64_t* const done = &mma_done[t == 0 ? 0 : 2];
      constexpr uint32_t ID_S = idesc(1, 0, 0, kBM, kBN);   // e4m3 x e4m3 -> f32, 128 x 64
      const uint32_t hi_qk = sdesc_hi(L::SBO_QK, L::LAYOUT_QK);
      const uint32_t lo_q = sdesc_lo(smem_u32(smem + L::OFF_Q));
      const uint32_t lo_op = sdesc_lo(smem_u32(smem + L::OFF_OP));
      bool ok = warp_wait(q_full, 0, lim);
      for (int j = 0; ok && j < nkb; ++j) {
        const int op = j % kOps;
        if (!warp_wait(&op_full[op], (j / kOps) & 1, lim)) { ok = false; break; }
        const uint32_t lk = lo_op + op * (L::OP_BYTES >> 4);
        if (!warp_wait(&s_empty[t], (j & 1) ^ 1, lim)) { ok = false; break; }
        tc_fence_after();
        if (p.inject_skip && j == 0 && t == 0) {   // fault injection: never committed
          __syncwarp();
          continue;
        }
        const uint32_t lq = lo_q + t * (L::Q_BYTES >> 4);
        const uint32_t d_s = tmem + L::T_S + t * kBN;
        if (elect_one()) {
          mma_f8f6f4_ss<0>(d_s, lq, hi_qk, lk, hi_qk, ID_S);
#pragma unroll
          for (int k = 1; k < D / 32; ++k) mma_f8f6f4_ss<1>(d_s, lq + 2 * k, hi_qk, lk + 2 * k, hi_qk, ID_S);
          mma_commit(&s_full[t]);
          mma_commit(&op_empty[op]);   // this tile's read of the stage's K tile
        }
        __syncwarp();
        if (warp_flag(sAbort)) { ok = false; break; }
      }
      if (!ok && lane == 0) *sAbort = 1;
      if (elect_one()) mma_commit(done);
      __syncwarp();
      warp_wait(done, 0, lim);
    } else if (warp == 2) {
      // ---- P V issuer: ACC^T = V_j^T P_t(j)^T, tile 0 then tile 1, into
      // the one ACC^T buffer ----
      constexpr uint32_t ID_PV = idesc(1, 0, 0, 128, kBM);  // e4m3 x e4m3 -> f32, 128 channels x 128 queries
      const uint32_t hi_64 = sdesc_hi(512, 4);               // 64-byte rows, 64B swizzle
      const uint32_t lo_p = sdesc_lo(smem_u32(smem + L::OFF_P));
      const uint32_t lo_v = sdesc_lo(smem_u32(smem + L::OFF_OP + L::K_BYTES));
      const uint32_t d_acc = tmem + L::T_ACC;
      bool ok = true;
      for (int j = 0; ok && j < nkb; ++j) {
        const int op = j % kOps, sl = j % kPSlots, pph = (j / kPSlots) & 1;
        if (!warp_wait(&op_full[op], (j / kOps) & 1, lim)) { ok = false; break; }
        const uint32_t lv = lo_v + op * (L::OP_BYTES >> 4);
        for (int t = 0; t < 2; ++t) {
          const int u = 2 * j + t;
          if (!warp_wait(&p_full[kPSlots * t + sl], pph, lim)) { ok = false; break; }
          if (!warp_wait(acc_empty, (u & 1) ^ 1, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t lp = lo_p + (kPSlots * t + sl) * (L::P_BYTES >> 4);
          if (elect_one()) {
            mma_f8f6f4_ss<0>(d_acc, lv, hi_64, lp, hi_64, ID_PV);
            mma_f8f6f4_ss<1>(d_acc, lv + 2, hi_64, lp + 2, hi_64, ID_PV);
            mma_commit(acc_full);
            mma_commit(&p_empty[kPSlots * t + sl]);  // the tile's codes of block j are read
            if (t == 1) mma_commit(&op_empty[op]);   // the stage's V^T tile is read
          }
          __syncwarp();
        }
        if (!ok) break;
        if (warp_flag(sAbort)) { ok = false; break; }
      }
      if (!ok && lane == 0) *sAbort = 1;
      if (elect_one()) mma_commit(&mma_done[1]);
      __syncwarp();
      warp_wait(&mma_done[1], 0, lim);
    }
  } else if (warp < 12) {
    // ======================================================== softmax warps
    setmaxnreg_softmax();
    const int t = (warp - 4) >> 2;            // tile 0 or 1
    const int r = tid & 127;                  // row within the tile = TMEM lane
    const int row = blockIdx.x * kRowsPerCta + t * kBM + r;
    const uint32_t t_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + L::T_S + t * kBN + t_lane;
    uint8_t* sQ = smem + L::OFF_Q + t * L::Q_BYTES;

    // own Q row: packed codes -> e4m3 subnormals, the swizzled row r of the
    // tile's shared-memory image (the A operand of the score MMA)
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
        *reinterpret_cast<uint4*>(sQ + swz<D>(r, cg * 32)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(sQ + swz<D>(r, cg * 32 + 16)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    }
    const float sq = row < npad ? __ldg(p.q_scale + head * p.nblk + row / kBN) : 0.f;
    const float* ksc = p.k_scale + head * p.nblk;
    const bool dumping = p.s_dump != nullptr;   // kernel argument: uniform
    const bool dump_rows = dumping && row >= p.dbg_r0 && row < p.dbg_r0 + p.dbg_nr;

    // S of block j -> registers, in two parts: start_s waits for the scores
    // and issues the TMEM loads, finish_s waits for the loads and releases the
    // buffer at once, so the MMA computes the tile's next scores while these
    // are coded.  With 64-key groups the next block's loads are started before
    // this block's codes are emitted (sr is dead by then), so their latency
    // overlaps the emit.
    auto start_s = [&](int j, uint32_t (&sr)[kBN]) -> bool {
      if (!warp_wait(&s_full[t], j & 1, lim)) return false;
      tc_fence_after();
      uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
      uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
      tmem_ld32(tS, s0);
      tmem_ld32(tS + 32, s1);
      return true;
    };
    auto finish_s = [&](int j, uint32_t (&sr)[kBN]) {
      uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
      uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
      tmem_wait_dep2(s0, s1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[t]);
      if (dumping) {
        const int nvalid = min(kBN, p.N - j * kBN);
#pragma unroll
        for (int k = 0; k < kBN; ++k)
          if (dump_rows && k < nvalid)
            p.s_dump[(size_t)(row - p.dbg_r0) * p.N + (size_t)j * kBN + k] =
                static_cast<int32_t>(__uint_as_float(sr[k]) * 262144.f);
      }
    };
    auto load_s = [&](int j, uint32_t (&sr)[kBN]) -> bool {
      if (!start_s(j, sr)) return false;
      finish_s(j, sr);
      return true;
    };
    // the codes of block j -> its P slot (the B operand of P V), with alpha
    // (the factor on O before the block is added) and the warp's flag
    auto emit = [&](int j, const uint32_t (&pw)[kBN / 4], float alpha) -> bool {
      const int ps = kPSlots * t + j % kPSlots, e = kAlphaRing * t + j % kAlphaRing;
      // the slot's previous codes (block j - kPSlots) are read by their P V,
      // and the entry's previous alpha (block j - kAlphaRing) by the correction
      if (j >= kPSlots && !warp_wait(&p_empty[ps], ((j / kPSlots) & 1) ^ 1, lim)) return false;
      if (j >= kAlphaRing && !warp_wait(&a_empty[e], ((j / kAlphaRing) & 1) ^ 1, lim)) return false;
      uint8_t* sP = smem + L::OFF_P + ps * L::P_BYTES;
#pragma unroll
      for (int i = 0; i < kBN / 16; ++i)
        *reinterpret_cast<uint4*>(sP + swz<64>(r, 16 * i)) =
            make_uint4(pw[4 * i], pw[4 * i + 1], pw[4 * i + 2], pw[4 * i + 3]);
      sAlpha[e * kBM + r] = alpha;
      const bool moved = __any_sync(0xffffffffu, alpha != 1.f);
      if (lane == 0) sFlag[e * 4 + (warp & 3)] = moved ? 1 : 0;
      if (dumping) {
        const int nvalid = min(kBN, p.N - j * kBN);
#pragma unroll
        for (int k = 0; k < kBN; ++k)
          if (dump_rows && k < nvalid)
            p.p_dump[(size_t)(row - p.dbg_r0) * p.N + (size_t)j * kBN + k] =
                static_cast<uint8_t>((pw[k >> 2] >> (8 * (k & 3))) & 0xFFu);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&p_full[ps]);
        mbar_arrive(&a_full[e]);
      }
      return true;
    };
    // alpha = 2^(m_old - m) for the rows whose max moved (exact 1 elsewhere; 0
    // before the first block, where O is not read)
    auto alpha_of = [&](bool first, float m_old, float m_new) -> float {
      if (first) return 0.f;
      float alpha = 1.f;
      if (__any_sync(0xffffffffu, m_new != m_old))
        if (m_new != m_old) alpha = exp2f(m_old - m_new);
      return alpha;
    };
    auto c18_of = [&](float sk) {   // S = S_int 2^-18, so c * 2^18 (exact) multiplies S
      return __fmul_rn(__fmul_rn(__fmul_rn(sq, sk), p.kappa), 262144.f);
    };
    // the key scales are read one block (pair) ahead
    float sk_next = __ldg(ksc), sk_next2 = nkb > 1 ? __ldg(ksc + 1) : 0.f;


    float m = -INFINITY, l = 0.f;
    bool aborted = false;
    if constexpr (G == 64) {
      uint32_t sr[kBN];
      aborted = !start_s(0, sr);
      for (int j = 0; j < nkb && !aborted; ++j) {
        const float c18 = c18_of(sk_next);
        if (j + 1 < nkb) sk_next = __ldg(ksc + j + 1);
        finish_s(j, sr);
        const int nvalid = min(kBN, p.N - j * kBN);
        const float smax = nvalid == kBN ? block_max<false>(sr, nvalid) : block_max<true>(sr, nvalid);
        const float m_old = m;
        m = fmaxf(m, __fmul_rn(smax, c18));
        uint32_t pw[kBN / 4];
        const float lsum = nvalid == kBN ? block_codes_l<false, R1>(sr, nvalid, c18, m, pw, sTau)
                                         : block_codes_l<true, R1>(sr, nvalid, c18, m, pw, sTau);
        const float alpha = alpha_of(j == 0, m_old, m);
        l = __fmaf_rn(l, alpha, lsum);
        if (j + 1 < nkb && !start_s(j + 1, sr)) { aborted = true; break; }
        if (!emit(j, pw, alpha)) { aborted = true; break; }
        if (warp_flag(sAbort)) { aborted = true; break; }
      }
      tmem_ld_wait();   // no TMEM load of this thread is left in flight
    } else {
      // 128-key groups: blocks j0 = 2g and j1 = 2g + 1 share the max over both,
      // so block j0's scores wait in shared memory while j1's come in; j1 is
      // coded first (from registers), then j0 (reloaded)
      float4* spill = reinterpret_cast<float4*>(smem + L::OFF_SPILL) + t * (kBN / 4) * kBM;
      for (int j0 = 0; j0 < nkb; j0 += 2) {
        const int j1 = j0 + 1;
        const bool has1 = j1 < nkb;
        const float c0 = c18_of(sk_next);
        const float c1 = has1 ? c18_of(sk_next2) : 0.f;
        if (j0 + 2 < nkb) sk_next = __ldg(ksc + j0 + 2);
        if (j0 + 3 < nkb) sk_next2 = __ldg(ksc + j0 + 3);
        const int nv0 = min(kBN, p.N - j0 * kBN), nv1 = has1 ? min(kBN, p.N - j1 * kBN) : 0;
        uint32_t sr[kBN];
        if (!load_s(j0, sr)) { aborted = true; break; }
        const float smax0 = nv0 == kBN ? block_max<false>(sr, nv0) : block_max<true>(sr, nv0);
#pragma unroll
        for (int i = 0; i < kBN / 4; ++i)
          spill[i * kBM + r] = make_float4(__uint_as_float(sr[4 * i]), __uint_as_float(sr[4 * i + 1]),
                                           __uint_as_float(sr[4 * i + 2]), __uint_as_float(sr[4 * i + 3]));
        float x1 = -INFINITY;
        if (has1) {
          if (!load_s(j1, sr)) { aborted = true; break; }
          const float smax1 = nv1 == kBN ? block_max<false>(sr, nv1) : block_max<true>(sr, nv1);
          x1 = __fmul_rn(smax1, c1);
        }
        const float m_old = m;
        m = fmaxf(fmaxf(m, __fmul_rn(smax0, c0)), x1);
        const float alpha = alpha_of(j0 == 0, m_old, m);
        uint32_t pw[kBN / 4];
        float lsum1 = 0.f;
        if (has1) {
          lsum1 = nv1 == kBN ? block_codes_l<false, R1>(sr, nv1, c1, m, pw, sTau)
                             : block_codes_l<true, R1>(sr, nv1, c1, m, pw, sTau);
          if (!emit(j1, pw, 1.f)) { aborted = true; break; }
        }
#pragma unroll
        for (int i = 0; i < kBN / 4; ++i) {
          const float4 x = spill[i * kBM + r];
          sr[4 * i] = __float_as_uint(x.x);
          sr[4 * i + 1] = __float_as_uint(x.y);
          sr[4 * i + 2] = __float_as_uint(x.z);
          sr[4 * i + 3] = __float_as_uint(x.w);
        }
        const float lsum0 = nv0 == kBN ? block_codes_l<false, R1>(sr, nv0, c0, m, pw, sTau)
                                       : block_codes_l<true, R1>(sr, nv0, c0, m, pw, sTau);
        l = __fadd_rn(__fmaf_rn(l, alpha, lsum0), lsum1);
        if (!emit(j0, pw, alpha)) { aborted = true; break; }
        if (warp_flag(sAbort)) { aborted = true; break; }
      }
    }
    if (aborted) *sAbort = 1;
    sL[t * kBM + r] = l;
    __syncwarp();
    if (lane == 0) mbar_arrive(l_full);
  } else {
    // ======================================================== correction warps
    setmaxnreg_corr();
    const int c = (warp & 3) * 32 + lane;     // channel = TMEM lane
    const uint32_t t_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tA = tmem + L::T_ACC + t_lane;
    const float* vsc = p.v_scale + head * p.nblk * D + (c < D ? c : 0);
    float s_next = c < D ? __ldg(vsc) : 0.f;
    bool aborted = false;
    for (int j = 0; j < nkb && !aborted; ++j) {
      const float s18 = __fmul_rn(s_next, 262144.f);   // ACC = sum u v * 2^-18; exact scaling
      if (j + 1 < nkb && c < D) s_next = __ldg(vsc + (size_t)(j + 1) * D);
      for (int t = 0; t < 2; ++t) {
        const int u = 2 * j + t, e = t * kAlphaRing + j % kAlphaRing;
        if (!warp_wait(acc_full, u & 1, lim)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t tO = tmem + L::T_O + t * kBM + t_lane;
        // the block's ACC, all 128 query columns, and the first half of O
        uint32_t a[kBM];
        uint32_t oh[64];
        {
          uint32_t(&aa)[64] = *reinterpret_cast<uint32_t(*)[64]>(&a[0]);
          uint32_t(&ab)[64] = *reinterpret_cast<uint32_t(*)[64]>(&a[64]);
          tmem_st_wait();   // this thread's O stores of the previous tile-block are complete
          tmem_ld64(tA, aa);   // 64-column loads and stores: fewer, larger TMEM accesses
          tmem_ld64(tA + 64, ab);
          if (j > 0) tmem_ld64(tO, oh);
          tmem_ld_wait();
          tmem_dep64(aa);
          tmem_dep64(ab);
          tmem_dep64(oh);
        }
        // ACC is in registers: the next P V may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        // alpha and the flags of (tile t, block j): written with the codes
        // the P V just used (already complete: no wait in effect)
        if (!warp_wait(&a_full[e], (j / kAlphaRing) & 1, lim)) { aborted = true; break; }
        const int* fl = sFlag + e * 4;
        const bool moved = j > 0 && (fl[0] | fl[1] | fl[2] | fl[3]) != 0;
        const float* al = sAlpha + e * kBM;
        // O in two 64-column halves (the first already loaded): FMAs, then two stores
        auto half = [&](int hb, uint32_t(&o)[64]) {
          if (j == 0) {
#pragma unroll
            for (int i = 0; i < 64; ++i) o[i] = __float_as_uint(__fmul_rn(__uint_as_float(a[64 * hb + i]), s18));
          } else if (moved) {
#pragma unroll
            for (int i = 0; i < 64; i += 4) {
              const float4 a4 = *reinterpret_cast<const float4*>(al + 64 * hb + i);
              float x0, x1, x2, x3;
              // O alpha (one rounding), then + s ACC (one rounding)
              fma2(x0, x1, __uint_as_float(o[i]), __uint_as_float(o[i + 1]), a4.x, a4.y, 0.f, 0.f);
              fma2(x2, x3, __uint_as_float(o[i + 2]), __uint_as_float(o[i + 3]), a4.z, a4.w, 0.f, 0.f);
              fma2(x0, x1, __uint_as_float(a[64 * hb + i]), __uint_as_float(a[64 * hb + i + 1]), s18, s18, x0, x1);
              fma2(x2, x3, __uint_as_float(a[64 * hb + i + 2]), __uint_as_float(a[64 * hb + i + 3]), s18, s18, x2, x3);
              o[i] = __float_as_uint(x0);
              o[i + 1] = __float_as_uint(x1);
              o[i + 2] = __float_as_uint(x2);
              o[i + 3] = __float_as_uint(x3);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
              float x0, x1;
              fma2(x0, x1, __uint_as_float(a[64 * hb + i]), __uint_as_float(a[64 * hb + i + 1]), s18, s18,
                   __uint_as_float(o[i]), __uint_as_float(o[i + 1]));
              o[i] = __float_as_uint(x0);
              o[i + 1] = __float_as_uint(x1);
            }
          }
          tmem_st64(tO + 64 * hb, o);
        };
        half(0, oh);
        {
          uint32_t o[64];
          if (j > 0) {
            tmem_ld64(tO + 64, o);
            tmem_ld_wait();
            tmem_dep64(o);
          }
          half(1, o);
        }
        // this tile's alpha and flags of block j are consumed (the O stores
        // may still be in flight: they are waited for before O is read again)
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_empty[e]);
      }
      if (warp_flag(sAbort)) aborted = true;
    }
    tmem_st_wait();
    // ---- epilogue: out = O / l once every row's l is final ----
    if (!aborted && !warp_wait(l_full, 0, lim)) aborted = true;
    if (aborted || warp_flag(sAbort)) {
      *sAbort = 1;
    } else {
      tc_fence_after();
#pragma unroll 1
      for (int t = 0; t < 2; ++t) {
        const int row0 = blockIdx.x * kRowsPerCta + t * kBM;
        const uint32_t tO = tmem + L::T_O + t * kBM + t_lane;
#pragma unroll 1
        for (int cb = 0; cb < kBM / 32; ++cb) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * cb, o);
          tmem_wait_dep(o);
          const float* lrow = sL + t * kBM + 32 * cb;
          float* dst = p.out + (head * p.N + (size_t)(row0 + 32 * cb)) * D + c;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (row0 + 32 * cb + i < p.N && c < D) dst[(size_t)i * D] = __fdiv_rn(__uint_as_float(o[i]), lrow[i]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// Widens the packed K / V codes of one (head, 64-key block) into the exact
// shared-memory images of the attention kernel's operand tiles: K as 64 rows
// x D e4m3 subnormals (K-major, 128B / 64B swizzle) and V^T as 128 channel
// rows x 64 keys of e4m3 subnormals (64B swizzle; rows >= D are zero).
template <int D>
__global__ void __launch_bounds__(256) widen_kv_kernel(const __grid_constant__ Int4Params p, uint8_t* work) {
  using L = Int4Smem<D, 64>;   // the images do not depend on the max group
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
    *reinterpret_cast<uint4*>(img + swz<D>(rr, cg * 32)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(img + swz<D>(rr, cg * 32 + 16)) = make_uint4(o[4], o[5], o[6], o[7]);
  }
  // V^T: channel c, keys 16q .. 16q+15 (two packed words) -> one 16-byte chunk
  const uint2* vp = reinterpret_cast<const uint2*>(p.v_codes + (head * p.nblk + j) * (size_t)D * 32);
  uint8_t* vt = img + L::K_BYTES;
  for (int i = threadIdx.x; i < 128 * 4; i += blockDim.x) {
    const int c = i >> 2, q = i & 3;
    uint4 o = make_uint4(0, 0, 0, 0);
    if (c < D) {
      const uint2 w = __ldg(vp + c * 4 + q);   // keys 16q .. 16q+7 and 16q+8 .. 16q+15
      codes8_to_e4m3(w.x, o.x, o.y);
      codes8_to_e4m3(w.y, o.z, o.w);
    }
    *reinterpret_cast<uint4*>(vt + swz<64>(c, 16 * q)) = o;
  }
}

// Exhaustive-check hook: the kernels' P-code function on an array.
template <bool FMA>
__global__ void pcode_kernel(const float* d, uint8_t* u, int64_t n, Int4Params p) {
  __shared__ float tau[16];
  if (threadIdx.x < 16) tau[threadIdx.x] = p.tau[threadIdx.x];
  __syncthreads();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    u[i] = static_cast<uint8_t>(FMA ? pcode_fma(d[i], tau) : pcode(d[i], tau));
}

}  // namespace rota
