// prologue.cuh -- fused 3D RoPE -> RoPE-aware rotation -> INT4 quantisation.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: Q and K carry 3D RoPE
// (head_dim split into temporal / height / width partitions), an orthogonal
// rotation inside each RoPE partition tames the partition-aligned outliers,
// and Q, K, V are quantised to INT4 before the INT4 FlashAttention.
//
// This file holds the prologue's arithmetic (RoPE of a pair, the Walsh-Hadamard
// units, the dense rotation of non-power-of-two blocks, the code of a value)
// and prologue_job, the prologue of one (64-token block, head, tensor) on
// tiles already in shared memory, which the fused QKV-projection kernel runs
// in its epilogue.  The standalone prologue runs prologue_stream.cuh's kernel
// when every rotation unit fits an 8-channel chunk, else prologue_kernel below.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "sm100.cuh"

namespace rota {

struct PrologueParams {
  const __half* q;
  const __half* k;
  const __half* v;
  uint8_t* q_codes;
  uint8_t* k_codes;
  float* q_scale;
  float* k_scale;
  uint8_t* v_codes;
  float* v_scale;
  __half* q_rope;
  __half* k_rope;
  const float* cos_tab;
  const float* sin_tab;
  int H, N, nblk;
  int grid_h, grid_w;
  int rope_dim[3];
  int had[3];
  int fused[3];      // partition a is rotated in registers while the tile is loaded
                     // (no rotation, or had[a] <= 8 and coff[a] % had[a] == 0: every
                     // unit then lies inside one 8-channel chunk)
  int any_unfused;   // some partition needs the shared-memory rotation pass
  int dense[3];      // partition a's block is not a power of two: a dense Hadamard product
  uint64_t hneg[3][64];  // its rows: bit j of row i set where H_ij = -1
  int coff[3];       // channel offset of each partition
  int toff[3];       // table offset of each axis
  float rnorm[3];    // RN(1 / sqrt(had[a]))
  uint32_t flags[8]; // bit h set: head h takes the FP16 fallback
};

constexpr int kPrologueThreads = 256;

__device__ __forceinline__ bool head_flagged(const PrologueParams& p, int h) {
  return (p.flags[h >> 5] >> (h & 31)) & 1u;
}

__device__ __forceinline__ void token_pos(const PrologueParams& p, int n, int pos[3]) {
  const int hw = p.grid_h * p.grid_w;
  pos[0] = n / hw;
  pos[1] = (n / p.grid_w) % p.grid_h;
  pos[2] = n % p.grid_w;
}

// RoPE of the pair (x0, x1) by the table angle, each product and the sum
// rounded separately (no contraction), as the quantiser definition requires.
__device__ __forceinline__ void rope_pair(float& x0, float& x1, float c, float s) {
  const float a0 = __fmul_rn(x0, c), b0 = __fmul_rn(x1, s);
  const float a1 = __fmul_rn(x0, s), b1 = __fmul_rn(x1, c);
  x0 = __fsub_rn(a0, b0);
  x1 = __fadd_rn(a1, b1);
}

// Walsh-Hadamard butterflies h = 1..G/2 and the normalisation of one rotation
// unit of G channels whose RoPE has been applied already, in place in the smem
// row.  Returns the unit's max |y|.
template <int G>
__device__ __forceinline__ float rotate_unit(float* xrow, int c0, float rnorm) {
  float y[G];
#pragma unroll
  for (int j = 0; j < G; ++j) y[j] = xrow[c0 + j];
#pragma unroll
  for (int h = 1; h < G; h <<= 1) {
#pragma unroll
    for (int j = 0; j < G; ++j) {
      if (j & h) continue;
      const float u = y[j], w = y[j + h];
      y[j] = __fadd_rn(u, w);
      y[j + h] = __fsub_rn(u, w);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < G; ++j) {
    y[j] = __fmul_rn(y[j], rnorm);
    xrow[c0 + j] = y[j];
    amax = fmaxf(amax, fabsf(y[j]));
  }
  return amax;
}

__device__ __noinline__ float rotate_unit_smem(float* xrow, int c0, int G, float rnorm) {
  float* y = xrow + c0;
  for (int h = 1; h < G; h <<= 1)
    for (int j = 0; j < G; ++j) {
      if (j & h) continue;
      const float u = y[j], w = y[j + h];
      y[j] = __fadd_rn(u, w);
      y[j + h] = __fsub_rn(u, w);
    }
  float amax = 0.f;
  for (int j = 0; j < G; ++j) {
    y[j] = __fmul_rn(y[j], rnorm);
    amax = fmaxf(amax, fabsf(y[j]));
  }
  return amax;
}

// The rotation units of one partition whose order G is not a power of two,
// by all threads of the CTA: y_i = sum_j H_ij x_j in fp32 in the order
// j = 0, 1, ..., G-1 (the first term exact, then one add of +-x_j per term),
// then y_i * rnorm.  One thread takes 8 output rows of one (token, unit); a
// round holds whole (token, unit) groups, so every input of a group is read
// before the barrier and every output stored after it.  The rows of H come as
// sign masks (bit j of row i set where H_ij = -1).  Returns the thread's max |y|.
template <int LD>
__device__ float rotate_partition_dense(float* X, int c_off, int G, int d_a, const uint64_t* neg, float rnorm,
                                        int rows) {
  const int nch = (G + 7) >> 3;
  const int per_round = (kPrologueThreads / nch) * nch;
  const int njobs = 64 * (d_a / G) * nch;          // (token, unit, 8 rows), tokens fastest within a unit
  float amax = 0.f;
#pragma unroll 1
  for (int base = 0; base < njobs; base += per_round) {
    const int job = base + static_cast<int>(threadIdx.x);
    const bool act = static_cast<int>(threadIdx.x) < per_round && job < njobs;
    int r = 0, c0 = 0, ch = 0;
    float acc[8];
    if (act) {
      const int g = job / nch;
      ch = job - g * nch;
      r = g & 63;
      c0 = c_off + (g >> 6) * G;
      if (r < rows) {
        const float* x = X + r * LD + c0;
        uint64_t m[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) m[k] = 8 * ch + k < G ? neg[8 * ch + k] : 0ull;
        const float x0 = x[0];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = (m[k] & 1ull) ? -x0 : x0;
#pragma unroll 1
        for (int j = 1; j < G; ++j) {
          const uint32_t xb = __float_as_uint(x[j]);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            acc[k] = __fadd_rn(acc[k], __uint_as_float(xb ^ (static_cast<uint32_t>(m[k] >> j) << 31)));
        }
      }
    }
    __syncthreads();
    if (act && r < rows) {
      float* x = X + r * LD + c0;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (8 * ch + k < G) {
          const float y = __fmul_rn(acc[k], rnorm);
          x[8 * ch + k] = y;
          amax = fmaxf(amax, fabsf(y));
        }
    }
    __syncthreads();
  }
  return amax;
}

// One butterfly (u, w) -> (u + w, u - w) where `on`, else unchanged.
__device__ __forceinline__ void bfly(float& u, float& w, bool on) {
  const float s = __fadd_rn(u, w), d = __fsub_rn(u, w);
  u = on ? s : u;
  w = on ? d : w;
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < kPrologueThreads / 32 ? red[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

// Sign-magnitude nibble of the code of y: c = RNE_int(RN(y * inv)) by adding
// 1.5 * 2^23 (the sum's integer part is the round-half-even integer of any
// |f| < 2^22).  |y| <= amax and inv = RN(7 / amax) bound |f| by 7 (1 + 2^-24),
// which rounds to at most 7: no clamp is needed.
__device__ __forceinline__ uint32_t code_nibble(float y, float inv) {
  const float f = __fmul_rn(y, inv);
  const int c = __float_as_int(__fadd_rn(f, 12582912.f)) - 0x4B400000;
  return static_cast<uint32_t>(abs(c)) | ((static_cast<uint32_t>(c) >> 28) & 8u);
}

// Codes of elements 0-3 (a) and 4-7 (b) -> one packed word (byte j: element j
// low, element j + 4 high).
__device__ __forceinline__ uint32_t pack8_f(float4 a, float4 b, float inv) {
  return (code_nibble(a.x, inv) | (code_nibble(b.x, inv) << 4)) |
         ((code_nibble(a.y, inv) | (code_nibble(b.y, inv) << 4)) << 8) |
         ((code_nibble(a.z, inv) | (code_nibble(b.z, inv) << 4)) << 16) |
         ((code_nibble(a.w, inv) | (code_nibble(b.w, inv) << 4)) << 24);
}

// 16 bytes of an fp16 tile row: read-only global loads, or plain loads from
// a shared-memory tile (the QKV-projection epilogue).
template <bool SMEM>
__device__ __forceinline__ uint4 load16(const __half* p) {
  if (SMEM) return *reinterpret_cast<const uint4*>(p);
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// fp16 tile [64, D] of one (head, block) -> fp32 smem rows of stride D + 4
// (16-byte aligned rows).  Every thread issues all of its 16-byte loads before
// it converts any, so a CTA waits for one memory latency rather than one per load.
template <int D, bool SMEM>
__device__ __forceinline__ void load_tile(const __half* src, int n0, int N, float* X) {
  constexpr int LD = D + 4;
  constexpr int PER = 64 * D / 8 / kPrologueThreads;
  static_assert(PER * kPrologueThreads * 8 == 64 * D, "tile split");
  uint4 u[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + k * kPrologueThreads;
    const int r = i / (D / 8), ch = i % (D / 8);
    const int n = n0 + r;
    u[k] = n < N ? load16<SMEM>(src + (size_t)n * D + ch * 8) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + k * kPrologueThreads;
    const int r = i / (D / 8), ch = i % (D / 8);
    const __half2* h2 = reinterpret_cast<const __half2*>(&u[k]);
    const float2 t0 = __half22float2(h2[0]), t1 = __half22float2(h2[1]);
    const float2 t2 = __half22float2(h2[2]), t3 = __half22float2(h2[3]);
    float4* xr = reinterpret_cast<float4*>(X + r * LD + ch * 8);
    xr[0] = make_float4(t0.x, t0.y, t1.x, t1.y);
    xr[1] = make_float4(t2.x, t2.y, t3.x, t3.y);
  }
}

// The prologue of one (64-token block blk, head (b, h), tensor which = Q / K
// / V), by all kPrologueThreads threads of the block.  src: the tensor's rows
// of this head, token n at src + n * D (SMEM: a shared-memory tile holding
// rows n0 .. n0 + 63, addressed the same way).  X, red, sPos: shared scratch.
// Not for a flagged head's V (the caller keeps the fp16 V itself).
template <int D, bool SMEM>
__device__ __forceinline__ void prologue_job(const PrologueParams& p, const __half* src, int blk, int h, int b,
                                             int which, float* X, float* red, int4* sPos) {
  constexpr int LD = D + 4;
  const size_t head = (size_t)b * p.H + h;
  const int n0 = blk * 64;
  const bool flagged = head_flagged(p, h);
  const int npad = p.nblk * 64;

  if (which < 2) {
    if (flagged) {
      // FP16 fallback head: RoPE only, stored as fp16 for the fallback kernel.
      __half* dst = (which == 0 ? p.q_rope : p.k_rope) + head * p.N * D;
      for (int i = threadIdx.x; i < 64 * D / 8; i += kPrologueThreads) {
        const int r = i / (D / 8), ch = i % (D / 8);
        const int n = n0 + r;
        if (n >= p.N) continue;
        int pos[3];
        token_pos(p, n, pos);
        uint4 u = load16<SMEM>(src + (size_t)n * D + ch * 8);
        __half2* h2 = reinterpret_cast<__half2*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = ch * 8 + 2 * j;
          const int a = c < p.coff[1] ? 0 : (c < p.coff[2] ? 1 : 2);
          const int half = p.rope_dim[a] >> 1;
          const int ti = p.toff[a] + pos[a] * half + ((c - p.coff[a]) >> 1);
          float2 t = __half22float2(h2[j]);
          rope_pair(t.x, t.y, __ldg(p.cos_tab + ti), __ldg(p.sin_tab + ti));
          h2[j] = __floats2half2_rn(t.x, t.y);
        }
        *reinterpret_cast<uint4*>(dst + (size_t)n * D + ch * 8) = u;
      }
      return;
    }
    // Each thread owns one 8-channel chunk ch of rows rb, rb + RSTEP, ...: RoPE
    // pairs never straddle a chunk, nor do the rotation units of the fused
    // partitions, so both are applied in registers before the row is stored.
    constexpr int CH = D / 8;
    constexpr int RSTEP = kPrologueThreads / CH;
    constexpr int PER = 64 / RSTEP;
    static_assert(CH * RSTEP == kPrologueThreads && PER * RSTEP == 64, "tile split");
    const int ch = threadIdx.x % CH, rb = threadIdx.x / CH;
    uint4 u[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int n = n0 + rb + k * RSTEP;
      u[k] = n < p.N ? load16<SMEM>(src + (size_t)n * D + ch * 8) : make_uint4(0, 0, 0, 0);
    }
    // token coordinates of the block's tokens, while the loads are in flight
    if (threadIdx.x < 64) {
      int pos[3];
      token_pos(p, n0 + threadIdx.x, pos);
      sPos[threadIdx.x] = make_int4(pos[0], pos[1], pos[2], 0);
    }
    // the chunk's four RoPE pairs: axis, table row base, rotation levels, norm
    int ax[4], tb[4], hf[4];
    float rn[4];
    bool l1[4], l2[4], fz[4];
    bool l3 = false, any2 = false;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = ch * 8 + 2 * q;
      const int a = c < p.coff[1] ? 0 : (c < p.coff[2] ? 1 : 2);
      const int G = p.had[a];
      ax[q] = a;
      tb[q] = p.toff[a] + ((c - p.coff[a]) >> 1);
      hf[q] = p.rope_dim[a] >> 1;
      fz[q] = p.fused[a] != 0;
      const bool rot = fz[q] && G > 1;
      l1[q] = rot;
      l2[q] = rot && G >= 4;
      if (q == 0) l3 = rot && G >= 8;
      any2 = any2 || l2[q];
      rn[q] = rot ? p.rnorm[a] : 1.f;
    }
    any2 = __any_sync(0xffffffffu, any2);
    const bool any3 = __any_sync(0xffffffffu, l3);
    __syncthreads();   // sPos

    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int r = rb + k * RSTEP;
      float y[8];
      {
        const __half2* h2 = reinterpret_cast<const __half2*>(&u[k]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 t = __half22float2(h2[j]);
          y[2 * j] = t.x;
          y[2 * j + 1] = t.y;
        }
      }
      if (n0 + r < p.N) {
        const int4 ps = sPos[r];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int pa = ax[q] == 0 ? ps.x : (ax[q] == 1 ? ps.y : ps.z);
          const int ti = tb[q] + pa * hf[q];
          rope_pair(y[2 * q], y[2 * q + 1], __ldg(p.cos_tab + ti), __ldg(p.sin_tab + ti));
        }
        // Walsh-Hadamard levels h = 1, 2, 4 inside the units of the fused partitions
#pragma unroll
        for (int q = 0; q < 4; ++q) bfly(y[2 * q], y[2 * q + 1], l1[q]);
        if (any2) {
          bfly(y[0], y[2], l2[0]);
          bfly(y[1], y[3], l2[0]);
          bfly(y[4], y[6], l2[2]);
          bfly(y[5], y[7], l2[2]);
        }
        if (any3) {
#pragma unroll
          for (int j = 0; j < 4; ++j) bfly(y[j], y[j + 4], l3);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          y[j] = __fmul_rn(y[j], rn[j >> 1]);
          if (fz[j >> 1]) amax = fmaxf(amax, fabsf(y[j]));
        }
      }
      float4* xr = reinterpret_cast<float4*>(X + r * LD + ch * 8);
      xr[0] = make_float4(y[0], y[1], y[2], y[3]);
      xr[1] = make_float4(y[4], y[5], y[6], y[7]);
    }

    // the other partitions' rotation units, (partition, unit, token) jobs in smem
    if (p.any_unfused) {
      __syncthreads();
#pragma unroll 1
      for (int a = 0; a < 3; ++a) {
        if (p.fused[a]) continue;
        const int G = p.had[a];
        if (p.dense[a]) {    // uniform: every thread takes part in the rounds
          amax = fmaxf(amax, rotate_partition_dense<LD>(X, p.coff[a], G, p.rope_dim[a], p.hneg[a], p.rnorm[a],
                                                        p.N - n0));
          continue;
        }
        const int njobs = 64 * (p.rope_dim[a] / G);
#pragma unroll 1
        for (int j = threadIdx.x; j < njobs; j += kPrologueThreads) {
          const int r = j & 63, un = j >> 6;
          if (n0 + r >= p.N) continue;
          float* xrow = X + r * LD;
          const int c0 = p.coff[a] + un * G;
          float m;
          switch (G) {
            case 2: m = rotate_unit<2>(xrow, c0, p.rnorm[a]); break;
            case 4: m = rotate_unit<4>(xrow, c0, p.rnorm[a]); break;
            case 8: m = rotate_unit<8>(xrow, c0, p.rnorm[a]); break;
            default: m = rotate_unit_smem(xrow, c0, G, p.rnorm[a]); break;
          }
          amax = fmaxf(amax, m);
        }
      }
    }
    amax = block_max(amax, red);  // includes the __syncthreads that publishes X
    const float scale = amax == 0.f ? 0.f : __fdiv_rn(amax, 7.f);
    const float inv = amax == 0.f ? 0.f : __fdiv_rn(7.f, amax);
    uint8_t* cdst = (which == 0 ? p.q_codes : p.k_codes) + (head * npad + n0) * (D / 2);
    for (int i = threadIdx.x; i < 64 * D / 16; i += kPrologueThreads) {
      const int r = i & 63, g = i >> 6;  // 16 channels -> 8 bytes
      uint2 w = make_uint2(0u, 0u);
      if (n0 + r < p.N) {
        const float4* xr = reinterpret_cast<const float4*>(X + r * LD + g * 16);
        const float4 v0 = xr[0], v1 = xr[1], v2 = xr[2], v3 = xr[3];
        w = make_uint2(pack8_f(v0, v1, inv), pack8_f(v2, v3, inv));
      }
      *reinterpret_cast<uint2*>(cdst + (size_t)r * (D / 2) + g * 8) = w;
    }
    if (threadIdx.x == 0) (which == 0 ? p.q_scale : p.k_scale)[head * p.nblk + blk] = scale;
    return;
  }

  // V: per (block, channel) scale, no RoPE, no rotation.
  if (flagged) return;
  load_tile<D, SMEM>(src, n0, p.N, X);
  __syncthreads();
  // kPrologueThreads / D neighbouring lanes share a channel, each taking 64 / TPC rows
  constexpr int TPC = kPrologueThreads / D;
  constexpr int RPT = 64 / TPC;
  static_assert(TPC * D == kPrologueThreads && RPT % 8 == 0, "V split");
  {
    const int c = threadIdx.x / TPC, part = threadIdx.x % TPC;
    const int r0 = part * RPT;
    float amax = 0.f;
#pragma unroll
    for (int r = 0; r < RPT; ++r) amax = fmaxf(amax, fabsf(X[(r0 + r) * LD + c]));
#pragma unroll
    for (int o = 1; o < TPC; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float scale = amax == 0.f ? 0.f : __fdiv_rn(amax, 7.f);
    const float inv = amax == 0.f ? 0.f : __fdiv_rn(7.f, amax);
    uint32_t w[RPT / 8];
#pragma unroll
    for (int j = 0; j < RPT / 8; ++j) {
      uint32_t wj = 0u;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int r = r0 + 8 * j + t;
        const uint32_t nb = (n0 + r < p.N) ? code_nibble(X[r * LD + c], inv) : 0u;
        wj |= nb << (t < 4 ? 8 * t : 8 * (t - 4) + 4);
      }
      w[j] = wj;
    }
    uint32_t* dst = reinterpret_cast<uint32_t*>(p.v_codes + ((head * p.nblk + blk) * D + c) * 32) + part * (RPT / 8);
#pragma unroll
    for (int j = 0; j < RPT / 8; j += 4)
      *reinterpret_cast<uint4*>(dst + j) = make_uint4(w[j], w[j + 1], w[j + 2], w[j + 3]);
    if (part == 0) p.v_scale[(head * p.nblk + blk) * D + c] = scale;
  }
}

// One CTA per (64-token block, head, tensor in {Q, K, V}), 5 per SM: the
// prologue of configurations with a partition whose rotation units do not fit
// an 8-channel chunk (they take the shared-memory rotation pass); the others
// run prologue_stream_kernel.
template <int D>
__global__ void __launch_bounds__(kPrologueThreads, 5) prologue_kernel(const __grid_constant__ PrologueParams p) {
  constexpr int LD = D + 4;
  __shared__ __align__(16) float X[64 * LD];
  __shared__ float red[kPrologueThreads / 32];
  __shared__ int4 sPos[64];
  const int h = blockIdx.y, b = blockIdx.z / 3, which = blockIdx.z % 3;
  const size_t head = (size_t)b * p.H + h;
  const __half* src = (which == 0 ? p.q : which == 1 ? p.k : p.v) + head * p.N * D;
  prologue_job<D, false>(p, src, blockIdx.x, h, b, which, X, red, sPos);
}

}  // namespace rota
