// prologue.cuh -- fused 3D RoPE -> RoPE-aware rotation -> INT4 quantisation.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: Q and K carry 3D RoPE
// (head_dim split into temporal / height / width partitions), an orthogonal
// rotation inside each RoPE partition tames the partition-aligned outliers,
// and Q, K, V are quantised to INT4 before the INT4 FlashAttention.
//
// One CTA per (64-token block, head, tensor in {Q, K, V}).  HBM-bound: each
// CTA reads 64 x head_dim fp16 values once (16-byte loads) and writes
// 64 x head_dim / 2 bytes of packed codes plus its scale(s).
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
  int unit[3];       // channels per rotation unit: max(2, had[a])
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

// One rotation unit of G channels of one token held in the smem row: RoPE on
// its G/2 pairs, then (if rot) the Walsh-Hadamard butterflies h = 1..G/2 and
// the normalisation.  Returns the unit's max |y|.
template <int G>
__device__ __forceinline__ float rope_rotate_unit(float* xrow, int c0, int pair0, const float* ct,
                                                  const float* st, bool rot, float rnorm) {
  float y[G];
#pragma unroll
  for (int j = 0; j < G; ++j) y[j] = xrow[c0 + j];
#pragma unroll
  for (int j = 0; j < G / 2; ++j) {
    rope_pair(y[2 * j], y[2 * j + 1], __ldg(ct + pair0 + j), __ldg(st + pair0 + j));
  }
  if (rot) {
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
#pragma unroll
    for (int j = 0; j < G; ++j) y[j] = __fmul_rn(y[j], rnorm);
  }
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < G; ++j) {
    xrow[c0 + j] = y[j];
    amax = fmaxf(amax, fabsf(y[j]));
  }
  return amax;
}

// The same unit for G >= 16, in place in the smem row (no register arrays).
__device__ __noinline__ float rope_rotate_unit_smem(float* xrow, int c0, int G, int pair0, const float* ct,
                                                   const float* st, bool rot, float rnorm) {
  float* y = xrow + c0;
  for (int j = 0; j < G / 2; ++j) {
    float x0 = y[2 * j], x1 = y[2 * j + 1];
    rope_pair(x0, x1, __ldg(ct + pair0 + j), __ldg(st + pair0 + j));
    y[2 * j] = x0;
    y[2 * j + 1] = x1;
  }
  if (rot) {
    for (int h = 1; h < G; h <<= 1)
      for (int j = 0; j < G; ++j) {
        if (j & h) continue;
        const float u = y[j], w = y[j + h];
        y[j] = __fadd_rn(u, w);
        y[j + h] = __fsub_rn(u, w);
      }
    for (int j = 0; j < G; ++j) y[j] = __fmul_rn(y[j], rnorm);
  }
  float amax = 0.f;
  for (int j = 0; j < G; ++j) amax = fmaxf(amax, fabsf(y[j]));
  return amax;
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

__device__ __forceinline__ int quant_code(float y, float inv) {
  const int c = __float2int_rn(__fmul_rn(y, inv));  // round half to even
  return max(-7, min(7, c));
}

// Sign-magnitude nibble of a code in [-7, 7]: bit 3 = sign, bits 0-2 = |v|.
__device__ __forceinline__ uint32_t nibble(int c) { return static_cast<uint32_t>(c < 0 ? 8 - c : c); }

// Eight codes -> one packed word: byte j holds element j (low nibble) and j+4 (high).
__device__ __forceinline__ uint32_t pack8(const int (&c)[8]) {
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) w |= (nibble(c[j]) | (nibble(c[j + 4]) << 4)) << (8 * j);
  return w;
}

// fp16 tile [64, D] of one (head, block) -> fp32 smem rows of stride D+1.
// Every thread issues all of its 16-byte loads before it converts any, so a
// CTA waits for one memory latency rather than one per load.
template <int D>
__device__ __forceinline__ void load_tile(const __half* src, int n0, int N, float* X) {
  constexpr int LD = D + 1;
  constexpr int PER = 64 * D / 8 / kPrologueThreads;
  static_assert(PER * kPrologueThreads * 8 == 64 * D, "tile split");
  uint4 u[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + k * kPrologueThreads;
    const int r = i / (D / 8), ch = i % (D / 8);
    const int n = n0 + r;
    u[k] = n < N ? __ldg(reinterpret_cast<const uint4*>(src + (size_t)n * D + ch * 8)) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + k * kPrologueThreads;
    const int r = i / (D / 8), ch = i % (D / 8);
    const __half2* h2 = reinterpret_cast<const __half2*>(&u[k]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 t = __half22float2(h2[j]);
      X[r * LD + ch * 8 + 2 * j] = t.x;
      X[r * LD + ch * 8 + 2 * j + 1] = t.y;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kPrologueThreads, 5) prologue_kernel(const PrologueParams p) {
  constexpr int LD = D + 1;
  __shared__ float X[64 * LD];
  __shared__ float red[kPrologueThreads / 32];

  const int blk = blockIdx.x, h = blockIdx.y;
  const int b = blockIdx.z / 3, which = blockIdx.z % 3;
  const size_t head = (size_t)b * p.H + h;
  const int n0 = blk * 64;
  const bool flagged = head_flagged(p, h);
  const int npad = p.nblk * 64;

  if (which < 2) {
    const __half* src = (which == 0 ? p.q : p.k) + head * p.N * D;
    if (flagged) {
      // FP16 fallback head: RoPE only, stored as fp16 for the fallback kernel.
      __half* dst = (which == 0 ? p.q_rope : p.k_rope) + head * p.N * D;
      for (int i = threadIdx.x; i < 64 * D / 8; i += kPrologueThreads) {
        const int r = i / (D / 8), ch = i % (D / 8);
        const int n = n0 + r;
        if (n >= p.N) continue;
        int pos[3];
        token_pos(p, n, pos);
        uint4 u = __ldg(reinterpret_cast<const uint4*>(src + (size_t)n * D + ch * 8));
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
    load_tile<D>(src, n0, p.N, X);
    __syncthreads();

    // RoPE + rotation, one (partition, unit, token) job per iteration, tokens fastest.
    float amax = 0.f;
    int pos_cache_n = -1;
    int pos[3] = {0, 0, 0};
    int jbase = 0;
#pragma unroll 1
    for (int a = 0; a < 3; ++a) {
      const int G = p.unit[a];
      const int nunits = p.rope_dim[a] / G;
      const int njobs = 64 * nunits;
      const int half = p.rope_dim[a] >> 1;
      const bool rot = p.had[a] > 1;
#pragma unroll 1
      for (int j = threadIdx.x; j < njobs; j += kPrologueThreads) {
        const int r = j & 63, u = j >> 6;
        const int n = n0 + r;
        if (n >= p.N) continue;
        if (n != pos_cache_n) {
          token_pos(p, n, pos);
          pos_cache_n = n;
        }
        float* xrow = X + r * LD;
        const int c0 = p.coff[a] + u * G;
        const float* ct = p.cos_tab + p.toff[a] + pos[a] * half;
        const float* st = p.sin_tab + p.toff[a] + pos[a] * half;
        const int pair0 = (u * G) >> 1;
        float m;
        switch (G) {
          case 2: m = rope_rotate_unit<2>(xrow, c0, pair0, ct, st, rot, p.rnorm[a]); break;
          case 4: m = rope_rotate_unit<4>(xrow, c0, pair0, ct, st, rot, p.rnorm[a]); break;
          case 8: m = rope_rotate_unit<8>(xrow, c0, pair0, ct, st, rot, p.rnorm[a]); break;
          default: m = rope_rotate_unit_smem(xrow, c0, G, pair0, ct, st, rot, p.rnorm[a]); break;
        }
        amax = fmaxf(amax, m);
      }
      jbase += njobs;
    }
    (void)jbase;
    amax = block_max(amax, red);  // includes the __syncthreads that publishes X
    const float scale = amax == 0.f ? 0.f : __fdiv_rn(amax, 7.f);
    const float inv = amax == 0.f ? 0.f : __fdiv_rn(7.f, amax);
    uint8_t* cdst = (which == 0 ? p.q_codes : p.k_codes) + (head * npad + n0) * (D / 2);
    for (int i = threadIdx.x; i < 64 * D / 16; i += kPrologueThreads) {
      const int r = i & 63, ch = i >> 6;  // 16 channels -> 8 bytes
      const float* xr = X + r * LD + ch * 16;
      uint32_t w[2] = {0u, 0u};
      if (n0 + r < p.N) {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          int c[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) c[j] = quant_code(xr[8 * g + j], inv);
          w[g] = pack8(c);
        }
      }
      *reinterpret_cast<uint2*>(cdst + (size_t)r * (D / 2) + ch * 8) = make_uint2(w[0], w[1]);
    }
    if (threadIdx.x == 0) (which == 0 ? p.q_scale : p.k_scale)[head * p.nblk + blk] = scale;
    return;
  }

  // V: per (block, channel) scale, no RoPE, no rotation.
  if (flagged) return;
  load_tile<D>(p.v + head * p.N * D, n0, p.N, X);
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
      int cs[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int r = r0 + 8 * j + t;
        cs[t] = (n0 + r < p.N) ? quant_code(X[r * LD + c], inv) : 0;
      }
      w[j] = pack8(cs);
    }
    uint32_t* dst = reinterpret_cast<uint32_t*>(p.v_codes + ((head * p.nblk + blk) * D + c) * 32) + part * (RPT / 8);
#pragma unroll
    for (int j = 0; j < RPT / 8; j += 4)
      *reinterpret_cast<uint4*>(dst + j) = make_uint4(w[j], w[j + 1], w[j + 2], w[j + 3]);
    if (part == 0) p.v_scale[(head * p.nblk + blk) * D + c] = scale;
  }
}

}  // namespace rota
