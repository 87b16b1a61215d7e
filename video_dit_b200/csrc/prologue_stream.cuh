// prologue_stream.cuh -- the standalone prologue (3D RoPE -> RoPE-aware
// rotation -> INT4 codes of Q, K, V) as a persistent, pipelined kernel.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: Q and K carry 3D RoPE,
// are rotated inside each RoPE partition, and Q, K, V are quantised to INT4
// for the INT4 FlashAttention.  The arithmetic is exactly that of prologue.cuh
// (same rounding steps in the same order, so the same codes byte for byte);
// only the data movement differs:
//
//  * a unit of work is one (batch, 64-token block, head): its Q, K and V tiles
//    (64 x D fp16 each, contiguous in memory) are streamed by cp.async.bulk
//    into a ring of NS shared-memory stages, NS tiles ahead of the compute;
//  * each CTA takes a contiguous range of units, heads fastest, so the
//    (token, RoPE pair) -> (cos, sin) table of a block is gathered once into
//    shared memory and reused by the Q and K of every head of that block;
//  * Q and K of a unit are processed together (one table read serves both),
//    rows of 8-channel chunks in registers: RoPE, the rotation units (every
//    unit lies inside one chunk: the kernel is used only when each partition's
//    block is at most 8 channels and aligned to the partition, otherwise
//    prologue_kernel of prologue.cuh runs), the block max, and the codes,
//    packed and stored straight from registers;
//  * V is read as channel pairs, its per-channel max reduced across row
//    groups in shared memory, its codes staged in a swizzled shared tile and
//    written with 16-byte stores.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "prologue.cuh"
#include "sm100.cuh"

namespace rota {

template <int D, int NT>
struct StreamSmem {
  static constexpr int NW = NT / 32;                // warps
  static constexpr int TILE = 64 * D * 2;           // one fp16 tile
  static constexpr int NS = D == 128 ? 4 : 6;       // ring stages
  static constexpr int RG = NW / (D / 64);          // V row groups (D / 64 warps each)
  static constexpr int OFF_TILE = 0;
  static constexpr int OFF_ANG = NS * TILE;         // float2 [64 tokens][D/2 pairs]: (cos, sin)
  static constexpr int OFF_VST = OFF_ANG + 64 * (D / 2) * 8;   // V codes [D channels][32 bytes], swizzled slots
  static constexpr int OFF_VRED = OFF_VST + D * 32;  // float [RG][D]: per row group channel max
  static constexpr int OFF_RED = OFF_VRED + RG * D * 4;         // float [2][2][NW]: Q/K warp max, two parities
  static constexpr int OFF_POS = OFF_RED + 2 * 2 * NW * 4;      // int4 [64]: token coordinates
  static constexpr int OFF_BAR = OFF_POS + 64 * 16;             // uint64 [NS]
  static constexpr int BYTES = OFF_BAR + NS * 8;
  static_assert(2 * (BYTES + 1024) <= 233472, "two CTAs per SM");
};

// The rotation levels of one thread's 8-channel chunk (fixed for the kernel).
struct ChunkRot {
  bool l1[4], l2[4], l3;
  float rn[4];
  bool any2, any3;   // warp-uniform: some lane has level 2 / 3
  bool all1;         // warp-uniform: every lane has level 1 on all four pairs
};

__device__ __forceinline__ ChunkRot chunk_rot(const PrologueParams& p, int ch) {
  ChunkRot c;
  c.l3 = false;
  bool any2 = false;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int ci = ch * 8 + 2 * q;
    const int a = ci < p.coff[1] ? 0 : (ci < p.coff[2] ? 1 : 2);
    const int G = p.had[a];
    const bool rot = p.fused[a] != 0 && G > 1;
    c.l1[q] = rot;
    c.l2[q] = rot && G >= 4;
    if (q == 0) c.l3 = rot && G >= 8;
    any2 = any2 || c.l2[q];
    c.rn[q] = rot ? p.rnorm[a] : 1.f;
  }
  c.any2 = __any_sync(0xffffffffu, any2);
  c.any3 = __any_sync(0xffffffffu, c.l3);
  c.all1 = __all_sync(0xffffffffu, c.l1[0] && c.l1[1] && c.l1[2] && c.l1[3]);
  return c;
}

// RoPE of the chunk's four pairs by the (cos, sin) of a0 = (c0, s0, c1, s1)
// and a1 = (c2, s2, c3, s3), then the Walsh-Hadamard levels h = 1, 2, 4 of the
// rotation units that lie inside the chunk and their normalisation.
__device__ __forceinline__ void rope_rotate8(float (&y)[8], float4 a0, float4 a1, const ChunkRot& c, bool rotate) {
  rope_pair(y[0], y[1], a0.x, a0.y);
  rope_pair(y[2], y[3], a0.z, a0.w);
  rope_pair(y[4], y[5], a1.x, a1.y);
  rope_pair(y[6], y[7], a1.z, a1.w);
  if (!rotate) return;
  if (c.all1) {   // the level every lane takes on every pair: no selects
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float u = y[2 * q], w = y[2 * q + 1];
      y[2 * q] = __fadd_rn(u, w);
      y[2 * q + 1] = __fsub_rn(u, w);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) bfly(y[2 * q], y[2 * q + 1], c.l1[q]);
  }
  if (c.any2) {
    bfly(y[0], y[2], c.l2[0]);
    bfly(y[1], y[3], c.l2[0]);
    bfly(y[4], y[6], c.l2[2]);
    bfly(y[5], y[7], c.l2[2]);
  }
  if (c.any3) {
#pragma unroll
    for (int j = 0; j < 4; ++j) bfly(y[j], y[j + 4], c.l3);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) y[j] = __fmul_rn(y[j], c.rn[j >> 1]);
}

// Eight codes -> one packed word (byte j: element j low nibble, element j + 4
// high), sign-magnitude.  Each code is c = RNE_int(RN(y * inv)), |c| <= 7: the
// sum RN(y * inv) + 1.5 * 2^23 holds c in its low bits, so its low nibble is c
// in two's complement; the eight nibbles are then turned to sign-magnitude
// together (a negative nibble x becomes (x ^ 7) + 1 = 8 | -c, which carries
// into no other nibble).
__device__ __forceinline__ uint32_t pack8_sm(const float (&y)[8], float inv) {
  uint32_t w = 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t lo = __float_as_uint(__fadd_rn(__fmul_rn(y[j], inv), 12582912.f)) & 0xFu;
    const uint32_t hi = __float_as_uint(__fadd_rn(__fmul_rn(y[j + 4], inv), 12582912.f)) & 0xFu;
    w |= (lo | (hi << 4)) << (8 * j);
  }
  const uint32_t neg = (w >> 3) & 0x11111111u;
  return (w ^ (neg * 7u)) + neg;
}

__device__ __forceinline__ void half8_to_float(uint4 u, float (&y)[8]) {
  const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 t = __half22float2(h2[j]);
    y[2 * j] = t.x;
    y[2 * j + 1] = t.y;
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <int D, int NT>
__global__ void __launch_bounds__(NT, 2)
    prologue_stream_kernel(const __grid_constant__ PrologueParams p, int units, uint64_t timeout_ns) {
  using L = StreamSmem<D, NT>;
  constexpr int NW = L::NW;
  constexpr int NS = L::NS;
  constexpr int CH = D / 8;                        // 8-channel chunks per row
  constexpr int RSTEP = NT / CH;     // rows between a thread's rows
  constexpr int PER = 64 / RSTEP;                  // rows per thread
  constexpr int WPR = D / 64;                      // V: warps per row group (32 channel pairs each)
  constexpr int RG = L::RG, RPG = 64 / RG;         // V: row groups, rows per group
  static_assert(CH * RSTEP == NT && PER * RSTEP == 64, "Q/K split");
  static_assert(WPR * RG == NT / 32 && RPG % 8 == 0, "V split");

  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* tiles = sm + L::OFF_TILE;
  float2* ang = reinterpret_cast<float2*>(sm + L::OFF_ANG);
  uint8_t* vst = sm + L::OFF_VST;
  float* vred = reinterpret_cast<float*>(sm + L::OFF_VRED);
  float* red = reinterpret_cast<float*>(sm + L::OFF_RED);
  int4* sPos = reinterpret_cast<int4*>(sm + L::OFF_POS);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * units / gridDim.x);
  const int u_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * units / gridDim.x);
  const int per_b = p.H * p.nblk;
  const int npad = p.nblk * 64;

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < NS; ++s) mbar_init(&bar[s], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // ---- producer (thread 0): the jobs Q, K and (unless the head is flagged) V
  // of each unit in order, one tile per job, job i into stage i % NS ----
  int pu = u_begin, pw = 0, issued = 0;
  auto issue = [&]() {
    if (pu < u_end && pw == 2 && head_flagged(p, pu % p.H)) {
      ++pu;
      pw = 0;
    }
    if (pu >= u_end) return;
    const int b = pu / per_b, blk = (pu / p.H) % p.nblk, h = pu % p.H;
    const int n0 = blk * 64;
    const uint32_t bytes = static_cast<uint32_t>(min(64, p.N - n0) * D * 2);
    const __half* src = (pw == 0 ? p.q : pw == 1 ? p.k : p.v) + ((static_cast<size_t>(b) * p.H + h) * p.N + n0) * D;
    const int st = issued % NS;
    mbar_arrive_expect_tx(&bar[st], bytes);
    bulk_g2s(tiles + st * L::TILE, src, bytes, &bar[st]);
    ++issued;
    if (++pw == 3) {
      ++pu;
      pw = 0;
    }
  };
  if (tid == 0)
    for (int i = 0; i < NS; ++i) issue();

  const int ch = tid % CH, rb = tid / CH;
  const ChunkRot rot = chunk_rot(p, ch);
  const int cp = (warp % WPR) * 32 + lane, rg = warp / WPR;   // V: channel pair, row group
  int jc = 0, cur_blk = -1, nred = 0;
  bool ok = true;

#pragma unroll 1
  for (int u = u_begin; u < u_end; ++u) {
    const int b = u / per_b, blk = (u / p.H) % p.nblk, h = u % p.H;
    const size_t head = static_cast<size_t>(b) * p.H + h;
    const int n0 = blk * 64;
    const bool flagged = head_flagged(p, h);

    if (blk != cur_blk) {
      // the block's (cos, sin) per (token, pair); rows past N take position 0
      __syncthreads();
      if (tid < 64) {
        int pos[3] = {0, 0, 0};
        if (n0 + tid < p.N) token_pos(p, n0 + tid, pos);
        sPos[tid] = make_int4(pos[0], pos[1], pos[2], 0);
      }
      __syncthreads();
#pragma unroll 4
      for (int e = tid; e < 64 * (D / 2); e += NT) {
        const int r = e / (D / 2), c = 2 * (e % (D / 2));
        const int a = c < p.coff[1] ? 0 : (c < p.coff[2] ? 1 : 2);
        const int4 ps = sPos[r];
        const int pa = a == 0 ? ps.x : (a == 1 ? ps.y : ps.z);
        const int ti = p.toff[a] + pa * (p.rope_dim[a] >> 1) + ((c - p.coff[a]) >> 1);
        ang[e] = make_float2(__ldg(p.cos_tab + ti), __ldg(p.sin_tab + ti));
      }
      __syncthreads();
      cur_blk = blk;
    }

    // ---------------- Q and K ----------------
    {
      const int sq = jc % NS, sk = (jc + 1) % NS;
      ok = mbar_wait(&bar[sq], (jc / NS) & 1, timeout_ns) && ok;
      ok = mbar_wait(&bar[sk], ((jc + 1) / NS) & 1, timeout_ns) && ok;
      const uint8_t* tq = tiles + sq * L::TILE;
      const uint8_t* tk = tiles + sk * L::TILE;
      float yq[PER][8], yk[PER][8];
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int r = rb + k * RSTEP;
        half8_to_float(*reinterpret_cast<const uint4*>(tq + r * (D * 2) + ch * 16), yq[k]);
        half8_to_float(*reinterpret_cast<const uint4*>(tk + r * (D * 2) + ch * 16), yk[k]);
        if (n0 + r >= p.N) {
#pragma unroll
          for (int j = 0; j < 8; ++j) yq[k][j] = yk[k][j] = 0.f;
        }
        const float4* ar = reinterpret_cast<const float4*>(ang + r * (D / 2) + ch * 4);
        const float4 a0 = ar[0], a1 = ar[1];
        rope_rotate8(yq[k], a0, a1, rot, !flagged);
        rope_rotate8(yk[k], a0, a1, rot, !flagged);
      }

      if (flagged) {
        // FP16 fallback head: the RoPE'd rows, fp16, for the fallback kernel
#pragma unroll
        for (int k = 0; k < PER; ++k) {
          const int n = n0 + rb + k * RSTEP;
          if (n >= p.N) continue;
          uint4 oq, ok4;
          __half2* hq = reinterpret_cast<__half2*>(&oq);
          __half2* hk = reinterpret_cast<__half2*>(&ok4);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            hq[j] = __floats2half2_rn(yq[k][2 * j], yq[k][2 * j + 1]);
            hk[j] = __floats2half2_rn(yk[k][2 * j], yk[k][2 * j + 1]);
          }
          *reinterpret_cast<uint4*>(p.q_rope + (head * p.N + n) * D + ch * 8) = oq;
          *reinterpret_cast<uint4*>(p.k_rope + (head * p.N + n) * D + ch * 8) = ok4;
        }
        if (!__syncthreads_and(ok)) return;
        if (tid == 0) {
          issue();
          issue();
        }
        jc += 2;
        continue;
      }

      float mq = 0.f, mk = 0.f;
#pragma unroll
      for (int k = 0; k < PER; ++k)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          mq = fmaxf(mq, fabsf(yq[k][j]));
          mk = fmaxf(mk, fabsf(yk[k][j]));
        }
      mq = warp_max(mq);
      mk = warp_max(mk);
      float* rd = red + (nred & 1) * 2 * NW;
      ++nred;
      if (lane == 0) {
        rd[warp] = mq;
        rd[NW + warp] = mk;
      }
      if (!__syncthreads_and(ok)) return;   // also: the Q and K stages are read
      if (tid == 0) {
        issue();
        issue();
      }
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        mq = fmaxf(mq, rd[w]);
        mk = fmaxf(mk, rd[NW + w]);
      }
      const float iq = mq == 0.f ? 0.f : __fdiv_rn(7.f, mq);
      const float ik = mk == 0.f ? 0.f : __fdiv_rn(7.f, mk);
      uint32_t* cq = reinterpret_cast<uint32_t*>(p.q_codes + (head * npad + n0) * (D / 2));
      uint32_t* ck = reinterpret_cast<uint32_t*>(p.k_codes + (head * npad + n0) * (D / 2));
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int r = rb + k * RSTEP;
        cq[r * (D / 8) + ch] = pack8_sm(yq[k], iq);
        ck[r * (D / 8) + ch] = pack8_sm(yk[k], ik);
      }
      if (tid == 0) {
        p.q_scale[head * p.nblk + blk] = mq == 0.f ? 0.f : __fdiv_rn(mq, 7.f);
        p.k_scale[head * p.nblk + blk] = mk == 0.f ? 0.f : __fdiv_rn(mk, 7.f);
      }
      jc += 2;
    }

    // ---------------- V: one scale per (block, channel) ----------------
    {
      const int sv = jc % NS;
      ok = mbar_wait(&bar[sv], (jc / NS) & 1, timeout_ns) && ok;
      const uint8_t* tv = tiles + sv * L::TILE;
      float x0[RPG], x1[RPG];
      float m0 = 0.f, m1 = 0.f;
#pragma unroll
      for (int i = 0; i < RPG; ++i) {
        const int r = rg * RPG + i;
        float2 t = __half22float2(*reinterpret_cast<const __half2*>(tv + r * (D * 2) + cp * 4));
        if (n0 + r >= p.N) t = make_float2(0.f, 0.f);
        x0[i] = t.x;
        x1[i] = t.y;
        m0 = fmaxf(m0, fabsf(t.x));
        m1 = fmaxf(m1, fabsf(t.y));
      }
      *reinterpret_cast<float2*>(vred + rg * D + 2 * cp) = make_float2(m0, m1);
      if (!__syncthreads_and(ok)) return;   // also: the V stage is read
      if (tid == 0) issue();
#pragma unroll
      for (int g = 0; g < RG; ++g) {
        const float2 t = *reinterpret_cast<const float2*>(vred + g * D + 2 * cp);
        m0 = fmaxf(m0, t.x);
        m1 = fmaxf(m1, t.y);
      }
      const float i0 = m0 == 0.f ? 0.f : __fdiv_rn(7.f, m0);
      const float i1 = m1 == 0.f ? 0.f : __fdiv_rn(7.f, m1);
      if (rg == 0)
        *reinterpret_cast<float2*>(p.v_scale + (head * p.nblk + blk) * D + 2 * cp) =
            make_float2(m0 == 0.f ? 0.f : __fdiv_rn(m0, 7.f), m1 == 0.f ? 0.f : __fdiv_rn(m1, 7.f));
      // codes of the row group's tokens, one word per 8 tokens, into the
      // staging tile: channel c's 32 bytes are RG slots of RPG / 2 bytes, slot
      // s stored at position s ^ (c / 2 mod RG) to spread the banks
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        const int c = 2 * cp + c2;
        const float inv = c2 == 0 ? i0 : i1;
        uint32_t wv[RPG / 8];
#pragma unroll
        for (int k = 0; k < RPG / 8; ++k) {
          float t8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) t8[j] = c2 == 0 ? x0[8 * k + j] : x1[8 * k + j];
          wv[k] = pack8_sm(t8, inv);
        }
        const int slot = rg ^ ((c >> 1) & (RG - 1));
        uint8_t* dst = vst + c * 32 + slot * (RPG / 2);
        if constexpr (RPG == 16)
          *reinterpret_cast<uint2*>(dst) = make_uint2(wv[0], wv[1]);
        else
          *reinterpret_cast<uint32_t*>(dst) = wv[0];
      }
      __syncthreads();
      // 16-byte pieces of the block's D x 32 code bytes, in memory order
      uint8_t* vdst = p.v_codes + (head * p.nblk + blk) * D * 32;
#pragma unroll
      for (int t = tid; t < D * 2; t += NT) {
        const int c = t >> 1, hh = t & 1;
        const int sw = (c >> 1) & (RG - 1);
        const uint8_t* src = vst + c * 32;
        uint4 o;
        if constexpr (RPG == 16) {
          const uint2 a = *reinterpret_cast<const uint2*>(src + ((2 * hh) ^ sw) * 8);
          const uint2 bq = *reinterpret_cast<const uint2*>(src + ((2 * hh + 1) ^ sw) * 8);
          o = make_uint4(a.x, a.y, bq.x, bq.y);
        } else {
          o.x = *reinterpret_cast<const uint32_t*>(src + ((4 * hh) ^ sw) * 4);
          o.y = *reinterpret_cast<const uint32_t*>(src + ((4 * hh + 1) ^ sw) * 4);
          o.z = *reinterpret_cast<const uint32_t*>(src + ((4 * hh + 2) ^ sw) * 4);
          o.w = *reinterpret_cast<const uint32_t*>(src + ((4 * hh + 3) ^ sw) * 4);
        }
        *reinterpret_cast<uint4*>(vdst + t * 16) = o;
      }
      jc += 1;
    }
  }
}

}  // namespace rota
