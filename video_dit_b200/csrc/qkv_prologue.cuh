// qkv_prologue.cuh -- the QKV projection of a DiT attention block with the
// RotateAttention prologue fused into its epilogue.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: the INT4 attention sits
// inside the DiT block, right after the projection that produces Q, K and V.
// Fusing the prologue (3D RoPE -> RoPE-aware rotation -> INT4 codes) into that
// projection's epilogue keeps the fp16 Q, K, V in shared memory: they are never
// written to and read back from HBM.
//
// [q | k | v] = x W^T per head: x fp16 [B*N, C] (token rows), W fp16
// [3*H*D, C] (rows h*D .. h*D+D-1 project Q of head h, H*D + h*D .. the K, and
// 2*H*D + h*D .. the V), fp32 accumulation, rounded to fp16 -- the fp16
// tensors the prologue takes -- then exactly the prologue of prologue.cuh.
//
// One CTA = 128 tokens of one head, 256 threads; the grid is (ntiles * H, B).  The K loop over C: warp 0
// loads the x tile (128 x 64) and the head's three W tiles (3 x D x 64) of each
// 64-channel step with TMA (128-byte swizzle) into a 3-stage ring; warp 1
// issues tcgen05.mma kind::f16 (Q and K as one N = 2D MMA, V as one N = D MMA,
// fp32 accumulators in TMEM, M = 128 tokens = TMEM lanes).  Then all eight
// warps move the accumulators to shared memory as fp16 tiles (token rows) and
// run the prologue on the CTA's two 64-token blocks and three tensors.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "prologue.cuh"
#include "sm100.cuh"

namespace rota {

struct QkvParams {
  CUtensorMap tm_x;   // x as [B*N rows, C], box 64 channels x 128 rows
  CUtensorMap tm_w;   // W as [3*H*D rows, C], box 64 channels x D rows
  PrologueParams pro; // the prologue's parameters (q, k, v unused)
  __half* v_out;      // fp16 V of the flagged heads [B,H,N,D] (NULL when none is flagged)
  int C;
  int ntiles;         // ceil(N / 128)
  int head_group;     // heads per raster group (see the kernel)
  uint64_t timeout_ns;
};

constexpr int kQkvThreads = kPrologueThreads;   // 256
constexpr int kQkvStages = 3;

template <int D>
struct QkvSmem {
  static constexpr int X_BYTES = 128 * 64 * 2;             // one stage of x
  static constexpr int W_BYTES = 3 * D * 64 * 2;           // the head's Q, K, V rows
  static constexpr int STAGE = X_BYTES + W_BYTES;
  static constexpr int OFF_STAGE = 0;
  // after the K loop the stages hold the fp16 tiles [3][128 tokens][D] and
  // the prologue's fp32 scratch
  static constexpr int OFF_TILE = 0;
  static constexpr int OFF_X = OFF_TILE + 3 * 128 * D * 2;
  static constexpr int SCRATCH_END = OFF_X + 64 * (D + 4) * 4;
  static constexpr int LOOP_END = kQkvStages * STAGE;
  static constexpr int OFF_RED = (SCRATCH_END > LOOP_END ? SCRATCH_END : LOOP_END);
  static constexpr int OFF_POS = OFF_RED + 64;
  static constexpr int OFF_BAR = OFF_POS + 64 * 16;
  static constexpr int NBAR = 2 * kQkvStages + 1;          // full[], empty[], done
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_TMEM + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static_assert(STAGE % 1024 == 0 && X_BYTES % 1024 == 0, "swizzle atom alignment");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

template <int D>
__global__ void __launch_bounds__(kQkvThreads, 1) qkv_prologue_kernel(const __grid_constant__ QkvParams p) {
  using L = QkvSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + kQkvStages;
  uint64_t* done = empty + kQkvStages;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  float* X = reinterpret_cast<float*>(smem + L::OFF_X);
  float* red = reinterpret_cast<float*>(smem + L::OFF_RED);
  int4* sPos = reinterpret_cast<int4*>(smem + L::OFF_POS);

  const PrologueParams& pro = p.pro;
  // Raster order: the heads are cut into groups of head_group; a group's CTAs
  // run tile by tile with the group's heads fastest, so the CTAs resident at
  // one time share few x tiles (each read from HBM once per group) and the
  // group's W rows (head_group x 3 x D x C fp16) stay in L2 for the whole
  // sweep over the tiles.
  const int b = blockIdx.y;
  int tile, h;
  {
    const int lin = blockIdx.x;
    const int g = lin / (p.head_group * p.ntiles);
    const int h0 = g * p.head_group;
    const int gh = min(p.head_group, p.pro.H - h0);
    const int r = lin - h0 * p.ntiles;
    h = h0 + r % gh;
    tile = r / gh;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = p.C / 64;
  const uint64_t lim = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQkvStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 2) {
    tmem_alloc(sTmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  bool ok = true;

  if (warp == 0) {
    // ---- TMA producer: x rows of the tile, W rows of the head's Q, K, V ----
    const int xrow = b * pro.N + tile * 128;
    for (int kk = 0; kk < nk; ++kk) {
      const int st = kk % kQkvStages;
      if (!warp_wait(&empty[st], ((kk / kQkvStages) & 1) ^ 1, lim)) { ok = false; break; }
      uint8_t* dst = smem + L::OFF_STAGE + st * L::STAGE;
      if (elect_one()) {
        mbar_arrive_expect_tx(&full[st], L::STAGE);
        tma_load_2d(dst, &p.tm_x, kk * 64, xrow, &full[st]);
#pragma unroll
        for (int m = 0; m < 3; ++m)
          tma_load_2d(dst + L::X_BYTES + m * D * 128, &p.tm_w, kk * 64, (m * pro.H + h) * D, &full[st]);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ---- MMA issuer: Q|K (N = 2D) and V (N = D), fp32 in TMEM columns [0, 3D) ----
    constexpr uint32_t ID_QK = idesc(1, 0, 0, 128, 2 * D);
    constexpr uint32_t ID_V = idesc(1, 0, 0, 128, D);
    const uint32_t hi = sdesc_hi(1024, 2);
    const uint32_t lo0 = sdesc_lo(smem_u32(smem + L::OFF_STAGE));
    for (int kk = 0; kk < nk; ++kk) {
      const int st = kk % kQkvStages;
      if (!warp_wait(&full[st], (kk / kQkvStages) & 1, lim)) { ok = false; break; }
      tc_fence_after();
      const uint32_t la = lo0 + st * (L::STAGE >> 4);
      const uint32_t lb = la + (L::X_BYTES >> 4);
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // 16 channels (32 bytes) per step inside the 128-byte rows
          const uint64_t a = (static_cast<uint64_t>(hi) << 32) | (la + 2 * k);
          const uint64_t bqk = (static_cast<uint64_t>(hi) << 32) | (lb + 2 * k);
          const uint64_t bv = (static_cast<uint64_t>(hi) << 32) | (lb + ((2 * D * 128) >> 4) + 2 * k);
          const uint32_t acc = (kk > 0 || k > 0) ? 1u : 0u;
          mma_f16(tmem, a, bqk, ID_QK, acc);
          mma_f16(tmem + 2 * D, a, bv, ID_V, acc);
        }
        mma_commit(&empty[st]);
        if (kk == nk - 1) mma_commit(done);
      }
      __syncwarp();
    }
    if (!ok && elect_one()) mma_commit(done);   // release the epilogue's wait (the result is not used)
    __syncwarp();
  }
  // ---- epilogue: accumulators -> fp16 tiles [tensor][token][D] in shared memory ----
  ok = __syncthreads_and(ok && warp_wait(done, 0, lim));
  if (ok) {
    tc_fence_after();
    const int r = (warp & 3) * 32 + lane;                   // token within the tile = TMEM lane
    const uint32_t t_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // warps 0-3: Q and the first half of V; warps 4-7: K and the second half of V
    const int col0 = warp < 4 ? 0 : D;
    __half* tiles = reinterpret_cast<__half*>(smem + L::OFF_TILE);
    auto put = [&](int tcol, __half* dst_row) {
      uint32_t v[32];
      tmem_ld32(tmem + t_lane + tcol, v);
      tmem_wait_dep(v);
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        const __half2 a = __floats2half2_rn(__uint_as_float(v[i]), __uint_as_float(v[i + 1]));
        const __half2 bb = __floats2half2_rn(__uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
        const __half2 c = __floats2half2_rn(__uint_as_float(v[i + 4]), __uint_as_float(v[i + 5]));
        const __half2 d = __floats2half2_rn(__uint_as_float(v[i + 6]), __uint_as_float(v[i + 7]));
        *reinterpret_cast<uint4*>(dst_row + i) =
            make_uint4(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&bb),
                       *reinterpret_cast<const uint32_t*>(&c), *reinterpret_cast<const uint32_t*>(&d));
      }
    };
    // the stage buffers are free: every MMA has completed (done)
    const int tq = warp < 4 ? 0 : 1;
    for (int cb = 0; cb < D; cb += 32) put(col0 + cb, tiles + ((size_t)tq * 128 + r) * D + cb);
    for (int cb = (warp < 4 ? 0 : D / 2); cb < (warp < 4 ? D / 2 : D); cb += 32)
      put(2 * D + cb, tiles + ((size_t)2 * 128 + r) * D + cb);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (!ok) {
    if (threadIdx.x == 0) set_error(kDevTimeout);
    return;
  }
  // ---- the prologue on the CTA's two 64-token blocks, Q, K and V ----
  const __half* tiles = reinterpret_cast<const __half*>(smem + L::OFF_TILE);
  const size_t head = (size_t)b * pro.H + h;
  const bool flagged = head_flagged(pro, h);
#pragma unroll 1
  for (int sb = 0; sb < 2; ++sb) {
    const int blk = tile * 2 + sb;
    if (blk >= pro.nblk) break;
#pragma unroll 1
    for (int which = 0; which < 3; ++which) {
      // the tile as the prologue addresses it: token n at src + n * D
      const __half* src = tiles + (size_t)which * 128 * D - (size_t)tile * 128 * D;
      if (which == 2 && flagged) {
        // a flagged head keeps its fp16 V for the FP16 fallback
        if (p.v_out)
          for (int i = threadIdx.x; i < 64 * D / 8; i += kQkvThreads) {
            const int rr = i / (D / 8), ch = i % (D / 8);
            const int n = blk * 64 + rr;
            if (n < pro.N)
              *reinterpret_cast<uint4*>(p.v_out + (head * pro.N + n) * D + ch * 8) =
                  *reinterpret_cast<const uint4*>(src + (size_t)n * D + ch * 8);
          }
        continue;
      }
      prologue_job<D, true>(pro, src, blk, h, b, which, X, red, sPos);
      __syncthreads();   // X, red and sPos are reused by the next job
    }
  }
}

}  // namespace rota
