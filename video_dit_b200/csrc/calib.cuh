// calib.cuh -- per-head output error for choosing the FP16-fallback heads.
//
// "RotateAttention: RoPE-Aware Rotation and Range Rectification for INT4
// Quantized Attention in Video Generation", abstract: the INT4 FlashAttention
// uses "selective FP16 fallback for accuracy-sensitive attention blocks and
// denoising steps".  The pages give no rule for which heads are sensitive;
// this kernel measures, per (b, h), how far one output (e.g. the INT4 path's)
// lies from another (e.g. the FP16 fallback's on the same inputs), and the
// host turns those numbers into flags.
#pragma once
#include <cstdint>

namespace rota {

constexpr int kCalibThreads = 256;

// sums[2 * head] += sum (test - ref)^2 and sums[2 * head + 1] += sum ref^2
// over the head's n4 float4 groups (fp64 accumulation; blockIdx.x = head,
// blockIdx.y = a slice of the head).  sums must start at zero.
__global__ void __launch_bounds__(kCalibThreads) head_error_kernel(const float* __restrict__ test,
                                                                   const float* __restrict__ ref, uint64_t n4,
                                                                   double* __restrict__ sums) {
  const uint64_t head = blockIdx.x;
  const float4* t = reinterpret_cast<const float4*>(test) + head * n4;
  const float4* r = reinterpret_cast<const float4*>(ref) + head * n4;
  double e = 0.0, q = 0.0;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.y) * kCalibThreads + threadIdx.x; i < n4;
       i += static_cast<uint64_t>(gridDim.y) * kCalibThreads) {
    const float4 a = __ldg(t + i), b = __ldg(r + i);
    const double d0 = static_cast<double>(a.x) - b.x, d1 = static_cast<double>(a.y) - b.y;
    const double d2 = static_cast<double>(a.z) - b.z, d3 = static_cast<double>(a.w) - b.w;
    e += d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
    q += static_cast<double>(b.x) * b.x + static_cast<double>(b.y) * b.y + static_cast<double>(b.z) * b.z +
         static_cast<double>(b.w) * b.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    e += __shfl_xor_sync(0xffffffffu, e, o);
    q += __shfl_xor_sync(0xffffffffu, q, o);
  }
  __shared__ double red[2][kCalibThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red[0][warp] = e;
    red[1][warp] = q;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double es = 0.0, qs = 0.0;
    for (int w = 0; w < kCalibThreads / 32; ++w) {
      es += red[0][w];
      qs += red[1][w];
    }
    atomicAdd(sums + 2 * head, es);
    atomicAdd(sums + 2 * head + 1, qs);
  }
}

}  // namespace rota
