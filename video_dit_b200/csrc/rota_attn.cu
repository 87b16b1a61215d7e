// rota_attn.cu -- the C ABI (include/rota_attn.h): argument checks, the
// host-side tables (3D RoPE angles, exact P-code thresholds) and the kernel
// launches.  Builds into librota_attn.so with the three kernels
// (prologue, INT4 attention, FP16 fallback).
#include <cmath>
#include <cstdio>
#include <cstring>
#include <limits>
#include <mutex>
#include <new>
#include <type_traits>
#include <vector>
#include <algorithm>

#include <cuda_runtime.h>

#include "../../include/rota_attn.h"
#include "attn_fp16.cuh"
#include "calib.cuh"
#include "attn_int4.cuh"
#include "prologue.cuh"
#include "prologue_stream.cuh"
#include "qkv_prologue.cuh"
#include "mma_rate.cuh"

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per mbarrier wait

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int npad_of(int N) { return ((N + 63) / 64) * 64; }

float sm_scale_of(const rota_attn_desc* d) {
  return d->sm_scale > 0.f ? d->sm_scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(d->head_dim)));
}

// kappa = RN(sm_scale * log2 e): scores are dequantised straight into base-2 exponents.
float kappa_of(const rota_attn_desc* d) {
  return static_cast<float>(static_cast<double>(sm_scale_of(d)) * 1.44269504088896340736);
}

// tau[k] (k = 1..15): the smallest fp32 d with rne(15 * 2^d) >= k, i.e. with
// 15 * 2^d >= k - 1/2 (ties only occur at k = 8, d = -1, and round up to the
// even code 8).  Found by rounding log2((k - 1/2) / 15) to fp32 and stepping
// one ulp at a time against a long-double evaluation.
struct TauTable {
  float tau[16];
  TauTable() {
    tau[0] = -INFINITY;
    for (int k = 1; k <= 15; ++k) {
      const long double target = (static_cast<long double>(k) - 0.5L) / 15.0L;
      auto reaches = [&](float d) { return exp2l(static_cast<long double>(d)) >= target; };
      float f = static_cast<float>(log2l(target));
      while (!reaches(f)) f = nextafterf(f, INFINITY);
      while (reaches(nextafterf(f, -INFINITY))) f = nextafterf(f, -INFINITY);
      tau[k] = f;
    }
  }
};

const TauTable& tau_table() {
  static const TauTable t;
  return t;
}

struct Injection {
  std::mutex mu;
  int armed = 0;
  uint64_t timeout_ns = kDefaultTimeoutNs;
} g_inject;

rota_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return ROTA_OK;
  std::fprintf(stderr, "rota_attn: CUDA error: %s\n", cudaGetErrorString(e));
  return ROTA_ERR_CUDA;
}

template <typename K>
rota_status set_smem(K kernel, int bytes) {
  return cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Hadamard matrices of orders that are not powers of two (rows as sign masks:
// bit j of row i set where H_ij = -1).  The first construction that applies:
// doubling [[H, H], [H, -H]] of a supported order >= 12; Paley I for a prime
// q = n - 1 = 3 (mod 4): H = I + [[0, 1^T], [-1, Q]]; Paley II for a prime
// q = n / 2 - 1 = 1 (mod 4): the conference matrix [[0, 1^T], [1, Q]] with
// every off-diagonal entry c replaced by c [[1, 1], [1, -1]] and every
// diagonal entry by [[1, -1], [-1, -1]].  Q_ij = chi(j - i), chi the quadratic
// character mod q.  Returns false for an unsupported order.
int quad_char(long a, int q) {
  a %= q;
  if (a < 0) a += q;
  if (a == 0) return 0;
  long r = 1, b = a;
  for (long e = (q - 1) / 2; e > 0; e >>= 1) {
    if (e & 1) r = r * b % q;
    b = b * b % q;
  }
  return r == 1 ? 1 : -1;
}

bool prime(int q) {
  if (q < 2) return false;
  for (int f = 2; f * f <= q; ++f)
    if (q % f == 0) return false;
  return true;
}

bool hadamard_rows(int n, uint64_t* neg) {
  if (n <= 1 || n > 64 || is_pow2(n)) return false;
  uint64_t half[64];
  if (n % 2 == 0 && n / 2 >= 12 && hadamard_rows(n / 2, half)) {
    const int m = n / 2;
    const uint64_t lo = (m == 64) ? ~0ull : ((1ull << m) - 1);
    for (int i = 0; i < m; ++i) {
      neg[i] = half[i] | (half[i] << m);                  // [H, H]
      neg[i + m] = half[i] | ((~half[i] & lo) << m);      // [H, -H]
    }
    return true;
  }
  auto put = [&](int i, int j, int v) {
    if (v < 0) neg[i] |= 1ull << j;
  };
  for (int i = 0; i < n; ++i) neg[i] = 0;
  int q = n - 1;
  if (q % 4 == 3 && prime(q)) {
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j)
        put(i, j, i == j ? 1 : i == 0 ? 1 : j == 0 ? -1 : quad_char(static_cast<long>(j) - i, q));
    return true;
  }
  q = n / 2 - 1;
  if (n % 2 == 0 && q % 4 == 1 && prime(q)) {
    const int m = q + 1;
    for (int i = 0; i < m; ++i)
      for (int j = 0; j < m; ++j) {
        const int c = i == j ? 0 : (i == 0 || j == 0) ? 1 : quad_char(static_cast<long>(j) - i, q);
        put(2 * i, 2 * j, c == 0 ? 1 : c);
        put(2 * i, 2 * j + 1, c == 0 ? -1 : c);
        put(2 * i + 1, 2 * j, c == 0 ? -1 : c);
        put(2 * i + 1, 2 * j + 1, c == 0 ? -1 : -c);
      }
    return true;
  }
  return false;
}
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// The buffers the INT4 path reads or writes: q_scale and k_scale are touched
// one float at a time (4-byte alignment), the others with 16-byte accesses.
bool int4_buffers_ok(const rota_attn_buffers* buf, bool with_work) {
  const void* v16[] = {buf->q_codes, buf->k_codes, buf->v_codes, buf->v_scale};
  for (const void* ptr : v16)
    if (!ptr || !aligned16(ptr)) return false;
  if (!buf->q_scale || !buf->k_scale || !aligned4(buf->q_scale) || !aligned4(buf->k_scale)) return false;
  return !with_work || (buf->int4_work && aligned16(buf->int4_work));
}

// The prologue's parameters for a descriptor, flags and buffers (the input
// pointers q, k, v are left to the caller).
void fill_prologue_params(const rota_attn_desc* d, const uint8_t* head_flags, const rota_attn_buffers* buf,
                          rota::PrologueParams* pp) {
  rota::PrologueParams& p = *pp;
  p.q_codes = buf->q_codes;
  p.k_codes = buf->k_codes;
  p.q_scale = buf->q_scale;
  p.k_scale = buf->k_scale;
  p.v_codes = buf->v_codes;
  p.v_scale = buf->v_scale;
  p.q_rope = reinterpret_cast<__half*>(buf->q_rope);
  p.k_rope = reinterpret_cast<__half*>(buf->k_rope);
  p.cos_tab = buf->rope_cos;
  p.sin_tab = buf->rope_sin;
  p.H = d->H;
  p.N = d->N;
  p.nblk = npad_of(d->N) / 64;
  p.grid_h = d->grid_h;
  p.grid_w = d->grid_w;
  const int extent[3] = {d->grid_t, d->grid_h, d->grid_w};
  int coff = 0, toff = 0;
  for (int a = 0; a < 3; ++a) {
    p.rope_dim[a] = d->rope_dim[a];
    p.had[a] = d->had_block[a];
    p.coff[a] = coff;
    p.toff[a] = toff;
    p.rnorm[a] = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d->had_block[a])));
    p.fused[a] = d->had_block[a] <= 1 || (d->had_block[a] <= 8 && coff % d->had_block[a] == 0);
    p.dense[a] = hadamard_rows(d->had_block[a], p.hneg[a]) ? 1 : 0;
    if (!p.fused[a]) p.any_unfused = 1;
    coff += d->rope_dim[a];
    toff += extent[a] * (d->rope_dim[a] / 2);
  }
  for (int h = 0; h < d->H; ++h)
    if (head_flags && head_flags[h]) p.flags[h >> 5] |= 1u << (h & 31);
}

// Heads with flag == want, written to `heads`; returns their count.
int select_heads(const rota_attn_desc* d, const uint8_t* flags, int want, int16_t* heads) {
  int n = 0;
  for (int h = 0; h < d->H; ++h) {
    const int f = flags ? (flags[h] ? 1 : 0) : 0;
    if (f == want) heads[n++] = static_cast<int16_t>(h);
  }
  return n;
}

// The INT4 kernel re-balances registers between its warpgroups with
// setmaxnreg; that only works if the build gave it exactly the register count
// the split was designed for, so any other count is refused before launch.
template <typename K>
rota_status launch_int4_kernel(K kernel, int smem, dim3 grid, cudaStream_t s, const rota::Int4Params& p) {
  cudaFuncAttributes fa{};
  rota_status st = cuda_status(cudaFuncGetAttributes(&fa, kernel));
  if (st != ROTA_OK) return st;
  if (fa.numRegs != rota::kLaunchRegs) {
    std::fprintf(stderr, "rota_attn: INT4 kernel built with %d registers/thread, expected %d; not launching\n",
                 fa.numRegs, rota::kLaunchRegs);
    return ROTA_ERR_UNSUPPORTED;
  }
  if ((st = set_smem(kernel, smem)) != ROTA_OK) return st;
  kernel<<<grid, rota::kInt4Threads, smem, s>>>(p);
  return cuda_status(cudaGetLastError());
}

// The INT4 kernel instantiation for a head dim, a max group and a row-sum reading.
template <int D>
rota_status launch_int4_variant(bool g128, bool r1, dim3 grid, cudaStream_t s, const rota::Int4Params& p) {
  if (g128)
    return r1 ? launch_int4_kernel(rota::attn_int4_kernel<D, 128, true>, rota::Int4Smem<D, 128>::ALLOC, grid, s, p)
              : launch_int4_kernel(rota::attn_int4_kernel<D, 128, false>, rota::Int4Smem<D, 128>::ALLOC, grid, s, p);
  return r1 ? launch_int4_kernel(rota::attn_int4_kernel<D, 64, true>, rota::Int4Smem<D, 64>::ALLOC, grid, s, p)
            : launch_int4_kernel(rota::attn_int4_kernel<D, 64, false>, rota::Int4Smem<D, 64>::ALLOC, grid, s, p);
}

// The persistent prologue: as many CTAs as fit on the device at once (at most
// one per unit), each taking a contiguous range of (batch, block, head) units.
// The standalone prologue.  When every partition's rotation units fit an
// 8-channel chunk: the persistent kernel, as many CTAs as fit on the device
// at once (at most one per unit), each taking a contiguous range of (batch,
// block, head) units.  Otherwise the kernel with one CTA per (block, head,
// tensor), whose shared-memory rotation pass those partitions need.
// Threads per CTA of the persistent prologue (two CTAs per SM; 512 measured
// slower than 256 at head_dim 128: 0.48 against 0.44 ms at 480p).
template <int D>
constexpr int kStreamThreads = 256;

template <int D>
rota_status launch_prologue(int units, cudaStream_t s, const rota::PrologueParams& p) {
  if (p.any_unfused) {
    const dim3 grid(p.nblk, p.H, units / (p.H * p.nblk) * 3);
    rota::prologue_kernel<D><<<grid, rota::kPrologueThreads, 0, s>>>(p);
    return cuda_status(cudaGetLastError());
  }
  constexpr int NT = kStreamThreads<D>;
  using L = rota::StreamSmem<D, NT>;
  auto kernel = rota::prologue_stream_kernel<D, NT>;
  rota_status st = set_smem(kernel, L::BYTES);
  if (st != ROTA_OK) return st;
  int dev = 0, nsm = 0, per_sm = 0;
  if ((st = cuda_status(cudaGetDevice(&dev))) != ROTA_OK) return st;
  if ((st = cuda_status(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev))) != ROTA_OK) return st;
  if ((st = cuda_status(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, NT, L::BYTES))) != ROTA_OK)
    return st;
  const int grid = std::max(1, std::min(units, nsm * std::max(per_sm, 1)));
  kernel<<<grid, NT, L::BYTES, s>>>(p, units, kDefaultTimeoutNs);
  return cuda_status(cudaGetLastError());
}

}  // namespace

namespace {

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// [rows, D] fp16 tensor, boxes of 64 channels x box_rows rows, 128-byte swizzle.
rota_status make_fp16_map(CUtensorMap* m, const void* base, uint64_t rows, int D, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return ROTA_ERR_CUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ROTA_OK : ROTA_ERR_CUDA;
}

template <int D>
rota_status launch_fp16_kernel(const rota::Fp16Params& p, dim3 grid, cudaStream_t s) {
  using L = rota::F16Smem<D>;
  rota_status st = set_smem(rota::attn_fp16_kernel<D>, L::ALLOC);
  if (st != ROTA_OK) return st;
  rota::attn_fp16_kernel<D><<<grid, rota::kF16Threads, L::ALLOC, s>>>(p);
  return cuda_status(cudaGetLastError());
}

}  // namespace

extern "C" {

const char* rota_attn_status_string(rota_status s) {
  switch (s) {
    case ROTA_OK: return "ok";
    case ROTA_ERR_INVALID_ARG: return "invalid argument";
    case ROTA_ERR_UNSUPPORTED: return "unsupported configuration";
    case ROTA_ERR_CUDA: return "CUDA runtime error";
    case ROTA_ERR_TIMEOUT: return "device wait timed out";
    case ROTA_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

rota_status rota_attn_validate(const rota_attn_desc* d) {
  if (!d) return ROTA_ERR_INVALID_ARG;
  if (d->B < 1 || d->H < 1 || d->N < 1 || d->head_dim < 1) return ROTA_ERR_INVALID_ARG;
  if (d->grid_t < 1 || d->grid_h < 1 || d->grid_w < 1) return ROTA_ERR_INVALID_ARG;
  if (static_cast<long long>(d->grid_t) * d->grid_h * d->grid_w != d->N) return ROTA_ERR_INVALID_ARG;
  int sum = 0;
  for (int a = 0; a < 3; ++a) {
    if (d->rope_dim[a] < 2 || d->rope_dim[a] % 2) return ROTA_ERR_INVALID_ARG;
    uint64_t rows[64];
    const int hb = d->had_block[a];
    if (hb < 1 || hb > 64 || d->rope_dim[a] % hb || !(is_pow2(hb) || hadamard_rows(hb, rows)))
      return ROTA_ERR_INVALID_ARG;
    sum += d->rope_dim[a];
  }
  if (sum != d->head_dim) return ROTA_ERR_INVALID_ARG;
  if (!(d->rope_theta > 0.f) || !std::isfinite(d->rope_theta)) return ROTA_ERR_INVALID_ARG;
  if (!(d->sm_scale >= 0.f) || !std::isfinite(d->sm_scale)) return ROTA_ERR_INVALID_ARG;
  for (int a = 0; a < 3; ++a)
    if (!std::isfinite(d->rope_phase[a])) return ROTA_ERR_INVALID_ARG;
  if (d->quant_block < 0 || d->max_group < 0 || d->row_sum < 0 || d->row_sum > 1) return ROTA_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return ROTA_ERR_UNSUPPORTED;
  if (d->quant_block != 0 && d->quant_block != 64) return ROTA_ERR_UNSUPPORTED;
  if (d->max_group != 0 && d->max_group != 64 && d->max_group != 128) return ROTA_ERR_UNSUPPORTED;
  if (d->H > 256) return ROTA_ERR_UNSUPPORTED;
  if (static_cast<long long>(d->B) * d->H * npad_of(d->N) * d->head_dim > (1ll << 40)) return ROTA_ERR_UNSUPPORTED;
  if (d->B > 65535) return ROTA_ERR_UNSUPPORTED;
  return ROTA_OK;
}

rota_status rota_attn_buffer_sizes(const rota_attn_desc* d, size_t* bytes) {
  const rota_status st = rota_attn_validate(d);
  if (st != ROTA_OK) return st;
  if (!bytes) return ROTA_ERR_INVALID_ARG;
  const size_t heads = static_cast<size_t>(d->B) * d->H;
  const size_t npad = npad_of(d->N), nblk = npad / 64, D = d->head_dim;
  bytes[ROTA_BUF_Q_CODES] = heads * npad * D / 2;
  bytes[ROTA_BUF_K_CODES] = heads * npad * D / 2;
  bytes[ROTA_BUF_Q_SCALE] = heads * nblk * 4;
  bytes[ROTA_BUF_K_SCALE] = heads * nblk * 4;
  bytes[ROTA_BUF_V_CODES] = heads * nblk * D * 32;
  bytes[ROTA_BUF_V_SCALE] = heads * nblk * D * 4;
  bytes[ROTA_BUF_Q_ROPE] = heads * d->N * D * 2;
  bytes[ROTA_BUF_K_ROPE] = heads * d->N * D * 2;
  bytes[ROTA_BUF_ROPE_TABLE] = 4 * (static_cast<size_t>(d->grid_t) * (d->rope_dim[0] / 2) +
                                    static_cast<size_t>(d->grid_h) * (d->rope_dim[1] / 2) +
                                    static_cast<size_t>(d->grid_w) * (d->rope_dim[2] / 2));
  bytes[ROTA_BUF_INT4_WORK] = heads * nblk * (D == 128 ? rota::Int4Smem<128, 64>::IMG_BYTES : rota::Int4Smem<64, 64>::IMG_BYTES);
  return ROTA_OK;
}

rota_status rota_attn_build_rope_tables(const rota_attn_desc* d, float* host_cos, float* host_sin) {
  const rota_status st = rota_attn_validate(d);
  if (st != ROTA_OK) return st;
  if (!host_cos || !host_sin) return ROTA_ERR_INVALID_ARG;
  const int extent[3] = {d->grid_t, d->grid_h, d->grid_w};
  const double theta = static_cast<double>(d->rope_theta);
  size_t base = 0;
  for (int a = 0; a < 3; ++a) {
    const int half = d->rope_dim[a] / 2;
    const double phase = static_cast<double>(d->rope_phase[a]);   // the merged per-pair rotation
    for (int i = 0; i < half; ++i) {
      // omega_i = theta^(-2i / d_a), evaluated in double
      const double omega = std::pow(theta, -static_cast<double>(2 * i) / static_cast<double>(d->rope_dim[a]));
      for (int pos = 0; pos < extent[a]; ++pos) {
        const double angle = static_cast<double>(pos) * omega + phase;
        host_cos[base + static_cast<size_t>(pos) * half + i] = static_cast<float>(std::cos(angle));
        host_sin[base + static_cast<size_t>(pos) * half + i] = static_cast<float>(std::sin(angle));
      }
    }
    base += static_cast<size_t>(extent[a]) * half;
  }
  return ROTA_OK;
}

rota_status rota_attn_prepare_qk(const rota_attn_desc* d, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 const uint8_t* head_flags, const rota_attn_buffers* buf, void* stream) {
  rota_status st = rota_attn_validate(d);
  if (st != ROTA_OK) return st;
  if (!buf || !q || !k || !v || !buf->rope_cos || !buf->rope_sin) return ROTA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return ROTA_ERR_INVALID_ARG;
  int16_t tmp[256];
  const int n_int4 = select_heads(d, head_flags, 0, tmp);
  const int n_fp16 = d->H - n_int4;
  if (n_int4 > 0 && !int4_buffers_ok(buf, false)) return ROTA_ERR_INVALID_ARG;
  if (n_fp16 > 0 && (!buf->q_rope || !buf->k_rope || !aligned16(buf->q_rope) || !aligned16(buf->k_rope)))
    return ROTA_ERR_INVALID_ARG;

  rota::PrologueParams p{};
  fill_prologue_params(d, head_flags, buf, &p);
  p.q = reinterpret_cast<const __half*>(q);
  p.k = reinterpret_cast<const __half*>(k);
  p.v = reinterpret_cast<const __half*>(v);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int units = d->B * d->H * p.nblk;
  return d->head_dim == 128 ? launch_prologue<128>(units, s, p) : launch_prologue<64>(units, s, p);
}

rota_status rota_attn_qkv_prepare(const rota_attn_desc* d, const uint16_t* x, const uint16_t* w, int32_t C,
                                  const uint8_t* head_flags, const rota_attn_buffers* buf, uint16_t* v_out,
                                  void* stream) {
  rota_status st = rota_attn_validate(d);
  if (st != ROTA_OK) return st;
  if (!buf || !x || !w || !buf->rope_cos || !buf->rope_sin) return ROTA_ERR_INVALID_ARG;
  if (C < 64 || C % 64 != 0 || !aligned16(x) || !aligned16(w)) return ROTA_ERR_INVALID_ARG;
  if (static_cast<long long>(C) > (1ll << 20)) return ROTA_ERR_UNSUPPORTED;
  int16_t tmp[256];
  const int n_int4 = select_heads(d, head_flags, 0, tmp);
  const int n_fp16 = d->H - n_int4;
  if (n_int4 > 0 && !int4_buffers_ok(buf, false)) return ROTA_ERR_INVALID_ARG;
  if (n_fp16 > 0 && (!buf->q_rope || !buf->k_rope || !v_out || !aligned16(buf->q_rope) || !aligned16(buf->k_rope) ||
                     !aligned16(v_out)))
    return ROTA_ERR_INVALID_ARG;
  static rota::QkvParams p;   // large (tensor maps, prologue tables); filled under a lock
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  p = rota::QkvParams{};
  fill_prologue_params(d, head_flags, buf, &p.pro);
  p.v_out = reinterpret_cast<__half*>(v_out);
  p.C = C;
  p.timeout_ns = kDefaultTimeoutNs;
  const int D = d->head_dim;
  if ((st = make_fp16_map(&p.tm_x, x, static_cast<uint64_t>(d->B) * d->N, C, 128)) != ROTA_OK) return st;
  if ((st = make_fp16_map(&p.tm_w, w, static_cast<uint64_t>(3) * d->H * D, C, static_cast<uint32_t>(D))) != ROTA_OK)
    return st;
  // heads per raster group: the group's W rows should take at most ~40 MB of L2
  const long long w_head = 3ll * D * C * 2;
  const int ngroups = static_cast<int>((d->H * w_head + (40ll << 20) - 1) / (40ll << 20));
  p.ntiles = (d->N + 127) / 128;
  p.head_group = (d->H + ngroups - 1) / ngroups;
  const dim3 grid(p.ntiles * d->H, d->B);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (D == 128) {
    if ((st = set_smem(rota::qkv_prologue_kernel<128>, rota::QkvSmem<128>::ALLOC)) != ROTA_OK) return st;
    rota::qkv_prologue_kernel<128><<<grid, rota::kQkvThreads, rota::QkvSmem<128>::ALLOC, s>>>(p);
  } else {
    if ((st = set_smem(rota::qkv_prologue_kernel<64>, rota::QkvSmem<64>::ALLOC)) != ROTA_OK) return st;
    rota::qkv_prologue_kernel<64><<<grid, rota::kQkvThreads, rota::QkvSmem<64>::ALLOC, s>>>(p);
  }
  return cuda_status(cudaGetLastError());
}

// part: 1 = widen only, 2 = attention only, 3 = both
static rota_status launch_int4(const rota_attn_desc* d, const rota_attn_buffers* buf, const uint8_t* head_flags,
                               float* out, void* stream, bool dump, int b, int h, int r0, int nr, int32_t* s_out,
                               uint8_t* p_out, int part = 3) {
  rota_status st = rota_attn_validate(d);
  if (st != ROTA_OK) return st;
  if (!buf || ((part & 2) && (!out || !aligned16(out)))) return ROTA_ERR_INVALID_ARG;
  if (!int4_buffers_ok(buf, true)) return ROTA_ERR_INVALID_ARG;

  static rota::Int4Params p;  // large (heads list); filled under a lock below
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  p = rota::Int4Params{};
  p.q_codes = buf->q_codes;
  p.k_codes = buf->k_codes;
  p.q_scale = buf->q_scale;
  p.k_scale = buf->k_scale;
  p.v_codes = buf->v_codes;
  p.v_scale = buf->v_scale;
  p.work = buf->int4_work;
  p.out = out;
  p.H = d->H;
  p.N = d->N;
  p.nblk = npad_of(d->N) / 64;
  p.kappa = kappa_of(d);
  std::memcpy(p.tau, tau_table().tau, sizeof(p.tau));
  {
    std::lock_guard<std::mutex> g(g_inject.mu);
    p.timeout_ns = g_inject.armed ? g_inject.timeout_ns : kDefaultTimeoutNs;
    p.inject_skip = g_inject.armed;
    g_inject.armed = 0;
  }
  int batches = d->B;
  if (dump) {
    if (b < 0 || b >= d->B || h < 0 || h >= d->H || r0 < 0 || nr < 1 || r0 + nr > d->N || !s_out || !p_out)
      return ROTA_ERR_INVALID_ARG;
    p.nheads = 1;
    p.heads[0] = static_cast<int16_t>(h);
    p.s_dump = s_out;
    p.p_dump = p_out;
    p.dbg_r0 = r0;
    p.dbg_nr = nr;
    batches = 1;
    // the kernel indexes batch by blockIdx.z; shift the base pointers to batch b
    const size_t hs = static_cast<size_t>(b) * d->H;
    const size_t npad = npad_of(d->N), nblk = npad / 64, D = d->head_dim;
    p.q_codes += hs * npad * D / 2;
    p.k_codes += hs * npad * D / 2;
    p.q_scale += hs * nblk;
    p.k_scale += hs * nblk;
    p.v_codes += hs * nblk * D * 32;
    p.v_scale += hs * nblk * D;
    p.work += hs * nblk * (D == 128 ? rota::Int4Smem<128, 64>::IMG_BYTES : rota::Int4Smem<64, 64>::IMG_BYTES);
    p.out += hs * d->N * D;
  } else {
    p.nheads = select_heads(d, head_flags, 0, p.heads);
    if (p.nheads == 0) return ROTA_OK;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // 1. widen the K / V codes of the selected heads once
  if (part & 1) {
    const dim3 wgrid(p.nblk, p.nheads, batches);
    if (d->head_dim == 128)
      rota::widen_kv_kernel<128><<<wgrid, 256, 0, s>>>(p, const_cast<uint8_t*>(p.work));
    else
      rota::widen_kv_kernel<64><<<wgrid, 256, 0, s>>>(p, const_cast<uint8_t*>(p.work));
    if ((st = cuda_status(cudaGetLastError())) != ROTA_OK) return st;
  }
  if (!(part & 2)) return ROTA_OK;
  // 2. attention
  const dim3 grid((d->N + rota::kRowsPerCta - 1) / rota::kRowsPerCta, p.nheads, batches);
  // the debug dump runs the same kernel with its dump pointers set
  const bool g128 = d->max_group == 128, r1 = d->row_sum != 0;
  if (d->head_dim == 128)
    st = launch_int4_variant<128>(g128, r1, grid, s, p);
  else
    st = launch_int4_variant<64>(g128, r1, grid, s, p);
  return st;
}

rota_status rota_attn_fwd_int4(const rota_attn_desc* d, const rota_attn_buffers* buf, const uint8_t* head_flags,
                               float* out, void* stream) {
  return launch_int4(d, buf, head_flags, out, stream, false, 0, 0, 0, 0, nullptr, nullptr);
}

rota_status rota_attn_int4_widen(const rota_attn_desc* d, const rota_attn_buffers* buf, const uint8_t* head_flags,
                                 void* stream) {
  return launch_int4(d, buf, head_flags, nullptr, stream, false, 0, 0, 0, 0, nullptr, nullptr, 1);
}

rota_status rota_attn_int4_attend(const rota_attn_desc* d, const rota_attn_buffers* buf, const uint8_t* head_flags,
                                  float* out, void* stream) {
  return launch_int4(d, buf, head_flags, out, stream, false, 0, 0, 0, 0, nullptr, nullptr, 2);
}

rota_status rota_attn_debug_dump_int4(const rota_attn_desc* d, const rota_attn_buffers* buf, int32_t b, int32_t h,
                                      int32_t r0, int32_t nr, int32_t* s_out, uint8_t* p_out, float* out,
                                      void* stream) {
  return launch_int4(d, buf, nullptr, out, stream, true, b, h, r0, nr, s_out, p_out);
}

rota_status rota_attn_fwd_fp16_fallback(const rota_attn_desc* d, const rota_attn_buffers* buf, const uint16_t* v,
                                        const uint8_t* head_flags, float* out, void* stream) {
  rota_status st = rota_attn_validate(d);
  if (st != ROTA_OK) return st;
  if (!buf || !v || !out || !aligned16(v) || !aligned16(out)) return ROTA_ERR_INVALID_ARG;
  static rota::Fp16Params p;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  p = rota::Fp16Params{};
  p.nheads = select_heads(d, head_flags, 1, p.heads);
  if (p.nheads == 0) return ROTA_OK;
  if (!buf->q_rope || !buf->k_rope || !aligned16(buf->q_rope) || !aligned16(buf->k_rope)) return ROTA_ERR_INVALID_ARG;
  const uint64_t rows = static_cast<uint64_t>(d->B) * d->H * d->N;
  if ((st = make_fp16_map(&p.tm_q, buf->q_rope, rows, d->head_dim, rota::kBM)) != ROTA_OK) return st;
  if ((st = make_fp16_map(&p.tm_k, buf->k_rope, rows, d->head_dim, rota::kBN)) != ROTA_OK) return st;
  if ((st = make_fp16_map(&p.tm_v, v, rows, d->head_dim, rota::kBN)) != ROTA_OK) return st;
  p.out = out;
  p.H = d->H;
  p.N = d->N;
  p.scale_log2 = kappa_of(d);
  p.timeout_ns = kDefaultTimeoutNs;
  const dim3 grid((d->N + 2 * rota::kBM - 1) / (2 * rota::kBM), p.nheads, d->B);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d->head_dim == 128 ? launch_fp16_kernel<128>(p, grid, s) : launch_fp16_kernel<64>(p, grid, s);
}

// ---------------------------------------------------------------------------
// Host-to-host forward: the heads are processed in chunks, with the copies of
// the neighbouring chunks on two copy streams while a chunk computes.
// ---------------------------------------------------------------------------
struct rota_attn_pipeline {
  int device = 0;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaStream_t comp2 = nullptr;       // odd chunks compute here, even ones on the caller's stream
  std::vector<cudaEvent_t> events;   // 2 per chunk + 2
};

rota_status rota_attn_pipeline_create(int32_t max_chunks, rota_attn_pipeline** out) {
  if (!out || max_chunks < 1 || max_chunks > (1 << 16)) return ROTA_ERR_INVALID_ARG;
  *out = nullptr;
  auto* pl = new (std::nothrow) rota_attn_pipeline;
  if (!pl) return ROTA_ERR_CUDA;
  cudaError_t e = cudaGetDevice(&pl->device);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&pl->h2d, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&pl->d2h, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&pl->comp2, cudaStreamNonBlocking);
  for (int i = 0; e == cudaSuccess && i < 2 * max_chunks + 2; ++i) {
    cudaEvent_t ev = nullptr;
    e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    if (e == cudaSuccess) pl->events.push_back(ev);
  }
  if (e != cudaSuccess) {
    rota_attn_pipeline_destroy(pl);
    return cuda_status(e);
  }
  *out = pl;
  return ROTA_OK;
}

rota_status rota_attn_pipeline_destroy(rota_attn_pipeline* pl) {
  if (!pl) return ROTA_OK;
  cudaError_t first = cudaSuccess;
  auto keep = [&](cudaError_t e) { if (first == cudaSuccess) first = e; };
  for (cudaEvent_t ev : pl->events) keep(cudaEventDestroy(ev));
  if (pl->h2d) keep(cudaStreamDestroy(pl->h2d));
  if (pl->d2h) keep(cudaStreamDestroy(pl->d2h));
  if (pl->comp2) keep(cudaStreamDestroy(pl->comp2));
  delete pl;
  return cuda_status(first);
}

int32_t rota_attn_pipeline_chunk_heads(const rota_attn_desc* d, int32_t num_sms) {
  if (rota_attn_validate(d) != ROTA_OK) return 0;
  if (num_sms < 1) num_sms = 148;
  // Consecutive chunks compute on two streams, so the attention waves of all
  // chunks pack about as tightly as one call on the whole problem and the
  // chunk size does not change them.  What it changes: the copies before the
  // first chunk and after the last are not hidden (about 1.4 heads of
  // attention per head of chunk: fp16 Q/K/V in and fp32 O out over PCIe
  // against one head's attention, in waves of cph / num_sms), and every chunk
  // pays its own prologue, widening and launches (about 0.05 waves).
  const double cph = static_cast<double>((d->N + rota::kRowsPerCta - 1) / rota::kRowsPerCta);
  int32_t best = 1;
  double best_cost = 1e300;
  for (int32_t h = 1; h <= d->H; ++h) {
    const double chunks = static_cast<double>(d->B) * ((d->H + h - 1) / h);
    const double cost = 1.4 * h * cph / num_sms + 0.05 * chunks;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = h;
    }
  }
  return best;
}

rota_status rota_attn_forward_host(const rota_attn_desc* d, const uint16_t* q_host, const uint16_t* k_host,
                                   const uint16_t* v_host, const uint8_t* head_flags, float* out_host,
                                   uint16_t* q_dev, uint16_t* k_dev, uint16_t* v_dev, float* out_dev,
                                   const rota_attn_buffers* buf, int32_t heads_per_chunk, rota_attn_pipeline* pl,
                                   void* stream) {
  rota_status st = rota_attn_validate(d);
  if (st != ROTA_OK) return st;
  if (!buf || !pl || !q_host || !k_host || !v_host || !out_host || !q_dev || !k_dev || !v_dev || !out_dev)
    return ROTA_ERR_INVALID_ARG;
  if (heads_per_chunk < 0) return ROTA_ERR_INVALID_ARG;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev != pl->device) return ROTA_ERR_INVALID_ARG;
  int nsm = 148;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int32_t hpc = heads_per_chunk ? std::min(heads_per_chunk, d->H) : rota_attn_pipeline_chunk_heads(d, nsm);
  const int32_t chunks_per_b = (d->H + hpc - 1) / hpc;
  const long long nchunks = static_cast<long long>(d->B) * chunks_per_b;
  if (2 * nchunks + 2 > static_cast<long long>(pl->events.size())) return ROTA_ERR_UNSUPPORTED;

  size_t sz[ROTA_BUF_COUNT];
  if ((st = rota_attn_buffer_sizes(d, sz)) != ROTA_OK) return st;
  const size_t heads = static_cast<size_t>(d->B) * d->H;
  const size_t elems_per_head = static_cast<size_t>(d->N) * d->head_dim;
  auto shift = [&](auto* ptr, int buf_index, size_t head) {
    using T = std::remove_pointer_t<decltype(ptr)>;
    if (!ptr) return ptr;
    return reinterpret_cast<T*>(reinterpret_cast<std::conditional_t<std::is_const_v<T>, const uint8_t*, uint8_t*>>(ptr) +
                                sz[buf_index] / heads * head);
  };

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaEvent_t* ev = pl->events.data();
  cudaEvent_t ev_start = ev[0], ev_end = ev[1];
  // everything already on `stream` (an earlier call reading q_dev ... out_dev) comes first
  if ((e = cudaEventRecord(ev_start, s)) != cudaSuccess) return cuda_status(e);
  if ((e = cudaStreamWaitEvent(pl->h2d, ev_start, 0)) != cudaSuccess) return cuda_status(e);
  if ((e = cudaStreamWaitEvent(pl->d2h, ev_start, 0)) != cudaSuccess) return cuda_status(e);
  if ((e = cudaStreamWaitEvent(pl->comp2, ev_start, 0)) != cudaSuccess) return cuda_status(e);

  rota_status result = ROTA_OK;
  long long c = 0;
  for (int32_t b = 0; b < d->B && result == ROTA_OK; ++b) {
    for (int32_t h0 = 0; h0 < d->H && result == ROTA_OK; h0 += hpc, ++c) {
      const int32_t nh = std::min(hpc, d->H - h0);
      const size_t head = static_cast<size_t>(b) * d->H + h0;
      const size_t off = head * elems_per_head, n_in = nh * elems_per_head;
      cudaEvent_t ev_in = ev[2 + 2 * c], ev_done = ev[3 + 2 * c];
      // consecutive chunks compute on two streams, so that the next chunk's
      // kernels fill the SMs the last wave of this chunk's attention leaves idle
      cudaStream_t cs = (c & 1) ? pl->comp2 : s;
      // inputs of the chunk
      e = cudaMemcpyAsync(q_dev + off, q_host + off, n_in * 2, cudaMemcpyHostToDevice, pl->h2d);
      if (e == cudaSuccess) e = cudaMemcpyAsync(k_dev + off, k_host + off, n_in * 2, cudaMemcpyHostToDevice, pl->h2d);
      if (e == cudaSuccess) e = cudaMemcpyAsync(v_dev + off, v_host + off, n_in * 2, cudaMemcpyHostToDevice, pl->h2d);
      if (e == cudaSuccess) e = cudaEventRecord(ev_in, pl->h2d);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_in, 0);
      if (e != cudaSuccess) { result = cuda_status(e); break; }
      // the chunk as a problem of its own: one batch entry, nh heads
      rota_attn_desc cd = *d;
      cd.B = 1;
      cd.H = nh;
      rota_attn_buffers cb = *buf;
      cb.q_codes = shift(buf->q_codes, ROTA_BUF_Q_CODES, head);
      cb.k_codes = shift(buf->k_codes, ROTA_BUF_K_CODES, head);
      cb.q_scale = shift(buf->q_scale, ROTA_BUF_Q_SCALE, head);
      cb.k_scale = shift(buf->k_scale, ROTA_BUF_K_SCALE, head);
      cb.v_codes = shift(buf->v_codes, ROTA_BUF_V_CODES, head);
      cb.v_scale = shift(buf->v_scale, ROTA_BUF_V_SCALE, head);
      cb.q_rope = shift(buf->q_rope, ROTA_BUF_Q_ROPE, head);
      cb.k_rope = shift(buf->k_rope, ROTA_BUF_K_ROPE, head);
      cb.int4_work = shift(buf->int4_work, ROTA_BUF_INT4_WORK, head);
      const uint8_t* flags = head_flags ? head_flags + h0 : nullptr;
      result = rota_attn_prepare_qk(&cd, q_dev + off, k_dev + off, v_dev + off, flags, &cb, cs);
      if (result == ROTA_OK) result = rota_attn_fwd_int4(&cd, &cb, flags, out_dev + off, cs);
      if (result == ROTA_OK) result = rota_attn_fwd_fp16_fallback(&cd, &cb, v_dev + off, flags, out_dev + off, cs);
      if (result != ROTA_OK) break;
      // its output
      e = cudaEventRecord(ev_done, cs);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(pl->d2h, ev_done, 0);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(out_host + off, out_dev + off, n_in * 4, cudaMemcpyDeviceToHost, pl->d2h);
      if (e != cudaSuccess) result = cuda_status(e);
    }
  }
  // `stream` continues after the last copy-out (also on an error path, so that
  // both copy streams are joined before the caller reuses the buffers)
  e = cudaEventRecord(ev_end, pl->d2h);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_end, 0);
  if (e == cudaSuccess) e = cudaEventRecord(ev_end, pl->h2d);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_end, 0);
  if (e == cudaSuccess) e = cudaEventRecord(ev_end, pl->comp2);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_end, 0);
  if (result == ROTA_OK && e != cudaSuccess) result = cuda_status(e);
  return result;
}

// ---------------------------------------------------------------------------
// Choosing the FP16-fallback heads from a calibration call.
// ---------------------------------------------------------------------------
rota_status rota_attn_head_error(const rota_attn_desc* d, const float* out_test, const float* out_ref,
                                 double* sums, void* stream) {
  rota_status st = rota_attn_validate(d);
  if (st != ROTA_OK) return st;
  if (!out_test || !out_ref || !sums || !aligned16(out_test) || !aligned16(out_ref) ||
      (reinterpret_cast<uintptr_t>(sums) & 7u))
    return ROTA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint64_t heads = static_cast<uint64_t>(d->B) * d->H;
  const uint64_t n4 = static_cast<uint64_t>(d->N) * d->head_dim / 4;
  cudaError_t e = cudaMemsetAsync(sums, 0, heads * 2 * sizeof(double), s);
  if (e != cudaSuccess) return cuda_status(e);
  const uint64_t slices = std::min<uint64_t>(64, (n4 + 8 * rota::kCalibThreads - 1) / (8 * rota::kCalibThreads));
  const dim3 grid(static_cast<unsigned>(heads), static_cast<unsigned>(std::max<uint64_t>(1, slices)));
  rota::head_error_kernel<<<grid, rota::kCalibThreads, 0, s>>>(out_test, out_ref, n4, sums);
  return cuda_status(cudaGetLastError());
}

rota_status rota_attn_select_fp16_heads(const double* sums, int32_t B, int32_t H, float max_rel_err,
                                        int32_t max_fp16_heads, float* rel_err, uint8_t* flags) {
  if (!sums || !flags || B < 1 || H < 1 || H > 256 || !(max_rel_err >= 0.f) || !std::isfinite(max_rel_err))
    return ROTA_ERR_INVALID_ARG;
  // per head: the worst batch entry's relative Frobenius error
  float rel[256];
  for (int32_t h = 0; h < H; ++h) {
    double worst = 0.0;
    for (int32_t b = 0; b < B; ++b) {
      const double e = sums[2 * (static_cast<size_t>(b) * H + h)];
      const double q = sums[2 * (static_cast<size_t>(b) * H + h) + 1];
      double r;
      if (std::isnan(e) || std::isnan(q)) r = std::numeric_limits<double>::infinity();
      else if (q > 0.0) r = std::sqrt(e / q);
      else r = e > 0.0 ? std::numeric_limits<double>::infinity() : 0.0;
      worst = std::max(worst, r);
    }
    rel[h] = static_cast<float>(worst);
    if (rel_err) rel_err[h] = rel[h];
    flags[h] = 0;
  }
  // candidates above the threshold, worst first (lower head index on ties)
  int32_t order[256], n = 0;
  for (int32_t h = 0; h < H; ++h)
    if (rel[h] > max_rel_err) order[n++] = h;
  std::stable_sort(order, order + n, [&](int32_t a, int32_t b) { return rel[a] > rel[b]; });
  const int32_t take = max_fp16_heads < 0 ? n : std::min(n, max_fp16_heads);
  for (int32_t i = 0; i < take; ++i) flags[order[i]] = 1;
  return ROTA_OK;
}

rota_status rota_attn_get_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_status(e);
  int v = 0, zero = 0;
  if ((e = cudaMemcpyFromSymbol(&v, rota::g_error, sizeof(int))) != cudaSuccess) return cuda_status(e);
  if ((e = cudaMemcpyToSymbol(rota::g_error, &zero, sizeof(int))) != cudaSuccess) return cuda_status(e);
  if (v == rota::kDevTimeout) return ROTA_ERR_TIMEOUT;
  if (v != 0) return ROTA_ERR_DEVICE;
  return ROTA_OK;
}

static rota_status debug_pcode(bool fma, const float* dvals, uint8_t* u, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!dvals || !u))) return ROTA_ERR_INVALID_ARG;
  if (n == 0) return ROTA_OK;
  rota::Int4Params p{};
  std::memcpy(p.tau, tau_table().tau, sizeof(p.tau));
  const int64_t blocks64 = (n + 255) / 256;
  const int blocks = static_cast<int>(blocks64 < 148 * 16 ? blocks64 : 148 * 16);
  if (fma)
    rota::pcode_kernel<true><<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(dvals, u, n, p);
  else
    rota::pcode_kernel<false><<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(dvals, u, n, p);
  return cuda_status(cudaGetLastError());
}

rota_status rota_attn_debug_pcode(const float* dvals, uint8_t* u, int64_t n, void* stream) {
  return debug_pcode(false, dvals, u, n, stream);
}

rota_status rota_attn_debug_pcode_fma(const float* dvals, uint8_t* u, int64_t n, void* stream) {
  return debug_pcode(true, dvals, u, n, stream);
}

rota_status rota_attn_debug_hadamard(int32_t n, int8_t* h) {
  if (!h || n < 2 || n > 64) return ROTA_ERR_INVALID_ARG;
  uint64_t neg[64];
  if (!hadamard_rows(n, neg)) return ROTA_ERR_UNSUPPORTED;
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) h[i * n + j] = ((neg[i] >> j) & 1ull) ? -1 : 1;
  return ROTA_OK;
}

rota_status rota_attn_debug_mma_cycles(int32_t kind, int32_t n, int32_t iters, uint64_t* cycles, void* stream) {
  if (kind < 0 || kind > 2 || (n != 64 && n != 128 && n != 256) || iters < 1 || iters > 65536 || !cycles ||
      reinterpret_cast<uintptr_t>(cycles) % 8 != 0)
    return ROTA_ERR_INVALID_ARG;
  rota_status st = set_smem(rota::mma_rate_kernel, rota::kRateSmem);
  if (st != ROTA_OK) return st;
  rota::mma_rate_kernel<<<1, rota::kRateThreads, rota::kRateSmem, static_cast<cudaStream_t>(stream)>>>(
      kind, n, iters, kDefaultTimeoutNs, reinterpret_cast<unsigned long long*>(cycles));
  return cuda_status(cudaGetLastError());
}

rota_status rota_attn_debug_inject_timeout(int32_t arm, uint64_t timeout_ns) {
  std::lock_guard<std::mutex> g(g_inject.mu);
  g_inject.armed = arm ? 1 : 0;
  g_inject.timeout_ns = timeout_ns ? timeout_ns : kDefaultTimeoutNs;
  return ROTA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free INT4 forward: the codes, scales and RoPE tables of one call
// live in a static device array instead of caller-allocated buffers.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[ROTA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct NoAllocState {
  std::mutex mu;
  void* scratch[kMaxDevices] = {};            // device address of g_noalloc_scratch, per device
  float host_cos[ROTA_NOALLOC_MAX_TABLE];     // staging for the RoPE tables (no heap allocation)
  float host_sin[ROTA_NOALLOC_MAX_TABLE];
} g_noalloc;

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Set-up, once per device, with that device current: the symbol's device address.
rota_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= kMaxDevices) return ROTA_ERR_UNSUPPORTED;
  if (!g_noalloc.scratch[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    g_noalloc.scratch[dev] = p;
  }
  *out = g_noalloc.scratch[dev];
  return ROTA_OK;
}

}  // namespace

extern "C" rota_status rota_attn_fwd_int4_noalloc(const rota_attn_desc* d, const uint16_t* q, const uint16_t* k,
                                                  const uint16_t* v, float* out, void* stream) {
  rota_status st = rota_attn_validate(d);
  if (st != ROTA_OK) return st;
  if (!q || !k || !v || !out) return ROTA_ERR_INVALID_ARG;
  size_t sz[ROTA_BUF_COUNT];
  if ((st = rota_attn_buffer_sizes(d, sz)) != ROTA_OK) return st;
  const size_t table_floats = sz[ROTA_BUF_ROPE_TABLE] / 4;
  const int order[] = {ROTA_BUF_Q_CODES, ROTA_BUF_K_CODES, ROTA_BUF_Q_SCALE, ROTA_BUF_K_SCALE,
                       ROTA_BUF_V_CODES, ROTA_BUF_V_SCALE, ROTA_BUF_ROPE_TABLE, ROTA_BUF_ROPE_TABLE,
                       ROTA_BUF_INT4_WORK};
  size_t off[9], total = 0;
  for (int i = 0; i < 9; ++i) {
    off[i] = total;
    total += round256(sz[order[i]]);
  }
  if (total > ROTA_NOALLOC_SCRATCH_BYTES || table_floats > ROTA_NOALLOC_MAX_TABLE) {
    std::fprintf(stderr,
                 "rota_attn_fwd_int4_noalloc: problem needs %zu bytes of scratch and %zu-entry RoPE tables; "
                 "the static scratch holds %u bytes and %u entries\n",
                 total, table_floats, ROTA_NOALLOC_SCRATCH_BYTES, ROTA_NOALLOC_MAX_TABLE);
    return ROTA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_noalloc.mu);
  void* base = nullptr;
  if ((st = noalloc_scratch(&base)) != ROTA_OK) return st;
  uint8_t* s = static_cast<uint8_t*>(base);
  if ((st = rota_attn_build_rope_tables(d, g_noalloc.host_cos, g_noalloc.host_sin)) != ROTA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // Pageable source: returns once the host buffer has been consumed.
  cudaError_t e = cudaMemcpyAsync(s + off[6], g_noalloc.host_cos, sz[ROTA_BUF_ROPE_TABLE], cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(s + off[7], g_noalloc.host_sin, sz[ROTA_BUF_ROPE_TABLE], cudaMemcpyHostToDevice, cs);
  if (e != cudaSuccess) return cuda_status(e);
  rota_attn_buffers b{};
  b.q_codes = s + off[0];
  b.k_codes = s + off[1];
  b.q_scale = reinterpret_cast<float*>(s + off[2]);
  b.k_scale = reinterpret_cast<float*>(s + off[3]);
  b.v_codes = s + off[4];
  b.v_scale = reinterpret_cast<float*>(s + off[5]);
  b.rope_cos = reinterpret_cast<const float*>(s + off[6]);
  b.rope_sin = reinterpret_cast<const float*>(s + off[7]);
  b.int4_work = s + off[8];
  if ((st = rota_attn_prepare_qk(d, q, k, v, nullptr, &b, stream)) != ROTA_OK) return st;
  return rota_attn_fwd_int4(d, &b, nullptr, out, stream);
}
