/*
 * rota_attn.h -- C ABI of the B200 (sm_100a) RotateAttention forward.
 *
 * The method: "RotateAttention: RoPE-Aware Rotation and Range Rectification
 * for INT4 Quantized Attention in Video Generation" (abstract and Key
 * Points): a mixed-precision INT4 FlashAttention for DiT video models with 3D
 * RoPE.  Q and K get 3D RoPE and then a RoPE-aware rotation (an orthogonal
 * matrix inside each RoPE partition, which leaves Q K^T unchanged) before
 * INT4 quantisation; P = exp(QK - max QK) is quantised with a fixed scale and
 * zero-point that use the whole unsigned 4-bit range; heads or denoising
 * steps flagged as accuracy-sensitive take an FP16 attention instead.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers allocated by the caller, except
 *     where a parameter is marked "host".  The library never allocates,
 *     never frees and never synchronises (except rota_attn_get_error), apart
 *     from the streams and events that rota_attn_pipeline_create makes
 *     on request and rota_attn_pipeline_destroy releases.
 *   - fp16 tensors are passed as their uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream); every
 *     device call is enqueued asynchronously on it.
 *   - Argument errors are detected on the host and returned synchronously,
 *     with nothing enqueued.  Faults detected on the device (a bounded wait
 *     that ran out, a failed bounds check) are recorded in a device error
 *     word and reported by rota_attn_get_error.
 *   - Layouts are row-major with the last index fastest.  INT4 codes (values
 *     in [-7, 7]) are sign-magnitude nibbles (bit 3 = sign, bits 0-2 =
 *     magnitude), packed along the last axis in groups of 8 elements per
 *     32-bit word: byte j of the word holds element j in its low nibble and
 *     element j + 4 in its high nibble (j = 0..3).
 *   - Npad = 64 * ceil(N / 64); nblk = Npad / 64.
 */
#ifndef ROTA_ATTN_H
#define ROTA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ROTA_OK = 0,
  ROTA_ERR_INVALID_ARG = 1,  /* a descriptor field, pointer, size or alignment is invalid */
  ROTA_ERR_UNSUPPORTED = 2,  /* valid, but outside what the kernels implement (e.g. head_dim) */
  ROTA_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch, symbol copy, sync) */
  ROTA_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out; the context stays usable */
  ROTA_ERR_DEVICE = 5        /* a device-side consistency check failed */
} rota_status;

/*
 * Problem descriptor.  Token n of the sequence sits at grid position
 * t = n / (grid_h * grid_w), h = (n / grid_w) % grid_h, w = n % grid_w
 * (t-major raster), N == grid_t * grid_h * grid_w.
 * rope_dim: channels of the temporal / height / width RoPE partitions, in
 *   that order at channel offsets 0, rope_dim[0], rope_dim[0]+rope_dim[1];
 *   each even, summing to head_dim (e.g. 44/42/42, 16/56/56, 16/24/24).
 * had_block: size of the Hadamard blocks of the rotation inside each
 *   partition, dividing rope_dim[a], <= 64: a power of two (1 = no rotation;
 *   Sylvester matrix, fast transform) or an order the library builds by
 *   doubling (of an order >= 12), Paley I (n - 1 a prime = 3 mod 4) or
 *   Paley II (n / 2 - 1 a prime = 1 mod 4), tried in that order -- 12, 20,
 *   24, 28, 36, 40, 44, 48, 56, 60 -- applied as a dense product summed in
 *   fp32 in column order.  Any other value is ROTA_ERR_INVALID_ARG.
 * rope_theta: RoPE base (10000).
 * sm_scale: softmax scale; 0 selects 1/sqrt(head_dim) (rounded to fp32).
 * rope_phase: per partition, an angle (radians, finite) added to every pair's
 *   RoPE angle: the "mergeable rotation fused into RoPE" of the abstract (a
 *   fixed 2-D rotation of each pair, the rotations that commute with RoPE),
 *   applied to Q and K alike and free at run time (it lives in the tables).
 *   0 = plain RoPE.  It composes with had_block (rotation after RoPE).
 * head_dim: 64 or 128.
 * quant_block: tokens per Q / K / V quantisation block; 0 or 64 (the only
 *   size implemented; anything else positive is ROTA_ERR_UNSUPPORTED).
 * max_group: keys per group of the running max the P codes are taken
 *   against (the codes of a group use the max over every key up to its
 *   end): 0 or 64 (= the quantisation block) or 128 (two blocks share one
 *   max); other positive values are ROTA_ERR_UNSUPPORTED.
 * row_sum: the softmax row sum l.  0: the sum of the P codes u (the values
 *   that multiply V, so the 1/15 scale cancels); 1: the sum of the
 *   unquantised 15 * 2^d the codes are rounded from.
 * A zeroed field selects the default (quant_block 64, max_group 64,
 * row_sum 0).
 */
typedef struct {
  int32_t B, H, N, head_dim;
  int32_t grid_t, grid_h, grid_w;
  int32_t rope_dim[3];
  int32_t had_block[3];
  float rope_theta;
  float sm_scale;
  float rope_phase[3];
  int32_t quant_block;
  int32_t max_group;
  int32_t row_sum;
} rota_attn_desc;

/*
 * Caller-owned device buffers written by rota_attn_prepare_qk and read by the
 * attention calls (sizes from rota_attn_buffer_sizes; every pointer 16-byte
 * aligned, except q_scale and k_scale, which need 4 bytes):
 *   q_codes, k_codes : uint8 [B,H,Npad,head_dim/2]  rotated, RoPE'd Q/K codes
 *   q_scale, k_scale : fp32  [B,H,nblk]               one scale per 64 tokens
 *   v_codes          : uint8 [B,H,nblk,head_dim,32]  64 tokens of one channel
 *   v_scale          : fp32  [B,H,nblk,head_dim]     per channel per 64 tokens
 *   q_rope, k_rope   : fp16  [B,H,N,head_dim]        RoPE'd Q/K of flagged heads
 *                      (may be NULL when no head is flagged)
 *   rope_cos, rope_sin: fp32 tables from rota_attn_build_rope_tables, copied
 *                      to the device by the caller.
 *   int4_work        : workspace of rota_attn_fwd_int4 (bytes[ROTA_BUF_INT4_WORK],
 *                      64 * head_dim + 8192 bytes per (head, 64-key block)): the
 *                      K and V codes of the INT4 heads widened once per call
 *                      into pre-swizzled tensor-core operand images of exact
 *                      e4m3 values -- K as 64 x head_dim, V transposed as 128
 *                      channel rows x 64 keys (rows past head_dim zero).
 *                      Transient: its contents are rewritten by every call.
 */
typedef struct {
  uint8_t* q_codes;
  uint8_t* k_codes;
  float* q_scale;
  float* k_scale;
  uint8_t* v_codes;
  float* v_scale;
  uint16_t* q_rope;
  uint16_t* k_rope;
  const float* rope_cos;
  const float* rope_sin;
  uint8_t* int4_work;
} rota_attn_buffers;

/* Indices into the `bytes` array of rota_attn_buffer_sizes. */
enum {
  ROTA_BUF_Q_CODES = 0,
  ROTA_BUF_K_CODES,
  ROTA_BUF_Q_SCALE,
  ROTA_BUF_K_SCALE,
  ROTA_BUF_V_CODES,
  ROTA_BUF_V_SCALE,
  ROTA_BUF_Q_ROPE,
  ROTA_BUF_K_ROPE,
  ROTA_BUF_ROPE_TABLE, /* each of rope_cos and rope_sin */
  ROTA_BUF_INT4_WORK,
  ROTA_BUF_COUNT
};

/* Checks a descriptor (fills nothing).  ROTA_ERR_INVALID_ARG with no side effects. */
rota_status rota_attn_validate(const rota_attn_desc* desc);

/* Host: byte size of each buffer (array of ROTA_BUF_COUNT entries, host). */
rota_status rota_attn_buffer_sizes(const rota_attn_desc* desc, size_t* bytes);

/*
 * Host: the 3D RoPE tables (3D RoPE of the abstract; RoFormer frequencies
 * restarted per partition).  For axis a (t, h, w) of extent P_a and
 * partition d_a, entry [pos][i] (i < d_a/2) holds cos / sin of
 * pos * rope_theta^(-2i/d_a), evaluated in double and rounded to fp32.  Axes
 * are concatenated t, h, w.  host_cos / host_sin: host arrays of
 * bytes[ROTA_BUF_ROPE_TABLE] / 4 floats.
 */
rota_status rota_attn_build_rope_tables(const rota_attn_desc* desc, float* host_cos, float* host_sin);

/*
 * The prologue (3D RoPE -> RoPE-aware rotation -> INT4 quantisation; the two
 * techniques of the abstract's pipeline up to the attention), one launch.
 *   q, k, v         : fp16 [B,H,N,head_dim] device inputs (after the QKV projection)
 *   head_flags      : host uint8 [H]; 1 = the head takes the FP16 fallback at this
 *                     call (per head, per denoising step), 0 = INT4.  NULL = all INT4.
 * INT4 heads: Q and K get RoPE (fp32, pair (2i, 2i+1) of each partition
 *   rotated by the table angle), then the normalised Hadamard matrix H_b/sqrt(b)
 *   (Sylvester for a power of two, else the one described at had_block) on
 *   consecutive blocks of had_block[a] channels inside each partition, then
 *   symmetric INT4 codes, one scale per 64 tokens x head_dim block:
 *   scale = amax/7, code = clamp(rne(y * (7/amax)), -7, 7).  V (no RoPE, no
 *   rotation) gets the same quantiser per channel per 64-token block.  Tokens
 *   >= N get code 0 and no weight in any amax.
 * FP16 heads: q_rope / k_rope = fp16(RoPE(q)), fp16(RoPE(k)); no codes.
 */
rota_status rota_attn_prepare_qk(const rota_attn_desc* desc, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, const uint8_t* head_flags,
                                 const rota_attn_buffers* buf, void* stream);

/*
 * The QKV projection of the DiT block with the prologue fused into its
 * epilogue (the abstract places the INT4 attention inside the DiT block, right
 * after this projection): fp16 Q, K, V are computed and quantised on chip and
 * never written to HBM.  Same results as the projection followed by
 * rota_attn_prepare_qk on its fp16 outputs.
 *   x    : fp16 [B, N, C] device, the block's input tokens (16-byte aligned)
 *   w    : fp16 [3 * H * head_dim, C] device, the projection weights: rows
 *          h*head_dim .. +head_dim-1 give Q of head h, rows H*head_dim + ...
 *          K, rows 2*H*head_dim + ... V (16-byte aligned)
 *   C    : input channels, a multiple of 64 (at most 2^20)
 *   q = x W_q^T, k = x W_k^T, v = x W_v^T per head with fp32 accumulation,
 *   each rounded to fp16; then, per head, exactly rota_attn_prepare_qk's
 *   prologue (codes and scales of INT4 heads; q_rope / k_rope of flagged
 *   heads).
 *   head_flags, buf: as for rota_attn_prepare_qk.
 *   v_out: fp16 [B, H, N, head_dim] device; the fp16 V of the flagged heads is
 *          written there (the FP16 fallback's v); may be NULL when no head is
 *          flagged.
 * ROTA_ERR_INVALID_ARG for a null / misaligned pointer or C not a positive
 * multiple of 64.
 */
rota_status rota_attn_qkv_prepare(const rota_attn_desc* desc, const uint16_t* x, const uint16_t* w, int32_t C,
                                  const uint8_t* head_flags, const rota_attn_buffers* buf, uint16_t* v_out,
                                  void* stream);

/*
 * INT4 attention (the abstract's mixed-precision INT4 FlashAttention) for the
 * heads whose flag is 0.  Exact integer Q K^T on the tensor cores (the codes
 * as exact e4m3 values, fp32 accumulation that stays integral); scores
 * dequantised with c = (sq * sk) * (sm_scale * log2 e); a running max m over
 * consecutive 64-key groups; range-optimised P codes u = rne(15 * 2^(S c - m))
 * in 0..15 (fixed scale 1/15, zero-point 0: the whole unsigned 4-bit range,
 * as the abstract's "Range-optimized P Quantization" asks); exact integer
 * P V per 64-key block on the tensor cores, the same way; then, in fp32 on
 * the CUDA cores, each block's per-channel V scales, the rescaling of O by
 * 2^(m_old - m_new) where a row's max moved, and the row sum of the codes;
 * out = O / l.  Two launches: the K / V codes are first widened once into
 * buf->int4_work, then the attention kernel streams the widened tiles with
 * bulk copies.
 *   out: fp32 [B,H,N,head_dim]; rows of flagged heads are not written.
 */
rota_status rota_attn_fwd_int4(const rota_attn_desc* desc, const rota_attn_buffers* buf,
                               const uint8_t* head_flags, float* out, void* stream);

/*
 * The two launches of rota_attn_fwd_int4 as separate calls (same arguments;
 * rota_attn_fwd_int4 == rota_attn_int4_widen then rota_attn_int4_attend on
 * the same stream), so that each kernel can be timed on its own:
 * rota_attn_int4_widen writes buf->int4_work from the K / V codes of the
 * INT4 heads; rota_attn_int4_attend reads it and writes out.  The attend call
 * must follow a widen call on the same codes and flags.
 */
rota_status rota_attn_int4_widen(const rota_attn_desc* desc, const rota_attn_buffers* buf,
                                 const uint8_t* head_flags, void* stream);
rota_status rota_attn_int4_attend(const rota_attn_desc* desc, const rota_attn_buffers* buf,
                                  const uint8_t* head_flags, float* out, void* stream);

/*
 * FP16 fallback (the abstract's "selective FP16 fallback") for the heads whose
 * flag is 1: softmax(sm_scale * q_rope k_rope^T) v with fp16 tensor-core
 * products, fp32 accumulation and an fp32 online softmax.
 *   v  : the fp16 V input of rota_attn_prepare_qk;  out: fp32 [B,H,N,head_dim]
 *   (rows of unflagged heads are not written).
 */
rota_status rota_attn_fwd_fp16_fallback(const rota_attn_desc* desc, const rota_attn_buffers* buf,
                                        const uint16_t* v, const uint8_t* head_flags, float* out,
                                        void* stream);

/*
 * Host-to-host forward (a packaging of the three calls above for inputs that
 * live in host memory; the paper has no counterpart).  q_host, k_host,
 * v_host: host fp16 [B,H,N,head_dim]; out_host: host fp32 [B,H,N,head_dim];
 * pinned (page-locked) host memory is needed for the copies to overlap the
 * kernels.  q_dev, k_dev, v_dev, out_dev: caller-owned device buffers of the
 * same shapes (16-byte aligned), used as staging; buf and head_flags as for
 * rota_attn_prepare_qk / rota_attn_fwd_int4 / rota_attn_fwd_fp16_fallback.
 *
 * The heads of each batch entry are taken in chunks of heads_per_chunk
 * (0 = rota_attn_pipeline_chunk_heads for this device): chunk c's inputs are
 * copied in on the pipeline's host-to-device stream, its prologue, INT4
 * attention and FP16 fallback run on `stream` (even c) or on the pipeline's
 * second compute stream (odd c), and its output is copied out on the
 * device-to-host stream.  So the copies of neighbouring chunks overlap chunk
 * c's kernels, and the next chunk's kernels fill the SMs that the last wave of
 * chunk c's attention leaves idle.  Every result is the one the three calls give on the
 * whole problem (heads are independent).  Ordering: the copies start after
 * the work already enqueued on `stream`, and `stream` continues only after
 * the last copy-out, so out_host is complete once `stream` has reached that
 * point (e.g. after rota_attn_get_error(stream)).  Neither host buffer may be
 * touched by the caller until then.  Errors: ROTA_ERR_INVALID_ARG for a null
 * pointer, a negative heads_per_chunk or a pipeline made on another device;
 * ROTA_ERR_UNSUPPORTED if the pipeline has too few events (2 per chunk + 2);
 * otherwise the first failing call's status (the streams are still joined).
 */
typedef struct rota_attn_pipeline rota_attn_pipeline;

/* Creates, on the current device, the two copy streams and the second compute
 * stream (all non-blocking) and the events for up to max_chunks chunks per
 * call.  *out receives the handle. */
rota_status rota_attn_pipeline_create(int32_t max_chunks, rota_attn_pipeline** out);

/* Releases what rota_attn_pipeline_create made (NULL is a no-op). */
rota_status rota_attn_pipeline_destroy(rota_attn_pipeline* pipeline);

/* The default chunk size for a device with num_sms SMs (0 on an invalid
 * descriptor): the heads per chunk that minimise the unhidden copies of the
 * first and last chunk plus a fixed cost per chunk (its prologue, widening and
 * launches), both counted in waves of the attention kernel. */
int32_t rota_attn_pipeline_chunk_heads(const rota_attn_desc* desc, int32_t num_sms);

rota_status rota_attn_forward_host(const rota_attn_desc* desc, const uint16_t* q_host, const uint16_t* k_host,
                                   const uint16_t* v_host, const uint8_t* head_flags, float* out_host,
                                   uint16_t* q_dev, uint16_t* k_dev, uint16_t* v_dev, float* out_dev,
                                   const rota_attn_buffers* buf, int32_t heads_per_chunk,
                                   rota_attn_pipeline* pipeline, void* stream);

/*
 * Choosing the FP16-fallback heads.  The paper keeps accuracy-sensitive
 * attention blocks and denoising steps in FP16 but gives no rule for which
 * ones; these two calls measure it on a calibration call and turn the result
 * into the host flag array the attention calls take.
 *
 * rota_attn_head_error: out_test, out_ref: device fp32 [B,H,N,head_dim]
 * (16-byte aligned), typically the output with every head on the INT4 path
 * and the output with every head on the FP16 fallback for the same inputs.
 * sums: device double [B*H*2] (8-byte aligned), overwritten with, per
 * (b, h), sum (out_test - out_ref)^2 and sum out_ref^2 (fp64 accumulation;
 * the summation order varies between runs, so the last bits may too).
 * Enqueued on `stream` (a memset and one kernel); no synchronisation.
 */
rota_status rota_attn_head_error(const rota_attn_desc* desc, const float* out_test, const float* out_ref,
                                 double* sums, void* stream);

/*
 * Host only.  sums: host double [B*H*2] as rota_attn_head_error writes them.
 * A head's error is the largest relative Frobenius error over the batch,
 * sqrt(sum diff^2 / sum ref^2) (infinite for NaN sums, or for a zero
 * reference with a non-zero difference; 0 when both are zero).  Heads whose
 * error exceeds max_rel_err are flagged, the largest errors first, at most
 * max_fp16_heads of them (< 0: no limit; ties go to the lower head index).
 * flags: host uint8 [H] (1 = FP16 fallback), overwritten; rel_err: host
 * float [H] receiving the errors, or NULL.  ROTA_ERR_INVALID_ARG for null
 * sums / flags, B < 1, H outside [1, 256] or a negative / non-finite
 * max_rel_err.
 */
rota_status rota_attn_select_fp16_heads(const double* sums, int32_t B, int32_t H, float max_rel_err,
                                        int32_t max_fp16_heads, float* rel_err, uint8_t* flags);

/* Synchronises `stream`, then returns and clears the device error word
 * (ROTA_OK, ROTA_ERR_TIMEOUT or ROTA_ERR_DEVICE), or ROTA_ERR_CUDA if the
 * synchronisation itself failed. */
rota_status rota_attn_get_error(void* stream);

/* Static string for a status code. */
const char* rota_attn_status_string(rota_status s);

/*
 * Allocation-free INT4 forward (the paper has no counterpart: this is a
 * packaging of rota_attn_prepare_qk + rota_attn_fwd_int4 for callers that
 * cannot allocate device memory -- a plugin inside a host application that
 * owns the device allocator, or a real-time loop where an allocation could
 * synchronise the device or fail).  The caller passes only the inputs
 * q, k, v (fp16 [B,H,N,head_dim]) and the output out (fp32 [B,H,N,head_dim]);
 * every head takes the INT4 path (no FP16 fallback).  The intermediate codes,
 * scales and RoPE tables live in one 16 MiB array in the library's static
 * device memory, which every GPU that loads the library holds until exit.
 * Its size bounds the problem: B*H*nblk*(164*head_dim + 8200) bytes of codes,
 * widened tiles and scales plus the RoPE tables (each entry padded to 256 bytes)
 * must fit in ROTA_NOALLOC_SCRATCH_BYTES, and each RoPE table in
 * ROTA_NOALLOC_MAX_TABLE floats; larger problems return
 * ROTA_ERR_UNSUPPORTED, with nothing enqueued.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and keeps it.  A device
 * reset (cudaDeviceReset) invalidates the kept address: after one, do not
 * call this entry point again in the same process.  The RoPE tables are copied from a static host
 * buffer with a pageable cudaMemcpyAsync, which synchronises `stream` first.
 * All calls share the one array and it keeps the last call's contents (every
 * byte a call reads is written earlier in the same call, so nothing has to
 * start at zero); calls whose device work overlaps -- on two streams, or from
 * two host threads -- race on it.  No cudaMalloc, cudaFree or other
 * allocating routine is called.
 */
#define ROTA_NOALLOC_SCRATCH_BYTES (16u << 20)
#define ROTA_NOALLOC_MAX_TABLE (1u << 14)
rota_status rota_attn_fwd_int4_noalloc(const rota_attn_desc* desc, const uint16_t* q, const uint16_t* k,
                                       const uint16_t* v, float* out, void* stream);

/* ---------------------------------------------------------- test hooks --- */

/*
 * Host only: the Hadamard matrix the prologue uses for a block of the
 * non-power-of-two order n (the construction described at had_block), as
 * +1 / -1 into h (host int8 [n*n], row-major).  ROTA_ERR_UNSUPPORTED for an
 * order it builds none of (powers of two included: those use the fast
 * Sylvester transform), ROTA_ERR_INVALID_ARG for h NULL or n outside [2, 64].
 */
rota_status rota_attn_debug_hadamard(int32_t n, int8_t* h);

/*
 * Runs the INT4 attention kernel for head (b, h) only, with its debug dump
 * enabled: for rows [r0, r0+nr) it also stores the s32 scores S (device int32
 * [nr, N]) and the P codes (device uint8 [nr, N]).  `out` as for
 * rota_attn_fwd_int4 (only that head's rows are written).
 */
rota_status rota_attn_debug_dump_int4(const rota_attn_desc* desc, const rota_attn_buffers* buf, int32_t b,
                                      int32_t h, int32_t r0, int32_t nr, int32_t* s_out, uint8_t* p_out,
                                      float* out, void* stream);

/* Applies the kernels' P-code function to n exponents d (device fp32 ->
 * device uint8), so it can be checked exhaustively against the definition. */
rota_status rota_attn_debug_pcode(const float* d, uint8_t* u, int64_t n, void* stream);

/* The same P-code function with the exponential taken on the FMA pipe
 * (Cody-Waite split and a fitted polynomial, the path the INT4 kernel can
 * route a share of the keys through) instead of the exponential unit; same
 * arguments, errors and result (the exact code) as rota_attn_debug_pcode. */
rota_status rota_attn_debug_pcode_fma(const float* d, uint8_t* u, int64_t n, void* stream);

/* Fault injection for the bounded waits: the next INT4 launch skips its first
 * score MMA, so every wait on it runs out after `timeout_ns` and the kernel
 * exits with ROTA_ERR_TIMEOUT.  One-shot; 0 disarms. */
rota_status rota_attn_debug_inject_timeout(int32_t arm, uint64_t timeout_ns);

/* Measurement of the tensor-core operand kinds the INT4 kernel chooses between
 * for Q K^T (the abstract's INT4 FlashAttention: an exact integer product).
 * One CTA issues `iters` x 4 tcgen05.mma of M = 128, N = n, 128 bytes of K per
 * operand row per 4 MMAs, back to back into one TMEM accumulator, operands in
 * shared memory.  kind: 0 = f8f6f4 (e4m3 x e4m3 -> f32), 1 = i8 (s8 x s8 ->
 * s32), 2 = f16 (f16 x f16 -> f32).  n: 64, 128 or 256.  iters: 1 .. 65536.
 * cycles (device, 8 bytes, 8-byte aligned, caller-owned): receives the SM
 * clock cycles from the first issue to the completion of the last MMA (0 if
 * the bounded wait ran out; ROTA_ERR_TIMEOUT is then recorded).  Argument
 * errors return ROTA_ERR_INVALID_ARG synchronously. */
rota_status rota_attn_debug_mma_cycles(int32_t kind, int32_t n, int32_t iters, uint64_t* cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ROTA_ATTN_H */
