/*
 * rota_oracle.c -- CPU oracle for RotateAttention's INT4 attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The
 * product path (video_dit_b200/) never links, imports or calls it, and this
 * file shares no code, header, table or constant generator with the CUDA
 * path.
 *
 * A plain, slow, single-threaded statement of what the method computes,
 * written from "RotateAttention: RoPE-Aware Rotation and Range Rectification
 * for INT4 Quantized Attention in Video Generation" (abstract and Key
 * Points).  The pages fix the pipeline (3D RoPE -> RoPE-aware rotation ->
 * INT4 Q/K/V -> INT4 FlashAttention with range-optimised P codes, FP16
 * fallback for flagged heads) but no rounding rule, block size or rotation
 * construction; the readings taken here are listed at each function.
 *
 * Precision.  The quantiser inputs (RoPE, rotation, scales) are DEFINED as
 * the fp32 operations written below, in the order written, each one IEEE
 * round-to-nearest-even (compiled with -ffp-contract=off, no fast-math);
 * that definition is what makes the integer codes reproducible bit for bit.
 * Everything downstream of the integer codes (P codes, softmax weights,
 * output) is exact or double precision: P codes come from long-double
 * exp2 with a tie margin check, outputs are accumulated in double.
 *
 * Parity status: every function below is pinned by tests under
 * tests/test_oracle_*.py against closed forms, library routines
 * (numpy fp16 casts, scipy's Hadamard matrix, torch fp64 attention,
 * mpmath thresholds) or brute force; none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ----------------------------------------------------------------------- */
/* fp16 <-> fp32, written from the IEEE 754 binary16 definition.            */
/* ----------------------------------------------------------------------- */

float oracle_half_to_float(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int mant = h & 0x3ff;
    double v;
    if (expo == 0) {
        v = ldexp((double)mant, -24);              /* subnormal: m * 2^-24 */
    } else if (expo == 31) {
        v = mant ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + mant), expo - 25);  /* (1 + m/1024) 2^(e-15) */
    }
    return (float)(sign ? -v : v);
}

/* Round-to-nearest-even fp32 -> fp16 (the cast the FP16 fallback inputs use). */
uint16_t oracle_float_to_half(float f)
{
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    double a = fabs((double)f);
    if (isnan(f)) return 0x7e00;
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) {                      /* subnormal range */
        double q = nearbyint(ldexp(a, 24));         /* RNE in default mode */
        return (uint16_t)(sign | (uint16_t)q);      /* q == 1024 is the smallest normal */
    }
    int e;
    double m = frexp(a, &e);                        /* a = m 2^e, m in [0.5,1) */
    m *= 2.0; e -= 1;                               /* m in [1,2) */
    double q = nearbyint(m * 1024.0);               /* 1024..2048 */
    if (q == 2048.0) { q = 1024.0; e += 1; }
    if (e + 15 >= 31) return sign | 0x7c00;         /* overflow to inf */
    return (uint16_t)(sign | ((e + 15) << 10) | ((uint16_t)q - 1024));
}

/* ----------------------------------------------------------------------- */
/* Step 1: 3D RoPE tables.                                                  */
/* Reading: standard RoFormer frequencies restarted in every partition:    */
/* pair i of axis a rotates by pos * theta^(-2i/d_a); the exponent and the  */
/* angle are evaluated in double, cos/sin in double (libm), then rounded    */
/* to fp32.  Table layout: axis t, then h, then w; inside an axis          */
/* [pos][pair].                                                            */
/* The "mergeable rotation matrices that can be fused into RoPE" of the     */
/* abstract: within a partition (distinct frequencies) the rotations that   */
/* commute with RoPE at every position are the fixed 2-D rotations of each  */
/* pair, so the plainest reading is one angle phase[a] per partition added  */
/* to every pair's angle, pos * omega + phase[a] (0 = plain RoPE).  Applied */
/* to Q and K alike it cancels in every q.k.                                */
/* ----------------------------------------------------------------------- */

static long rope_table_len(const int grid[3], const int rope_dim[3])
{
    return (long)grid[0] * (rope_dim[0] / 2) + (long)grid[1] * (rope_dim[1] / 2) +
           (long)grid[2] * (rope_dim[2] / 2);
}

long oracle_rope_table_len(const int grid[3], const int rope_dim[3])
{
    return rope_table_len(grid, rope_dim);
}

void oracle_rope_tables(const int grid[3], const int rope_dim[3], double theta, const double phase[3],
                        float *cos_tab, float *sin_tab)
{
    long off = 0;
    for (int a = 0; a < 3; ++a) {
        int half = rope_dim[a] / 2;
        for (int pos = 0; pos < grid[a]; ++pos) {
            for (int i = 0; i < half; ++i) {
                double expo = -(double)(2 * i) / (double)rope_dim[a];
                double omega = pow(theta, expo);
                double ang = (double)pos * omega + phase[a];
                cos_tab[off + (long)pos * half + i] = (float)cos(ang);
                sin_tab[off + (long)pos * half + i] = (float)sin(ang);
            }
        }
        off += (long)grid[a] * half;
    }
}

/* ----------------------------------------------------------------------- */
/* Step 2: RoPE on one token row (fp32, no fused multiply-add).             */
/* Token n sits at t = n / (Hh W), h = (n / W) mod Hh, w = n mod W          */
/* (t-major raster; reading).  Partition a occupies channels                */
/* [off_a, off_a + d_a) with off = (0, d_t, d_t + d_h); pair i of the      */
/* partition is channels (off_a + 2i, off_a + 2i + 1) (interleaved; reading).*/
/*   y0 = RN(RN(x0 c) - RN(x1 s)),  y1 = RN(RN(x0 s) + RN(x1 c))            */
/* ----------------------------------------------------------------------- */

static void rope_row(const float *x, float *y, long n, const int grid[3], const int rope_dim[3],
                     const float *cos_tab, const float *sin_tab)
{
    int Hh = grid[1], W = grid[2];
    int pos[3];
    pos[0] = (int)(n / ((long)Hh * W));
    pos[1] = (int)((n / W) % Hh);
    pos[2] = (int)(n % W);
    long toff = 0;
    int coff = 0;
    for (int a = 0; a < 3; ++a) {
        int half = rope_dim[a] / 2;
        for (int i = 0; i < half; ++i) {
            float c = cos_tab[toff + (long)pos[a] * half + i];
            float s = sin_tab[toff + (long)pos[a] * half + i];
            float x0 = x[coff + 2 * i], x1 = x[coff + 2 * i + 1];
            float a0 = x0 * c, b0 = x1 * s;
            float a1 = x0 * s, b1 = x1 * c;
            y[coff + 2 * i] = a0 - b0;
            y[coff + 2 * i + 1] = a1 + b1;
        }
        toff += (long)grid[a] * half;
        coff += rope_dim[a];
    }
}

/* ----------------------------------------------------------------------- */
/* Step 3: RoPE-aware rotation ("negligible-overhead matrices" variant).    */
/* Inside each partition, consecutive blocks of b_a channels are multiplied */
/* by the normalised Sylvester Hadamard matrix H_b / sqrt(b): an in-place  */
/* fast Walsh-Hadamard transform with stages h = 1, 2, ..., b/2 (each      */
/* butterfly one fp32 add and one fp32 subtract), then every element times  */
/* r_b = RN(1/sqrt(b)) (skipped for b = 1).  Same matrix for Q and K, so   */
/* Q K^T is unchanged in exact arithmetic; V is not rotated.               */
/* ----------------------------------------------------------------------- */

/* Blocks whose size is not a power of two (a numerics option: e.g. the    */
/* partition's own size, 44 for a 44-channel partition) take a            */
/* Hadamard matrix of that order from the classical constructions:          */
/*   Paley I  (q prime, q = 3 mod 4), order q + 1:  H = I + S,             */
/*            S = [[0, 1^T], [-1, Q]],  Q_ij = chi(j - i);                  */
/*   Paley II (q prime, q = 1 mod 4), order 2(q + 1):  from the conference */
/*            matrix C = [[0, 1^T], [1, Q]], every off-diagonal entry c ->  */
/*            c [[1, 1], [1, -1]], every diagonal entry -> [[1, -1], [-1, -1]];*/
/*   doubling: H_2n = [[H, H], [H, -H]].                                   */
/* chi is the quadratic character mod q (chi(0) = 0).  For an order n <= 64 */
/* that is not a power of two the first rule that applies is used:          */
/* doubling (n / 2 >= 12 and supported), Paley I (q = n - 1), Paley II      */
/* (q = n / 2 - 1); e.g. 12, 20, 44, 60 by Paley I (q = 11, 19, 43, 59),    */
/* 28, 36 by Paley II (q = 13, 17), 24, 40, 48, 56 by doubling.  Other     */
/* orders (6, 10, 14, ...) are unsupported.  Such a block is applied as a dense */
/* product, y_i = sum_j H_ij x_j accumulated in fp32 in the order          */
/* j = 0, 1, ..., b-1 (the first term exact, then one add or subtract per  */
/* term), then y_i * r_b.                                                  */
static int chi(long a, int q)
{
    a %= q;
    if (a < 0) a += q;
    if (a == 0) return 0;
    long r = 1, base = a, e = (q - 1) / 2;
    while (e > 0) {
        if (e & 1) r = r * base % q;
        base = base * base % q;
        e >>= 1;
    }
    return r == 1 ? 1 : -1;
}

static int is_prime(int q)
{
    if (q < 2) return 0;
    for (int f = 2; f * f <= q; ++f)
        if (q % f == 0) return 0;
    return 1;
}

/* H (n x n, row-major, entries +1 / -1) for a supported non-power-of-two    */
/* order n <= 64; returns 0 for any other n.                                */
int oracle_hadamard(int n, signed char *H)
{
    if (n <= 1 || n > 64 || (n & (n - 1)) == 0) return 0;
    if (n % 2 == 0 && n / 2 >= 12 && oracle_hadamard(n / 2, NULL)) {
        if (H) {
            int m = n / 2;
            signed char *h = (signed char *)malloc((size_t)m * m);
            if (!h) return 0;
            oracle_hadamard(m, h);
            for (int i = 0; i < m; ++i)
                for (int j = 0; j < m; ++j) {
                    H[i * n + j] = h[i * m + j];
                    H[i * n + j + m] = h[i * m + j];
                    H[(i + m) * n + j] = h[i * m + j];
                    H[(i + m) * n + j + m] = (signed char)-h[i * m + j];
                }
            free(h);
        }
        return 1;
    }
    int q = n - 1;
    if (q % 4 == 3 && is_prime(q)) {           /* Paley I */
        if (H)
            for (int i = 0; i < n; ++i)
                for (int j = 0; j < n; ++j) {
                    int sv;
                    if (i == j) sv = 1;                      /* I + S, S_ii = 0 */
                    else if (i == 0) sv = 1;                 /* first row of S: 1 */
                    else if (j == 0) sv = -1;                /* first column of S: -1 */
                    else sv = chi((long)(j - 1) - (i - 1), q);
                    H[i * n + j] = (signed char)sv;
                }
        return 1;
    }
    if (n % 2 == 0) {
        q = n / 2 - 1;
        if (q % 4 == 1 && is_prime(q)) {       /* Paley II */
            if (H) {
                int m = q + 1;
                for (int i = 0; i < m; ++i)
                    for (int j = 0; j < m; ++j) {
                        int c;
                        if (i == j) c = 0;
                        else if (i == 0 || j == 0) c = 1;
                        else c = chi((long)(j - 1) - (i - 1), q);
                        int e00, e01, e10, e11;
                        if (c == 0) { e00 = 1; e01 = -1; e10 = -1; e11 = -1; }
                        else { e00 = c; e01 = c; e10 = c; e11 = -c; }
                        H[(2 * i) * n + 2 * j] = (signed char)e00;
                        H[(2 * i) * n + 2 * j + 1] = (signed char)e01;
                        H[(2 * i + 1) * n + 2 * j] = (signed char)e10;
                        H[(2 * i + 1) * n + 2 * j + 1] = (signed char)e11;
                    }
            }
            return 1;
        }
    }
    return 0;
}

static void rotate_row(float *y, const int rope_dim[3], const int had_block[3])
{
    int coff = 0;
    for (int a = 0; a < 3; ++a) {
        int b = had_block[a];
        if (b > 1 && (b & (b - 1)) != 0) {       /* dense block of a non-power-of-two order */
            float r = (float)(1.0 / sqrt((double)b));
            signed char H[64 * 64];
            float t[64];
            if (!oracle_hadamard(b, H)) { coff += rope_dim[a]; continue; }
            for (int blk = coff; blk < coff + rope_dim[a]; blk += b) {
                for (int i = 0; i < b; ++i) {
                    float acc = H[i * b] > 0 ? y[blk] : -y[blk];
                    for (int j = 1; j < b; ++j) acc = H[i * b + j] > 0 ? acc + y[blk + j] : acc - y[blk + j];
                    t[i] = acc;
                }
                for (int i = 0; i < b; ++i) y[blk + i] = t[i] * r;
            }
        } else if (b > 1) {
            float r = (float)(1.0 / sqrt((double)b));
            for (int blk = coff; blk < coff + rope_dim[a]; blk += b) {
                for (int h = 1; h < b; h <<= 1) {
                    for (int j = 0; j < b; ++j) {
                        if (j & h) continue;
                        float u = y[blk + j], w = y[blk + j + h];
                        y[blk + j] = u + w;
                        y[blk + j + h] = u - w;
                    }
                }
                for (int j = 0; j < b; ++j) y[blk + j] = y[blk + j] * r;
            }
        }
        coff += rope_dim[a];
    }
}

/* Exposed for the pins: RoPE then (optionally) the rotation, one row. */
void oracle_rope_rotate_row(const float *x, float *y, long n, const int grid[3],
                            const int rope_dim[3], const int had_block[3],
                            const float *cos_tab, const float *sin_tab, int do_rope, int do_rotate)
{
    int d = rope_dim[0] + rope_dim[1] + rope_dim[2];
    if (do_rope) rope_row(x, y, n, grid, rope_dim, cos_tab, sin_tab);
    else memcpy(y, x, sizeof(float) * (size_t)d);
    if (do_rotate) rotate_row(y, rope_dim, had_block);
}

/* ----------------------------------------------------------------------- */
/* Step 4: symmetric INT4 quantisation of a set of fp32 values.             */
/* Reading: range +-7 (-8 unused), scale = RN(amax / 7),                    */
/* code = clamp(RNE(RN(y * RN(7 / amax))), -7, 7); amax == 0 gives scale 0  */
/* and all-zero codes.                                                      */
/* ----------------------------------------------------------------------- */

void oracle_quant_params(float amax, float *scale, float *inv)
{
    if (amax == 0.0f) { *scale = 0.0f; *inv = 0.0f; return; }
    *scale = amax / 7.0f;
    *inv = 7.0f / amax;
}

int oracle_quant_code(float y, float inv)
{
    float t = y * inv;
    float r = nearbyintf(t);                      /* ties to even */
    if (r > 7.0f) r = 7.0f;
    if (r < -7.0f) r = -7.0f;
    return (int)r;
}

static uint8_t nibble(int v) { return (uint8_t)(v < 0 ? (8 | -v) : v); }

/* Packs n (multiple of 8) codes into n/2 bytes in the layout above. */
static void pack_codes(const int *v, long n, uint8_t *out)
{
    for (long g = 0; g < n; g += 8)
        for (int j = 0; j < 4; ++j)
            out[g / 2 + j] = (uint8_t)(nibble(v[g + j]) | (nibble(v[g + j + 4]) << 4));
}

/* Element i of a packed row. */
static int code_at(const uint8_t *row, long i)
{
    uint8_t byte = row[(i / 8) * 4 + (i % 4)];
    int nib = (i % 8) < 4 ? (byte & 0xf) : (byte >> 4);
    return (nib & 8) ? -(nib & 7) : (nib & 7);
}

void oracle_pack_codes(const int *v, long n, uint8_t *out) { pack_codes(v, n, out); }
int oracle_code_at(const uint8_t *row, long i) { return code_at(row, i); }

void oracle_quant_codes(const float *y, long n, float inv, int8_t *codes)
{
    for (long i = 0; i < n; ++i) codes[i] = (int8_t)oracle_quant_code(y[i], inv);
}

/* ----------------------------------------------------------------------- */
/* The prologue for one attention call.                                     */
/*   q, k, v        : fp16 bits [B,H,N,d]                                   */
/*   flags          : [H], 1 = head takes the FP16 fallback                 */
/* Outputs (layouts are the library's interface):                         */
/*   a code v in [-7, 7] is a sign-magnitude nibble (bit 3 = sign,          */
/*   bits 0-2 = |v|; zero is 0000); along the packed axis every 8           */
/*   consecutive elements e0..e7 form one little-endian 32-bit word whose   */
/*   byte j (0..3) holds e_j in its low nibble and e_{j+4} in its high one. */
/*   q_codes,k_codes: [B,H,Npad,d/2]   q_scale,k_scale : [B,H,Npad/64]      */
/*   v_codes        : [B,H,Npad/64,d,32] (64 tokens of one channel)         */
/*   v_scale        : [B,H,Npad/64,d]                                       */
/*   q_rope,k_rope  : fp16 bits [B,H,N,d], RoPE only, flagged heads only    */
/* Unflagged heads get codes; flagged heads get q_rope/k_rope (their code   */
/* buffers are left untouched).  Tokens >= N get code 0 and do not enter    */
/* any amax.                                                                */
/* ----------------------------------------------------------------------- */

int oracle_prepare(int B, int H, int N, int d, const int grid[3], const int rope_dim[3],
                   const int had_block[3], double theta, const double phase[3],
                   const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint8_t *flags,
                   uint8_t *q_codes, uint8_t *k_codes, float *q_scale, float *k_scale,
                   uint8_t *v_codes, float *v_scale, uint16_t *q_rope, uint16_t *k_rope)
{
    const int QB = 64;
    int nblk = (N + QB - 1) / QB;
    long npad = (long)nblk * QB;
    long tlen = rope_table_len(grid, rope_dim);
    float *cos_tab = (float *)malloc(sizeof(float) * (size_t)tlen);
    float *sin_tab = (float *)malloc(sizeof(float) * (size_t)tlen);
    float *x = (float *)malloc(sizeof(float) * (size_t)d);
    float *blk = (float *)malloc(sizeof(float) * (size_t)QB * d);
    int *codes = (int *)malloc(sizeof(int) * (size_t)(d > QB ? d : QB));
    if (!cos_tab || !sin_tab || !x || !blk || !codes) return -1;
    oracle_rope_tables(grid, rope_dim, theta, phase, cos_tab, sin_tab);

    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            long head = (long)b * H + h;
            const uint16_t *srcs[2] = {q + head * N * d, k + head * N * d};
            if (flags && flags[h]) {
                uint16_t *dsts[2] = {q_rope + head * N * d, k_rope + head * N * d};
                for (int t = 0; t < 2; ++t) {
                    for (long n = 0; n < N; ++n) {
                        float y[1024];
                        for (int c = 0; c < d; ++c) x[c] = oracle_half_to_float(srcs[t][n * d + c]);
                        rope_row(x, y, n, grid, rope_dim, cos_tab, sin_tab);
                        for (int c = 0; c < d; ++c) dsts[t][n * d + c] = oracle_float_to_half(y[c]);
                    }
                }
                continue;
            }
            uint8_t *cdst[2] = {q_codes + head * npad * (d / 2), k_codes + head * npad * (d / 2)};
            float *sdst[2] = {q_scale + head * nblk, k_scale + head * nblk};
            for (int t = 0; t < 2; ++t) {
                for (int j = 0; j < nblk; ++j) {
                    float amax = 0.0f;
                    for (int r = 0; r < QB; ++r) {
                        long n = (long)j * QB + r;
                        float *y = blk + (long)r * d;
                        if (n >= N) { memset(y, 0, sizeof(float) * (size_t)d); continue; }
                        for (int c = 0; c < d; ++c) x[c] = oracle_half_to_float(srcs[t][n * d + c]);
                        rope_row(x, y, n, grid, rope_dim, cos_tab, sin_tab);
                        rotate_row(y, rope_dim, had_block);
                        for (int c = 0; c < d; ++c) {
                            float av = fabsf(y[c]);
                            if (av > amax) amax = av;
                        }
                    }
                    float scale, inv;
                    oracle_quant_params(amax, &scale, &inv);
                    sdst[t][j] = scale;
                    for (int r = 0; r < QB; ++r) {
                        long n = (long)j * QB + r;
                        for (int c = 0; c < d; ++c)
                            codes[c] = (n < N) ? oracle_quant_code(blk[(long)r * d + c], inv) : 0;
                        pack_codes(codes, d, cdst[t] + n * (d / 2));
                    }
                }
            }
            /* V: per (64-token block, channel), no RoPE, no rotation. */
            const uint16_t *vs = v + head * N * d;
            uint8_t *vc = v_codes + head * nblk * (long)d * 32;
            float *vsc = v_scale + head * nblk * (long)d;
            for (int j = 0; j < nblk; ++j) {
                for (int c = 0; c < d; ++c) {
                    float vals[64];
                    float amax = 0.0f;
                    for (int r = 0; r < QB; ++r) {
                        long n = (long)j * QB + r;
                        vals[r] = (n < N) ? oracle_half_to_float(vs[n * d + c]) : 0.0f;
                        if (n < N && fabsf(vals[r]) > amax) amax = fabsf(vals[r]);
                    }
                    float scale, inv;
                    oracle_quant_params(amax, &scale, &inv);
                    vsc[(long)j * d + c] = scale;
                    for (int r = 0; r < QB; ++r)
                        codes[r] = ((long)j * QB + r < N) ? oracle_quant_code(vals[r], inv) : 0;
                    pack_codes(codes, QB, vc + ((long)j * d + c) * 32);
                }
            }
        }
    }
    free(cos_tab); free(sin_tab); free(x); free(blk); free(codes);
    return 0;
}

/* ----------------------------------------------------------------------- */
/* The QKV projection in front of the path (the abstract places the INT4    */
/* attention inside the DiT block, right after it): per head h and token n, */
/* q[b,h,n,c] = sum_k x[b,n,k] w[h*D + c, k], k[...] with rows H*D + h*D + c,*/
/* v[...] with rows 2*H*D + h*D + c; each sum accumulated exactly (double:   */
/* the fp16 products are exact, and the sums of the pinned inputs too),     */
/* rounded to fp32 (reading: an fp32 accumulation whose order the pages do  */
/* not fix, taken as the correctly rounded fp32 value of the sum) and then  */
/* to fp16 -- the fp16 Q, K, V the prologue takes.  x [B,N,C], w [3HD,C],   */
/* outputs fp16 bit patterns [B,H,N,D].                                      */
/* ----------------------------------------------------------------------- */

void oracle_qkv_project(int B, int N, int C, int H, int D, const uint16_t *x, const uint16_t *w,
                        uint16_t *q, uint16_t *k, uint16_t *v)
{
    uint16_t *outs[3] = {q, k, v};
    double *xrow = (double *)malloc(sizeof(double) * (size_t)C);
    double *wrow = (double *)malloc(sizeof(double) * (size_t)C);
    if (!xrow || !wrow) { free(xrow); free(wrow); return; }
    for (int m = 0; m < 3; ++m)
        for (int h = 0; h < H; ++h)
            for (int c = 0; c < D; ++c) {
                const uint16_t *wr = w + ((long)(m * H + h) * D + c) * C;
                for (int kk = 0; kk < C; ++kk) wrow[kk] = (double)oracle_half_to_float(wr[kk]);
                for (int b = 0; b < B; ++b)
                    for (int n = 0; n < N; ++n) {
                        const uint16_t *xr = x + ((long)b * N + n) * C;
                        double acc = 0.0;
                        for (int kk = 0; kk < C; ++kk) acc += (double)oracle_half_to_float(xr[kk]) * wrow[kk];
                        outs[m][(((long)b * H + h) * N + n) * D + c] = oracle_float_to_half((float)acc);
                    }
            }
    free(xrow); free(wrow);
}

/* ----------------------------------------------------------------------- */
/* Step 5: range-optimised P code of one exponent d (fp32, d <= ~0).        */
/* P = 2^d in (0,1] is mapped to the unsigned code u = RNE(15 P) with the   */
/* fixed scale 1/15 and zero-point 0, in exact real arithmetic on the fp32  */
/* d.  15 * 2^d equals a half-integer only at d = -1 (7.5 -> 8), because    */
/* 2^d is irrational for every non-integer rational d; the long-double      */
/* evaluation is therefore exact in effect, and a margin check reports any  */
/* case that would be too close to call (*bad set to 1).                   */
/* ----------------------------------------------------------------------- */

int oracle_pcode(float d, int *bad)
{
    long double p = 15.0L * exp2l((long double)d);
    long double fl = floorl(p);
    long double gap = fabsl(p - (fl + 0.5L));
    if (gap < 1e-15L && d != -1.0f && bad) *bad = 1;
    long double r = nearbyintl(p);                /* ties to even */
    if (r > 15.0L) r = 15.0L;
    if (r < 0.0L) r = 0.0L;
    return (int)r;
}

void oracle_pcode_array(const float *d, uint8_t *u, long n, int *bad)
{
    for (long i = 0; i < n; ++i) u[i] = (uint8_t)oracle_pcode(d[i], bad);
}

/* ----------------------------------------------------------------------- */
/* Steps 6-9: the INT4 attention for rows [r0, r0+nr) of head (b, h).       */
/*  S_int[i,k] = sum_c qcode[i,c] kcode[k,c]              (exact integer)   */
/*  c_ij       = RN(RN(sq_i sk_j) kappa), kappa = RN(sm_scale log2 e)       */
/*  m_g        = max(m_{g-1}, max_{k in g} RN(S_int c))  (running max over  */
/*               64-key groups, in order; reading: the online max of        */
/*               FlashAttention at the quant-block granularity)             */
/*  d          = fmaf(S_int, c, -m_g);   u = RNE(15 * 2^d)                  */
/*  out[c]     = sum_g 2^(m_g - M) sv[g,c] sum_{k in g} u_k vcode[k,c]      */
/*               / sum_g 2^(m_g - M) sum_{k in g} u_k        (double)       */
/* The row sum uses the quantised P, the same values that multiply V        */
/* (reading R2, rowsum = 0); the 1/15 scale cancels.  rowsum = 1 takes the  */
/* other reading of the page's row sum, the unquantised P (R1):            */
/*  out[c]     = sum_g 2^(m_g - M) sv[g,c] sum_{k in g} u_k vcode[k,c]      */
/*               / sum_g 2^(m_g - M) sum_{k in g} 15 * 2^(d_k)  (double)    */
/* with d_k the same fp32 exponent the code u_k is taken from (15 P_k      */
/* unrounded, so P = u / 15 in the numerator).  `group` is the key group   */
/* of the running max (64 = the quant block; 128 spans two blocks, whose    */
/* codes then share one max).  `online` selects the recurrence form */
/* O <- O 2^(m_{g-1}-m_g) + ..., l <- l 2^(m_{g-1}-m_g) + ... instead of the */
/* closed form; both are kept so they can be checked against each other.    */
/* s_dump [nr,N] and p_dump [nr,N] may be NULL.  Returns the number of      */
/* margin violations in the P codes (0 expected).                          */
/* ----------------------------------------------------------------------- */

int oracle_attn_int4(int B, int H, int N, int d, float sm_scale, int group, int rowsum,
                     const uint8_t *q_codes, const uint8_t *k_codes, const float *q_scale,
                     const float *k_scale, const uint8_t *v_codes, const float *v_scale,
                     int b, int h, int r0, int nr, int online,
                     int32_t *s_dump, uint8_t *p_dump, double *out)
{
    (void)B;
    const int QB = 64;
    int nblk = (N + QB - 1) / QB;
    long npad = (long)nblk * QB;
    long head = (long)b * H + h;
    const uint8_t *qc = q_codes + head * npad * (d / 2);
    const uint8_t *kc = k_codes + head * npad * (d / 2);
    const float *qs = q_scale + head * nblk;
    const float *ks = k_scale + head * nblk;
    const uint8_t *vc = v_codes + head * nblk * (long)d * 32;
    const float *vsc = v_scale + head * nblk * (long)d;
    float kappa = (float)((double)sm_scale * 1.4426950408889634074);
    int ngroup = (N + group - 1) / group;
    int bad = 0;

    int32_t *S = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    float *cs = (float *)malloc(sizeof(float) * (size_t)N);
    uint8_t *U = (uint8_t *)malloc((size_t)N);
    float *mg = (float *)malloc(sizeof(float) * (size_t)ngroup);
    int *qrow = (int *)malloc(sizeof(int) * (size_t)d);
    double *num = (double *)malloc(sizeof(double) * (size_t)d);
    double *rs = (double *)malloc(sizeof(double) * (size_t)N);   /* row-sum weight of each key */
    if (!S || !cs || !U || !mg || !qrow || !num || !rs) return -1;

    for (int i = r0; i < r0 + nr; ++i) {
        for (int c = 0; c < d; ++c) qrow[c] = code_at(qc + (long)i * (d / 2), c);
        float sq = qs[i / QB];
        for (long kk = 0; kk < N; ++kk) {
            long acc = 0;
            for (int c = 0; c < d; ++c) acc += (long)qrow[c] * code_at(kc + kk * (d / 2), c);
            if (acc > 49L * d || acc < -49L * d) bad++;
            S[kk] = (int32_t)acc;
            float t = sq * ks[kk / QB];
            cs[kk] = t * kappa;
        }
        /* running group max */
        float m = -INFINITY;
        for (int g = 0; g < ngroup; ++g) {
            for (long kk = (long)g * group; kk < N && kk < (long)(g + 1) * group; ++kk) {
                float x = (float)S[kk] * cs[kk];
                if (x > m) m = x;
            }
            mg[g] = m;
        }
        float M = mg[ngroup - 1];
        for (long kk = 0; kk < N; ++kk) {
            float dd = fmaf((float)S[kk], cs[kk], -mg[kk / group]);
            U[kk] = (uint8_t)oracle_pcode(dd, &bad);
            rs[kk] = rowsum ? 15.0 * exp2((double)dd) : (double)U[kk];
        }
        double den = 0.0;
        for (int c = 0; c < d; ++c) num[c] = 0.0;
        if (!online) {
            for (long kk = 0; kk < N; ++kk) {
                double wg = exp2((double)mg[kk / group] - (double)M);
                double w = wg * (double)U[kk];
                den += wg * rs[kk];
                if (U[kk] == 0) continue;
                long j = kk / QB, t = kk % QB;
                for (int c = 0; c < d; ++c) {
                    int vcode = code_at(vc + (j * d + c) * 32, t);
                    num[c] += w * (double)vsc[j * d + c] * (double)vcode;
                }
            }
        } else {
            float mprev = -INFINITY;
            for (int g = 0; g < ngroup; ++g) {
                double alpha = (g == 0) ? 0.0 : exp2((double)mprev - (double)mg[g]);
                den *= alpha;
                for (int c = 0; c < d; ++c) num[c] *= alpha;
                for (long kk = (long)g * group; kk < N && kk < (long)(g + 1) * group; ++kk) {
                    den += rs[kk];
                    long j = kk / QB, t = kk % QB;
                    for (int c = 0; c < d; ++c) {
                        int vcode = code_at(vc + (j * d + c) * 32, t);
                        num[c] += (double)U[kk] * (double)vsc[j * d + c] * (double)vcode;
                    }
                }
                mprev = mg[g];
            }
        }
        for (int c = 0; c < d; ++c) out[(long)(i - r0) * d + c] = num[c] / den;
        if (s_dump) memcpy(s_dump + (long)(i - r0) * N, S, sizeof(int32_t) * (size_t)N);
        if (p_dump) memcpy(p_dump + (long)(i - r0) * N, U, (size_t)N);
    }
    free(S); free(cs); free(U); free(mg); free(qrow); free(num); free(rs);
    return bad;
}

/* ----------------------------------------------------------------------- */
/* FP16 fallback statement: textbook softmax attention in double over the   */
/* RoPE'd fp16 Q/K (no rotation: it is an identity in exact arithmetic;     */
/* reading) and the fp16 V, for rows [r0, r0+nr) of head (b, h).            */
/* ----------------------------------------------------------------------- */

int oracle_attn_fp16(int B, int H, int N, int d, float sm_scale,
                     const uint16_t *q_rope, const uint16_t *k_rope, const uint16_t *v,
                     int b, int h, int r0, int nr, double *out)
{
    (void)B;
    long head = (long)b * H + h;
    const uint16_t *qh = q_rope + head * N * d, *kh = k_rope + head * N * d, *vh = v + head * N * d;
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *qrow = (double *)malloc(sizeof(double) * (size_t)d);
    if (!s || !qrow) return -1;
    for (int i = r0; i < r0 + nr; ++i) {
        for (int c = 0; c < d; ++c) qrow[c] = oracle_half_to_float(qh[(long)i * d + c]);
        double mx = -INFINITY;
        for (long kk = 0; kk < N; ++kk) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += qrow[c] * (double)oracle_half_to_float(kh[kk * d + c]);
            s[kk] = acc * (double)sm_scale;
            if (s[kk] > mx) mx = s[kk];
        }
        double den = 0.0;
        for (long kk = 0; kk < N; ++kk) { s[kk] = exp(s[kk] - mx); den += s[kk]; }
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (long kk = 0; kk < N; ++kk) acc += s[kk] * (double)oracle_half_to_float(vh[kk * d + c]);
            out[(long)(i - r0) * d + c] = acc / den;
        }
    }
    free(s); free(qrow);
    return 0;
}

/* ----------------------------------------------------------------------- */
/* Unquantised attention for the accuracy report: RoPE (fp32, step 2) on    */
/* the fp16 inputs, no rotation, no fp16 rounding, textbook softmax in      */
/* double.  Rows [r0, r0+nr) of head (b, h).                                */
/* ----------------------------------------------------------------------- */

int oracle_attn_ref(int B, int H, int N, int d, const int grid[3], const int rope_dim[3],
                    double theta, const double phase[3], float sm_scale, const uint16_t *q, const uint16_t *k,
                    const uint16_t *v, int b, int h, int r0, int nr, double *out)
{
    (void)B;
    long head = (long)b * H + h;
    long tlen = rope_table_len(grid, rope_dim);
    float *cos_tab = (float *)malloc(sizeof(float) * (size_t)tlen);
    float *sin_tab = (float *)malloc(sizeof(float) * (size_t)tlen);
    float *kr = (float *)malloc(sizeof(float) * (size_t)N * d);
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    float x[1024], qr[1024];
    if (!cos_tab || !sin_tab || !kr || !s) return -1;
    oracle_rope_tables(grid, rope_dim, theta, phase, cos_tab, sin_tab);
    const uint16_t *qh = q + head * N * d, *kh = k + head * N * d, *vh = v + head * N * d;
    for (long kk = 0; kk < N; ++kk) {
        for (int c = 0; c < d; ++c) x[c] = oracle_half_to_float(kh[kk * d + c]);
        rope_row(x, kr + kk * d, kk, grid, rope_dim, cos_tab, sin_tab);
    }
    for (int i = r0; i < r0 + nr; ++i) {
        for (int c = 0; c < d; ++c) x[c] = oracle_half_to_float(qh[(long)i * d + c]);
        rope_row(x, qr, i, grid, rope_dim, cos_tab, sin_tab);
        double mx = -INFINITY;
        for (long kk = 0; kk < N; ++kk) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += (double)qr[c] * (double)kr[kk * d + c];
            s[kk] = acc * (double)sm_scale;
            if (s[kk] > mx) mx = s[kk];
        }
        double den = 0.0;
        for (long kk = 0; kk < N; ++kk) { s[kk] = exp(s[kk] - mx); den += s[kk]; }
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (long kk = 0; kk < N; ++kk) acc += s[kk] * (double)oracle_half_to_float(vh[kk * d + c]);
            out[(long)(i - r0) * d + c] = acc / den;
        }
    }
    free(cos_tab); free(sin_tab); free(kr); free(s);
    return 0;
}
