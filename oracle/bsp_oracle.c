/*
 * bsp_oracle.c -- plain, slow CPU oracle for the block-scaled precision linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the test-suite, the smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code, header, table or constant generator with
 * the CUDA library.
 *
 * What it computes (sources are the pages the method is described on):
 *   - "BFL (fp8r / nvfp4)" (Diffusers quantization doc), format bullets:
 *       nvfp4: packed E2M1 weight (two values per byte), E4M3 scale per block of
 *              16 (`weight_scale`), fp32 global `weight_scale_2`, fp32 calibrated
 *              `input_scale`;
 *       fp8r : E4M3 weight plus one fp32 `weight_scale` per row; activations are
 *              quantized to E4M3 per row at run time.
 *   - same page, "Kernels" table: the fused NVFP4 path quantizes the activations
 *     (nvfp4_quantize) and then runs a block-scaled GEMM; the fp8r path runs a
 *     row-scaled FP8 GEMM.  The closing paragraph of that section says the
 *     dequantise-only fallback does NOT quantize activations, so its outputs differ;
 *     this oracle follows the fused path.
 *   - "NVFP4 vs FP8 vs BF16" article: NVFP4 carries a per-block scale factor, which
 *     is what separates it from plain 4-bit integers.
 *
 * The pages give no formulas.  The readings taken here (rounding, operation order,
 * zero/saturation rules, packing order, scale layouts) are the build's own and are
 * listed, one by one, in the design notes.  In short:
 *   E2M1 : sign | 2-bit exponent (bias 1) | 1-bit mantissa; magnitudes
 *          {0,0.5,1,1.5,2,3,4,6}; encode = round to nearest, ties to the even code,
 *          saturating at 6; the sign bit is kept (so -0 and small negatives give 0x8).
 *   E4M3 : the "FN" variant: bias 7, no infinities, S.1111.111 = NaN, max 448;
 *          encode = round to nearest even, saturating at 448, sign kept.
 *   Codes are packed two per byte, element 2j in the low nibble.
 *   NVFP4 block quantizer (decode-side global scale g, fp32, every step one IEEE
 *   binary32 operation with round-to-nearest-even):
 *          t  = 6*g ;  s = (t > 0) ? amax_b / t : 0 ;  sb = E4M3(s) ; sd = dec(sb)
 *          d  = sd*g ; if d == 0: all codes 0
 *          r  = 1/d (clamped to FLT_MAX) ; code_i = E2M1(x_i * r)
 *   fp8r row quantizer: s = amax_r / 448 ; if s == 0: all codes 0 ;
 *          r = 1/s (clamped) ; q_i = E4M3(x_i * r)
 *   GEMMs: sum over k of the dequantised products in fp64, times the fp64 product
 *          of the global scales, plus bias, in fp64.
 *
 * Build: plain C11, -O2 -ffp-contract=off (no FMA contraction, no fast-math), so
 * every float expression is one correctly rounded binary32 operation.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <math.h>
#include <float.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* E2M1: explicit decode table, written out from the bit definition.         */
/* code = s e1 e0 m ; e = 0: value m * 0.5 ; e > 0: 2^(e-1) * (1 + m/2)       */
/* ------------------------------------------------------------------------- */
static const float E2M1_VALUE[16] = {
    0.0f,  0.5f,  1.0f,  1.5f,  2.0f,  3.0f,  4.0f,  6.0f,
   -0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f,
};

float oracle_e2m1_decode(uint8_t code) { return E2M1_VALUE[code & 0xF]; }

/* Round-to-nearest over the 8 magnitudes by table search; a tie between two
 * neighbours goes to the one whose code is even (mantissa bit 0); anything
 * above 6 saturates to 6.  The sign bit is copied from the input. */
uint8_t oracle_e2m1_encode(float y)
{
    uint8_t sign = signbit(y) ? 0x8 : 0x0;
    float a = fabsf(y);
    if (isnan(a)) return (uint8_t)(sign | 0x7);        /* unspecified; finite inputs only */
    if (a >= 6.0f) return (uint8_t)(sign | 0x7);
    int best = 0;
    for (int c = 1; c < 8; ++c) {
        float lo = E2M1_VALUE[c - 1], hi = E2M1_VALUE[c];
        if (a < lo) break;
        if (a > hi) { best = c; continue; }
        /* lo <= a <= hi: pick the nearer, ties to the even code */
        float dlo = a - lo, dhi = hi - a;               /* exact: both on a fine grid */
        if (dlo < dhi) best = c - 1;
        else if (dhi < dlo) best = c;
        else best = ((c - 1) % 2 == 0) ? c - 1 : c;
        break;
    }
    return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------------- */
/* E4M3 (FN): decode table of all 256 codes, from the bit definition.        */
/* ------------------------------------------------------------------------- */
static float E4M3_VALUE[256];
static int e4m3_ready = 0;

static void e4m3_build(void)
{
    if (e4m3_ready) return;
    for (int c = 0; c < 256; ++c) {
        int s = (c >> 7) & 1, e = (c >> 3) & 0xF, m = c & 7;
        double v;
        if (e == 0xF && m == 7) v = NAN;
        else if (e == 0)        v = ldexp((double)m / 8.0, -6);
        else                    v = ldexp(1.0 + (double)m / 8.0, e - 7);
        E4M3_VALUE[c] = (float)(s ? -v : v);
    }
    e4m3_ready = 1;
}

float oracle_e4m3_decode(uint8_t code) { e4m3_build(); return E4M3_VALUE[code]; }

/* Nearest of the 127 finite non-negative codes (0x00..0x7E) by binary search on
 * the monotone table; ties to the even code; above 448 saturates to 448. */
uint8_t oracle_e4m3_encode(float y)
{
    e4m3_build();
    uint8_t sign = signbit(y) ? 0x80 : 0x00;
    float a = fabsf(y);
    if (isnan(a)) return (uint8_t)(sign | 0x7F);       /* unspecified; finite inputs only */
    if (a >= 448.0f) return (uint8_t)(sign | 0x7E);
    int lo = 0, hi = 0x7E;                              /* E4M3_VALUE[lo] <= a < E4M3_VALUE[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (E4M3_VALUE[mid] <= a) lo = mid; else hi = mid;
    }
    double dlo = (double)a - (double)E4M3_VALUE[lo];
    double dhi = (double)E4M3_VALUE[hi] - (double)a;    /* exact in double */
    int best;
    if (dlo < dhi) best = lo;
    else if (dhi < dlo) best = hi;
    else best = (lo % 2 == 0) ? lo : hi;
    return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------------- */
/* bf16 helpers                                                               */
/* ------------------------------------------------------------------------- */
static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ------------------------------------------------------------------------- */
/* Scale-factor layouts                                                       */
/*   LINEAR: [R][K/16] row-major (the reading of the checkpoint tensor).      */
/*   MMA   : tiles of 128 rows x 4 block-columns, 512 bytes each, tiles       */
/*           ordered K-fastest; inside a tile, row r and block-column c sit   */
/*           at (r%32)*16 + ((r/32)%4)*4 + c%4.                               */
/* ------------------------------------------------------------------------- */
int64_t oracle_sf_bytes(int64_t R, int64_t K, int mma)
{
    int64_t nb = K / 16;
    if (!mma) return R * nb;
    int64_t rt = (R + 127) / 128, ct = (nb + 3) / 4;
    return rt * ct * 512;
}

int64_t oracle_sf_mma_offset(int64_t r, int64_t c, int64_t K)
{
    int64_t ct = (K / 16 + 3) / 4;
    int64_t tile = (r / 128) * ct + c / 4;
    return tile * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4);
}

/* Copy a linear-layout scale array into the MMA layout; padding bytes are 0. */
/* The encoders above applied to every fp32 whose bit pattern is first, first+1, ...,
 * first+n-1 (an exhaustive pin of a converter walks all 2^32 patterns in ranges).
 * kind 0: E2M1, kind 1: E4M3. */
void oracle_encode_range(int kind, uint32_t first, int64_t n, uint8_t* out)
{
    e4m3_build();                       /* the table once, before the threads read it */
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint32_t bits = first + (uint32_t)i;
        float y;
        memcpy(&y, &bits, sizeof y);
        out[i] = kind == 0 ? oracle_e2m1_encode(y) : oracle_e4m3_encode(y);
    }
}

void oracle_sf_linear_to_mma(const uint8_t* lin, int64_t R, int64_t K, uint8_t* mma)
{
    memset(mma, 0, (size_t)oracle_sf_bytes(R, K, 1));
    int64_t nb = K / 16;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < nb; ++c)
            mma[oracle_sf_mma_offset(r, c, K)] = lin[r * nb + c];
}

/* ------------------------------------------------------------------------- */
/* Global scale: g = amax(X) / (448*6).                                       */
/* ------------------------------------------------------------------------- */
float oracle_amax_bf16(const uint16_t* x, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(bf16_to_f32(x[i]));
        if (a > m) m = a;
    }
    return m;
}

float oracle_nvfp4_global_scale(const uint16_t* x, int64_t n)
{
    float amax = oracle_amax_bf16(x, n);
    return amax / 2688.0f;
}

/* ------------------------------------------------------------------------- */
/* NVFP4 quantizer (one tensor X [R][K], K % 16 == 0).                        */
/* codes: [R][K/2] (element 2j low nibble); sf_lin: [R][K/16] E4M3.           */
/* ------------------------------------------------------------------------- */
static void nvfp4_quantize_row(const uint16_t* xr, int64_t K, float g,
                               uint8_t* cr, uint8_t* sr)
{
    for (int64_t b = 0; b < K / 16; ++b) {
        const uint16_t* xb = xr + b * 16;
        float amax = 0.0f;
        for (int i = 0; i < 16; ++i) {
            float a = fabsf(bf16_to_f32(xb[i]));
            if (a > amax) amax = a;
        }
        float t = 6.0f * g;
        float s = (t > 0.0f) ? amax / t : 0.0f;
        uint8_t sb = oracle_e4m3_encode(s);
        float sd = oracle_e4m3_decode(sb);
        float d = sd * g;
        sr[b] = sb;
        uint8_t q[16];
        if (d == 0.0f) {
            for (int i = 0; i < 16; ++i) q[i] = 0;
        } else {
            float r = 1.0f / d;
            if (r > FLT_MAX) r = FLT_MAX;
            for (int i = 0; i < 16; ++i) {
                float y = bf16_to_f32(xb[i]) * r;
                q[i] = oracle_e2m1_encode(y);
            }
        }
        for (int j = 0; j < 8; ++j)
            cr[b * 8 + j] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
    }
}

void oracle_nvfp4_quantize(const uint16_t* x, int64_t R, int64_t K, float g,
                           uint8_t* codes, uint8_t* sf_lin, int threads)
{
    e4m3_build();                       /* the table once, before the threads read it */
#ifdef _OPENMP
    if (threads < 1) threads = 1;
    #pragma omp parallel for num_threads(threads) schedule(static)
#endif
    for (int64_t r = 0; r < R; ++r)
        nvfp4_quantize_row(x + r * K, K, g, codes + r * (K / 2), sf_lin + r * (K / 16));
    (void)threads;
}

/* Dequantise: xhat = e2m1(code) * e4m3(sb) * g, written in fp64 (exact). */
void oracle_nvfp4_dequant(const uint8_t* codes, const uint8_t* sf_lin, int64_t R, int64_t K,
                          double g, double* out)
{
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t c = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            double sd = (double)oracle_e4m3_decode(sf_lin[r * (K / 16) + k / 16]);
            out[r * K + k] = (double)oracle_e2m1_decode(c) * sd * g;
        }
}

/* Dequantise to bf16, the weight decode of the dequantise-only fallback that the
 * closing paragraph of the "Kernels" section describes (weights back to bf16, then a
 * bf16 GEMM on activations that are not quantized).  Reading taken here: the decode
 * is done in binary32 and rounded once to bf16, nearest-even:
 *     p = e2m1(code) * e4m3(sb)      (exact in binary32: at most 6 significant bits)
 *     y = p * g                      (one binary32 rounding)
 *     out = bf16_rne(y)
 * sf_lin is [R][K/16]; out is [R][K] bf16 bit patterns. */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u);          /* NaN stays NaN (quiet) */
    /* round to nearest, ties to even, on the 16 bits dropped */
    uint32_t lsb = (u >> 16) & 1u;
    uint32_t rounded = u + 0x7FFFu + lsb;
    return (uint16_t)(rounded >> 16);
}

void oracle_nvfp4_dequant_bf16(const uint8_t* codes, const uint8_t* sf_lin, int64_t R,
                               int64_t K, float g, uint16_t* out)
{
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t c = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            float p = oracle_e2m1_decode(c) * oracle_e4m3_decode(sf_lin[r * (K / 16) + k / 16]);
            float y = p * g;
            out[r * K + k] = f32_to_bf16_rne(y);
        }
}

/* ------------------------------------------------------------------------- */
/* fp8r row quantizer: q [R][K] E4M3, s [R] fp32.                             */
/* ------------------------------------------------------------------------- */
static void fp8r_quantize_row(const uint16_t* xr, int64_t K, uint8_t* qr, float* sr)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(bf16_to_f32(xr[k]));
        if (a > amax) amax = a;
    }
    float s = amax / 448.0f;
    *sr = s;
    if (s == 0.0f) {
        for (int64_t k = 0; k < K; ++k) qr[k] = 0;
        return;
    }
    float r = 1.0f / s;
    if (r > FLT_MAX) r = FLT_MAX;
    for (int64_t k = 0; k < K; ++k)
        qr[k] = oracle_e4m3_encode(bf16_to_f32(xr[k]) * r);
}

void oracle_fp8r_quantize(const uint16_t* x, int64_t R, int64_t K, uint8_t* q, float* s,
                          int threads)
{
    e4m3_build();                       /* the table once, before the threads read it */
#ifdef _OPENMP
    if (threads < 1) threads = 1;
    #pragma omp parallel for num_threads(threads) schedule(static)
#endif
    for (int64_t r = 0; r < R; ++r)
        fp8r_quantize_row(x + r * K, K, q + r * K, s + r);
    (void)threads;
}

/* ------------------------------------------------------------------------- */
/* GEMM oracles, fp64.  Y[m][n] = alpha * sum_k A[m][k] * W[n][k] + bias[n].  */
/* rows[] selects which rows of A to compute (NULL = all M rows, in order).   */
/* ------------------------------------------------------------------------- */
void oracle_gemm_f64(const double* A, const double* W, const double* bias,
                     double alpha, const int64_t* rows, int64_t nrows,
                     int64_t N, int64_t K, double* Y, int threads)
{
#ifdef _OPENMP
    if (threads < 1) threads = 1;
    #pragma omp parallel for num_threads(threads) schedule(static)
#endif
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        const double* a = A + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const double* w = W + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += a[k] * w[k];
            Y[i * N + n] = alpha * acc + (bias ? bias[n] : 0.0);
        }
    }
    (void)threads;
}

/* Decode helpers used to build the fp64 operands of the GEMM oracles. */
void oracle_nvfp4_unscaled(const uint8_t* codes, const uint8_t* sf_lin, int64_t R, int64_t K,
                           double* out)
{
    oracle_nvfp4_dequant(codes, sf_lin, R, K, 1.0, out);
}

void oracle_e4m3_decode_array(const uint8_t* q, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = (double)oracle_e4m3_decode(q[i]);
}

/* NVFP4 linear: Y = (gA*gW) * sum_k (e2m1*sd)_A (e2m1*sd)_W + bias. */
void oracle_nvfp4_linear(const uint8_t* a_codes, const uint8_t* a_sf_lin, float a_global,
                         const uint8_t* w_codes, const uint8_t* w_sf_lin, float w_global,
                         const double* bias, const int64_t* rows, int64_t nrows,
                         int64_t M, int64_t N, int64_t K, double* Y,
                         double* scratch_a, double* scratch_w, int threads)
{
    oracle_nvfp4_unscaled(a_codes, a_sf_lin, M, K, scratch_a);
    oracle_nvfp4_unscaled(w_codes, w_sf_lin, N, K, scratch_w);
    double alpha = (double)a_global * (double)w_global;
    oracle_gemm_f64(scratch_a, scratch_w, bias, alpha, rows, nrows, N, K, Y, threads);
}

/* fp8r linear: Y = (sum_k e4m3(a) e4m3(w)) * sA[m] * sW[n] + bias. */
void oracle_fp8r_linear(const uint8_t* a_q, const float* a_s, const uint8_t* w_q,
                        const float* w_s, const double* bias, const int64_t* rows,
                        int64_t nrows, int64_t M, int64_t N, int64_t K, double* Y,
                        double* scratch_a, double* scratch_w, int threads)
{
    oracle_e4m3_decode_array(a_q, M * K, scratch_a);
    oracle_e4m3_decode_array(w_q, N * K, scratch_w);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) scratch_a[m * K + k] *= (double)a_s[m];
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) scratch_w[n * K + k] *= (double)w_s[n];
    oracle_gemm_f64(scratch_a, scratch_w, bias, 1.0, rows, nrows, N, K, Y, threads);
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
