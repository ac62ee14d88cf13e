/*
 * lbq_oracle.c -- plain, slow, scalar CPU oracle for the low-bit weight GEMV.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline leg of bench.py may load this file's library.  It shares no
 * code, header, table or constant with the CUDA library; it only receives
 * the same input bytes.  Build: gcc -O2 -fno-fast-math -ffp-contract=off
 * -fopenmp -shared -fPIC (see oracle/build.py).  Floating point on x86-64
 * is SSE binary32/binary64 with round-to-nearest-even, so every `float`
 * operation below is one correctly rounded IEEE operation.
 *
 * What each function follows (pages are cited by title and section):
 *
 *  - "Métodos de cuantización de LLM para ejecutar un modelo de 70B en una
 *    sola GPU" (gotburnout.io), section "RTN (Round-To-Nearest)": every
 *    weight is rounded to the nearest level of its grid, with no
 *    calibration data.
 *  - "TurboQuant: cuantizar modelos grandes para que quepan en local"
 *    (quellm.com), section "Cómo funciona la compresión" / "Compresión por
 *    bloques": blocks of 32 or 64 weights share one scale and one offset;
 *    "Asignación de bits por capa": 5-6 bits for attention, 2 for MLP.
 *  - "70B en 4GB de VRAM: la compresión neural de 2026, ¿es real?"
 *    (nramos.dev), section "1. NanoQuant — sub-1-bit PTQ", bullet
 *    "Formulación": W ≈ s1 ⊙ (U±1 · V±1ᵀ) ⊙ s2ᵀ with binary low-rank U, V.
 *
 * Readings where the pages are silent:
 *  R1  the group offset is an integer zero-point z with w_hat = s*(q - z);
 *      the grid range is forced to contain 0, so z lies in [0, 2^b-1];
 *  R2  the fp32 scale is rounded UP to fp16, so (hi-lo)/s <= 2^b-1 and
 *      |w - w_hat| <= s/2 holds;
 *  R3  rint = round half to even;
 *  R4  an all-zero group gets s = 1, z = 0;
 *  R5  non-finite weights are rejected (return code -1);
 *  R6  groups run along K (in-features) of a row-major [n x k] weight;
 *  R7  canonical packing: LSB-first bitstream per row (code j, bit t at
 *      stream bit j*b+t); sign packing: element c at bit c%32 of word
 *      c/32, bit 1 meaning +1;
 *  R8  the fragment-interleaved kernel layout is a permutation of the same
 *      bits (tiles of 16 rows x 256 columns in integer tensor-core fragment
 *      order); its index map is written out in orc_kernel_pos() below from
 *      the written specification restated above it, independently of the
 *      CUDA packer.
 *
 * Parity pins for every function live in tests/test_oracle_*.py; there is
 * no function here whose parity is unpinned.
 */
#include <stdint.h>
#include <stddef.h>
#include <math.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* IEEE 754 binary16 and bfloat16, from their definitions.                    */
/* ------------------------------------------------------------------------- */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Subnormals: fraction * 2^-24. */
double orc_f16_decode(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int f = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = (f == 0) ? INFINITY : NAN;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return sign ? -v : v;
}

/* bfloat16 is the upper half of a binary32 word. */
double orc_bf16_decode(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Encode a value that is exactly representable in binary16 (finite). */
static uint16_t f16_encode_exact(double v)
{
    uint16_t sign = 0;
    if (v < 0 || (v == 0 && signbit(v))) { sign = 0x8000; v = -v; }
    if (v == 0) return sign;
    if (v < ldexp(1.0, -14))                       /* subnormal */
        return sign | (uint16_t)(v / ldexp(1.0, -24));
    int ex;
    double fr = frexp(v, &ex);                     /* v = fr * 2^ex, fr in [0.5,1) */
    int E = ex - 1;                                /* v = 1.m * 2^E */
    uint16_t mant = (uint16_t)((fr * 2.0 - 1.0) * 1024.0);
    return sign | (uint16_t)((E + 15) << 10) | mant;
}

/* Round a binary32 value toward +infinity into binary16 (IEEE "roundTowardPositive").
 * For x > 0 the result is the smallest binary16 value >= x; for x < 0 it is
 * the negative of the largest binary16 magnitude <= |x|. */
uint16_t orc_f32_to_f16_ru(float xf)
{
    double x = (double)xf;                         /* exact */
    if (isnan(x)) return 0x7E00;
    if (x == 0) return signbit(x) ? 0x8000 : 0x0000;
    double ax = fabs(x);
    const double maxf = 65504.0;
    if (ax > maxf) {
        if (x > 0) return 0x7C00;                  /* +inf */
        return 0xFBFF;                             /* -65504 */
    }
    /* quantum of the binade containing ax */
    double q;
    if (ax < ldexp(1.0, -14)) {
        q = ldexp(1.0, -24);
    } else {
        int ex;
        frexp(ax, &ex);
        q = ldexp(1.0, (ex - 1) - 10);
    }
    double m = ax / q;                             /* exact: q is a power of two */
    double mag = (x > 0) ? ceil(m) * q : floor(m) * q;
    if (mag > maxf) return (x > 0) ? 0x7C00 : 0xFBFF;
    if (mag == 0) return 0x8000;                   /* tiny negative rounds up to -0 */
    return f16_encode_exact(x > 0 ? mag : -mag);
}

/* ------------------------------------------------------------------------- */
/* RTN group quantization (readings R1-R6).                                   */
/* ------------------------------------------------------------------------- */

static float load_w(const uint16_t* W, int w_is_bf16, int64_t idx)
{
    double d = w_is_bf16 ? orc_bf16_decode(W[idx]) : orc_f16_decode(W[idx]);
    return (float)d;                               /* exact widening */
}

/* W: [n x k] row-major fp16 (or bf16) bit patterns.
 * codes: [n x k] u8; scales, zeros: [n x k/group] fp16 bit patterns.
 * Returns 0, or -1 on a non-finite weight, or -2 on bad arguments. */
int orc_quantize_rtn(const uint16_t* W, int w_is_bf16, int64_t n, int64_t k,
                     int bits, int group, uint8_t* codes,
                     uint16_t* scales, uint16_t* zeros)
{
    if (bits < 2 || bits > 6) return -2;
    if (group <= 0 || k % group != 0) return -2;
    const int qmax = (1 << bits) - 1;
    const float qmaxf = (float)qmax;
    const int64_t G = k / group;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t i = 0; i < n; i++) {
        for (int64_t j = 0; j < G; j++) {
            const int64_t base = i * k + j * group;
            /* step 1: range over the group, forced to contain zero */
            float lo = 0.0f, hi = 0.0f;
            for (int t = 0; t < group; t++) {
                float w = load_w(W, w_is_bf16, base + t);
                if (!isfinite(w)) bad = 1;
                if (w < lo) lo = w;
                if (w > hi) hi = w;
            }
            /* steps 2-4: fp32 step, rounded up to fp16 */
            float d = hi - lo;
            float s32 = d / qmaxf;
            uint16_t sbits = orc_f32_to_f16_ru(s32);
            float s = (float)orc_f16_decode(sbits);
            if (s == 0.0f) { sbits = 0x3C00; s = 1.0f; }
            /* step 5: integer zero-point */
            float zr = rintf(-lo / s);
            int z = (int)zr;
            if (z < 0) z = 0;
            if (z > qmax) z = qmax;
            scales[i * G + j] = sbits;
            zeros[i * G + j] = f16_encode_exact((double)z);
            /* step 6: codes, rounded first, then the zero added */
            for (int t = 0; t < group; t++) {
                float w = load_w(W, w_is_bf16, base + t);
                int q = (int)rintf(w / s) + z;
                if (q < 0) q = 0;
                if (q > qmax) q = qmax;
                codes[base + t] = (uint8_t)q;
            }
        }
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------- */
/* Canonical packing (reading R7).                                            */
/* ------------------------------------------------------------------------- */

int orc_pack_canonical(const uint8_t* codes, int64_t n, int64_t k, int bits, uint8_t* out)
{
    if (bits < 1 || bits > 8 || (k * bits) % 8 != 0) return -2;
    const int64_t stride = k * bits / 8;
    memset(out, 0, (size_t)(n * stride));
    for (int64_t i = 0; i < n; i++)
        for (int64_t j = 0; j < k; j++)
            for (int t = 0; t < bits; t++) {
                int64_t sb = j * bits + t;          /* stream bit */
                if ((codes[i * k + j] >> t) & 1)
                    out[i * stride + sb / 8] |= (uint8_t)(1u << (sb % 8));
            }
    return 0;
}

int orc_unpack_canonical(const uint8_t* in, int64_t n, int64_t k, int bits, uint8_t* codes)
{
    if (bits < 1 || bits > 8 || (k * bits) % 8 != 0) return -2;
    const int64_t stride = k * bits / 8;
    for (int64_t i = 0; i < n; i++)
        for (int64_t j = 0; j < k; j++) {
            int q = 0;
            for (int t = 0; t < bits; t++) {
                int64_t sb = j * bits + t;
                q |= ((in[i * stride + sb / 8] >> (sb % 8)) & 1) << t;
            }
            codes[i * k + j] = (uint8_t)q;
        }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Kernel (fragment-interleaved) layout for group codes (reading R8).         */
/*                                                                            */
/* Specification of the layout:                                             */
/*  * a b-bit code is split into a low plane of width w0 and a high plane    */
/*    of width w1 = b - w0: b=2 -> (2), b=3 -> (2,1), b=4 -> (4),              */
/*    b=5 -> (4,1), b=6 -> (4,2).  Low plane value = q mod 2^w0, high plane   */
/*    value = q >> w0.                                                        */
/*  * rows are cut into tiles of 16 and k into superblocks of 256.  Tile T,   */
/*    superblock S occupies 512*b bytes at byte offset (T*(k/256) + S)*512*b: */
/*    first the low plane (512*w0 bytes), then the high plane (512*w1).       */
/*  * element (row r = 16T + g + 8u, column k = 256S + 32*kappa + 8c + nu),   */
/*    g in 0..7, u in 0..1, kappa in 0..7, c in 0..3, nu in 0..7, belongs to  */
/*    lane L = 4g + c and octet eta = 2*kappa + u of that lane; nu = 2j + e.  */
/*  * in a plane of width w a 32-bit word holds O = 4/w octets: octet        */
/*    eta sits in word omega = eta / O as slot o = eta % O, and its code     */
/*    nu = 2j + e occupies bits 8j + 2w*o + w*e .. +w-1.  Word omega of lane  */
/*    L is at byte (omega/4)*512 + 16L + 4*(omega%4) of the plane.            */
/*    (Masking a word with 0x0F0F0F0F-style byte masks after a shift yields   */
/*    the m16n8k32 u8 A-fragment registers of lane L directly.)               */
/* ------------------------------------------------------------------------- */

static void plane_widths(int bits, int* w0, int* w1)
{
    switch (bits) {
    case 2: *w0 = 2; *w1 = 0; break;
    case 3: *w0 = 2; *w1 = 1; break;
    case 4: *w0 = 4; *w1 = 0; break;
    case 5: *w0 = 4; *w1 = 1; break;
    default: *w0 = 4; *w1 = 2; break;              /* 6 */
    }
}

static int superblock_k(int bits)
{
    (void)bits;
    return 256;
}

/* For element (row i, column kk) and plane index pl (0 low, 1 high), return
 * the absolute bit offset of its first bit within the packed buffer. */
static int64_t orc_kernel_pos(int64_t i, int64_t kk, int64_t k, int bits, int pl)
{
    int w0, w1;
    plane_widths(bits, &w0, &w1);
    const int w = pl == 0 ? w0 : w1;
    const int64_t T = i / 16, r = i % 16;
    const int g = (int)(r % 8), u = (int)(r / 8);
    const int64_t S = kk / 256, ks = kk % 256;
    const int kappa = (int)(ks / 32), c = (int)((ks % 32) / 8), nu = (int)(ks % 8);
    const int j = nu / 2, e = nu % 2;
    const int lane = 4 * g + c;
    const int eta = 2 * kappa + u;
    const int O = 4 / w;
    const int omega = eta / O, o = eta % O;
    int64_t byte = (T * (k / 256) + S) * 512 * bits;
    if (pl == 1) byte += 512 * w0;
    byte += (omega / 4) * 512 + 16 * lane + 4 * (omega % 4);
    return byte * 8 + 8 * j + 2 * w * o + w * e;
}

int orc_pack_kernel(const uint8_t* codes, int64_t n, int64_t k, int bits, uint8_t* out)
{
    if (bits < 2 || bits > 6) return -2;
    const int64_t SB = superblock_k(bits);
    if (n % 16 != 0 || k % SB != 0) return -2;
    int w0, w1;
    plane_widths(bits, &w0, &w1);
    memset(out, 0, (size_t)(n * k * bits / 8));
    for (int64_t i = 0; i < n; i++)
        for (int64_t kk = 0; kk < k; kk++) {
            int q = codes[i * k + kk];
            for (int pl = 0; pl < (w1 ? 2 : 1); pl++) {
                int w = pl ? w1 : w0;
                int v = pl ? (q >> w0) : (q & ((1 << w0) - 1));
                int64_t pos = orc_kernel_pos(i, kk, k, bits, pl);
                for (int t = 0; t < w; t++)
                    if ((v >> t) & 1)
                        out[(pos + t) / 8] |= (uint8_t)(1u << ((pos + t) % 8));
            }
        }
    return 0;
}

int orc_unpack_kernel(const uint8_t* in, int64_t n, int64_t k, int bits, uint8_t* codes)
{
    if (bits < 2 || bits > 6) return -2;
    const int64_t SB = superblock_k(bits);
    if (n % 16 != 0 || k % SB != 0) return -2;
    int w0, w1;
    plane_widths(bits, &w0, &w1);
    for (int64_t i = 0; i < n; i++)
        for (int64_t kk = 0; kk < k; kk++) {
            int q = 0;
            for (int pl = 0; pl < (w1 ? 2 : 1); pl++) {
                int w = pl ? w1 : w0;
                int64_t pos = orc_kernel_pos(i, kk, k, bits, pl);
                int v = 0;
                for (int t = 0; t < w; t++)
                    v |= ((in[(pos + t) / 8] >> ((pos + t) % 8)) & 1) << t;
                q |= pl ? (v << w0) : v;
            }
            codes[i * k + kk] = (uint8_t)q;
        }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Group GEMV / GEMM in fp64: y[m,i] = sum_k x[m,k] * s[i,k/g] * (q[i,k]-z).  */
/* ------------------------------------------------------------------------- */

/* x: [M x k] fp16/bf16 bits; packed: canonical (layout 0) or kernel (1);
 * rows: optional list of output rows (NULL = all n rows, in order);
 * y: [M x nrows] fp64, column j for rows[j]. */
int orc_gemv_group(const uint16_t* x, int x_is_bf16, int64_t M,
                   const uint8_t* packed, int layout,
                   const uint16_t* scales, const uint16_t* zeros,
                   int64_t n, int64_t k, int bits, int group,
                   const int64_t* rows, int64_t nrows, double* y)
{
    if (bits < 2 || bits > 6 || group <= 0 || k % group) return -2;
    if (layout == 1 && (n % 16 || k % superblock_k(bits))) return -2;
    if (rows == NULL) nrows = n;
    const int64_t G = k / group;
    double* xd = (double*)malloc(sizeof(double) * (size_t)(M * k));
    if (!xd) return -3;
    for (int64_t e = 0; e < M * k; e++)
        xd[e] = x_is_bf16 ? orc_bf16_decode(x[e]) : orc_f16_decode(x[e]);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(|:err)
    for (int64_t jr = 0; jr < nrows; jr++) {
        int64_t i = rows ? rows[jr] : jr;
        uint8_t* q = (uint8_t*)malloc((size_t)k);
        double* wh = (double*)malloc(sizeof(double) * (size_t)k);
        if (!q || !wh) { err = 1; free(q); free(wh); continue; }
        /* unpack row i */
        for (int64_t kk = 0; kk < k; kk++) {
            int v = 0;
            if (layout == 0) {
                for (int t = 0; t < bits; t++) {
                    int64_t sb = i * (k * bits) + kk * bits + t;
                    v |= ((packed[sb / 8] >> (sb % 8)) & 1) << t;
                }
            } else {
                int w0, w1;
                plane_widths(bits, &w0, &w1);
                for (int pl = 0; pl < (w1 ? 2 : 1); pl++) {
                    int w = pl ? w1 : w0;
                    int64_t pos = orc_kernel_pos(i, kk, k, bits, pl);
                    int pv = 0;
                    for (int t = 0; t < w; t++)
                        pv |= ((packed[(pos + t) / 8] >> ((pos + t) % 8)) & 1) << t;
                    v |= pl ? (pv << w0) : pv;
                }
            }
            q[kk] = (uint8_t)v;
        }
        /* dequantize (fp64) */
        for (int64_t kk = 0; kk < k; kk++) {
            double s = orc_f16_decode(scales[i * G + kk / group]);
            double z = orc_f16_decode(zeros[i * G + kk / group]);
            wh[kk] = s * ((double)q[kk] - z);
        }
        /* sequential fp64 dot products */
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0;
            for (int64_t kk = 0; kk < k; kk++)
                acc += xd[m * k + kk] * wh[kk];
            y[m * nrows + jr] = acc;
        }
        free(q);
        free(wh);
    }
    free(xd);
    return err ? -3 : 0;
}

/* Dense reference y = x W^T with W given as fp16 bits, fp64 sequential sums. */
int orc_gemv_dense(const uint16_t* x, int x_is_bf16, int64_t M, const uint16_t* W,
                   int64_t n, int64_t k, const int64_t* rows, int64_t nrows, double* y)
{
    if (rows == NULL) nrows = n;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t jr = 0; jr < nrows; jr++) {
        int64_t i = rows ? rows[jr] : jr;
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0;
            for (int64_t kk = 0; kk < k; kk++) {
                double xv = x_is_bf16 ? orc_bf16_decode(x[m * k + kk]) : orc_f16_decode(x[m * k + kk]);
                acc += xv * orc_f16_decode(W[i * k + kk]);
            }
            y[m * nrows + jr] = acc;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Binary low-rank form W_hat = diag(s1) U V^T diag(s2).                      */
/* U: [d_out x r/32] u32 words, Vt = V^T: [r x d_in/32] u32 words, canonical  */
/* sign packing (R7): element c at bit c%32 of word c/32, bit 1 -> +1.        */
/* ------------------------------------------------------------------------- */

int orc_sign_bit(const uint32_t* words, int64_t words_per_row, int64_t row, int64_t col)
{
    return (int)((words[row * words_per_row + col / 32] >> (col % 32)) & 1u);
}

static double sgn(const uint32_t* w, int64_t wpr, int64_t row, int64_t col)
{
    return orc_sign_bit(w, wpr, row, col) ? 1.0 : -1.0;
}

/* Explicit form: reconstruct W_hat [d_out x d_in] in fp64, then y = x W_hat^T. */
int orc_binlr_dense(const uint16_t* x, int x_is_bf16, int64_t M,
                    const uint32_t* U, const uint32_t* Vt,
                    const uint16_t* s1, const uint16_t* s2,
                    int64_t d_out, int64_t d_in, int64_t r, double* y)
{
    if (r % 32 || d_in % 32) return -2;
    double* Wh = (double*)malloc(sizeof(double) * (size_t)(d_out * d_in));
    if (!Wh) return -3;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d_out; i++)
        for (int64_t kk = 0; kk < d_in; kk++) {
            double acc = 0.0;
            for (int64_t j = 0; j < r; j++)
                acc += sgn(U, r / 32, i, j) * sgn(Vt, d_in / 32, j, kk);
            Wh[i * d_in + kk] = orc_f16_decode(s1[i]) * acc * orc_f16_decode(s2[kk]);
        }
    for (int64_t m = 0; m < M; m++)
        for (int64_t i = 0; i < d_out; i++) {
            double acc = 0.0;
            for (int64_t kk = 0; kk < d_in; kk++) {
                double xv = x_is_bf16 ? orc_bf16_decode(x[m * d_in + kk]) : orc_f16_decode(x[m * d_in + kk]);
                acc += xv * Wh[i * d_in + kk];
            }
            y[m * d_out + i] = acc;
        }
    free(Wh);
    return 0;
}

/* Factored form y = s1 ⊙ U (V^T (s2 ⊙ x)), fp64; optional row subset of y.
 * t_out (optional, [M x r]) receives the intermediate V^T (s2 ⊙ x). */
int orc_binlr_factored(const uint16_t* x, int x_is_bf16, int64_t M,
                       const uint32_t* U, const uint32_t* Vt,
                       const uint16_t* s1, const uint16_t* s2,
                       int64_t d_out, int64_t d_in, int64_t r,
                       const int64_t* rows, int64_t nrows, double* y, double* t_out)
{
    if (r % 32 || d_in % 32) return -2;
    if (rows == NULL) nrows = d_out;
    double* xs = (double*)malloc(sizeof(double) * (size_t)(M * d_in));
    double* t = (double*)malloc(sizeof(double) * (size_t)(M * r));
    if (!xs || !t) { free(xs); free(t); return -3; }
    for (int64_t m = 0; m < M; m++)
        for (int64_t kk = 0; kk < d_in; kk++) {
            double xv = x_is_bf16 ? orc_bf16_decode(x[m * d_in + kk]) : orc_f16_decode(x[m * d_in + kk]);
            xs[m * d_in + kk] = orc_f16_decode(s2[kk]) * xv;
        }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < r; j++)
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0;
            for (int64_t kk = 0; kk < d_in; kk++)
                acc += sgn(Vt, d_in / 32, j, kk) * xs[m * d_in + kk];
            t[m * r + j] = acc;
        }
#pragma omp parallel for schedule(static)
    for (int64_t jr = 0; jr < nrows; jr++) {
        int64_t i = rows ? rows[jr] : jr;
        for (int64_t m = 0; m < M; m++) {
            double acc = 0.0;
            for (int64_t j = 0; j < r; j++)
                acc += sgn(U, r / 32, i, j) * t[m * r + j];
            y[m * nrows + jr] = orc_f16_decode(s1[i]) * acc;
        }
    }
    if (t_out) memcpy(t_out, t, sizeof(double) * (size_t)(M * r));
    free(xs);
    free(t);
    return 0;
}

/* Canonical sign packing from +-1 bytes: [rows x cols] int8 -> [rows x cols/32] u32. */
int orc_pack_signs(const int8_t* pm1, int64_t rows, int64_t cols, uint32_t* out)
{
    if (cols % 32) return -2;
    for (int64_t i = 0; i < rows; i++)
        for (int64_t w = 0; w < cols / 32; w++) {
            uint32_t v = 0;
            for (int b = 0; b < 32; b++)
                if (pm1[i * cols + w * 32 + b] > 0) v |= 1u << b;
            out[i * (cols / 32) + w] = v;
        }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Kernel (fragment-interleaved) layout for sign matrices (reading R8).       */
/*                                                                            */
/* Specification of the layout: a sign                                      */
/* matrix [rows x cols] (rows % 16 == 0) has its columns padded with bit 0   */
/* up to cols_pad = 256*ceil(cols/256).  Tile T (16 rows) and superblock S    */
/* (256 columns) occupy 512 bytes at byte offset (T*(cols_pad/256) + S)*512.  */
/* Lane L (g = L/4, c = L%4) owns bytes [16L, 16L+16) = words W0..W3: W0 row  */
/* g, W1 row g+8, W2 row g, W3 row g+8.  Bit 8j+p (p = 0..7, j = 0..3) of W0  */
/* and W1 is column S*256 + 32p + 4c + j; of W2 and W3 column                 */
/* S*256 + 32p + 16 + 4c + j.  (These are the m16n8k32 u8 A-fragment bytes of */
/* lane L for the p-th 32-column slice, one bit per byte at bit p.)           */
/* ------------------------------------------------------------------------- */

int64_t orc_sign_cols_pad(int64_t cols) { return (cols + 255) / 256 * 256; }

static int64_t orc_sign_kernel_pos(int64_t row, int64_t col, int64_t cols)
{
    const int64_t cp = orc_sign_cols_pad(cols);
    const int64_t T = row / 16, r = row % 16;
    const int64_t S = col / 256, cs = col % 256;
    const int64_t p = cs / 32, s = cs % 32;        /* slice, slot */
    const int second = s >= 16;                    /* W2/W3 */
    const int64_t s16 = s % 16;
    const int c = (int)(s16 / 4), j = (int)(s16 % 4);
    const int g = (int)(r % 8), upper = (int)(r / 8);
    const int lane = 4 * g + c;
    const int word = 2 * second + upper;
    const int64_t byte = (T * (cp / 256) + S) * 512 + 16 * lane + 4 * word;
    return byte * 8 + 8 * j + p;
}

/* canonical words [rows x cols/32] -> kernel bytes [rows x cols_pad/8] */
int orc_pack_signs_kernel(const uint32_t* canon, int64_t rows, int64_t cols, uint8_t* out)
{
    if (rows % 16 || cols % 32) return -2;
    const int64_t cp = orc_sign_cols_pad(cols);
    memset(out, 0, (size_t)(rows * cp / 8));
    for (int64_t i = 0; i < rows; i++)
        for (int64_t cc = 0; cc < cols; cc++)
            if (orc_sign_bit(canon, cols / 32, i, cc)) {
                int64_t pos = orc_sign_kernel_pos(i, cc, cols);
                out[pos / 8] |= (uint8_t)(1u << (pos % 8));
            }
    return 0;
}

/* kernel bytes -> canonical words (padding dropped) */
int orc_unpack_signs_kernel(const uint8_t* in, int64_t rows, int64_t cols, uint32_t* canon)
{
    if (rows % 16 || cols % 32) return -2;
    memset(canon, 0, (size_t)(rows * cols / 8));
    for (int64_t i = 0; i < rows; i++)
        for (int64_t cc = 0; cc < cols; cc++) {
            int64_t pos = orc_sign_kernel_pos(i, cc, cols);
            if ((in[pos / 8] >> (pos % 8)) & 1)
                canon[i * (cols / 32) + cc / 32] |= 1u << (cc % 32);
        }
    return 0;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Array helpers for the pins (elementwise applications of the above). */
void orc_f16_decode_array(const uint16_t* in, int64_t n, double* out)
{
    for (int64_t e = 0; e < n; e++) out[e] = orc_f16_decode(in[e]);
}

void orc_f32_to_f16_ru_array(const float* in, int64_t n, uint16_t* out)
{
    for (int64_t e = 0; e < n; e++) out[e] = orc_f32_to_f16_ru(in[e]);
}
