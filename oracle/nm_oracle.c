/*
 * nm_oracle.c -- plain, slow, obviously-correct CPU oracle for N:M
 * fine-grained structured sparsity (mask selection, 2:4 compression,
 * decompression, the tensor-core metadata permutation, and the fp64
 * sparse x dense product).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load
 * or call this file; only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * constant with the CUDA library: every definition here is written out
 * again from the sources cited next to it.
 *
 * Sources (web pages on N:M sparsity; section names as printed there):
 *  [SRSTE]  "SR-STE sparse training (quantisation-friendly)",
 *           blog.bakeneko-kuro.com: section "N:M sparsity / concept",
 *           Apex static mask listing (mn_1d_best / m4n2_1d) and its
 *           explanation, SR-STE forward (argsort top-N of |w| per group).
 *  [ASDNN]  Medium review of "Accelerating Sparse Deep Neural Networks":
 *           "Benefits of 2:4 sparsity" (compressed matrix R*C/2 values,
 *           2-bit metadata per kept value, groups with more zeros still
 *           store 2 values, 36 vs 64 bits per 4 16-bit values),
 *           "Structured sparse GEMM on tensor cores" (sparse x dense =
 *           dense), "Network pruning workflow, Step-2" (drop the two
 *           smallest of every 4).
 *  [SPGPT]  "sparsegpt.py" source page (ken1301225.github.io, code_math
 *           articles): fasterprune, semi-structured branch (prunen of
 *           every prunem columns pruned by the score w^2 / d^2, d the
 *           diagonal of the upper Cholesky factor of the damped inverse
 *           Hessian; weights and Hessian in float32).
 *  [TRANS]  nubint.ai review of "Accelerated Sparse Neural Training: A
 *           Provable and Efficient Method to Find N:M Transposable Masks":
 *           in every MxM block keep the largest L1 norm with N non-zeros
 *           per row and per column (W and W^T both N:M); an exact min-cost
 *           flow and a fast greedy 2-approximation.
 *  [PTX]    NVIDIA PTX ISA, tcgen05 "Sparse matrices" (metadata of
 *           .kind::f16 sparse MMA in tensor memory) -- the pages give no
 *           hardware layout; this is the public ISA description.
 *
 * Readings of points the pages leave open (each is also listed in the
 * design notes):
 *  - N is the number of KEPT entries per group of M.
 *  - Magnitude order: the IEEE bit pattern with the sign cleared, read as
 *    an unsigned integer (+0 == -0, subnormals below normals, Inf above
 *    every finite value, NaN above Inf).
 *  - Ties: equal magnitude -> the lower in-group index is kept.
 *  - decompress writes +0.0 at pruned positions.
 *
 * Floating point: oracle_spmm works in double from exactly-decoded
 * inputs; oracle_srste's step (one binary32 rounding per operation) and
 * oracle_mask_scored's scores are binary32, as their sources compute
 * them.  Magnitude masks use exact integers.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <stdlib.h>
#include <math.h>
#include <pthread.h>

/* element type codes used by this file's callers (tests pass these);
 * OR_S8 is two's-complement int8, whose magnitude is |x| */
enum { OR_F32 = 0, OR_BF16 = 1, OR_F16 = 2, OR_S8 = 3 };

/* status codes */
enum { OR_OK = 0, OR_BAD_ARG = 1, OR_NONFINITE = 2, OR_BAD_MASK = 3 };

static size_t elem_size(int dtype) { return dtype == OR_F32 ? 4 : (dtype == OR_S8 ? 1 : 2); }

static uint32_t load_bits(const void *base, int dtype, size_t i)
{
    if (dtype == OR_F32) return ((const uint32_t *)base)[i];
    if (dtype == OR_S8) return ((const uint8_t *)base)[i];
    return ((const uint16_t *)base)[i];
}

static void store_bits(void *base, int dtype, size_t i, uint32_t v)
{
    if (dtype == OR_F32) ((uint32_t *)base)[i] = v;
    else if (dtype == OR_S8) ((uint8_t *)base)[i] = (uint8_t)v;
    else ((uint16_t *)base)[i] = (uint16_t)v;
}

/* the int8 value of an 8-bit two's-complement pattern */
static int s8_value(uint32_t bits) { return (bits & 0x80u) ? (int)(bits & 0xFFu) - 256 : (int)(bits & 0xFFu); }

/* --------------------------------------------------------------------- */
/* IEEE-754 decoding, written from the format definitions.                */
/*   binary32: 1 sign, 8 exponent (bias 127), 23 fraction                 */
/*   bfloat16: the upper 16 bits of a binary32                            */
/*   binary16: 1 sign, 5 exponent (bias 15), 10 fraction                  */
/* --------------------------------------------------------------------- */
static double decode_generic(uint32_t sign, uint32_t e, uint32_t f,
                             int ebits, int fbits, int bias)
{
    double v;
    uint32_t emax = (1u << ebits) - 1u;
    if (e == emax) {
        if (f != 0) return NAN;
        v = INFINITY;
    } else if (e == 0) {
        v = ldexp((double)f, 1 - bias - fbits);          /* subnormal */
    } else {
        v = ldexp((double)(f | (1u << fbits)), (int)e - bias - fbits);
    }
    return sign ? -v : v;
}

double oracle_decode(uint32_t bits, int dtype)
{
    if (dtype == OR_S8) return (double)s8_value(bits);
    if (dtype == OR_F16)
        return decode_generic(bits >> 15, (bits >> 10) & 0x1Fu, bits & 0x3FFu, 5, 10, 15);
    if (dtype == OR_BF16) bits <<= 16;
    return decode_generic(bits >> 31, (bits >> 23) & 0xFFu, bits & 0x7FFFFFu, 8, 23, 127);
}

/* Round a double to the nearest representable value of a binary format
 * with `fbits` fraction bits, exponent bias `bias` and `ebits` exponent
 * bits, ties to even; overflow to Inf (round-to-nearest semantics).
 * Returns the encoded bit pattern. */
static uint32_t encode_rne(double x, int ebits, int fbits, int bias)
{
    uint32_t sign = signbit(x) ? 1u : 0u;
    uint32_t emax = (1u << ebits) - 1u;
    uint32_t sbit = 1u << (ebits + fbits);
    if (isnan(x)) return (sign ? sbit : 0u) | (emax << fbits) | (1u << (fbits - 1));
    double a = fabs(x);
    if (isinf(a)) return (sign ? sbit : 0u) | (emax << fbits);
    if (a == 0.0) return sign ? sbit : 0u;
    int e2;
    frexp(a, &e2);                 /* a = m * 2^e2, m in [0.5, 1) */
    int exp_unb = e2 - 1;          /* a in [2^exp_unb, 2^(exp_unb+1)) */
    int emin = 1 - bias;
    int q = (exp_unb < emin ? emin : exp_unb) - fbits;  /* quantum exponent */
    double scaled = ldexp(a, -q);  /* exact: power-of-two scaling */
    double fl = floor(scaled);
    double rem = scaled - fl;
    uint64_t n = (uint64_t)fl;
    if (rem > 0.5 || (rem == 0.5 && (n & 1u))) n += 1;
    /* n * 2^q is the rounded magnitude */
    uint32_t E, F;
    if (q == emin - fbits && n < (1ull << fbits)) {
        E = 0; F = (uint32_t)n;                          /* subnormal */
    } else {
        int ee = q + fbits;
        if (n >= (2ull << fbits)) { n >>= 1; ee += 1; }  /* carried into next binade */
        if (ee + bias >= (int)emax) return (sign ? sbit : 0u) | (emax << fbits);
        E = (uint32_t)(ee + bias);
        F = (uint32_t)(n - (1ull << fbits));
    }
    return (sign ? sbit : 0u) | (E << fbits) | F;
}

uint32_t oracle_encode(double x, int dtype)
{
    if (dtype == OR_F16) return encode_rne(x, 5, 10, 15);
    if (dtype == OR_BF16) return encode_rne(x, 8, 7, 127);
    return encode_rne(x, 8, 23, 127);
}

/* Magnitude key: sign bit cleared, read as unsigned. */
uint32_t oracle_mag(uint32_t bits, int dtype)
{
    if (dtype == OR_S8) {
        const int v = s8_value(bits);
        return (uint32_t)(v < 0 ? -v : v);
    }
    return dtype == OR_F32 ? (bits & 0x7FFFFFFFu) : (bits & 0x7FFFu);
}

/* --------------------------------------------------------------------- */
/* Mask, variant S: rank rule.                                           */
/* [SRSTE] SR-STE forward: argsort |w| inside each group of M and zero   */
/* the M-N smallest; [ASDNN] Step-2: drop the smallest of every group.   */
/* Element i is kept iff fewer than N elements of its group beat it,     */
/* where j beats i when mag_j > mag_i, or mag_j == mag_i and j < i.       */
/* Groups are M consecutive entries of a row (the reduction dimension).  */
/* --------------------------------------------------------------------- */
int oracle_mask_rank(const void *W, int dtype, int64_t R, int64_t C, int64_t ldw,
                     int N, int M, uint8_t *mask, int64_t ldm)
{
    if (M < 2 || M > 8 || N < 1 || N >= M || C % M != 0 || R < 0 || C < 0)
        return OR_BAD_ARG;
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t g = 0; g < C / M; ++g) {
            uint32_t mag[8];
            for (int i = 0; i < M; ++i)
                mag[i] = oracle_mag(load_bits(W, dtype, (size_t)(r * ldw + g * M + i)), dtype);
            for (int i = 0; i < M; ++i) {
                int beaten_by = 0;
                for (int j = 0; j < M; ++j) {
                    if (j == i) continue;
                    if (mag[j] > mag[i] || (mag[j] == mag[i] && j < i)) beaten_by++;
                }
                mask[r * ldm + g * M + i] = (uint8_t)(beaten_by < N ? 1 : 0);
            }
        }
    }
    return OR_OK;
}

/* --------------------------------------------------------------------- */
/* Saliency-scored mask.  [SPGPT] semi-structured branch: inside every    */
/* group of M consecutive columns the score of w is w^2 / d^2, with d the */
/* entry of its column in the caller's vector (the diagonal of the upper  */
/* Cholesky factor of the inverse Hessian there), and the M-N smallest    */
/* scores are pruned (topk with largest=False).  In binary32, as there:   */
/*   s = fl( fl(w*w) / fl(d*d) )                                          */
/* each product and the quotient rounded once to nearest even.  Scores    */
/* are ranked by their bit pattern with the sign cleared (the magnitude   */
/* order above; 0/0 gives NaN, which ranks highest); equal scores keep    */
/* the lower in-group index.                                              */
/* --------------------------------------------------------------------- */
static uint32_t f32_bits(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    return u;
}

int oracle_mask_scored(const void *W, int dtype, const float *d, int64_t R, int64_t C, int64_t ldw,
                       int N, int M, uint8_t *mask, int64_t ldm)
{
    if (M < 2 || M > 8 || N < 1 || N >= M || C % M != 0 || R < 0 || C < 0)
        return OR_BAD_ARG;
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t g = 0; g < C / M; ++g) {
            uint32_t key[8];
            for (int i = 0; i < M; ++i) {
                const int64_t c = g * M + i;
                const float w = (float)oracle_decode(load_bits(W, dtype, (size_t)(r * ldw + c)), dtype);
                volatile float ww = w * w;          /* binary32, rounded once */
                volatile float dd = d[c] * d[c];
                volatile float sc = ww / dd;
                key[i] = f32_bits(sc) & 0x7FFFFFFFu;
            }
            for (int i = 0; i < M; ++i) {
                int beaten_by = 0;
                for (int j = 0; j < M; ++j) {
                    if (j == i) continue;
                    if (key[j] > key[i] || (key[j] == key[i] && j < i)) beaten_by++;
                }
                mask[r * ldm + g * M + i] = (uint8_t)(beaten_by < N ? 1 : 0);
            }
        }
    }
    return OR_OK;
}

/* --------------------------------------------------------------------- */
/* Transposable N:M mask, greedy.  [TRANS]: inside every MxM block (rows  */
/* r0..r0+M-1, columns c0..c0+M-1) the mask should keep as much |w| as     */
/* possible with at most N kept entries in each row and in each column,    */
/* so that W and its transpose are both N:M.  The page names a fast        */
/* 2-approximation without printing it; the reading here is the standard   */
/* greedy for this weighted b-matching:                                    */
/*   1. order the M*M entries by magnitude (as oracle_mag), largest first, */
/*      equal magnitudes by row-major position within the block;           */
/*   2. walk that order and keep an entry when its row and its column each */
/*      hold fewer than N kept entries.                                    */
/* The result keeps at least half of the optimum's |w| (each optimal entry */
/* left out is blocked by a kept entry at least as large in its row or     */
/* column, and each kept entry blocks at most two such).                   */
/* --------------------------------------------------------------------- */
typedef struct { uint32_t key; int pos; } tr_entry;

static int tr_cmp(const void *pa, const void *pb)
{
    const tr_entry *a = (const tr_entry *)pa, *b = (const tr_entry *)pb;
    if (a->key != b->key) return a->key > b->key ? -1 : 1;   /* larger magnitude first */
    return a->pos - b->pos;                                  /* then lower position    */
}

int oracle_mask_transposable(const void *W, int dtype, int64_t R, int64_t C, int64_t ldw,
                             int N, int M, uint8_t *mask, int64_t ldm)
{
    if (M < 2 || M > 8 || N < 1 || N >= M || R % M != 0 || C % M != 0 || R < 0 || C < 0)
        return OR_BAD_ARG;
    for (int64_t br = 0; br < R / M; ++br) {
        for (int64_t bc = 0; bc < C / M; ++bc) {
            tr_entry e[64];
            int row_kept[8] = {0}, col_kept[8] = {0};
            for (int i = 0; i < M; ++i)
                for (int j = 0; j < M; ++j) {
                    const int64_t r = br * M + i, c = bc * M + j;
                    e[i * M + j].key = oracle_mag(load_bits(W, dtype, (size_t)(r * ldw + c)), dtype);
                    e[i * M + j].pos = i * M + j;
                    mask[r * ldm + c] = 0;
                }
            qsort(e, (size_t)(M * M), sizeof e[0], tr_cmp);
            for (int t = 0; t < M * M; ++t) {
                const int i = e[t].pos / M, j = e[t].pos % M;
                if (row_kept[i] < N && col_kept[j] < N) {
                    row_kept[i]++;
                    col_kept[j]++;
                    mask[(br * M + i) * ldm + bc * M + j] = 1;
                }
            }
        }
    }
    return OR_OK;
}

/* --------------------------------------------------------------------- */
/* Mask, variant E: exhaustive pattern search.                           */
/* [SRSTE] Apex listing (mn_1d_best): enumerate every pattern with N     */
/* ones among M places, score each by the L1 sum of the |w| it keeps,    */
/* take the argmax.  Here the sums are EXACT (multi-limb integers in     */
/* units of 2^-149, the smallest binary32 subnormal) so no rounding can  */
/* create a false tie, patterns are visited in lexicographic order of    */
/* their ascending index tuples, and the first strictly greater score    */
/* wins.  Only finite inputs are accepted.                                */
/* --------------------------------------------------------------------- */
#define LIMBS 5  /* 320 bits >= 277-bit magnitude + 3 bits of carry */
typedef struct { uint64_t w[LIMBS]; } big_t;

static void big_zero(big_t *a) { memset(a, 0, sizeof *a); }

static void big_add_shifted(big_t *a, uint64_t m, int shift)
{
    /* a += m << shift, m < 2^24 */
    int limb = shift / 64, off = shift % 64;
    uint64_t lo = m << off;
    uint64_t hi = off ? (m >> (64 - off)) : 0;
    uint64_t carry = 0;
    for (int i = limb; i < LIMBS; ++i) {
        uint64_t add = (i == limb) ? lo : (i == limb + 1 ? hi : 0);
        uint64_t s = a->w[i] + add;
        uint64_t c1 = s < add;
        uint64_t s2 = s + carry;
        uint64_t c2 = s2 < carry;
        a->w[i] = s2;
        carry = c1 + c2;
        if (i > limb + 1 && carry == 0) break;
    }
}

static int big_cmp(const big_t *a, const big_t *b)
{
    for (int i = LIMBS - 1; i >= 0; --i) {
        if (a->w[i] != b->w[i]) return a->w[i] > b->w[i] ? 1 : -1;
    }
    return 0;
}

/* |w| = m * 2^(shift-149): returns 0 on success, -1 if non-finite */
static int exact_magnitude(uint32_t bits, int dtype, uint64_t *m, int *shift)
{
    if (dtype == OR_S8) { *m = oracle_mag(bits, OR_S8); *shift = 149; return 0; }   /* |x| * 2^0 */
    if (dtype == OR_BF16) { bits <<= 16; dtype = OR_F32; }
    if (dtype == OR_F32) {
        uint32_t e = (bits >> 23) & 0xFFu, f = bits & 0x7FFFFFu;
        if (e == 0xFFu) return -1;
        if (e == 0) { *m = f; *shift = 0; }
        else { *m = f | (1u << 23); *shift = (int)e - 1; }
        return 0;
    }
    /* binary16: subnormal f * 2^-24 ; normal (1.f) * 2^(e-15) */
    uint32_t e = (bits >> 10) & 0x1Fu, f = bits & 0x3FFu;
    if (e == 0x1Fu) return -1;
    if (e == 0) { *m = f; *shift = 125; }                 /* 2^-24 = 2^(125-149) */
    else { *m = f | (1u << 10); *shift = (int)e + 124; }   /* 2^(e-25) */
    return 0;
}

int oracle_mask_exhaustive(const void *W, int dtype, int64_t R, int64_t C, int64_t ldw,
                           int N, int M, uint8_t *mask, int64_t ldm)
{
    if (M < 2 || M > 8 || N < 1 || N >= M || C % M != 0 || R < 0 || C < 0)
        return OR_BAD_ARG;
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t g = 0; g < C / M; ++g) {
            uint64_t m[8]; int sh[8];
            for (int i = 0; i < M; ++i) {
                uint32_t b = load_bits(W, dtype, (size_t)(r * ldw + g * M + i));
                if (exact_magnitude(b, dtype, &m[i], &sh[i]) != 0) return OR_NONFINITE;
            }
            int idx[8], best[8];
            for (int i = 0; i < N; ++i) idx[i] = i;   /* first combination */
            big_t best_score; int have_best = 0;
            for (;;) {
                big_t s; big_zero(&s);
                for (int i = 0; i < N; ++i) big_add_shifted(&s, m[idx[i]], sh[idx[i]]);
                if (!have_best || big_cmp(&s, &best_score) > 0) {
                    best_score = s; have_best = 1;
                    memcpy(best, idx, sizeof(int) * (size_t)N);
                }
                /* next combination in lexicographic order */
                int p = N - 1;
                while (p >= 0 && idx[p] == M - N + p) --p;
                if (p < 0) break;
                idx[p]++;
                for (int q = p + 1; q < N; ++q) idx[q] = idx[q - 1] + 1;
            }
            for (int i = 0; i < M; ++i) mask[r * ldm + g * M + i] = 0;
            for (int i = 0; i < N; ++i) mask[r * ldm + g * M + best[i]] = 1;
        }
    }
    return OR_OK;
}

/* --------------------------------------------------------------------- */
/* 2:4 compression. [ASDNN] "Benefits of 2:4 sparsity": the compressed   */
/* matrix holds R*C/2 values, and 2-bit metadata gives the in-group      */
/* position of each kept value; every group stores exactly 2 values even */
/* when it holds more zeros.                                              */
/* Canonical layout (this library's documented choice):                   */
/*   values[r][2g+j] = W[r][4g+idx_j], idx_0 < idx_1, bits copied as-is   */
/*   meta: kept entry k = 2g+j of row r -> its 2-bit idx_j in bits        */
/*   2*(k%4) .. 2*(k%4)+1 of byte r*(C/8) + k/4 (LSB first).              */
/* The mask holds 0/1 bytes with at most 2 ones per group; otherwise     */
/* OR_BAD_MASK.  A group with fewer than 2 ones (a 1:4 mask, a greedy     */
/* transposable mask) still stores two values, as the page says of groups */
/* with more zeros: the pair is the kept positions plus the lowest unkept */
/* ones, in ascending order, and an unkept position's value is +0.0, so   */
/* decompression gives W where kept and +0.0 elsewhere.                   */
/* --------------------------------------------------------------------- */
int oracle_compress24(const void *W, const uint8_t *mask, int dtype, int64_t R, int64_t C,
                      void *values, uint8_t *meta)
{
    if (C % 8 != 0 || R < 0) return OR_BAD_ARG;
    memset(meta, 0, (size_t)(R * C / 8));
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t g = 0; g < C / 4; ++g) {
            int keep[4], nk = 0;
            for (int i = 0; i < 4; ++i) {
                uint8_t mv = mask[r * C + g * 4 + i];
                if (mv > 1) return OR_BAD_MASK;
                keep[i] = mv;
                nk += mv;
            }
            if (nk > 2) return OR_BAD_MASK;
            /* fill up to two positions with the lowest unkept indices */
            int take[4];
            for (int i = 0; i < 4; ++i) take[i] = keep[i];
            for (int i = 0; i < 4 && nk < 2; ++i)
                if (!take[i]) { take[i] = 1; ++nk; }
            int j = 0;
            for (int i = 0; i < 4; ++i) {
                if (!take[i]) continue;
                int64_t k = 2 * g + j;
                uint32_t b = keep[i] ? load_bits(W, dtype, (size_t)(r * C + g * 4 + i)) : 0u;
                store_bits(values, dtype, (size_t)(r * (C / 2) + k), b);
                meta[r * (C / 8) + k / 4] |= (uint8_t)(i << (2 * (k % 4)));
                ++j;
            }
        }
    }
    return OR_OK;
}

/* Inverse of the above: kept positions get their value, others +0.0. */
int oracle_decompress24(const void *values, const uint8_t *meta, int dtype, int64_t R, int64_t C,
                        void *W_out)
{
    if (C % 8 != 0 || R < 0) return OR_BAD_ARG;
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t c = 0; c < C; ++c) store_bits(W_out, dtype, (size_t)(r * C + c), 0u);
        for (int64_t k = 0; k < C / 2; ++k) {
            int idx = (meta[r * (C / 8) + k / 4] >> (2 * (k % 4))) & 3;
            int64_t g = k / 2;
            uint32_t b = load_bits(values, dtype, (size_t)(r * (C / 2) + k));
            store_bits(W_out, dtype, (size_t)(r * C + g * 4 + idx), b);
        }
    }
    return OR_OK;
}

/* --------------------------------------------------------------------- */
/* 1:2 compression.  [ASDNN] "Structured sparse GEMM on tensor cores":    */
/* sparse TF32 works only with a 1:2 pattern (one of every two values).   */
/* Layout (this library's choice, as the 2:4 one): values[r][p] is the    */
/* kept element of pair p (columns 2p, 2p+1) of row r, bits as stored;    */
/* its index (0 or 1) is bit p%8 of byte r*(C/16) + p/8 (LSB first).     */
/* The mask must hold exactly one 1 per pair; otherwise OR_BAD_MASK.      */
/* --------------------------------------------------------------------- */
int oracle_compress12(const void *W, const uint8_t *mask, int dtype, int64_t R, int64_t C,
                      void *values, uint8_t *meta)
{
    if (C % 16 != 0 || R < 0) return OR_BAD_ARG;
    memset(meta, 0, (size_t)(R * C / 16));
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t p = 0; p < C / 2; ++p) {
            const uint8_t m0 = mask[r * C + 2 * p], m1 = mask[r * C + 2 * p + 1];
            if (m0 > 1 || m1 > 1 || m0 + m1 != 1) return OR_BAD_MASK;
            const int idx = m1 ? 1 : 0;
            store_bits(values, dtype, (size_t)(r * (C / 2) + p), load_bits(W, dtype, (size_t)(r * C + 2 * p + idx)));
            meta[r * (C / 16) + p / 8] |= (uint8_t)(idx << (p % 8));
        }
    }
    return OR_OK;
}

/* Inverse: the kept position of each pair gets its value, the other +0.0. */
int oracle_decompress12(const void *values, const uint8_t *meta, int dtype, int64_t R, int64_t C,
                        void *W_out)
{
    if (C % 16 != 0 || R < 0) return OR_BAD_ARG;
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t p = 0; p < C / 2; ++p) {
            const int idx = (meta[r * (C / 16) + p / 8] >> (p % 8)) & 1;
            const uint32_t b = load_bits(values, dtype, (size_t)(r * (C / 2) + p));
            store_bits(W_out, dtype, (size_t)(r * C + 2 * p + idx), b);
            store_bits(W_out, dtype, (size_t)(r * C + 2 * p + 1 - idx), 0u);
        }
    }
    return OR_OK;
}

/* --------------------------------------------------------------------- */
/* Tensor-core metadata layout for the sm_100 sparse MMA (.kind::f16).    */
/* [PTX] tcgen05 sparse matrices: for an MMA of 128 rows x 32 (logical)  */
/* K, each row's metadata is 32 bits: 8 groups of 4, a 4-bit field per   */
/* group holding idx_0 | idx_1 << 2.  In tensor memory, lane L of the     */
/* 32-bit column holds, for m2 = L/16, h = (L%16)/8, m0 = L%8:            */
/*     bits  0..15: row 16*m2 + m0,     groups 4h..4h+3 of the 32-K slice */
/*     bits 16..31: row 16*m2 + 8 + m0, groups 4h..4h+3 of the 32-K slice */
/* This library stores, per block of 128 rows x 128 logical K, the exact  */
/* 2048-byte image that one 128-lane x 128-bit copy puts in tensor memory:*/
/*   block (rt, kt) at byte ((rt * ceil(C/128)) + kt) * 2048              */
/*   16 bytes per lane L, 4 bytes per 32-K slice s = (c%128)/32.          */
/* Rows are padded to a multiple of 128 and C to a multiple of 128; the   */
/* padding carries the valid pattern (0,1), nibble 0x4.                   */
/* --------------------------------------------------------------------- */
int64_t oracle_meta_sm100_bytes(int64_t R, int64_t C)
{
    int64_t Rp = (R + 127) / 128 * 128, Cp = (C + 127) / 128 * 128;
    return Rp * Cp / 8;
}

int oracle_meta_sm100(const uint8_t *meta, int64_t R, int64_t C, uint8_t *out)
{
    if (C % 8 != 0 || R < 0) return OR_BAD_ARG;
    int64_t Rp = (R + 127) / 128 * 128, Cp = (C + 127) / 128 * 128;
    int64_t kblocks = Cp / 128;
    memset(out, 0, (size_t)(Rp * Cp / 8));
    for (int64_t r = 0; r < Rp; ++r) {
        for (int64_t g = 0; g < Cp / 4; ++g) {
            uint32_t nib;
            if (r < R && g < C / 4) {
                /* group g holds kept entries 2g and 2g+1 */
                int i0 = (meta[r * (C / 8) + (2 * g) / 4] >> (2 * ((2 * g) % 4))) & 3;
                int i1 = (meta[r * (C / 8) + (2 * g + 1) / 4] >> (2 * ((2 * g + 1) % 4))) & 3;
                nib = (uint32_t)(i0 | (i1 << 2));
            } else {
                nib = 0x4u;
            }
            int64_t c = 4 * g;                       /* first logical column of the group */
            int64_t rt = r / 128, kt = c / 128;
            int64_t rr = r % 128, cc = c % 128;
            int64_t lane = (rr % 8) + 8 * ((cc % 32) / 16) + 16 * (rr / 16);
            int64_t slice = cc / 32;
            int64_t bit = 16 * ((rr % 16) / 8) + 4 * ((cc % 16) / 4);
            int64_t byte = (rt * kblocks + kt) * 2048 + lane * 16 + slice * 4 + bit / 8;
            out[byte] |= (uint8_t)(nib << (bit % 8));
        }
    }
    return OR_OK;
}

/* --------------------------------------------------------------------- */
/* Tensor-core metadata for the int8 sparse MMA (.kind::i8).  [PTX]       */
/* tcgen05 sparse matrices: an i8 MMA covers 64 logical K per row, 16     */
/* groups of 4 with the same 4-bit field idx_0 | idx_1 << 2 per group,    */
/* and its metadata fills two 32-bit tensor-memory columns of the row's   */
/* own lane, group g at bit 4*(g%8) of column g/8 -- the canonical         */
/* row-major order of this library's metadata, read as little-endian      */
/* words.  The image holds, per block of 128 rows x 128 logical K, the    */
/* 2048 bytes one 128-lane x 128-bit copy moves: lane L = r%128 gets the  */
/* 16 canonical bytes of row r for those 128 columns.  Blocks are stored   */
/* row-tile major, block (rt, kt) at byte (rt*nk + kt)*2048 with           */
/* nk = 2*ceil(C/256) (K is padded to the product's 256-column stage).    */
/* Padding rows and columns hold the valid pattern (0,1), byte 0x44.      */
/* --------------------------------------------------------------------- */
int64_t oracle_meta_sm100_s8_bytes(int64_t R, int64_t C)
{
    int64_t Rp = (R + 127) / 128 * 128, Cp = (C + 255) / 256 * 256;
    return Rp * Cp / 8;
}

int oracle_meta_sm100_s8(const uint8_t *meta, int64_t R, int64_t C, uint8_t *out)
{
    if (C % 8 != 0 || R < 0) return OR_BAD_ARG;
    int64_t nk = (C + 255) / 256 * 2;
    memset(out, 0x44, (size_t)oracle_meta_sm100_s8_bytes(R, C));
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t b = 0; b < C / 8; ++b) {      /* canonical byte b: groups 2b, 2b+1 */
            int64_t rt = r / 128, kt = b / 16;      /* 16 bytes = 128 logical columns */
            out[(rt * nk + kt) * 2048 + (r % 128) * 16 + (b % 16)] = meta[r * (C / 8) + b];
        }
    }
    return OR_OK;
}

/* --------------------------------------------------------------------- */
/* Tensor-core metadata for the 1:2 TF32 sparse MMA (.kind::tf32).  [PTX] */
/* tcgen05 sparse matrices: a tf32 MMA covers 16 logical K per row (one  */
/* of each pair kept), and its metadata has the .kind::f16 layout for the */
/* row seen as 16-bit halves: pair p of 32-bit elements is the group of   */
/* four halves 4p..4p+3, and its field is 0x4 (halves 0,1: element 0      */
/* kept) or 0xE (halves 2,3: element 1 kept).  The image is therefore the */
/* .kind::f16 image above for the R x 2C matrix of halves: per block of   */
/* 128 rows x 64 fp32 columns, 2048 bytes, lane L = r%8 + 8*((h%32)/16)   */
/* + 16*((r%128)/16), bits 16*((r%16)/8) + 4*((h%16)/4) of slice          */
/* (h%128)/32, with h = 4p the pair's first half-column.  Blocks row-tile */
/* major, block (rt, kt) at byte (rt*ceil(C/64) + kt)*2048; padding pairs */
/* hold 0x4.                                                               */
/* --------------------------------------------------------------------- */
int64_t oracle_meta12_sm100_bytes(int64_t R, int64_t C)
{
    return (R + 127) / 128 * ((C + 63) / 64) * 2048;
}

int oracle_meta12_sm100(const uint8_t *meta, int64_t R, int64_t C, uint8_t *out)
{
    if (C % 16 != 0 || R < 0) return OR_BAD_ARG;
    int64_t Rp = (R + 127) / 128 * 128, Cp = (C + 63) / 64 * 64, kblocks = Cp / 64;
    memset(out, 0, (size_t)oracle_meta12_sm100_bytes(R, C));
    for (int64_t r = 0; r < Rp; ++r) {
        for (int64_t p = 0; p < Cp / 2; ++p) {
            uint32_t nib = 0x4u;
            if (r < R && p < C / 2 && ((meta[r * (C / 16) + p / 8] >> (p % 8)) & 1)) nib = 0xEu;
            int64_t h = 4 * p;                       /* first half-column of the pair */
            int64_t rt = r / 128, kt = h / 128;
            int64_t rr = r % 128, hh = h % 128;
            int64_t lane = (rr % 8) + 8 * ((hh % 32) / 16) + 16 * (rr / 16);
            int64_t slice = hh / 32;
            int64_t bit = 16 * ((rr % 16) / 8) + 4 * ((hh % 16) / 4);
            out[(rt * kblocks + kt) * 2048 + lane * 16 + slice * 4 + bit / 8] |= (uint8_t)(nib << (bit % 8));
        }
    }
    return OR_OK;
}

/* --------------------------------------------------------------------- */
/* Sparse x dense product in double.  [ASDNN] "Structured sparse GEMM on  */
/* tensor cores": sparse matrix x dense matrix = dense matrix; only the  */
/* kept values are multiplied.                                            */
/*   Y[r][t] = alpha * sum_k values[r][k] * X[col(r, k)][t]               */
/*             + beta * Y_in[r][t]        (Y_in not read when beta == 0)  */
/* 2:4 (oracle_spmm): col(r, k) = 4*(k/2) + idx_k from the canonical 2:4  */
/* metadata.  1:2 (oracle_spmm12): col(r, k) = 2*k + idx_k from the 1:2    */
/* metadata (one index bit per pair).  X is K x T row-major, Y_in R x T    */
/* row-major (y_dtype).  Floating-point inputs are decoded exactly and     */
/* summed in double.  int8 inputs (OR_S8) are summed exactly in int64      */
/* (every product is an integer of magnitude <= 2^14) and the sum is then  */
/* exact in double for |sum| < 2^53.  Only the listed rows are computed    */
/* (rows == NULL means all R rows); Y_out is nrows x T doubles.            */
/* --------------------------------------------------------------------- */
typedef struct {
    const void *values; const uint8_t *meta; int ab_dtype;
    const void *X; int64_t T; const void *Y_in; int y_dtype;
    int64_t R, K; double alpha, beta;
    const int64_t *rows; int64_t nrows; double *Y_out;
    int64_t lo, hi; int pattern;   /* 24: 2:4 metadata, 12: 1:2 metadata */
} spmm_job;

/* exact decode of one element to double: a 65536-entry table for the
 * 16-bit formats (filled by oracle_decode), a plain float->double
 * conversion (exact in C) for binary32 */
static double *g_tab[3];
static pthread_once_t g_tab_once = PTHREAD_ONCE_INIT;
static void build_tables(void)
{
    for (int d = OR_BF16; d <= OR_F16; ++d) {
        g_tab[d] = (double *)malloc(sizeof(double) * 65536);
        for (uint32_t b = 0; b < 65536; ++b) g_tab[d][b] = oracle_decode(b, d);
    }
}

static double decode_fast(const void *base, int dtype, size_t i)
{
    if (dtype == OR_S8) return (double)s8_value(((const uint8_t *)base)[i]);
    if (dtype == OR_F32) {
        float f;
        memcpy(&f, (const char *)base + 4 * i, 4);
        return (double)f;
    }
    return g_tab[dtype][((const uint16_t *)base)[i]];
}

/* logical column of kept value k of row r */
static int64_t kept_column(const spmm_job *j, int64_t r, int64_t k)
{
    if (j->pattern == 12) {
        int idx = (j->meta[r * (j->K / 16) + k / 8] >> (k % 8)) & 1;
        return 2 * k + idx;
    }
    int idx = (j->meta[r * (j->K / 8) + k / 4] >> (2 * (k % 4))) & 3;
    return 4 * (k / 2) + idx;
}

static void *spmm_worker(void *arg)
{
    spmm_job *j = (spmm_job *)arg;
    size_t n = (size_t)(j->T > 0 ? j->T : 1);
    double *acc = (double *)malloc(sizeof(double) * n);
    int64_t *iacc = (int64_t *)malloc(sizeof(int64_t) * n);
    const int ints = j->ab_dtype == OR_S8;
    for (int64_t i = j->lo; i < j->hi; ++i) {
        int64_t r = j->rows ? j->rows[i] : i;
        for (int64_t t = 0; t < j->T; ++t) { acc[t] = 0.0; iacc[t] = 0; }
        for (int64_t k = 0; k < j->K / 2; ++k) {
            int64_t kk = kept_column(j, r, k);
            size_t vi = (size_t)(r * (j->K / 2) + k);
            if (ints) {
                int64_t v = s8_value(((const uint8_t *)j->values)[vi]);
                const uint8_t *xrow = (const uint8_t *)j->X + kk * j->T;
                for (int64_t t = 0; t < j->T; ++t) iacc[t] += v * s8_value(xrow[t]);
            } else {
                double v = decode_fast(j->values, j->ab_dtype, vi);
                for (int64_t t = 0; t < j->T; ++t)
                    acc[t] += v * decode_fast(j->X, j->ab_dtype, (size_t)(kk * j->T + t));
            }
        }
        for (int64_t t = 0; t < j->T; ++t) {
            double sum = ints ? (double)iacc[t] : acc[t];
            double y = j->alpha * sum;
            if (j->beta != 0.0)
                y += j->beta * decode_fast(j->Y_in, j->y_dtype, (size_t)(r * j->T + t));
            j->Y_out[i * j->T + t] = y;
        }
    }
    free(acc);
    free(iacc);
    return NULL;
}

static int spmm_run(int pattern, const void *values, const uint8_t *meta, int ab_dtype,
                    const void *X, int64_t T, const void *Y_in, int y_dtype,
                    int64_t R, int64_t K, double alpha, double beta,
                    const int64_t *rows, int64_t nrows, int nthreads, double *Y_out)
{
    if (K % (pattern == 12 ? 16 : 8) != 0 || R < 0 || T < 0) return OR_BAD_ARG;
    if (rows == NULL) nrows = R;
    for (int64_t i = 0; rows && i < nrows; ++i) if (rows[i] < 0 || rows[i] >= R) return OR_BAD_ARG;
    pthread_once(&g_tab_once, build_tables);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nrows < nthreads) nthreads = (int)(nrows > 0 ? nrows : 1);
    spmm_job jobs[256];
    pthread_t th[256];
    for (int i = 0; i < nthreads; ++i) {
        spmm_job j = { values, meta, ab_dtype, X, T, Y_in, y_dtype, R, K, alpha, beta,
                       rows, nrows, Y_out, nrows * i / nthreads, nrows * (i + 1) / nthreads, pattern };
        jobs[i] = j;
    }
    if (nthreads == 1) { spmm_worker(&jobs[0]); return OR_OK; }
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, spmm_worker, &jobs[i]);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    return OR_OK;
}

int oracle_spmm(const void *values, const uint8_t *meta, int ab_dtype,
                const void *X, int64_t T, const void *Y_in, int y_dtype,
                int64_t R, int64_t K, double alpha, double beta,
                const int64_t *rows, int64_t nrows, int nthreads, double *Y_out)
{
    return spmm_run(24, values, meta, ab_dtype, X, T, Y_in, y_dtype, R, K, alpha, beta, rows, nrows,
                    nthreads, Y_out);
}

int oracle_spmm12(const void *values, const uint8_t *meta, int ab_dtype,
                  const void *X, int64_t T, const void *Y_in, int y_dtype,
                  int64_t R, int64_t K, double alpha, double beta,
                  const int64_t *rows, int64_t nrows, int nthreads, double *Y_out)
{
    return spmm_run(12, values, meta, ab_dtype, X, T, Y_in, y_dtype, R, K, alpha, beta, rows, nrows,
                    nthreads, Y_out);
}

/* --------------------------------------------------------------------- */
/* Row-parallel drivers for timing the oracle on many cores (the mask and */
/* compress steps are independent per row).                               */
/* --------------------------------------------------------------------- */
typedef struct {
    const void *W; int dtype; int64_t C; int N, M; uint8_t *mask;
    void *values; uint8_t *meta; int64_t lo, hi; int what; int status;
} rows_job;

static void *rows_worker(void *arg)
{
    rows_job *j = (rows_job *)arg;
    int64_t n = j->hi - j->lo;
    const char *Wr = (const char *)j->W + (size_t)(j->lo * j->C) * elem_size(j->dtype);
    uint8_t *mr = j->mask + j->lo * j->C;
    if (j->what == 0) {
        j->status = oracle_mask_rank(Wr, j->dtype, n, j->C, j->C, j->N, j->M, mr, j->C);
    } else {
        j->status = oracle_mask_rank(Wr, j->dtype, n, j->C, j->C, 2, 4, mr, j->C);
        if (j->status == OR_OK)
            j->status = oracle_compress24(Wr, mr, j->dtype, n, j->C,
                                          (char *)j->values + (size_t)(j->lo * j->C / 2) * elem_size(j->dtype),
                                          j->meta + j->lo * j->C / 8);
    }
    return NULL;
}

/* what = 0: mask only (N:M); what = 1: 2:4 mask then compress. */
int oracle_rows_parallel(int what, const void *W, int dtype, int64_t R, int64_t C, int N, int M,
                         uint8_t *mask, void *values, uint8_t *meta, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (R < nthreads) nthreads = (int)(R > 0 ? R : 1);
    rows_job jobs[256];
    pthread_t th[256];
    for (int i = 0; i < nthreads; ++i) {
        rows_job j = { W, dtype, C, N, M, mask, values, meta, R * i / nthreads, R * (i + 1) / nthreads, what, 0 };
        jobs[i] = j;
    }
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, rows_worker, &jobs[i]);
    int st = OR_OK;
    for (int i = 0; i < nthreads; ++i) { pthread_join(th[i], NULL); if (jobs[i].status) st = jobs[i].status; }
    return st;
}

/* --------------------------------------------------------------------- */
/* SR-STE step.  [SRSTE] "SR-STE sparse training", SR-STE forward and     */
/* backward.  The forward recomputes the N:M mask of |w| every step and   */
/* returns output * w_b; the backward returns                              */
/*     grad_output + decay * (1 - mask) * weight                           */
/* (the page's default decay is 0.0002).  Both are evaluated here the way */
/* PyTorch evaluates that listing: w_b is made by torch.ones with no      */
/* dtype, so it is float32, and type promotion carries every product and  */
/* the sum in binary32:                                                    */
/*   forward   ws = fl32(w * m)             (exact: w, or a signed zero)   */
/*   backward  c  = decay * (1 - m)          (decay or 0, exact)           */
/*             t  = fl32(c * w)              rounding 1                    */
/*             y  = fl32(g + t)              rounding 2                    */
/* two separate roundings, never one fused multiply-add; the results are  */
/* returned in the weight's dtype (autograd hands a parameter its         */
/* gradient in the parameter's dtype), one more rounding to nearest even  */
/* for 16-bit weights.  Kept entries therefore get g + (+-0): g itself,   */
/* except that g = -0 with w >= +0 gives +0.  Pruned negative weights     */
/* give -0 in the forward.  Inf / NaN inputs are outside the contract     */
/* (their NaN results carry no defined payload).  mask may be NULL.       */
/* --------------------------------------------------------------------- */
int oracle_srste(const void *W, const void *grad, int dtype, int64_t R, int64_t C, int N, int M, float decay,
                 void *W_sparse, void *grad_out, uint8_t *mask_out)
{
    if (M < 2 || M > 8 || N < 1 || N >= M || C % M != 0 || R < 0) return OR_BAD_ARG;
    if (dtype == OR_S8) return OR_BAD_ARG;
    uint8_t *m = (uint8_t *)malloc((size_t)(C > 0 ? C : 1));
    for (int64_t r = 0; r < R; ++r) {
        int st = oracle_mask_rank((const char *)W + (size_t)(r * C) * elem_size(dtype), dtype, 1, C, C, N, M, m, C);
        if (st != OR_OK) { free(m); return st; }
        for (int64_t c = 0; c < C; ++c) {
            size_t i = (size_t)(r * C + c);
            uint32_t wb = load_bits(W, dtype, i), gb = load_bits(grad, dtype, i);
            if (mask_out) mask_out[i] = m[c];
            float w = (float)oracle_decode(wb, dtype);   /* exact: every element type fits binary32 */
            float g = (float)oracle_decode(gb, dtype);
            float keep = m[c] ? 1.0f : 0.0f;              /* the listing's float32 mask */
            float ws = w * keep;                          /* forward product */
            float coef = decay * (1.0f - keep);           /* decay * (1 - mask) */
            float t = coef * w;                           /* binary32, rounded once */
            float y = g + t;                              /* binary32, rounded once */
            store_bits(W_sparse, dtype, i, oracle_encode((double)ws, dtype));
            store_bits(grad_out, dtype, i, oracle_encode((double)y, dtype));
        }
    }
    free(m);
    return OR_OK;
}
