/*
 * mxs_oracle.c -- plain, single-threaded CPU oracle for the MXSens hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  The
 * product path (the CUDA library under mx_microscaling_mixed_b200/) never
 * links, imports or calls it, and shares no code, header, table or constant
 * generator with it.
 *
 * Sources (MXSens: Sensitivity-Aware Mixed-Precision Quantization for
 * Efficient LLM Inference, arXiv 2607.17733, as summarised on five web pages):
 *   [TS]  gist.science technical summary ("Technische Samenvatting"), sections
 *         1 (problem), 2.1 (sensitivity), 2.2 (triplet 4/6/8 strategy),
 *         2.3 (allocation algorithm), 4 (results / hardware overhead).
 *   [ABS] the paper's abstract (insight.artgrammer.co.kr).
 *   [RP]  researchpod.app summary (widths go to weights and activations).
 * Where the pages leave a step open, the reading used here is stated at the
 * function and listed with the other readings in the repository's design
 * notes.
 *
 * Arithmetic: fp64 throughout, IEEE round-to-nearest-even, no contraction
 * (build with -O2 -ffp-contract=off, never -ffast-math).
 *
 * Every function is pinned by tests (tests/test_oracle_*.py) against brute
 * force, exact rational arithmetic, closed forms or invariants.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BLOCK 32          /* MXINT block: 32 values share one scale [TS §1, §2.2] */
#define ORC_SUM_CHUNK 64      /* rows per partial sum in the sensitivity reductions   */

/* ------------------------------------------------------------------------ */
/* C1. MXINT block format                                                   */
/* ------------------------------------------------------------------------ */

/* Shared exponent of one block: e = floor(log2(max_i |x_i|)), clamped to the
 * E8M0 range [-127, 127]; an all-zero block takes e = -127 (scale byte 0).
 * [TS §1: blocks of 32 values share a power-of-two scale.]  The exponent is
 * read from frexp, never from a log2 approximation. */
int orc_block_exp(const double *x, int n)
{
    double amax = 0.0;
    for (int i = 0; i < n; ++i) {
        double a = fabs(x[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0) return -127;
    int ex;
    frexp(amax, &ex);           /* amax = f * 2^ex, f in [0.5, 1) */
    int e = ex - 1;             /* 2^e <= amax < 2^(e+1)          */
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* Largest code magnitude of an m-bit signed code: 2^(m-1) - 1. */
static int orc_qmax(int m) { return (1 << (m - 1)) - 1; }

/* Quantise one block to m-bit codes:
 *   q_i = clamp(round_half_even(x_i / 2^(e - m + 2)), -(2^(m-1)-1), 2^(m-1)-1).
 * Division by a power of two is exact, so the rounding acts on the exact
 * quotient.  Returns e through *e_out. */
void orc_quant_block(const double *x, int n, int m, int32_t *q, int *e_out)
{
    int e = orc_block_exp(x, n);
    int L = orc_qmax(m);
    for (int i = 0; i < n; ++i) {
        double y = ldexp(x[i], m - 2 - e);   /* exact */
        double r = nearbyint(y);             /* ties to even (default mode) */
        if (r > L) r = L;
        if (r < -L) r = -L;
        q[i] = (int32_t)r;
    }
    *e_out = e;
}

/* Value of code q under shared exponent e at width m: q * 2^(e - m + 2). */
double orc_dequant(int32_t q, int e, int m)
{
    return ldexp((double)q, e - m + 2);
}

/* Packed byte count of n codes at width m (n a multiple of 32). */
int64_t orc_packed_bytes(int64_t n, int m)
{
    return n * m / 8;
}

/* Pack n codes (n a multiple of 4) of width m into bytes, two's complement:
 *   m = 4: code 2k in the low nibble of byte k, code 2k+1 in the high nibble;
 *   m = 6: codes 4g..4g+3 form one 24-bit little-endian word, code 4g+i in
 *          bits [6i, 6i+6), stored as bytes 3g, 3g+1, 3g+2;
 *   m = 8: one byte per code. */
void orc_pack(const int32_t *q, int64_t n, int m, uint8_t *out)
{
    if (m == 8) {
        for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)(q[i] & 0xFF);
    } else if (m == 4) {
        for (int64_t k = 0; k < n / 2; ++k)
            out[k] = (uint8_t)((q[2 * k] & 0xF) | ((q[2 * k + 1] & 0xF) << 4));
    } else { /* m == 6 */
        for (int64_t g = 0; g < n / 4; ++g) {
            uint32_t w = 0;
            for (int i = 0; i < 4; ++i) w |= ((uint32_t)q[4 * g + i] & 0x3Fu) << (6 * i);
            out[3 * g + 0] = (uint8_t)(w & 0xFF);
            out[3 * g + 1] = (uint8_t)((w >> 8) & 0xFF);
            out[3 * g + 2] = (uint8_t)((w >> 16) & 0xFF);
        }
    }
}

/* Inverse of orc_pack: sign-extend each m-bit field. */
void orc_unpack(const uint8_t *in, int64_t n, int m, int32_t *q)
{
    for (int64_t i = 0; i < n; ++i) {
        uint32_t field;
        if (m == 8) {
            field = in[i];
        } else if (m == 4) {
            field = (in[i / 2] >> (4 * (i & 1))) & 0xF;
        } else {
            int64_t g = i / 4;
            uint32_t w = (uint32_t)in[3 * g] | ((uint32_t)in[3 * g + 1] << 8) |
                         ((uint32_t)in[3 * g + 2] << 16);
            field = (w >> (6 * (i % 4))) & 0x3F;
        }
        int32_t v = (int32_t)field;
        if (v >= (1 << (m - 1))) v -= (1 << m);
        q[i] = v;
    }
}

/* ------------------------------------------------------------------------ */
/* C2. Column sensitivity                                                   */
/* ------------------------------------------------------------------------ */

/* Column-wise sensitivity [TS §2.1: the Hessian diagonal of H = X^T X marks
 * columns whose quantisation noise costs most]:
 *   H_jj = (2/T) * sum_t X_tj^2,
 *   E_j  = sum_i (W_ij - Q4(W)_ij)^2   (Q4: 4-bit MXINT of each W row, blocks
 *                                      of 32 columns in the original order,
 *                                      a short last block zero-padded),
 *   s_j  = H_jj * E_j.
 * The 2/T factor (absent on the pages) scales every column of a layer alike
 * and does not change its ranking.
 * Rounding order (a reading: the pages fix none): rows are taken in chunks of
 * ORC_SUM_CHUNK; each chunk is summed from zero in increasing row order, and
 * the chunk sums are added in chunk order.  Every term (a square of an fp32
 * or bf16 value, or of an exact fp64 difference) is formed with one fp64
 * multiply.
 * X is T x K, W is N x K, both row-major, given as fp64 copies of the fp32 /
 * bf16 inputs (exact). */
void orc_sensitivity(const double *X, int64_t T, int64_t K,
                     const double *W, int64_t N,
                     double *H, double *E, double *s)
{
    for (int64_t j = 0; j < K; ++j) {
        double total = 0.0;
        for (int64_t c0 = 0; c0 < T; c0 += ORC_SUM_CHUNK) {
            int64_t c1 = c0 + ORC_SUM_CHUNK < T ? c0 + ORC_SUM_CHUNK : T;
            double part = 0.0;
            for (int64_t t = c0; t < c1; ++t) {
                double x = X[t * K + j];
                part = part + x * x;
            }
            total = total + part;
        }
        H[j] = (2.0 * total) / (double)T;
    }

    /* Q4 error per element, then the same chunked column sums over rows. */
    int64_t nblk = (K + ORC_BLOCK - 1) / ORC_BLOCK;
    double *err2 = (double *)malloc(sizeof(double) * (size_t)(N * K));
    double blk[ORC_BLOCK];
    int32_t q[ORC_BLOCK];
    for (int64_t i = 0; i < N; ++i) {
        for (int64_t b = 0; b < nblk; ++b) {
            for (int t = 0; t < ORC_BLOCK; ++t) {
                int64_t j = b * ORC_BLOCK + t;
                blk[t] = j < K ? W[i * K + j] : 0.0;
            }
            int e;
            orc_quant_block(blk, ORC_BLOCK, 4, q, &e);
            for (int t = 0; t < ORC_BLOCK; ++t) {
                int64_t j = b * ORC_BLOCK + t;
                if (j >= K) break;
                double d = blk[t] - orc_dequant(q[t], e, 4);
                err2[i * K + j] = d * d;
            }
        }
    }
    for (int64_t j = 0; j < K; ++j) {
        double total = 0.0;
        for (int64_t c0 = 0; c0 < N; c0 += ORC_SUM_CHUNK) {
            int64_t c1 = c0 + ORC_SUM_CHUNK < N ? c0 + ORC_SUM_CHUNK : N;
            double part = 0.0;
            for (int64_t i = c0; i < c1; ++i) part = part + err2[i * K + j];
            total = total + part;
        }
        E[j] = total;
        s[j] = H[j] * E[j];
    }
    free(err2);
}

/* ------------------------------------------------------------------------ */
/* C3. Bit allocation                                                       */
/* ------------------------------------------------------------------------ */

static const double *g_sort_key;
static int orc_rank_cmp(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    double sa = g_sort_key[a], sb = g_sort_key[b];
    if (sa > sb) return -1;         /* descending sensitivity */
    if (sa < sb) return 1;
    return (a < b) ? -1 : (a > b);  /* ties: lower column index first */
}

/* order[r] = column of rank r: descending s, ties to the lower index
 * [TS §2.3 "Sorteren": columns are sorted by their sensitivity]. */
void orc_rank_order(const double *s, int64_t K, int32_t *order)
{
    for (int64_t j = 0; j < K; ++j) order[j] = (int32_t)j;
    g_sort_key = s;
    qsort(order, (size_t)K, sizeof(int32_t), orc_rank_cmp);
    g_sort_key = NULL;
}

/* floor(p * K + 1/2) for p = num/den, in exact integer arithmetic. */
static int64_t orc_round_frac(int64_t num, int64_t den, int64_t K)
{
    return (2 * num * K + den) / (2 * den);
}

/* The layer-score rule's steps.  Layer l with score w_l > 0 reaches its
 * k-th 32-column 6-bit group when R * w_l >= 32 k, i.e. at R = 32 k / w_l.
 * Steps are ordered by that R, compared exactly: k_a / w_a < k_b / w_b iff
 * k_a * w_b < k_b * w_a, each product taken exactly as the pair (rounded
 * product, its rounding error from fma), compared lexicographically. */
typedef struct {
    int layer;
    int64_t k;        /* group index, 1-based */
    int64_t cols;     /* 32, or fewer for the last group */
} orc_rstep;

static const double *g_rscore = NULL;

static int orc_rstep_cmp_values(const orc_rstep *a, const orc_rstep *b)
{
    double ka = (double)a->k, kb = (double)b->k;
    double wa = g_rscore[a->layer], wb = g_rscore[b->layer];
    double p1 = ka * wb, e1 = fma(ka, wb, -p1);     /* k_a * w_b exactly = p1 + e1 */
    double p2 = kb * wa, e2 = fma(kb, wa, -p2);     /* k_b * w_a exactly = p2 + e2 */
    if (p1 != p2) return p1 < p2 ? -1 : 1;
    if (e1 != e2) return e1 < e2 ? -1 : 1;
    return 0;
}

static int orc_rstep_cmp(const void *pa, const void *pb)
{
    const orc_rstep *a = (const orc_rstep *)pa, *b = (const orc_rstep *)pb;
    int c = orc_rstep_cmp_values(a, b);
    if (c) return c;
    if (a->layer != b->layer) return a->layer < b->layer ? -1 : 1;   /* fixes qsort's order only */
    return a->k < b->k ? -1 : (a->k > b->k);
}

/* Bit allocation for n_layers linear layers.
 *   mode 0 (fractions): n8 = round(p8*K), n6 = round(p6*K) (half up, exact),
 *                       the rest 4-bit.
 *   mode 1 (budget):    n8 = min(fixed8, K) -- the 32 most sensitive
 *                       columns, one MXINT block [TS §2.2, §2.3 fixed block];
 *                       then 6-bit upgrades in groups of the next 32 ranked
 *                       4-bit columns of a layer (fewer at the tail), taken
 *                       greedily by gain/cost, gain = w_l * sum of s over the
 *                       group (fp64, rank order), cost = 2 * N_l * count bits,
 *                       comparing gain_a*cost_b > gain_b*cost_a in fp64, ties
 *                       to the lower layer; the greedy stops at the first
 *                       candidate that does not fit [TS §2.3: the 6-bit count
 *                       follows the layer's sensitivity, scaled to meet the
 *                       global average budget].
 *   mode 2 (layer score): n8 as in mode 1; the 6-bit count of layer l is
 *                       proportional to its layer score w_l = layer_w[l],
 *                       scaled by one global R [TS §2.3 "Dynamische 6-bit
 *                       Allocatie"], in whole 32-column groups:
 *                         n6_l(R) = min(K_l - n8_l, 32 * floor(R * w_l / 32)),
 *                       with R the largest value whose counts meet the
 *                       budget.  n6_l(R) only changes at R = 32 k / w_l, so
 *                       R is found by taking those steps in increasing R
 *                       (all steps at one R value together) until the next
 *                       value's steps no longer fit.  A layer with w_l = 0
 *                       gets no 6-bit columns.
 *   Budget accounting: average mantissa bits over all weight elements, E8M0
 *   scales excluded; with B = num/den the test is
 *     sum_l N_l (4 K_l + 4 n8_l + 2 n6_l) * den <= num * sum_l N_l K_l.
 *   ([TS §4: at a 4.03-bit budget about 1% of the work is wider; with K=4096
 *   the fixed block alone gives 4 + 4*32/4096 = 4.03125.])
 * Outputs: perm[l][0..K_l) = columns of the 8-bit, then 6-bit, then 4-bit
 * segment, each in ascending column order; counts[3l..3l+2] = n8, n6, n4.
 * Returns 0, or 1 if the fixed 8-bit blocks alone exceed the budget,
 * or 2 on a bad argument. */
int orc_allocate(int n_layers, const int64_t *K, const int64_t *N,
                 const double *const *s, const double *layer_w,
                 int mode, int64_t num, int64_t den,
                 int64_t p8_num, int64_t p8_den, int64_t p6_num, int64_t p6_den,
                 int64_t fixed8, int32_t *const *perm, int64_t *counts)
{
    if (n_layers <= 0 || den <= 0) return 2;
    if (mode == 2) {
        if (!layer_w) return 2;
        for (int l = 0; l < n_layers; ++l)
            if (!(layer_w[l] >= 0.0) || !isfinite(layer_w[l])) return 2;
    }
    int32_t **order = (int32_t **)calloc((size_t)n_layers, sizeof(int32_t *));
    for (int l = 0; l < n_layers; ++l) {
        order[l] = (int32_t *)malloc(sizeof(int32_t) * (size_t)(K[l] > 0 ? K[l] : 1));
        orc_rank_order(s[l], K[l], order[l]);
    }
    int rc = 0;
    int64_t *n8 = (int64_t *)calloc((size_t)n_layers, sizeof(int64_t));
    int64_t *n6 = (int64_t *)calloc((size_t)n_layers, sizeof(int64_t));
    if (mode == 0) {
        for (int l = 0; l < n_layers; ++l) {
            n8[l] = orc_round_frac(p8_num, p8_den, K[l]);
            n6[l] = orc_round_frac(p6_num, p6_den, K[l]);
            if (n8[l] > K[l]) n8[l] = K[l];
            if (n6[l] > K[l] - n8[l]) n6[l] = K[l] - n8[l];
        }
    } else {
        __int128 cap = 0, used = 0;
        for (int l = 0; l < n_layers; ++l) {
            n8[l] = fixed8 < K[l] ? fixed8 : K[l];
            cap += (__int128)num * N[l] * K[l];
            used += (__int128)den * N[l] * (4 * K[l] + 4 * n8[l]);
        }
        if (used > cap) {
            rc = 1;
        } else if (mode == 2) {
            int64_t nsteps = 0;
            for (int l = 0; l < n_layers; ++l)
                if (layer_w[l] > 0.0) nsteps += (K[l] - n8[l] + 31) / 32;
            orc_rstep *st = (orc_rstep *)malloc(sizeof(orc_rstep) * (size_t)(nsteps + 1));
            int64_t i = 0;
            for (int l = 0; l < n_layers; ++l) {
                if (!(layer_w[l] > 0.0)) continue;
                int64_t avail = K[l] - n8[l];
                for (int64_t k = 1; 32 * (k - 1) < avail; ++k) {
                    st[i].layer = l;
                    st[i].k = k;
                    st[i].cols = avail - 32 * (k - 1) < 32 ? avail - 32 * (k - 1) : 32;
                    ++i;
                }
            }
            g_rscore = layer_w;
            qsort(st, (size_t)nsteps, sizeof(orc_rstep), orc_rstep_cmp);
            for (int64_t a = 0; a < nsteps;) {
                int64_t b = a + 1;
                while (b < nsteps && orc_rstep_cmp_values(&st[a], &st[b]) == 0) ++b;
                __int128 add = 0;
                for (int64_t j = a; j < b; ++j) add += (__int128)den * 2 * N[st[j].layer] * st[j].cols;
                if (used + add > cap) break;          /* R stays below this step value */
                used += add;
                for (int64_t j = a; j < b; ++j) n6[st[j].layer] += st[j].cols;
                a = b;
            }
            g_rscore = NULL;
            free(st);
        } else {
            for (;;) {
                int best = -1;
                double best_gain = 0.0, best_cost = 0.0;
                for (int l = 0; l < n_layers; ++l) {
                    int64_t r0 = n8[l] + n6[l];
                    if (r0 >= K[l]) continue;
                    int64_t r1 = r0 + 32 < K[l] ? r0 + 32 : K[l];
                    double sum = 0.0;
                    for (int64_t r = r0; r < r1; ++r) sum = sum + s[l][order[l][r]];
                    double w = layer_w ? layer_w[l] : 1.0;
                    double gain = w * sum;
                    double cost = (double)(2 * N[l] * (r1 - r0));
                    if (best < 0 || gain * best_cost > best_gain * cost) {
                        best = l;
                        best_gain = gain;
                        best_cost = cost;
                    }
                }
                if (best < 0) break;
                int64_t r0 = n8[best] + n6[best];
                int64_t cnt = (r0 + 32 < K[best] ? 32 : K[best] - r0);
                __int128 add = (__int128)den * 2 * N[best] * cnt;
                if (used + add > cap) break;
                used += add;
                n6[best] += cnt;
            }
        }
    }
    if (rc == 0) {
        for (int l = 0; l < n_layers; ++l) {
            int64_t k = K[l];
            uint8_t *seg = (uint8_t *)malloc((size_t)(k > 0 ? k : 1));
            for (int64_t r = 0; r < k; ++r)
                seg[order[l][r]] = (uint8_t)(r < n8[l] ? 0 : (r < n8[l] + n6[l] ? 1 : 2));
            int64_t pos = 0;
            for (int g = 0; g < 3; ++g)
                for (int64_t j = 0; j < k; ++j)
                    if (seg[j] == g) perm[l][pos++] = (int32_t)j;
            free(seg);
            counts[3 * l + 0] = n8[l];
            counts[3 * l + 1] = n6[l];
            counts[3 * l + 2] = k - n8[l] - n6[l];
        }
    }
    for (int l = 0; l < n_layers; ++l) free(order[l]);
    free(order);
    free(n8);
    free(n6);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* C4. Quantise rows (weights, activations, K/V cache)                      */
/* ------------------------------------------------------------------------ */

static const int orc_seg_bits[3] = {8, 6, 4};

static int64_t orc_pad32(int64_t n) { return (n + ORC_BLOCK - 1) / ORC_BLOCK * ORC_BLOCK; }

/* Quantise `rows` rows of a row-major rows x K matrix into the mixed-width
 * layout: columns are gathered by perm (8-bit segment, then 6-bit, then
 * 4-bit, each zero-padded to a multiple of 32 positions) and each segment is
 * coded in blocks of 32 with its own width [TS §2.2 triplet strategy; §2.3
 * last paragraph: the mixed widths ride on MXINT's block structure; RP: the
 * widths apply to weights and activations].  perm == NULL means the
 * identity (K/V cache: one 4-bit segment, counts = {0, 0, K}).
 * Outputs are compact: codes[g] is rows x (k_pad_g * bits_g / 8) bytes,
 * scales[g] is rows x (k_pad_g / 32) bytes (E8M0: e + 127). */
void orc_quantize_rows(const double *src, int64_t rows, int64_t K,
                       const int32_t *perm, const int64_t *counts,
                       uint8_t *const *codes, uint8_t *const *scales)
{
    double blk[ORC_BLOCK];
    int32_t q[ORC_BLOCK];
    for (int64_t r = 0; r < rows; ++r) {
        int64_t real_off = 0;
        for (int g = 0; g < 3; ++g) {
            int m = orc_seg_bits[g];
            int64_t kr = counts[g], kp = orc_pad32(kr);
            int64_t row_bytes = kp * m / 8, nb = kp / ORC_BLOCK;
            for (int64_t b = 0; b < nb; ++b) {
                for (int t = 0; t < ORC_BLOCK; ++t) {
                    int64_t p = b * ORC_BLOCK + t;
                    if (p < kr) {
                        int64_t col = perm ? perm[real_off + p] : real_off + p;
                        blk[t] = src[r * K + col];
                    } else {
                        blk[t] = 0.0;
                    }
                }
                int e;
                orc_quant_block(blk, ORC_BLOCK, m, q, &e);
                orc_pack(q, ORC_BLOCK, m, codes[g] + r * row_bytes + b * ORC_BLOCK * m / 8);
                scales[g][r * nb + b] = (uint8_t)(e + 127);
            }
            real_off += kr;
        }
    }
}

/* Decode compact mixed-width rows back to fp64 values in padded-position
 * order: out is rows x K' with K' = sum of padded segment lengths. */
void orc_dequantize_rows(int64_t rows, const int64_t *counts,
                         const uint8_t *const *codes, const uint8_t *const *scales,
                         double *out)
{
    int64_t kpad_total = 0;
    for (int g = 0; g < 3; ++g) kpad_total += orc_pad32(counts[g]);
    int32_t q[ORC_BLOCK];
    for (int64_t r = 0; r < rows; ++r) {
        int64_t off = 0;
        for (int g = 0; g < 3; ++g) {
            int m = orc_seg_bits[g];
            int64_t kp = orc_pad32(counts[g]);
            int64_t row_bytes = kp * m / 8, nb = kp / ORC_BLOCK;
            for (int64_t b = 0; b < nb; ++b) {
                orc_unpack(codes[g] + r * row_bytes + b * ORC_BLOCK * m / 8, ORC_BLOCK, m, q);
                int e = (int)scales[g][r * nb + b] - 127;
                for (int t = 0; t < ORC_BLOCK; ++t)
                    out[r * kpad_total + off + b * ORC_BLOCK + t] = orc_dequant(q[t], e, m);
            }
            off += kp;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* C5. Mixed-width linear layer                                             */
/* ------------------------------------------------------------------------ */

/* Y[i][j] = sum_k deq(A)[row_i][k] * deq(W)[col_j][k] over all padded
 * positions k (pads contribute zero), fp64, summed in position order, for the
 * requested output rows (A rows) and columns (W rows).  A and W share one
 * segment table [TS §2.3 last paragraph, §4 hardware overhead: the layer
 * runs on the MXINT blocks directly].  Y is n_rows x n_cols. */
void orc_gemm(int64_t M, int64_t N, const int64_t *counts,
              const uint8_t *const *a_codes, const uint8_t *const *a_scales,
              const uint8_t *const *w_codes, const uint8_t *const *w_scales,
              const int64_t *row_idx, int64_t n_rows,
              const int64_t *col_idx, int64_t n_cols, double *Y)
{
    int64_t kp = 0;
    for (int g = 0; g < 3; ++g) kp += orc_pad32(counts[g]);
    double *a = (double *)malloc(sizeof(double) * (size_t)(n_rows * kp + 1));
    double *w = (double *)malloc(sizeof(double) * (size_t)(n_cols * kp + 1));
    const uint8_t *c[3], *sc[3];
    /* decode the requested A rows and W rows once */
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t r = row_idx[i];
        for (int g = 0; g < 3; ++g) {
            int64_t kpg = orc_pad32(counts[g]);
            c[g] = a_codes[g] + r * (kpg * orc_seg_bits[g] / 8);
            sc[g] = a_scales[g] + r * (kpg / ORC_BLOCK);
        }
        orc_dequantize_rows(1, counts, c, sc, a + i * kp);
    }
    for (int64_t jj = 0; jj < n_cols; ++jj) {
        int64_t r = col_idx[jj];
        for (int g = 0; g < 3; ++g) {
            int64_t kpg = orc_pad32(counts[g]);
            c[g] = w_codes[g] + r * (kpg * orc_seg_bits[g] / 8);
            sc[g] = w_scales[g] + r * (kpg / ORC_BLOCK);
        }
        orc_dequantize_rows(1, counts, c, sc, w + jj * kp);
    }
    for (int64_t i = 0; i < n_rows; ++i) {
        for (int64_t jj = 0; jj < n_cols; ++jj) {
            double acc = 0.0;
            for (int64_t k = 0; k < kp; ++k) acc = acc + a[i * kp + k] * w[jj * kp + k];
            Y[i * n_cols + jj] = acc;
        }
    }
    (void)M;
    (void)N;
    free(a);
    free(w);
}

/* ------------------------------------------------------------------------ */
/* Decode-step attention over the 4-bit MXINT K/V cache                     */
/* ------------------------------------------------------------------------ */

/* One decoding step of grouped-query attention whose key and value caches
 * are kept as MXINT4: the uniform 4-bit layout {0, 0, d}, blocks of 32 along
 * the head dimension, one E8M0 byte per block [TS §4: the W4A4KV4 setting
 * quantises the K/V cache to 4 bits; RV Validation: A4W4KV4 against
 * A4W4KV16].  The pages do not spell out the attention arithmetic; it is the
 * textbook scaled dot-product attention of one query token, read on the
 * decoded cache:
 *   query head h uses kv head g = h / (n_qh / n_kvh);
 *   cache row t * n_kvh + g holds token t of kv head g (a [T][n_kvh][d]
 *   cache flattened token-major);
 *   s_t = sm_scale * sum_d q[h][d] * deq(K)[t n_kvh + g][d]
 *   p_t = exp(s_t - max_u s_u) / sum_u exp(s_u - max_u s_u)
 *   out[h][d] = sum_t p_t * deq(V)[t n_kvh + g][d]
 * fp64 throughout; every sum runs in index order.  q is n_qh x d (row-major),
 * the caches are compact (rows x d/2 code bytes, rows x d/32 scale bytes),
 * out is n_qh x d. */
void orc_attn_decode(const double *q, int64_t n_qh, int64_t d,
                     const uint8_t *k_codes, const uint8_t *k_scales,
                     const uint8_t *v_codes, const uint8_t *v_scales,
                     int64_t T, int64_t n_kvh, double sm_scale, double *out)
{
    const int64_t counts[3] = {0, 0, d};
    const int64_t rows = T * n_kvh;
    const int64_t rep = n_qh / n_kvh;
    double *kd = (double *)malloc(sizeof(double) * (size_t)(rows * d + 1));
    double *vd = (double *)malloc(sizeof(double) * (size_t)(rows * d + 1));
    double *s = (double *)malloc(sizeof(double) * (size_t)(T + 1));
    const uint8_t *c[3], *sc[3];
    c[0] = c[1] = sc[0] = sc[1] = NULL;
    c[2] = k_codes;
    sc[2] = k_scales;
    orc_dequantize_rows(rows, counts, c, sc, kd);
    c[2] = v_codes;
    sc[2] = v_scales;
    orc_dequantize_rows(rows, counts, c, sc, vd);
    for (int64_t h = 0; h < n_qh; ++h) {
        const int64_t g = h / rep;
        double smax = -INFINITY;
        for (int64_t t = 0; t < T; ++t) {
            const double *k = kd + (t * n_kvh + g) * d;
            double dot = 0.0;
            for (int64_t i = 0; i < d; ++i) dot = dot + q[h * d + i] * k[i];
            s[t] = sm_scale * dot;
            if (s[t] > smax) smax = s[t];
        }
        double denom = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            s[t] = exp(s[t] - smax);
            denom = denom + s[t];
        }
        for (int64_t i = 0; i < d; ++i) out[h * d + i] = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            const double p = s[t] / denom;
            const double *v = vd + (t * n_kvh + g) * d;
            for (int64_t i = 0; i < d; ++i) out[h * d + i] = out[h * d + i] + p * v[i];
        }
    }
    free(kd);
    free(vd);
    free(s);
}
