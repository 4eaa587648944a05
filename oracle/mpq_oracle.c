/*
 * mpq_oracle.c -- the fp64 CPU oracle for the block-wise mixed-precision
 * weight-only quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the CUDA library computes.  Only the test suite, the smoke
 * check and the CPU-baseline leg of the benchmark load it.  It shares no code,
 * header, table or constant with the CUDA path, and the CUDA path never calls it.
 *
 * Sources (web pages on the method; cited by title and section):
 *   [SB-abs]  "ScaleBITS: Scalable Bitwidth Search for Hardware-Aligned
 *             Mixed-Precision LLMs", abstract.
 *   [SB-app]  same paper, AI-written summary page, section "Approach":
 *             bits are assigned per 64x128 block under a global budget after
 *             rows and columns are reordered.
 *   [SB-res]  same summary, "Key results": uniform RTN-g128 is the baseline
 *             quantizer (round-to-nearest, groups of 128 weights).
 *   [SB-lim]  same summary, "Limitations": only scalar RTN with group 128.
 *   [SB-sur]  same summary, "Surprising findings": a 0- or 1-bit minimum.
 *   [SFMP]    "SFMP: Fine-Grained, Hardware-Friendly and Search-Free
 *             Mixed-Precision Quantization for Large Language Models",
 *             abstract: block-wise mixed precision, row-column reordering with
 *             an activation reordering step at inference.
 *   [TQ]      "TileQuant: Tile as the Precision-Allocation Unit for LLM
 *             Mixed-Precision Post-Training Quantization", abstract: the
 *             precision map guides the layout of compact weight buffers.
 *
 * Readings where the pages are silent:
 *   - a block is 64 output rows x 128 input columns, so each block row is one
 *     quantization group of 128 weights;
 *   - RTN is asymmetric with the range widened to include 0; the fp16 scale is
 *     the SMALLEST fp16 value h with h*qmax >= (hi - lo); z = rne(-lo/s);
 *     q = clamp(rne(w/s) + z, 0, qmax); dequant = (q - z)*s;
 *   - bits are in {0,1,2,3,4,5,6,8,16}; a 0-bit block dequantizes to zero;
 *     a 16-bit block keeps its bf16 weights unquantized ([TQ]: the
 *     highest-scoring tiles stay at 16 bits while the rest are quantized);
 *     its payload is the 64 x 128 bf16 bit patterns of the block, row-major,
 *     and its scales/zeros are 1 and 0 (unused);
 *   - W'[i][j] = W[row_perm[i]][col_perm[j]]; blocks are defined on W';
 *   - the packed format ("format v1") is this library's own; see
 *     mpqo_pack below for the byte layout.
 *
 * Everything is IEEE fp64 with round-to-nearest-even (nearbyint in the default
 * rounding mode).  Compile without -ffast-math.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "mpq_oracle.h"

int mpqo_set_threads(int n) {
    const int prev = omp_get_max_threads();
    omp_set_num_threads(n < 1 ? 1 : n);
    return prev;
}

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* bf16 bit pattern -> exact double. */
double mpqo_bf16_to_f64(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16 bit pattern -> exact double (normals, subnormals, inf, nan). */
double mpqo_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24);            /* subnormal: m * 2^-24 */
    } else if (e == 31) {
        v = (m == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Exact encoding of a small non-negative integer (0..2048) as binary16. */
static uint16_t f16_from_small_int(int v)
{
    if (v == 0) return 0;
    int e = 0;
    while ((v >> (e + 1)) != 0) e++;          /* v in [2^e, 2^(e+1)) */
    /* mantissa holds the 10 bits below the leading one */
    int m = (v << (10 - e)) & 0x3ff;           /* exact for e <= 10 */
    return (uint16_t)(((e + 15) << 10) | m);
}

/* ------------------------------------------------------------------------ */
/* Bit widths and their pieces                                               */
/* ------------------------------------------------------------------------ */

int mpqo_bits_valid(int b)
{
    return b == 0 || b == 1 || b == 2 || b == 3 || b == 4 || b == 5 ||
           b == 6 || b == 8 || b == 16;
}

/* A b-bit code is stored as one or two "pieces"; the low piece comes first.
 * q = low_piece | (high_piece << width(low_piece)).                         */
int mpqo_pieces(int b, int widths[2])
{
    switch (b) {
    case 1: widths[0] = 1; return 1;
    case 2: widths[0] = 2; return 1;
    case 3: widths[0] = 2; widths[1] = 1; return 2;
    case 4: widths[0] = 4; return 1;
    case 5: widths[0] = 4; widths[1] = 1; return 2;
    case 6: widths[0] = 4; widths[1] = 2; return 2;
    case 8: widths[0] = 8; return 1;
    default: return 0;
    }
}

/* ------------------------------------------------------------------------ */
/* Plan: block table and segment offsets                                     */
/* ------------------------------------------------------------------------ */

/* Segments hold the payloads of all blocks of one bit width, in ascending
 * block id t = nb*KB + kb; segments are ordered b = 1,2,3,4,5,6,8,16.  Each
 * payload is 1024*b bytes (64 rows x 128 codes x b bits).  table[4t..4t+3] =
 * {code_off, sz_off, bits, bit_prefix}: byte offset of the payload in the
 * codes buffer, index of the block's first scale/zero, the width, and the sum
 * of the widths of all blocks before t in row-major block order.            */
int mpqo_plan(int32_t N, int32_t K, const uint8_t *bits, mpqo_layout *L,
              uint32_t *table)
{
    if (N <= 0 || K <= 0 || N % 64 != 0 || K % 128 != 0) return MPQO_ERR_SHAPE;
    int NB = N / 64, KB = K / 128;
    int64_t T = (int64_t)NB * KB;
    memset(L, 0, sizeof *L);
    L->N = N; L->K = K; L->NB = NB; L->KB = KB;

    int64_t count[17] = {0};
    for (int64_t t = 0; t < T; t++) {
        if (!mpqo_bits_valid(bits[t])) return MPQO_ERR_BITS;
        count[bits[t]]++;
    }
    static const int order[8] = {1, 2, 3, 4, 5, 6, 8, 16};
    uint64_t off = 0;
    for (int i = 0; i < 8; i++) {
        int b = order[i];
        L->seg_off[b] = off;
        L->seg_bytes[b] = (uint64_t)count[b] * 1024u * (uint64_t)b;
        off += L->seg_bytes[b];
    }
    L->codes_bytes = off;
    if (off >= ((uint64_t)1 << 32)) return MPQO_ERR_SHAPE;

    uint64_t seen[17] = {0};
    uint64_t nz = 0, prefix = 0;
    for (int64_t t = 0; t < T; t++) {
        int b = bits[t];
        uint32_t *e = table ? table + 4 * t : NULL;
        if (b == 0) {
            if (e) { e[0] = 0; e[1] = 0; e[2] = 0; e[3] = (uint32_t)prefix; }
        } else {
            if (e) {
                e[0] = (uint32_t)(L->seg_off[b] + seen[b] * 1024u * (uint64_t)b);
                e[1] = (uint32_t)(64u * nz);
                e[2] = (uint32_t)b;
                e[3] = (uint32_t)prefix;
            }
            seen[b]++;
            nz++;
        }
        prefix += (uint64_t)b;
    }
    L->n_sz = 64u * nz;
    L->bit_total = prefix;
    return MPQO_OK;
}

/* ------------------------------------------------------------------------ */
/* RTN of one group                                                          */
/* ------------------------------------------------------------------------ */

/* Round-to-nearest asymmetric quantization of one group of n weights to b
 * bits ([SB-res], [SB-lim]: RTN with group size 128).
 *   lo = min(min w, 0), hi = max(max w, 0), d = hi - lo
 *   d == 0 -> s = 1, z = 0, every q = 0
 *   else   s = smallest fp16 h with h*qmax >= d  (h*qmax is exact in fp64)
 *          z = rne(-lo/s)
 *          q = clamp(rne(w/s) + z, 0, qmax)
 * Returns MPQO_ERR_NONFINITE for a NaN/Inf weight and MPQO_ERR_RANGE when no
 * finite fp16 scale exists or qmax*s exceeds the fp16 maximum 65504.        */
int mpqo_quantize_group(const double *w, int n, int b, uint16_t *s_bits,
                        uint16_t *z_bits, uint8_t *q)
{
    if (b < 1 || b > 8 || !mpqo_bits_valid(b)) return MPQO_ERR_BITS;
    double qmax = (double)((1 << b) - 1);
    double lo = 0.0, hi = 0.0;
    for (int j = 0; j < n; j++) {
        if (!isfinite(w[j])) return MPQO_ERR_NONFINITE;
        if (w[j] < lo) lo = w[j];
        if (w[j] > hi) hi = w[j];
    }
    double d = hi - lo;
    if (d == 0.0) {
        *s_bits = 0x3C00;                      /* 1.0 */
        *z_bits = 0;
        for (int j = 0; j < n; j++) q[j] = 0;
        return MPQO_OK;
    }
    /* smallest positive finite fp16 h with h*qmax >= d: positive binary16
     * values increase with their bit patterns, so bisect on 0x0001..0x7BFF. */
    uint16_t a = 1, c = 0x7BFF;
    if (mpqo_f16_to_f64(c) * qmax < d) return MPQO_ERR_RANGE;
    while (a < c) {
        uint16_t mid = (uint16_t)(a + (c - a) / 2);
        if (mpqo_f16_to_f64(mid) * qmax >= d) c = mid; else a = (uint16_t)(mid + 1);
    }
    double s = mpqo_f16_to_f64(a);
    if (s * qmax > 65504.0) return MPQO_ERR_RANGE;
    double z = nearbyint(-lo / s);
    for (int j = 0; j < n; j++) {
        double v = nearbyint(w[j] / s) + z;
        if (v < 0.0) v = 0.0;
        if (v > qmax) v = qmax;
        q[j] = (uint8_t)v;
    }
    *s_bits = a;
    *z_bits = f16_from_small_int((int)z);
    return MPQO_OK;
}

/* ------------------------------------------------------------------------ */
/* Pack                                                                      */
/* ------------------------------------------------------------------------ */

/* Byte layout of one block payload (format v1, this library's own choice;
 * the pages only say the precision map guides compact weight buffers [TQ]):
 *   pieces in low-first order; piece of width p is 64 rows x (16*p) bytes,
 *   row-major; within a row, the p-bit field of code j (column j of the
 *   block, 0..127) sits in little-endian 32-bit word j / (32/p) at bit
 *   (j % (32/p)) * p.                                                       */
static void put_field(uint8_t *row, int p, int j, unsigned v)
{
    int per_word = 32 / p;
    int word = j / per_word;
    int bit = (j % per_word) * p;
    uint32_t wv;
    memcpy(&wv, row + 4 * word, 4);           /* host is little-endian */
    wv |= ((uint32_t)v & ((1u << p) - 1u)) << bit;
    memcpy(row + 4 * word, &wv, 4);
}

static unsigned get_field(const uint8_t *row, int p, int j)
{
    int per_word = 32 / p;
    uint32_t wv;
    memcpy(&wv, row + 4 * (j / per_word), 4);
    return (wv >> ((j % per_word) * p)) & ((1u << p) - 1u);
}

static int check_perm(const int32_t *p, int n)
{
    if (!p) return 1;
    char *seen = (char *)calloc((size_t)n, 1);
    if (!seen) return 0;
    int ok = 1;
    for (int i = 0; i < n && ok; i++) {
        if (p[i] < 0 || p[i] >= n || seen[p[i]]) ok = 0;
        else seen[p[i]] = 1;
    }
    free(seen);
    return ok;
}

int mpqo_pack(int32_t N, int32_t K, const uint16_t *W, const uint8_t *bits,
              const int32_t *row_perm, const int32_t *col_perm,
              uint8_t *codes, uint32_t *table, uint16_t *scales,
              uint16_t *zeros)
{
    mpqo_layout L;
    int st = mpqo_plan(N, K, bits, &L, table);
    if (st != MPQO_OK) return st;
    if (!check_perm(row_perm, N) || !check_perm(col_perm, K)) return MPQO_ERR_PERM;
    memset(codes, 0, (size_t)L.codes_bytes);

    double w[128];
    uint8_t q[128];
    for (int nb = 0; nb < L.NB; nb++) {
        for (int kb = 0; kb < L.KB; kb++) {
            int64_t t = (int64_t)nb * L.KB + kb;
            int b = bits[t];
            if (b == 0) continue;
            const uint32_t *e = table + 4 * t;
            uint8_t *payload = codes + e[0];
            if (b == 16) {
                /* passthrough: the bf16 weights, row-major; scale 1, zero 0;
                 * every weight finite and within the binary16 range (the
                 * tensor-core path multiplies in fp16) */
                for (int r = 0; r < 64; r++) {
                    int i = nb * 64 + r;
                    int src_row = row_perm ? row_perm[i] : i;
                    for (int j = 0; j < 128; j++) {
                        int col = kb * 128 + j;
                        int src_col = col_perm ? col_perm[col] : col;
                        uint16_t wb = W[(int64_t)src_row * K + src_col];
                        double v = mpqo_bf16_to_f64(wb);
                        if (!isfinite(v)) return MPQO_ERR_NONFINITE;
                        if (fabs(v) > 65504.0) return MPQO_ERR_RANGE;
                        memcpy(payload + r * 256 + 2 * j, &wb, 2);
                    }
                    scales[e[1] + r] = 0x3C00;
                    zeros[e[1] + r] = 0;
                }
                continue;
            }
            int widths[2];
            int np = mpqo_pieces(b, widths);
            for (int r = 0; r < 64; r++) {
                int i = nb * 64 + r;                     /* row of W' */
                int src_row = row_perm ? row_perm[i] : i;
                for (int j = 0; j < 128; j++) {
                    int col = kb * 128 + j;              /* column of W' */
                    int src_col = col_perm ? col_perm[col] : col;
                    w[j] = mpqo_bf16_to_f64(W[(int64_t)src_row * K + src_col]);
                }
                uint16_t sb, zb;
                st = mpqo_quantize_group(w, 128, b, &sb, &zb, q);
                if (st != MPQO_OK) return st;
                scales[e[1] + r] = sb;
                zeros[e[1] + r] = zb;
                int piece_base = 0, shift = 0;
                for (int pi = 0; pi < np; pi++) {
                    int p = widths[pi];
                    uint8_t *row = payload + piece_base + r * 16 * p;
                    for (int j = 0; j < 128; j++)
                        put_field(row, p, j, (unsigned)(q[j] >> shift));
                    piece_base += 64 * 16 * p;
                    shift += p;
                }
            }
        }
    }
    return MPQO_OK;
}

/* ------------------------------------------------------------------------ */
/* Dequant and linear                                                        */
/* ------------------------------------------------------------------------ */

/* Codes of row r (0..63) of a block, decoded from its payload. */
static void unpack_row(const uint8_t *payload, int b, int r, uint8_t *q)
{
    int widths[2];
    int np = mpqo_pieces(b, widths);
    for (int j = 0; j < 128; j++) q[j] = 0;
    int piece_base = 0, shift = 0;
    for (int pi = 0; pi < np; pi++) {
        int p = widths[pi];
        const uint8_t *row = payload + piece_base + r * 16 * p;
        for (int j = 0; j < 128; j++)
            q[j] = (uint8_t)(q[j] | (get_field(row, p, j) << shift));
        piece_base += 64 * 16 * p;
        shift += p;
    }
}

/* Dequantized row i of W' (reordered order), K values: (q - z) * s, exact. */
static void dequant_row_reordered(const mpqo_packed *P, int i, double *out)
{
    int nb = i / 64, r = i % 64, KB = P->K / 128;
    uint8_t q[128];
    for (int kb = 0; kb < KB; kb++) {
        const uint32_t *e = P->table + 4 * ((int64_t)nb * KB + kb);
        int b = (int)e[2];
        if (b == 0) {
            for (int j = 0; j < 128; j++) out[kb * 128 + j] = 0.0;
            continue;
        }
        if (b == 16) {              /* passthrough: the stored bf16 weights */
            for (int j = 0; j < 128; j++) {
                uint16_t wb;
                memcpy(&wb, P->codes + e[0] + r * 256 + 2 * j, 2);
                out[kb * 128 + j] = mpqo_bf16_to_f64(wb);
            }
            continue;
        }
        unpack_row(P->codes + e[0], b, r, q);
        double s = mpqo_f16_to_f64(P->scales[e[1] + r]);
        double z = mpqo_f16_to_f64(P->zeros[e[1] + r]);
        for (int j = 0; j < 128; j++) out[kb * 128 + j] = ((double)q[j] - z) * s;
    }
}

/* What = dequantized weights in the ORIGINAL order, N x K row-major:
 * What[row_perm[i]][col_perm[j]] = dequant(W')[i][j].                       */
void mpqo_dequant(const mpqo_packed *P, double *What)
{
    double *tmp = (double *)malloc(sizeof(double) * (size_t)P->K);
    for (int i = 0; i < P->N; i++) {
        dequant_row_reordered(P, i, tmp);
        int n = P->row_perm ? P->row_perm[i] : i;
        for (int j = 0; j < P->K; j++) {
            int k = P->col_perm ? P->col_perm[j] : j;
            What[(int64_t)n * P->K + k] = tmp[j];
        }
    }
    free(tmp);
}

/* y[m][n] = sum_k x[m][k] * What[n][k] (fp64), bound[m][n] = sum_k |x*What|.
 * x is bf16, M x K row-major, read exactly.                                 */
void mpqo_linear_dense(int32_t M, int32_t N, int32_t K, const uint16_t *x,
                       const double *What, double *y, double *bound)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; n++) {
        for (int m = 0; m < M; m++) {
            double acc = 0.0, mag = 0.0;
            for (int k = 0; k < K; k++) {
                double p = mpqo_bf16_to_f64(x[(int64_t)m * K + k]) *
                           What[(int64_t)n * K + k];
                acc += p;
                mag += fabs(p);
            }
            y[(int64_t)m * N + n] = acc;
            if (bound) bound[(int64_t)m * N + n] = mag;
        }
    }
}

/* The same product for a chosen set of ORIGINAL output rows only (for large
 * layers): y[m][c] and bound[m][c] for n = rows[c], c < nrows (M x nrows).  */
void mpqo_linear_rows(const mpqo_packed *P, int32_t M, const uint16_t *x,
                      const int32_t *rows, int32_t nrows, double *y,
                      double *bound)
{
    int N = P->N, K = P->K;
    int32_t *inv = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    for (int i = 0; i < N; i++) inv[P->row_perm ? P->row_perm[i] : i] = i;
#pragma omp parallel for schedule(dynamic, 1)
    for (int c = 0; c < nrows; c++) {
        double *wr = (double *)malloc(sizeof(double) * (size_t)K);
        dequant_row_reordered(P, inv[rows[c]], wr);
        for (int m = 0; m < M; m++) {
            double acc = 0.0, mag = 0.0;
            for (int j = 0; j < K; j++) {
                int k = P->col_perm ? P->col_perm[j] : j;
                double p = mpqo_bf16_to_f64(x[(int64_t)m * K + k]) * wr[j];
                acc += p;
                mag += fabs(p);
            }
            y[(int64_t)m * nrows + c] = acc;
            if (bound) bound[(int64_t)m * nrows + c] = mag;
        }
        free(wr);
    }
    free(inv);
}
