/*
 * mpq_oracle.h -- declarations of the fp64 CPU oracle (test infrastructure
 * only; see mpq_oracle.c).  Independent of the library header: the oracle and
 * the CUDA path share no header, table or helper.
 */
#ifndef MPQ_ORACLE_H
#define MPQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    MPQO_OK = 0,
    MPQO_ERR_ARG = 1,
    MPQO_ERR_SHAPE = 2,
    MPQO_ERR_BITS = 3,
    MPQO_ERR_PERM = 4,
    MPQO_ERR_NONFINITE = 5,
    MPQO_ERR_RANGE = 6
};

typedef struct {
    int32_t N, K, NB, KB;
    uint64_t codes_bytes, n_sz, bit_total;
    uint64_t seg_off[17], seg_bytes[17];   /* index = bit width */
} mpqo_layout;

typedef struct {
    int32_t N, K;
    const uint8_t *codes;
    const uint32_t *table;      /* 4 words per block */
    const uint16_t *scales, *zeros;
    const int32_t *row_perm, *col_perm;   /* NULL = identity */
} mpqo_packed;

/* Threads of the OpenMP loops (n >= 1); returns the previous count.  Only
 * the timing of the oracle uses it; results do not depend on it. */
int mpqo_set_threads(int n);

double mpqo_bf16_to_f64(uint16_t b);
double mpqo_f16_to_f64(uint16_t h);
int mpqo_bits_valid(int b);
int mpqo_pieces(int b, int widths[2]);
int mpqo_plan(int32_t N, int32_t K, const uint8_t *bits, mpqo_layout *L,
              uint32_t *table);
int mpqo_quantize_group(const double *w, int n, int b, uint16_t *s_bits,
                        uint16_t *z_bits, uint8_t *q);
int mpqo_pack(int32_t N, int32_t K, const uint16_t *W, const uint8_t *bits,
              const int32_t *row_perm, const int32_t *col_perm,
              uint8_t *codes, uint32_t *table, uint16_t *scales,
              uint16_t *zeros);
void mpqo_dequant(const mpqo_packed *P, double *What);
void mpqo_linear_dense(int32_t M, int32_t N, int32_t K, const uint16_t *x,
                       const double *What, double *y, double *bound);
void mpqo_linear_rows(const mpqo_packed *P, int32_t M, const uint16_t *x,
                      const int32_t *rows, int32_t nrows, double *y,
                      double *bound);

#ifdef __cplusplus
}
#endif
#endif
