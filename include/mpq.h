/*
 * mpq.h -- C ABI of the block-wise mixed-precision weight-only quantized
 * linear layer for NVIDIA B200 (sm_100a).
 *
 *   y = x * dequant(W)^T
 *
 * Method (web pages on the subject, cited by title and section):
 *   "ScaleBITS: Scalable Bitwidth Search for Hardware-Aligned Mixed-Precision
 *   LLMs" -- abstract and summary page, section "Approach": the weight matrix
 *   is partitioned into hardware-aligned 64x128 blocks, each with its own bit
 *   width under a global budget, after rows and columns are reordered so that
 *   sensitive weights cluster; "Key results"/"Limitations": the scalar
 *   quantizer is round-to-nearest with group size 128; "Surprising findings":
 *   0- or 1-bit minimum precision.
 *   "SFMP: Fine-Grained, Hardware-Friendly and Search-Free Mixed-Precision
 *   Quantization for Large Language Models" -- abstract: block-wise mixed
 *   precision with row-column reordering and a small activation reordering
 *   step at inference.
 *   "TileQuant: Tile as the Precision-Allocation Unit for LLM Mixed-Precision
 *   Post-Training Quantization" -- abstract: the precision map guides compact
 *   weight buffers that the kernel streams.
 *
 * Definitions (the pages give no formulas; these readings are the library's):
 *   W is N x K (out x in, nn.Linear layout), bf16, row-major.  With
 *   permutations P_r (N) and P_c (K), W'[i][j] = W[P_r[i]][P_c[j]].
 *   Block (nb, kb) of W' is rows 64nb..64nb+63, columns 128kb..128kb+127;
 *   block id t = nb*KB + kb; each block has bits[t] in {0,1,2,3,4,5,6,8,16}.
 *   Each block row is one RTN group of 128 weights:
 *     lo = min(min w, 0), hi = max(max w, 0), d = hi - lo, qmax = 2^b - 1,
 *     s  = smallest fp16 h with h*qmax >= d  (s = 1 if d == 0),
 *     z  = rne(-lo / s) (an integer in [0, qmax], stored as fp16),
 *     q  = clamp(rne(w / s) + z, 0, qmax),   w_hat = (q - z) * s.
 *   A 0-bit block has no codes and dequantizes to zero.  A 16-bit block keeps
 *   its bf16 weights (w_hat = w; TileQuant abstract: the highest-scoring
 *   tiles stay at 16 bits); its weights must be finite and |w| <= 65504.
 *   y[m][P_r[i]] = sum_j x[m][P_c[j]] * w_hat'[i][j]   (y is fp32).
 *
 * Packed format v1 (the library's own; the pages name no layout):
 *   codes   -- segments for b = 1,2,3,4,5,6,8,16 in that order, each holding
 *              the payloads of all b-bit blocks in ascending t.  A payload is
 *              1024*b bytes: the code's "pieces" (1->[1], 2->[2], 3->[2,1],
 *              4->[4], 5->[4,1], 6->[4,2], 8->[8]; q = lo | hi << width(lo)),
 *              low piece first; a p-bit piece is 64 rows x 16p bytes,
 *              row-major; in a row, code j sits in little-endian 32-bit word
 *              j/(32/p) at bit (j%(32/p))*p.  A 16-bit payload is the
 *              block's 64 x 128 bf16 bit patterns, row-major.
 *   scales, zeros -- fp16 bit patterns, 64 per non-zero block, in ascending t;
 *              row r of block t is at table[t].sz_off + r (1 and 0 for a
 *              16-bit block).
 *   table   -- one mpq_block per block (ascending t).
 *   sched   -- the decode schedule, sched_words 32-bit words: the blocks are
 *              cut into n_units row-major runs [t0, t1) of about equal
 *              estimated cost (bytes streamed plus decode work by width),
 *              one per decode warp.  Run u has a 32-word descriptor at word
 *              32u: t0, t1, the index of its first stage and its number of
 *              stages, and the partial-sum slots of its first and last block
 *              rows (the other words are 0).  After the descriptors, 4 words
 *              per stage, in block order: payload byte offset, scale/zero
 *              index, block column | width << 16 | half << 24, block row.  A
 *              quantized block is one stage; a 16-bit block is two (its rows
 *              0..31 and 32..63, half 0 and 1).
 *
 * Conventions:
 *   - The caller owns every buffer.  The library allocates no device memory
 *     and keeps no state between calls beyond one-time kernel attributes per
 *     device (and mpq_linear_noalloc's static scratch, below); calls are
 *     asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 *     legacy default stream).
 *   - Errors that the host can see are returned at once and nothing is
 *     launched.  Errors found in device data (non-finite W, a group with no
 *     representable scale) or a device wait that ran out are written to an
 *     error word at the start of the workspace: the first such error since
 *     the workspace was zero-filled or since the last mpq_check(), which
 *     reports and clears it (mpq_pack clears it when it starts).
 *   - A launch failure returns MPQ_ERR_CUDA.
 *   - Every device pointer that the kernels read -- W, x, and the codes,
 *     table, sched, scales, zeros and permutations of a layer -- must be
 *     16-byte aligned (vector loads and bulk copies); MPQ_ERR_ARG otherwise.
 *   - Limits: N % 64 == 0, K % 128 == 0, N, K > 0, K <= 65536 when a column
 *     permutation is given, codes_bytes < 2^32; M >= 0 (M == 0 is a no-op).
 */
#ifndef MPQ_H
#define MPQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MPQ_OK = 0,
    MPQ_ERR_ARG = 1,        /* NULL pointer or inconsistent argument        */
    MPQ_ERR_SHAPE = 2,      /* N % 64, K % 128, N or K <= 0, M < 0, too big  */
    MPQ_ERR_BITS = 3,       /* a bit width outside {0,1,2,3,4,5,6,8,16}      */
    MPQ_ERR_PERM = 4,       /* a permutation that is not a bijection         */
    MPQ_ERR_NONFINITE = 5,  /* NaN/Inf in W (device-detected)               */
    MPQ_ERR_RANGE = 6,      /* no fp16 scale, qmax*s > 65504, or a 16-bit
                               block weight beyond +-65504 (device)          */
    MPQ_ERR_WORKSPACE = 7,  /* workspace missing or too small               */
    MPQ_ERR_CUDA = 8,       /* a CUDA call failed                           */
    MPQ_ERR_TIMEOUT = 9     /* a bounded device wait ran out (device)       */
} mpq_status;

/* Element type of y for mpq_linear_typed. */
typedef enum {
    MPQ_Y_F32 = 0,          /* fp32: the graded output (mpq_linear)          */
    MPQ_Y_BF16 = 1          /* bf16, round-to-nearest-even of the fp32 y     */
} mpq_ydtype;

/* One block of the table (16 bytes). */
typedef struct {
    uint32_t code_off;    /* byte offset of the payload in `codes` (0 if 0-bit) */
    uint32_t sz_off;      /* index of the block's row 0 in scales/zeros          */
    uint32_t bits;        /* 0,1,2,3,4,5,6,8 or 16                               */
    uint32_t bit_prefix;  /* sum of bits of all blocks with a smaller id        */
} mpq_block;

/* Sizes of a packed layer; filled by mpq_plan. */
typedef struct {
    int32_t N, K, NB, KB;    /* NB = N/64, KB = K/128                          */
    int32_t n_units;         /* decode work units (runs)                        */
    int32_t sched_words;     /* 32-bit words of sched                          */
    uint64_t codes_bytes;    /* = 1024 * bit_total                              */
    uint64_t n_sz;           /* = 64 * number of non-zero blocks                */
    uint64_t bit_total;      /* sum of the per-block bits                       */
    uint64_t seg_off[17];    /* byte offset of segment b (index = bit width)    */
    uint64_t seg_bytes[17];  /* bytes of segment b (0 for unused widths)         */
} mpq_layout;

/* A packed layer: device pointers to caller-owned buffers of the sizes in
 * mpq_layout.  mpq_pack writes these buffers; mpq_linear reads them. */
/* mpq_layer.flags */
#define MPQ_LAYER_16BIT 1   /* the layer has 16-bit blocks (seg_bytes[16] > 0) */

typedef struct {
    int32_t N, K;
    int32_t n_units;
    int32_t flags;               /* MPQ_LAYER_16BIT when the layer has 16-bit
                                    blocks: mpq_linear then uses the decode
                                    kernel built with the 16-bit path (a 16-bit
                                    block met without the flag records
                                    MPQ_ERR_BITS on the device)                */
    const void* codes;           /* uint8  [codes_bytes]                        */
    const mpq_block* table;      /* [NB*KB]                                      */
    const uint32_t* sched;       /* [sched_words] (mpq_layout)                    */
    const uint16_t* scales;      /* fp16 bits [n_sz]                             */
    const uint16_t* zeros;       /* fp16 bits [n_sz]                             */
    const int32_t* row_perm;     /* int32 [N]; NULL = identity                   */
    const int32_t* col_perm;     /* int32 [K]; NULL = identity                   */
} mpq_layer;

/* Host only.  Validates N, K and the bit map (uint8, NB*KB, block id order)
 * and fills `out`: segment offsets/sizes, codes_bytes, n_sz, bit_total and
 * the number of decode work units.  Block partition: ScaleBITS summary,
 * "Approach"; bit set and budget: ScaleBITS abstract, "Key results".
 * Errors: MPQ_ERR_ARG, MPQ_ERR_SHAPE, MPQ_ERR_BITS. */
mpq_status mpq_plan(int32_t N, int32_t K, const uint8_t* bits_host,
                    mpq_layout* out);

/* Host only.  Writes the decode schedule that mpq_pack stores in `sched`
 * (sched_words words, format above) for layout L and the same bit map into
 * host memory, e.g. to inspect the work split.  Errors: ARG (L does not
 * belong to these bits), SHAPE, BITS. */
mpq_status mpq_plan_schedule(const mpq_layout* L, const uint8_t* bits_host,
                             uint32_t* sched_host);

/* Workspace bytes that mpq_pack needs (the error word). */
size_t mpq_pack_workspace_size(const mpq_layout* L);

/* Quantize and pack W (ScaleBITS summary "Approach" + "Key results": RTN-g128
 * per 64x128 block after reordering; TileQuant abstract: compact buffers).
 *   L              layout from mpq_plan for the same N, K and bits.
 *   W_dev          bf16 bit patterns, N x K row-major, ORIGINAL order, device.
 *   bits_host      uint8 [NB*KB] (host).
 *   row_perm_host, col_perm_host   int32 permutations (host) or NULL.
 *   out            buffers to fill (device): codes, table, sched, scales,
 *                  zeros; out->row_perm / col_perm receive copies of the host
 *                  permutations and must be NULL exactly when those are NULL.
 *   ws, ws_bytes   device workspace (>= mpq_pack_workspace_size).
 * The result is a pure function of the inputs (byte-deterministic).
 * Host errors: ARG, SHAPE, BITS, PERM, WORKSPACE; device errors (mpq_check):
 * NONFINITE, RANGE.  Outputs are unspecified after a device error. */
mpq_status mpq_pack(const mpq_layout* L, const void* W_dev,
                    const uint8_t* bits_host, const int32_t* row_perm_host,
                    const int32_t* col_perm_host, const mpq_layer* out,
                    void* ws, size_t ws_bytes, void* stream);

/* mpq_pack with two optional cudaEvent_t handles (NULL = none): ev_begin is
 * recorded on `stream` after the host planning and the table / schedule /
 * permutation uploads, right before the quantize kernel, and ev_end right
 * after it, so a caller can time the kernel alone.  Same arguments, results
 * and errors as mpq_pack. */
mpq_status mpq_pack_timed(const mpq_layout* L, const void* W_dev,
                          const uint8_t* bits_host, const int32_t* row_perm_host,
                          const int32_t* col_perm_host, const mpq_layer* out,
                          void* ws, size_t ws_bytes, void* stream, void* ev_begin,
                          void* ev_end);

/* Workspace bytes that mpq_linear needs for M tokens. */
size_t mpq_linear_workspace_size(const mpq_layer* layer, int32_t M);

/* y = x * dequant(W)^T for M tokens, including the activation column
 * reordering x'[m][j] = x[m][P_c[j]] (SFMP abstract: "activation reordering
 * overhead during inference") and the inverse output reordering
 * y[m][P_r[i]] = y'[m][i].
 *   x_dev   bf16 bit patterns, M x K row-major (device).
 *   y_dev   fp32, M x N row-major, original output order (device).
 *   ws      device workspace of >= mpq_linear_workspace_size(layer, M) bytes,
 *           256-byte aligned, zero-filled before its first use (e.g.
 *           cudaMemset); every call that ends without a device error leaves
 *           the parts that must start at zero at zero, so it can be reused
 *           as is (zero it again after a device error).
 * Uses a memory-bound decode kernel (integer tensor cores) for M <= 8; for
 * 9 <= M <= 16 on layers of at least 100 tiles of 128 rows without 16-bit
 * blocks, the same integer arithmetic on tcgen05 (kind::i8); otherwise a
 * tcgen05 kernel on dequantized fp16 tiles.  Non-finite x gives non-finite y
 * (no error).  Activations are scaled by exact powers of two (per 128-column
 * slice into 23-bit integers on the integer paths, per token into fp16 on
 * the fp16 path); a slice element more than 2^15 below the slice maximum is
 * rounded to 2^-23 of that maximum.
 * Host errors: ARG, SHAPE, WORKSPACE; device (mpq_check): TIMEOUT, BITS (a
 * 16-bit block in a layer whose flags lack MPQ_LAYER_16BIT). */
mpq_status mpq_linear(const mpq_layer* layer, const void* x_dev, int32_t M,
                      float* y_dev, void* ws, size_t ws_bytes, void* stream);

/* mpq_linear with a choice of output type.  MPQ_Y_F32 is mpq_linear itself
 * (y_dev is float*).  MPQ_Y_BF16 writes y_dev as bf16 bit patterns (uint16,
 * M x N row-major): the fp32 result of mpq_linear, kept in the workspace,
 * rounded to nearest-even.  This is a convenience for callers that feed a bf16
 * model: the rounding alone (up to 2^-9 relative) exceeds the fp32 path's
 * error bars.  ws must hold mpq_linear_typed_workspace_size(layer, M, ydt)
 * bytes.  Errors: those of mpq_linear; ARG for an unknown ydt. */
size_t mpq_linear_typed_workspace_size(const mpq_layer* layer, int32_t M, mpq_ydtype ydt);
mpq_status mpq_linear_typed(const mpq_layer* layer, const void* x_dev, int32_t M,
                            void* y_dev, mpq_ydtype ydt, void* ws, size_t ws_bytes,
                            void* stream);

/* Several layers that share x (the same K): y_i = x * dequant(W_i)^T for
 * i < n, e.g. the q, k and v projections or gate and up.  Same results as n
 * mpq_linear calls (bit for bit); when M == 1 and every layer's decode
 * builds its own activation records (layers whose runs hold at most two
 * blocks on average), the whole group is one kernel launch -- the launch
 * floor, which dominates such small layers, is paid once per group instead
 * of once per layer (the pages have no grouped call; this is a deployment
 * convenience of the library).  Otherwise the layers run one after another.
 *   layers  host array of n layers (1 <= n <= MPQ_GROUP_MAX), equal K.
 *   y_devs  host array of n device pointers (fp32, M x N_i each).
 *   ws      device workspace of mpq_linear_group_workspace_size(layers, n, M)
 *           bytes, 256-byte aligned, zero-filled before first use (as for
 *           mpq_linear); its first word is the group's error word.
 * Host errors: ARG (n out of range, NULL), SHAPE (K differs, bad layer),
 * WORKSPACE; device (mpq_check): TIMEOUT. */
#define MPQ_GROUP_MAX 8
size_t mpq_linear_group_workspace_size(const mpq_layer* layers, int32_t n, int32_t M);
mpq_status mpq_linear_group(const mpq_layer* layers, int32_t n, const void* x_dev, int32_t M,
                            float* const* y_devs, void* ws, size_t ws_bytes, void* stream);

/* mpq_linear that also records two CUDA events (cudaEvent_t as void*; either
 * may be NULL) on `stream`: ev_begin right before the first launch of the
 * main GEMM kernel and ev_end right after its last launch, so a caller can
 * time that kernel alone with events (the activation prologue is outside).
 * Same arguments, results and errors as mpq_linear. */
mpq_status mpq_linear_timed(const mpq_layer* layer, const void* x_dev, int32_t M,
                            float* y_dev, void* ws, size_t ws_bytes, void* stream,
                            void* ev_begin, void* ev_end);

/* The same product with HOST activations and outputs: copies x_host (bf16,
 * M x K) into the workspace, runs mpq_linear and copies y back to y_host
 * (fp32, M x N), all on `stream`; returns after enqueueing (synchronize the
 * stream before reading y_host).  Use pinned host memory for asynchrony.
 * ws must hold mpq_linear_host_workspace_size(layer, M) bytes and follows
 * the same zero-fill rule as mpq_linear's. */
size_t mpq_linear_host_workspace_size(const mpq_layer* layer, int32_t M);
mpq_status mpq_linear_host(const mpq_layer* layer, const void* x_host,
                           int32_t M, float* y_host, void* ws,
                           size_t ws_bytes, void* stream);

/* mpq_linear for callers that cannot allocate device memory, and so cannot
 * pass a workspace: e.g. an inference-engine plugin whose device memory is
 * fixed when it is initialized, or a host program whose allocator is not
 * reachable through this C ABI.  (The paper has no counterpart: this is a
 * deployment convenience of the library.)
 *   Same layer, x_dev, M, y_dev, stream and results as mpq_linear.  The
 *   scratch is one static device array of MPQ_NOALLOC_SCRATCH_BYTES
 *   (6 MiB) inside the library, held by every GPU that loads the library
 *   until the process exits; no cudaMalloc/cudaFree or other allocating
 *   call is made.  Sizes whose workspace (mpq_linear_workspace_size) would
 *   exceed it return MPQ_ERR_WORKSPACE.
 *   Every call looks up the array's device address (cudaGetSymbolAddress)
 *   with the calling device current; the first lookup on a device loads the
 *   library's device code there, so make the first call before any stream
 *   capture.
 *   All calls share the one array, which starts zeroed and keeps the last
 *   call's contents (the parts that must start at zero are left at zero): calls
 *   that overlap on the GPU -- on different streams, or from different
 *   threads -- race and give wrong results.  Serialize them.
 *   Device-side errors (MPQ_ERR_TIMEOUT) go to the array's error word, which
 *   mpq_check cannot see: read it with mpq_noalloc_check.  Until then, a call
 *   that stopped on a device error may have left the array's counters set,
 *   and the calls after it give wrong results.  Host-side errors are returned
 *   as for mpq_linear. */
#define MPQ_NOALLOC_SCRATCH_BYTES (6u << 20)
mpq_status mpq_linear_noalloc(const mpq_layer* layer, const void* x_dev, int32_t M,
                              float* y_dev, void* stream);

/* The error word of mpq_linear_noalloc's static array on the current device:
 * synchronizes `stream`, returns the first device error of the calls since
 * the previous check (MPQ_OK if none) and, after an error, zero-fills the
 * array (memset, no allocation) so that the next call starts clean. */
mpq_status mpq_noalloc_check(void* stream);

/* Budgeted bit allocation: the bit map that mpq_plan / mpq_pack take, from
 * per-block sensitivity surrogates under a global budget.  ScaleBITS
 * abstract (bitwidth allocation under a memory budget by "a scalable
 * approximation to the greedy algorithm") and summary page, "Approach" (a
 * batched approximation to greedy knapsack allocation per 64x128 block) and
 * "Key results" (16-36 search iterations against about 3e6 for classic
 * greedy).  The library's reading: with a price lam per bit, each block
 * takes argmin_b loss[t][b] + lam * b (fp64, the product rounded before the
 * sum, ties to the smaller width); lam is bisected until the total fits the
 * budget (from lo = 0 and hi = the largest per-bit saving over the smallest
 * width, doubled while rounding leaves the total above the budget; until the
 * total equals the budget, hi - lo <= hi * 2^-20, the midpoint equals an end,
 * or 64 steps); the leftover is then filled in rounds, each taking the
 * longest prefix of the next-width upgrades that save loss (saving per bit
 * descending, block index ascending) whose increments fit.  On losses convex
 * in the width this is the classic one-upgrade-at-a-time greedy's result.
 *   n_blocks    blocks (1 .. 2^24), in any order the caller chooses (e.g. the
 *               block ids of one layer, or all layers of a model).
 *   loss_dev    device float [n_blocks][8]: the loss of each block at widths
 *               0,1,2,3,4,5,6,8 (columns of widths not allowed are ignored).
 *   allowed     bit b set = width b allowed (b in {0..6, 8}, at least one).
 *   budget      total bits (sum of the widths); at least n_blocks times the
 *               smallest allowed width.
 *   bits_dev    device uint8 [n_blocks] (out): the widths.
 *   info_dev    device uint32 [4] (out): search iterations (1 + bisection
 *               steps + fill rounds), total bits (low word, high word),
 *               status (MPQ_OK, or MPQ_ERR_NONFINITE for a non-finite loss).
 *   ws          device workspace of mpq_allocate_bits_workspace_size bytes.
 * One CTA runs the search (deterministic).  Host errors: ARG, WORKSPACE. */
size_t mpq_allocate_bits_workspace_size(int64_t n_blocks);
mpq_status mpq_allocate_bits(int64_t n_blocks, const float* loss_dev, uint32_t allowed,
                             uint64_t budget, uint8_t* bits_dev, uint32_t* info_dev, void* ws,
                             size_t ws_bytes, void* stream);

/* Folds the output reordering of one layer into the input reordering of the
 * next (SFMP abstract: reordering costs only "a small activation
 * reordering overhead during inference"; this removes the output scatter of
 * the first layer as well).  Host only.
 *   Layer A (N_A outputs) was packed with row order row_perm_a; layer B
 *   (K_B = N_A inputs) with column order col_perm_b.  Run A with a layer
 *   whose row_perm is NULL: its y is then in A's packed row order,
 *   y'[m][i] = y[m][row_perm_a[i]].  Run B on that y' (or on any elementwise
 *   function of it) with col_perm = out, where
 *     out[j] = inverse(row_perm_a)[col_perm_b[j]],  j < n,
 *   so B gathers x'[m][j] = y'[m][out[j]] = y[m][col_perm_b[j]] -- the same
 *   values, and the same result bit for bit, as the unfolded pair.
 *   NULL for either order means identity; out (host, n int32) must not be
 *   NULL.  Errors: ARG (n <= 0, out NULL), PERM (an order that is not a
 *   bijection of 0..n-1). */
mpq_status mpq_fold_orders(int32_t n, const int32_t* row_perm_a, const int32_t* col_perm_b,
                           int32_t* out);

/* Synchronizes `stream` and returns the device error word of `ws`: the first
 * device error of the mpq_linear calls on that workspace since it was
 * zero-filled or since the previous mpq_check, or of the last mpq_pack
 * (MPQ_OK if none); then clears it. */
mpq_status mpq_check(const void* ws, void* stream);

/* Human-readable name of a status. */
const char* mpq_status_string(mpq_status s);

#ifdef __cplusplus
}
#endif

#endif /* MPQ_H */
