// k_decode.cuh -- memory-bound mixed-precision GEMV/GEMM for small M.
//
// y'[m][i] = sum_kb s[i,kb] * sum_{j in kb} x'[m][j] * (q[i][j] - z[i,kb])
// (the blocks' RTN dequantization, ScaleBITS summary "Approach" / "Key
// results"; 0-bit blocks are skipped -- they hold no bytes), then
// y[m][row_perm[i]] = y'[m][i].
//
// Work split.  At pack time the blocks are cut into `n_units` row-major runs
// of about equal estimated cost (bytes moved plus decode work per bit
// width); each run is one warp's work.  A run descriptor of 128 bytes holds
// its blocks [t0, t1), where its non-zero blocks start in the stage list and
// how many there are, and where the partial sums of its first and last block
// rows go.  The stage list holds, per non-zero block, everything its copies
// need (payload offset, scale/zero index, block column and width, block
// row): a warp loads 32 of them with one coalesced 16-byte load per lane.
//
// Each warp streams its non-zero blocks through a private ring of shared
// memory with 1-D bulk async copies (payload + 64 scales + 64 zeros + the
// activation record(s) of the block's slice), several blocks ahead of the
// one it computes.
//
// Arithmetic (exact up to the final fp32 steps).  The activation slice is
// held as integers X (k_xprep.cuh: X = rne(x' 2^e), |X| < 2^23, three s8
// digits) and the codes as unsigned bytes: one AND of a code word gives four
// codes of one "plane" (piece_regs).  The integer tensor cores
// (mma.m16n8k32.u8.s8, s32 accumulation) form C_d = sum_j q_j d_d(X_j) per
// digit d with no rounding, so the zero point is taken out exactly:
//   E_d = C_d - z T_d,   T_d = sum_j d_d(X_j),
//   V   = E_0 + 256 E_1 + 65536 E_2 = sum_j (q_j - z) X_j,
// and each block adds s * 2^-e * V to its output row in fp32.  The only
// roundings are X (for slice elements more than 2^15 below the slice
// maximum), the conversion of V to fp32 and the fp32 accumulation -- all
// relative to sum |x * w_hat|, never to the cancelled sum q*x.
// 16-bit passthrough blocks (TileQuant abstract) take bf16 mma.m16n8k16 on
// the block's weights and the slice's bf16 values (a separate build of the
// kernel, chosen by the layer's MPQ_LAYER_16BIT flag).
//
// A block row that lies inside one run is written straight to y.  A block
// row shared by several runs (the first and last row of a run) is finished
// by the last warp to arrive (a per-row arrival counter): it adds the
// contributors' partial sums -- a contiguous range of slots -- in run order,
// so results are deterministic.
//
// Every wait is bounded: after ~2 s it records MPQ_ERR_TIMEOUT and the warp
// stops computing (its arithmetic is skipped, its bookkeeping still runs);
// before it leaves it waits, again bounded, for the copies it has in flight.
#pragma once
#include "common.cuh"
#include "k_xprep.cuh"   // XQD_*

namespace mpq {

// Wait-test build (-DMPQ_WAIT_TEST, a separate library used only by the
// timeout test, never the default build): waits give up after 2 ms, and the
// producers arm their barriers without issuing any copy, so every first wait
// runs out with nothing in flight.
#ifdef MPQ_WAIT_TEST
constexpr bool kWaitTest = true;
constexpr uint64_t DEC_WAIT_NS = 2000000ull;
#else
constexpr bool kWaitTest = false;
constexpr uint64_t DEC_WAIT_NS = 2000000000ull;
#endif

// Run descriptor: 32 words (the unused ones are zero).
enum DescWord {
    DW_T0 = 0, DW_T1 = 1,  // the run's blocks [t0, t1)
    DW_S0 = 2,             // index of its first non-zero block in the stage list
    DW_NS = 3,             // number of non-zero blocks
    DW_A_SLOT = 10,        // first block row of the run: first partial slot of the row,
    DW_A_NC = 11,          //   number of runs that meet the row, this run's index among them
    DW_A_IDX = 12,
    DW_B_SLOT = 13,        // last block row of the run: the same three
    DW_B_NC = 14,
    DW_B_IDX = 15,
    DESC_WORDS = 32
};
// Stage descriptor: one per non-zero block (block order), 4 words.
enum StageWord {
    SW_CODE = 0,           // byte offset of the payload in the codes buffer
    SW_SZ = 1,             // index of the block's row 0 in scales / zeros
    SW_KB_BITS = 2,        // block column | bit width << 16
    SW_NB = 3,             // block row
    STAGE_WORDS = 4
};

struct DecodeParams {
    const uint8_t* codes;
    const uint32_t* desc;     // [n_units][32]
    const uint4* stages;      // [non-zero blocks] stage descriptors
    const uint16_t* scales;
    const uint16_t* zeros;
    const int32_t* row_perm;
    const uint8_t* xq;        // k_xprep_decode records: [KB][XQD_REC * M_total]
    const uint16_t* x;        // bf16 x [M_total][K] (the fused one-token path reads it)
    const int32_t* col_perm;  // [K] or null (fused path)
    float* y;                 // [M_total][N]
    float* partial;           // [slots][Mg][64]
    uint32_t* counters;       // [NB] arrivals per block row
    uint32_t* err;
    int N, K, NB, KB;
    int M_total;              // tokens in xq / y
    int m0, Mg;               // this launch's token group [m0, m0+Mg), Mg <= 8
    int n_units;
};

constexpr int DEC_WARPS = 4;
constexpr int DEC_THREADS = DEC_WARPS * 32;
constexpr int DEC_CTAS_PER_SM = 4;   // 16 resident warps per SM
constexpr int DEC_MAX_REGS = 112;
constexpr int DEC_RING = 12800;      // bytes of ring per warp (>= largest stage)
constexpr int DEC_SLOTS = 8;         // stages in flight per warp
constexpr int DEC_MAX_TOKENS = 8;

struct DecWarp {
    uint8_t ring[DEC_RING];
    int32_t rows[64];         // output index of each row of the current block row (16-byte aligned)
    uint64_t full[DEC_SLOTS];
    uint4 zero32[2];          // zero B fragments for lanes beyond the token count
};
struct DecSmem {
    DecWarp w[DEC_WARPS];
};

// DEC_CTAS_PER_SM x (smem + 1 KB reserved) must fit the SM's 228 KB
static_assert(DEC_CTAS_PER_SM * (sizeof(DecSmem) + 1024) <= 228 * 1024, "decode smem too large");
// largest stages: an 8-bit payload, or a 6-bit one with two activation variants
static_assert(DEC_RING >= 8 * 1024 + 256 + DEC_MAX_TOKENS * XQD_VAR, "ring too small");
static_assert(DEC_RING >= 6 * 1024 + 256 + 2 * DEC_MAX_TOKENS * XQD_VAR, "ring too small");
static_assert(DEC_RING >= 8192 + DEC_MAX_TOKENS * (XQD_VAR + 128), "ring too small");

__host__ __device__ constexpr int lo_width(int b) { return (b == 3) ? 2 : (b == 5 || b == 6) ? 4 : b; }
__host__ __device__ constexpr int hi_width(int b) { return (b == 3 || b == 5) ? 1 : (b == 6) ? 2 : 0; }
// activation variant of a piece width (16: the bf16 slice for passthrough blocks)
__host__ __device__ constexpr int variant_of(int p) { return p == 1 ? 0 : p == 2 ? 1 : p == 4 ? 2 : p == 16 ? 4 : 3; }
// index of width b in the descriptor's code offsets (1,2,3,4,5,6,8 -> 0..6)
__host__ __device__ constexpr int width_index(int b) { return b == 8 ? 6 : b - 1; }

// ---------------------------------------------------------------------------
// Code extraction.  piece_regs<P, W> turns this lane's quarter of one row of
// a P-bit piece (columns 32t .. 32t+31 of the block) into the eight A-operand
// registers of the four k-tiles of mma.m16n8k32 (index 2j + hf): four codes
// per register, one per byte, each register one AND (and at most one shift)
// of a code word -- a "plane" of the word.  The column that byte b of
// register (j, hf) holds is xqd_col(variant of P, 32j + 16hf + 4t + b); the
// activation records use the same order.  W shifts the codes left by W bits:
// the high piece of a split code is worth 2^(low width) (3 = 2 + 1 bits,
// 5 = 4 + 1, 6 = 4 + 2), so its planes carry that weight and both pieces
// accumulate into the same sums (q = lo + 2^w(lo) hi <= 63 fits a byte).
// ---------------------------------------------------------------------------
template <int S, int W>
__device__ __forceinline__ uint32_t plane_shift(uint32_t w) {   // (w >> S) << W, as one shift
    return (S >= W) ? (w >> (S - W)) : (w << (W - S));
}

template <int P, int W>
__device__ __forceinline__ void piece_regs(const uint8_t* rowp, int t, uint32_t (&a)[8]) {
    if (P == 1) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(rowp + 4 * t);
        constexpr uint32_t m = 0x01010101u << W;
        a[0] = plane_shift<0, W>(w) & m;
        a[1] = plane_shift<1, W>(w) & m;
        a[2] = plane_shift<2, W>(w) & m;
        a[3] = plane_shift<3, W>(w) & m;
        a[4] = plane_shift<4, W>(w) & m;
        a[5] = plane_shift<5, W>(w) & m;
        a[6] = plane_shift<6, W>(w) & m;
        a[7] = plane_shift<7, W>(w) & m;
    } else if (P == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(rowp + 8 * t);
        constexpr uint32_t m = 0x03030303u << W;
        // register (j, hf): word j / 2, plane 2 (j % 2) + hf (bits 2 plane)
        a[0] = plane_shift<0, W>(v.x) & m;
        a[1] = plane_shift<2, W>(v.x) & m;
        a[2] = plane_shift<4, W>(v.x) & m;
        a[3] = plane_shift<6, W>(v.x) & m;
        a[4] = plane_shift<0, W>(v.y) & m;
        a[5] = plane_shift<2, W>(v.y) & m;
        a[6] = plane_shift<4, W>(v.y) & m;
        a[7] = plane_shift<6, W>(v.y) & m;
    } else if (P == 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(rowp + 16 * t);
        a[0] = v.x & 0x0F0F0F0Fu; a[1] = (v.x >> 4) & 0x0F0F0F0Fu;
        a[2] = v.y & 0x0F0F0F0Fu; a[3] = (v.y >> 4) & 0x0F0F0F0Fu;
        a[4] = v.z & 0x0F0F0F0Fu; a[5] = (v.z >> 4) & 0x0F0F0F0Fu;
        a[6] = v.w & 0x0F0F0F0Fu; a[7] = (v.w >> 4) & 0x0F0F0F0Fu;
    } else {
        const uint4 v0 = reinterpret_cast<const uint4*>(rowp + 32 * t)[0];
        const uint4 v1 = reinterpret_cast<const uint4*>(rowp + 32 * t)[1];
        a[0] = v0.x; a[1] = v0.y; a[2] = v0.z; a[3] = v0.w;
        a[4] = v1.x; a[5] = v1.y; a[6] = v1.z; a[7] = v1.w;
    }
}

// D(16x8, s32) += A(16x32, u8 codes) * B(32x8, s8 activation digits)
__device__ __forceinline__ void imma_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void load8(const uint8_t* src, uint32_t (&b)[8]) {
    const uint4 v0 = reinterpret_cast<const uint4*>(src)[0];
    const uint4 v1 = reinterpret_cast<const uint4*>(src)[1];
    b[0] = v0.x; b[1] = v0.y; b[2] = v0.z; b[3] = v0.w;
    b[4] = v1.x; b[5] = v1.y; b[6] = v1.z; b[7] = v1.w;
}

// One block of width B, added into acc.  The mma's rows are the block's rows
// in an order that keeps each lane's rows together: in row tile rt, mma row
// g is block row 8g + 2rt and mma row g + 8 is block row 8g + 2rt + 1 (two
// adjacent rows: their scales and zero points are one fp16 pair).  mma
// column 4u + d (d < 3) is digit d of token 2 grp + u; column 4u + 3 is zero.
// Lane (g, t) accumulates columns 2t, 2t+1 -- digits (0, 1) of token
// 2 grp + t/2 for even t, digit 2 for odd t -- of both rows; the lane pair
// (t, t^1) swaps one partial sum so that the even lane finishes row
// 8g + 2rt and the odd lane row 8g + 2rt + 1:
//   V = (E_0 + 256 E_1) + 65536 E_2,  E_d = C_d - z T_d  (exact int32 parts)
//   acc[rt][grp] += s * F * V        (lane row 8g + 2rt + (t & 1))
template <int B, int G>
__device__ __forceinline__ void block_accumulate(const uint8_t* stage, const uint8_t* xlo,
                                                 const uint8_t* xhi, const uint8_t* zero32, int g,
                                                 int t, uint32_t Mg, float (&acc)[4][G]) {
    constexpr int P0 = lo_width(B), P1 = hi_width(B);
    const uint8_t* lo = stage;                       // 64 rows x 16 P0 bytes
    const uint8_t* hi = stage + 64 * 16 * P0;        // 64 rows x 16 P1 bytes
    const uint8_t* sz = stage + 1024 * B;            // scales[64], zeros[64] (fp16)
    const bool odd = (t & 1) != 0;
    // Four token groups: groups outermost, the codes unpacked again for each
    // (fewer live registers); otherwise every group reuses a tile's codes.
    constexpr bool kGroupOuter = G >= 4;
    // B-fragment source of group grp: column g = token 2 grp + g/4, digit g%4
    auto bsrc = [&](const uint8_t* x, int grp) -> const uint8_t* {
        const uint32_t tb = 2u * grp + (uint32_t)(g >> 2), dg = (uint32_t)(g & 3);
        return (dg < 3u && tb < Mg) ? x + tb * XQD_VAR + dg * 128 + t * 32 : zero32;
    };
    // digit sums and F of the lane's columns 2t, 2t+1 (token 2 grp + t/2)
    constexpr int GT = G >= 4 ? 1 : G;   // four groups read theirs per group (below)
    int Ta[GT], Tb[GT];
    float F[GT];
#pragma unroll
    for (int grp = 0; grp < GT; ++grp) {
        const uint32_t tc = 2u * grp + (uint32_t)(t >> 1);
        uint4 tf = make_uint4(0u, 0u, 0u, 0u);
        if (tc < Mg) tf = *reinterpret_cast<const uint4*>(xlo + tc * XQD_VAR + XQD_DIGITS * 128);
        Ta[grp] = (int)(odd ? tf.z : tf.x);
        Tb[grp] = odd ? 0 : (int)tf.y;
        F[grp] = __uint_as_float(tf.w);
    }
    uint32_t bl[8], bh[8];
    if (G == 1) {
        load8(bsrc(xlo, 0), bl);
        if (P1) load8(bsrc(xhi, 0), bh);
    }
#pragma unroll 1
    for (int go = 0; go < (kGroupOuter ? G : 1); ++go) {
        // the group's digit sums and F, and its accumulators (selected
        // without run-time register indexing)
        int Tag = 0, Tbg = 0;
        float Fg = 0.f;
        if (kGroupOuter) {
            const uint32_t tc = 2u * go + (uint32_t)(t >> 1);
            uint4 tf = make_uint4(0u, 0u, 0u, 0u);
            if (tc < Mg) tf = *reinterpret_cast<const uint4*>(xlo + tc * XQD_VAR + XQD_DIGITS * 128);
            Tag = (int)(odd ? tf.z : tf.x);
            Tbg = odd ? 0 : (int)tf.y;
            Fg = __uint_as_float(tf.w);
        }
        float cur[4];
        if (kGroupOuter) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                cur[i] = acc[i][0];
#pragma unroll
                for (int k = 1; k < G; ++k) cur[i] = (go == k) ? acc[i][k] : cur[i];
            }
        }
#pragma unroll
        for (int rt = 0; rt < 4; ++rt) {
            const int r0 = 8 * g + 2 * rt;
            const __half2 sh = bits_h2(*reinterpret_cast<const uint32_t*>(sz + 2 * r0));
            const __half2 zh = bits_h2(*reinterpret_cast<const uint32_t*>(sz + 128 + 2 * r0));
            // z is an fp16 integer <= 255: z + 1024 has the bits 0x6400 | z
            const uint32_t zb = h2_bits(__hadd2(zh, bits_h2(0x64006400u)));
            const int z0 = (int)(zb & 0x3FFu), z1 = (int)((zb >> 16) & 0x3FFu);
            const float s_own = __half2float(odd ? __high2half(sh) : __low2half(sh));
            uint32_t a0[8], a1[8];
            piece_regs<P0, 0>(lo + r0 * 16 * P0, t, a0);
            piece_regs<P0, 0>(lo + (r0 + 1) * 16 * P0, t, a1);
            uint32_t h0[8], h1[8];
            if (P1) {
                piece_regs<P1, P0>(hi + r0 * 16 * P1, t, h0);
                piece_regs<P1, P0>(hi + (r0 + 1) * 16 * P1, t, h1);
            }
#pragma unroll
            for (int gi = 0; gi < (kGroupOuter ? 1 : G); ++gi) {
                const int grp = kGroupOuter ? 0 : gi;     // register index (group-outer: cur[])
                const int gsel = kGroupOuter ? go : gi;   // the token group
                if (G > 1) {
                    load8(bsrc(xlo, gsel), bl);
                    if (P1) load8(bsrc(xhi, gsel), bh);
                }
                int c[4] = {0, 0, 0, 0}, d[4] = {0, 0, 0, 0};
#pragma unroll
                for (int j = 0; j < 4; j += 2) {
                    imma_16832(c, a0[2 * j], a1[2 * j], a0[2 * j + 1], a1[2 * j + 1], bl[2 * j], bl[2 * j + 1]);
                    imma_16832(d, a0[2 * j + 2], a1[2 * j + 2], a0[2 * j + 3], a1[2 * j + 3], bl[2 * j + 2],
                               bl[2 * j + 3]);
                }
                if (P1) {
#pragma unroll
                    for (int j = 0; j < 4; j += 2) {
                        imma_16832(c, h0[2 * j], h1[2 * j], h0[2 * j + 1], h1[2 * j + 1], bh[2 * j],
                                   bh[2 * j + 1]);
                        imma_16832(d, h0[2 * j + 2], h1[2 * j + 2], h0[2 * j + 3], h1[2 * j + 3],
                                   bh[2 * j + 2], bh[2 * j + 3]);
                    }
                }
                // exact int32 parts of rows r0 (c0, c1) and r0 + 1 (c2, c3):
                // even lanes E_0 + 256 E_1, odd lanes E_2
                const int ta = kGroupOuter ? Tag : Ta[grp], tb = kGroupOuter ? Tbg : Tb[grp];
                const int p0 = (c[0] + d[0] - z0 * ta) + 256 * (c[1] + d[1] - z0 * tb);
                const int p1 = (c[2] + d[2] - z1 * ta) + 256 * (c[3] + d[3] - z1 * tb);
                // even lane keeps row r0 and gets its E_2; odd lane keeps row r0 + 1
                const int other = __shfl_xor_sync(0xffffffffu, odd ? p0 : p1, 1);
                const float lo01 = (float)(odd ? other : p0);
                const float e2 = (float)(odd ? p1 : other);
                if (kGroupOuter)
                    cur[rt] = fmaf(s_own * Fg, fmaf(65536.f, e2, lo01), cur[rt]);
                else
                    acc[rt][grp] = fmaf(s_own * F[grp], fmaf(65536.f, e2, lo01), acc[rt][grp]);
            }
        }
        if (kGroupOuter) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int k = 0; k < G; ++k) acc[i][k] = (go == k) ? cur[i] : acc[i][k];
        }
    }
}

// bf16 MMA: D(16x8, fp32) += A(16x16, bf16) * B(16x8, bf16)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Half `half` (block rows 32 half .. +31) of a 16-bit passthrough block
// (TileQuant abstract: the highest-scoring tiles stay at 16 bits): the bf16
// weights times the bf16 activations, exact products, fp32 accumulation.  The
// mma's k order is the lane's quarter of the row: for k-step ks quad lane t
// holds columns 32t + 4ks .. +3, so each lane reads 64 contiguous bytes of a
// row and of the activation slice (the bf16 variant is x' in column order).
// mma rows: tile tt, row g = half row 16tt + g, row g + 8 = 16tt + g + 8;
// columns = tokens 0..7.  The sums go to the stage's fix-up area
// (fix[half row][token]); block_add16 hands them to the lanes that own the
// rows in the quantized path.  Kept out of line: 16-bit blocks are few, and
// the hot loop's code stays small.
__device__ __noinline__ void block_mma16(const uint8_t* stage, const uint8_t* xb, float* fix, int g, int t,
                                         uint32_t Mg) {
    uint32_t b[16];
    {
        const uint8_t* src = (uint32_t)g < Mg ? xb + g * XQD_VAR + 64 * t : nullptr;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 v = src ? reinterpret_cast<const uint4*>(src)[c] : make_uint4(0u, 0u, 0u, 0u);
            b[4 * c] = v.x; b[4 * c + 1] = v.y; b[4 * c + 2] = v.z; b[4 * c + 3] = v.w;
        }
    }
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
        uint32_t a0[16], a1[16];
        const uint8_t* r0 = stage + (16 * tt + g) * 256 + 64 * t;
        const uint8_t* r1 = r0 + 8 * 256;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 v0 = reinterpret_cast<const uint4*>(r0)[c];
            const uint4 v1 = reinterpret_cast<const uint4*>(r1)[c];
            a0[4 * c] = v0.x; a0[4 * c + 1] = v0.y; a0[4 * c + 2] = v0.z; a0[4 * c + 3] = v0.w;
            a1[4 * c] = v1.x; a1[4 * c + 1] = v1.y; a1[4 * c + 2] = v1.z; a1[4 * c + 3] = v1.w;
        }
        float c[4] = {0.f, 0.f, 0.f, 0.f}, d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 8; ks += 2) {
            mma_bf16_16816(c, a0[2 * ks], a1[2 * ks], a0[2 * ks + 1], a1[2 * ks + 1], b[2 * ks], b[2 * ks + 1]);
            mma_bf16_16816(d, a0[2 * ks + 2], a1[2 * ks + 2], a0[2 * ks + 3], a1[2 * ks + 3], b[2 * ks + 2],
                           b[2 * ks + 3]);
        }
        const int ra = 16 * tt + g, rb = ra + 8;
        const uint32_t t0 = 2u * t, t1 = 2u * t + 1u;
        if (t0 < Mg) { fix[ra * Mg + t0] = c[0] + d[0]; fix[rb * Mg + t0] = c[2] + d[2]; }
        if (t1 < Mg) { fix[ra * Mg + t1] = c[1] + d[1]; fix[rb * Mg + t1] = c[3] + d[3]; }
    }
    __syncwarp();
}

// The owners of the half's rows add the fix-up area's sums (rows 8g + 2i +
// (t & 1) lie in half `half` when g / 4 == half).
template <int G>
__device__ __forceinline__ void block_add16(const float* fix, int half, int g, int t, uint32_t Mg,
                                            float (&acc)[4][G]) {
    if ((g >> 2) != half) return;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int rl = 8 * g + 2 * i + (t & 1) - 32 * half;
#pragma unroll
        for (int grp = 0; grp < G; ++grp) {
            const uint32_t tok = 2u * grp + (uint32_t)(t >> 1);
            if (tok < Mg) acc[i][grp] += fix[rl * Mg + tok];
        }
    }
}

// Stage layout in the ring (all parts 16-byte multiples):
//   payload 1024*b | scales 128 | zeros 128 | activation variant of the low
//   piece, 272 bytes per token | (split widths) the high piece's variant
__host__ __device__ constexpr bool split_width(int b) { return hi_width(b) != 0; }
//   16-bit block: one half (32 rows x 256 bytes) | the bf16 activation
//   variant | a fix-up area of 32 rows x Mg fp32 (no scales or zeros)
__device__ __forceinline__ uint32_t stage_bytes(uint32_t b, uint32_t Mg) {
    if (b == 16) return 8192u + XQD_VAR * Mg + 128u * Mg;
    return 1024u * b + 256u + XQD_VAR * Mg * (split_width((int)b) ? 2u : 1u);
}

// Last arriver of a shared block row: y[m][rows[r]] = sum over the row's nc
// runs (in run order) of their partial sums.  The slots are contiguous
// ([nc][Mg tokens][64 rows] floats at `slots`); lanes read float4 vectors of
// them, sixteen slots per batch with every load of a batch in flight.  With one
// token a slot is 16 vectors, so two lane groups take the even and odd slots
// and are combined in that order (the sum stays deterministic).  Kept out of
// line: it runs once per shared row, and its registers must not weigh on the
// block loop.
__device__ __noinline__ void finish_shared_row(const float* __restrict__ slots, uint32_t Mg, uint32_t nc,
                                               float* __restrict__ y, int N, const int32_t* rows, int lane) {
    const float4* pv = reinterpret_cast<const float4*>(slots);
    const uint32_t V = Mg * 16u;
    const uint32_t groups = (V == 16u) ? 2u : 1u;
    const uint32_t grp = (V == 16u) ? (uint32_t)lane >> 4 : 0u;
    for (uint32_t v = (V == 16u) ? ((uint32_t)lane & 15u) : (uint32_t)lane; v < V; v += 32u) {
        float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
        for (uint32_t c0 = grp; c0 < nc; c0 += 16u * groups) {
            float4 q[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t c = c0 + (uint32_t)k * groups;
                q[k] = c < nc ? __ldcg(pv + (size_t)c * V + v) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                tot.x += q[k].x; tot.y += q[k].y; tot.z += q[k].z; tot.w += q[k].w;
            }
        }
        if (groups == 2u) {   // even slots' sum + odd slots' sum
            const int lo = (int)(v & 15u);
            float4 all;
            all.x = __shfl_sync(0xffffffffu, tot.x, lo) + __shfl_sync(0xffffffffu, tot.x, lo + 16);
            all.y = __shfl_sync(0xffffffffu, tot.y, lo) + __shfl_sync(0xffffffffu, tot.y, lo + 16);
            all.z = __shfl_sync(0xffffffffu, tot.z, lo) + __shfl_sync(0xffffffffu, tot.z, lo + 16);
            all.w = __shfl_sync(0xffffffffu, tot.w, lo) + __shfl_sync(0xffffffffu, tot.w, lo + 16);
            tot = all;
        }
        if (grp == 0u) {   // vector v: token v / 16, rows 4 (v % 16) .. +3
            const uint32_t r = 4u * (v & 15u);
            float* yr = y + (size_t)(v >> 4) * N;
            yr[rows[r]] = tot.x;
            yr[rows[r + 1]] = tot.y;
            yr[rows[r + 2]] = tot.z;
            yr[rows[r + 3]] = tot.w;
        }
    }
}

// ---------------------------------------------------------------------------
// Fused activation records (one token, no prologue kernel): the records that
// k_xprep_decode would write for block column kb, built by the warp in the
// stage -- the slice x[m][col_perm[128kb + c]], c = 0..127, turned into
// integers X with its power of two (xqd_integerize), then the digits of the
// low piece's variant and, for a split width, the high piece's, each
// followed by the digit sums and F -- the same arithmetic as k_xprep_decode.  cp holds the column indices 128kb + 4 lane .. +3 (after
// col_perm).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int4 fused_cols(const DecodeParams& p, uint32_t kb, int lane) {
    const int c0 = (int)kb * 128 + 4 * lane;
    if (!p.col_perm) return make_int4(c0, c0 + 1, c0 + 2, c0 + 3);
    return __ldg(reinterpret_cast<const int4*>(p.col_perm + c0));
}

template <bool W16>
__device__ __forceinline__ void fused_records(const DecodeParams& p, int4 cp, int b, uint8_t* rec, int lane) {
    const uint16_t* xr = p.x + (size_t)p.m0 * p.K;
    float v[4];
    v[0] = __uint_as_float((uint32_t)xr[cp.x] << 16);
    v[1] = __uint_as_float((uint32_t)xr[cp.y] << 16);
    v[2] = __uint_as_float((uint32_t)xr[cp.z] << 16);
    v[3] = __uint_as_float((uint32_t)xr[cp.w] << 16);
    if (W16 && b == 16) {   // the bf16 slice, column order
        *reinterpret_cast<uint2*>(rec + 8 * lane) =
            make_uint2((uint32_t)xr[cp.x] | ((uint32_t)xr[cp.y] << 16), (uint32_t)xr[cp.z] | ((uint32_t)xr[cp.w] << 16));
        fence_proxy_async_smem();
        __syncwarp();
        return;
    }
    int X[4], T[3];
    float F;
    xqd_integerize(v, X, T, F);
    xqd_scatter_variant(X, T, F, variant_of(lo_width(b)), rec, lane);
    if (split_width(b)) xqd_scatter_variant(X, T, F, variant_of(hi_width(b)), rec + XQD_VAR, lane);
    // generic writes into the ring, later overwritten by bulk copies
    fence_proxy_async_smem();
    __syncwarp();
}

// ---------------------------------------------------------------------------
// One warp's run u of the layer p (the body of the decode kernels below).
// G token groups of two: the launch's tokens Mg <= 2G.
// ---------------------------------------------------------------------------
template <int G, bool FUSED_X, bool W16>
__device__ __forceinline__ void decode_warp(const DecodeParams& p, DecWarp& W, int u, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const uint32_t KB = (uint32_t)p.KB;
    if (u >= p.n_units) return;

    // ---- the run descriptor: lane i holds word i ----
    const uint32_t dw = __ldg(p.desc + (size_t)u * DESC_WORDS + lane);
    const uint32_t t0 = __shfl_sync(0xffffffffu, dw, DW_T0);
    const uint32_t t1 = __shfl_sync(0xffffffffu, dw, DW_T1);
    const uint32_t s0 = __shfl_sync(0xffffffffu, dw, DW_S0);
    const uint32_t ns = __shfl_sync(0xffffffffu, dw, DW_NS);

    const uint32_t Mg = (uint32_t)p.Mg;
    // xq offsets fit 32 bits: KB * M * XQD_REC < 2^32 (the host checks it)
    const uint32_t rec_bytes = (uint32_t)p.M_total * XQD_REC;
    const uint32_t var_bytes = (uint32_t)p.M_total * XQD_VAR;
    const uint32_t x_tok_off = (uint32_t)p.m0 * XQD_VAR;
    const uint32_t x_bytes = XQD_VAR * Mg;     // one variant of the launch's tokens

    // ---- stage descriptors of the current chunk: lane l holds stage 32 chunk + l ----
    uint32_t chunk = 0;
    uint4 cs = make_uint4(0u, 0u, 0u, 0u);
    auto load_chunk = [&]() {
        const uint32_t j = 32u * chunk + (uint32_t)lane;
        if (j < ns) cs = __ldg(p.stages + s0 + j);
    };
    load_chunk();
    uint32_t next = 0;               // stages issued

    bool aborted = false;            // a bounded wait ran out: stop computing
    // variant of piece width p's activation record: 1, 2, 4, 8 -> 0, 1, 2, 3;
    // the low piece of width b is variant (0x302221100 >> 4b) & 15
    auto var_lo = [](uint32_t b) -> uint32_t {
        return b == 16 ? 4u : (uint32_t)(0x302221100ull >> (4 * b)) & 15u;
    };
    auto var_hi = [](uint32_t b) -> uint32_t { return (uint32_t)(0x001010000ull >> (4 * b)) & 15u; };
    auto issue_x = [&](uint8_t* dst, uint32_t b, uint32_t xo, uint64_t* bar) {
        bulk_g2s(dst, p.xq + xo, x_bytes, bar);
        // the high piece is narrower: its variant comes first in the record
        if (split_width((int)b))
            bulk_g2s(dst + x_bytes, p.xq + (xo - (var_lo(b) - var_hi(b)) * var_bytes), x_bytes, bar);
    };

    // ---- stage queue: entry k lives in lane k % DEC_SLOTS ----
    uint32_t q_head = 0, q_tail = 0;     // consumed / issued stages
    uint32_t r_head = 0, r_tail = 0;     // ring bytes issued / freed (monotone)
    uint32_t r_pos = 0;                  // physical ring offset of r_head
    uint32_t qe_nb = 0, qe_bits = 0, qe_off = 0, qe_end = 0, qe_x = 0, qe_kb = 0;
    bool xq_ready = false;               // x' is written by the prologue kernel
    auto issue_more = [&]() {
        while (q_tail - q_head < (uint32_t)DEC_SLOTS && next < ns && !aborted && !(kWaitTest && q_tail > 0)) {
            const int l = (int)(next & 31u);
            // the stage's size first: when the ring is full nothing else is needed
            const uint32_t kbb = __shfl_sync(0xffffffffu, cs.z, l);
            const uint32_t b = (kbb >> 16) & 0xFFu;
            if (!W16 && b == 16u) {   // a 16-bit block in a layer not flagged for them
                if (lane == 0) set_error(p.err, MPQ_ERR_BITS);
                next = ns;   // issue nothing more; the stages in flight are consumed as usual
                break;
            }
            const bool b16 = W16 && b == 16u;
            const uint32_t xb = split_width((int)b) ? 2u * x_bytes : x_bytes;
            const uint32_t pay = b16 ? 8192u : 1024u * b + 256u;   // payload (+ scales, zeros)
            const uint32_t size = pay + xb + (b16 ? 128u * Mg : 0u);   // stage_bytes(b, Mg)
            if (q_head == q_tail) { r_head = 0; r_tail = 0; r_pos = 0; }   // empty ring: restart at 0
            // a stage never wraps: when the ring's tail end is too short, skip to 0
            const bool skip = r_pos + size > (uint32_t)DEC_RING;
            const uint32_t start = skip ? r_head + ((uint32_t)DEC_RING - r_pos) : r_head;
            if (start + size - r_tail > (uint32_t)DEC_RING) break;   // ring full: compute first
            const uint32_t coff = __shfl_sync(0xffffffffu, cs.x, l);
            const uint32_t szo = __shfl_sync(0xffffffffu, cs.y, l);
            const uint32_t nbs = __shfl_sync(0xffffffffu, cs.w, l);
            const uint32_t hb = kbb >> 24;                 // 16-bit blocks: which row half
            const uint32_t xo = (kbb & 0xFFFFu) * rec_bytes + var_lo(b) * var_bytes + x_tok_off;
            const uint32_t slot = q_tail % DEC_SLOTS;
            const uint32_t off = skip ? 0u : r_pos;
            if (lane == 0) {
                // the fused path writes activation records into the ring
                if (FUSED_X) fence_proxy_async_smem();
                uint64_t* bar = &W.full[slot];
                mbar_arrive_expect_tx(bar, FUSED_X ? pay : pay + xb);
                uint8_t* dst = W.ring + off;
                if (!kWaitTest) {
                    if (b16) {
                        bulk_g2s(dst, p.codes + coff, 8192u, bar);
                    } else {
                        bulk_g2s(dst, p.codes + coff, 1024u * b, bar);
                        bulk_g2s(dst + 1024u * b, p.scales + szo, 128u, bar);
                        bulk_g2s(dst + 1024u * b + 128u, p.zeros + szo, 128u, bar);
                    }
                    if (!FUSED_X && xq_ready) issue_x(dst + pay, b, xo, bar);
                }
            }
            if (lane == (int)slot) {
                qe_nb = nbs; qe_bits = b | (hb << 8); qe_off = off; qe_end = start + size; qe_x = xo;
                if (FUSED_X) qe_kb = kbb & 0xFFFFu;
            }
            r_head = start + size;
            r_pos = off + size;
            ++q_tail;
            ++next;
            if ((next & 31u) == 0u) { ++chunk; load_chunk(); }
        }
    };

    // Weights do not depend on the prologue kernel: start streaming them, then
    // wait for x' (programmatic dependent launch) and add its copies.
    issue_more();
    // fused path: the column order of the first block's slice is static, so
    // it is read before waiting for the kernel that writes x
    int4 cp_pref = make_int4(0, 0, 0, 0);
    uint32_t cp_kb = 0xFFFFFFFFu;
    if (FUSED_X && q_head != q_tail) {
        cp_kb = __shfl_sync(0xffffffffu, cs.z, 0) & 0xFFFFu;   // the run's first non-zero block
        cp_pref = fused_cols(p, cp_kb, lane);
    }
    pdl_wait();
    xq_ready = true;
    if (!FUSED_X) {
        for (uint32_t k = q_head; k < q_tail; ++k) {
            const uint32_t slot = k % DEC_SLOTS;
            const uint32_t kbits = __shfl_sync(0xffffffffu, qe_bits, slot) & 0xFFu;
            const uint32_t ko = __shfl_sync(0xffffffffu, qe_off, slot);
            const uint32_t kx = __shfl_sync(0xffffffffu, qe_x, slot);
            const uint32_t kpay = (W16 && kbits == 16) ? 8192u : 1024u * kbits + 256u;
            if (lane == 0 && !kWaitTest) issue_x(W.ring + ko + kpay, kbits, kx, &W.full[slot]);
        }
    }

    const uint32_t nb_first = t0 / KB, nb_last = (t1 - 1) / KB;
    for (uint32_t nb = nb_first; nb <= nb_last; ++nb) {
        // output indices of the block row's 64 rows, kept in shared memory
        // (fetched early; read back when the row is written)
        __syncwarp();
        if (lane < 16) {
            const int i0 = (int)nb * 64 + 4 * lane;
            const int4 r4 = p.row_perm ? __ldg(reinterpret_cast<const int4*>(p.row_perm + i0))
                                       : make_int4(i0, i0 + 1, i0 + 2, i0 + 3);
            *reinterpret_cast<int4*>(&W.rows[4 * lane]) = r4;
        }
        float acc[4][G];      // rows 8g + 2i + (t & 1), token 2 grp + t / 2
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < G; ++c) acc[i][c] = 0.f;

        while (true) {
            issue_more();
            if (q_head == q_tail) break;    // nothing left for this warp at all
            const uint32_t slot = q_head % DEC_SLOTS;
            const uint32_t fnb = __shfl_sync(0xffffffffu, qe_nb, slot);
            if (fnb != nb) break;           // the next block is in a later row
            const uint32_t fbh = __shfl_sync(0xffffffffu, qe_bits, slot);
            const uint32_t fb = fbh & 0xFFu;
            const uint32_t foff = __shfl_sync(0xffffffffu, qe_off, slot);
            const uint32_t fend = __shfl_sync(0xffffffffu, qe_end, slot);
            if (!aborted) {
                const bool ok = mbar_wait_bounded(&W.full[slot], (q_head / DEC_SLOTS) & 1u, DEC_WAIT_NS);
                if (!__all_sync(0xffffffffu, ok)) {
                    aborted = true;
                    if (lane == 0) set_error(p.err, MPQ_ERR_TIMEOUT);
                }
            }
            if (!aborted) {
                const uint8_t* stage = W.ring + foff;
                uint8_t* xs = W.ring + foff + ((W16 && fb == 16) ? 8192u : 1024u * fb + 256u);
                if (FUSED_X) {
                    const uint32_t kb = __shfl_sync(0xffffffffu, qe_kb, slot);
                    const int4 cp = (kb == cp_kb) ? cp_pref : fused_cols(p, kb, lane);
                    fused_records<W16>(p, cp, (int)fb, xs, lane);
                }
                const uint8_t* xh = xs + x_bytes;
                const uint8_t* z32 = reinterpret_cast<const uint8_t*>(W.zero32);
                if (W16 && fb == 16) {
                    float* fix = reinterpret_cast<float*>(xs + x_bytes);
                    block_mma16(stage, xs, fix, g, t, Mg);
                    block_add16<G>(fix, (int)(fbh >> 8), g, t, Mg, acc);
                } else switch (fb) {
                    case 1: block_accumulate<1, G>(stage, xs, xh, z32, g, t, Mg, acc); break;
                    case 2: block_accumulate<2, G>(stage, xs, xh, z32, g, t, Mg, acc); break;
                    case 3: block_accumulate<3, G>(stage, xs, xh, z32, g, t, Mg, acc); break;
                    case 4: block_accumulate<4, G>(stage, xs, xh, z32, g, t, Mg, acc); break;
                    case 5: block_accumulate<5, G>(stage, xs, xh, z32, g, t, Mg, acc); break;
                    case 6: block_accumulate<6, G>(stage, xs, xh, z32, g, t, Mg, acc); break;
                    default: block_accumulate<8, G>(stage, xs, xh, z32, g, t, Mg, acc); break;
                }
            }
            __syncwarp();
            ++q_head;
            r_tail = fend;
        }

        // ---- end of block row nb ----
        uint32_t slot_base = 0, nc = 1, idx = 0;
        if (nb == nb_first) {
            slot_base = __shfl_sync(0xffffffffu, dw, DW_A_SLOT);
            nc = __shfl_sync(0xffffffffu, dw, DW_A_NC);
            idx = __shfl_sync(0xffffffffu, dw, DW_A_IDX);
        } else if (nb == nb_last) {
            slot_base = __shfl_sync(0xffffffffu, dw, DW_B_SLOT);
            nc = __shfl_sync(0xffffffffu, dw, DW_B_NC);
            idx = __shfl_sync(0xffffffffu, dw, DW_B_IDX);
        }
        // this lane's values: rows 8g + 2i + (t & 1) of token 2 grp + t / 2
        __syncwarp();
        const int row0 = 8 * g + (t & 1);
        if (nc == 1u) {
#pragma unroll
            for (int grp = 0; grp < G; ++grp) {
                const uint32_t tok = 2u * grp + (uint32_t)(t >> 1);
                if (tok < Mg) {
                    float* yr = p.y + (size_t)(p.m0 + tok) * p.N;
#pragma unroll
                    for (int i = 0; i < 4; ++i) yr[W.rows[row0 + 2 * i]] = acc[i][grp];
                }
            }
            continue;
        }
        // shared row: deposit this run's partial sums, then count the arrival
        {
            float* part = p.partial + (size_t)(slot_base + idx) * Mg * 64;
#pragma unroll
            for (int grp = 0; grp < G; ++grp) {
                const uint32_t tok = 2u * grp + (uint32_t)(t >> 1);
                if (tok < Mg) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) part[tok * 64 + row0 + 2 * i] = acc[i][grp];
                }
            }
        }
        // __syncwarp orders every lane's partial before lane 0's release; the
        // acquire side is lane 0's atomic + __syncwarp, then L2 (.cg) loads
        __syncwarp();
        uint32_t last = 0;
        if (lane == 0) last = (atomic_add_acq_rel_gpu(&p.counters[nb], 1u) + 1u == nc) ? 1u : 0u;
        last = __shfl_sync(0xffffffffu, last, 0);
        __syncwarp();
        if (!last) continue;
        finish_shared_row(p.partial + (size_t)slot_base * Mg * 64, Mg, nc, p.y + (size_t)p.m0 * p.N,
                          p.N, W.rows, lane);
        if (lane == 0) p.counters[nb] = 0u;   // ready for the next launch
    }
    // after a wait ran out, copies may still be landing in this warp's ring:
    // wait (bounded) for the last stage issued on each slot before leaving
    if (aborted && lane == 0)
        for (uint32_t k = q_tail > (uint32_t)DEC_SLOTS ? q_tail - DEC_SLOTS : 0u; k < q_tail; ++k)
            mbar_wait_bounded(&W.full[k % DEC_SLOTS], (k / DEC_SLOTS) & 1u, DEC_WAIT_NS);
}


// ---------------------------------------------------------------------------
// The kernels.  G: token groups of four (Mg <= 4G).  FUSED_X (one token): no
// prologue kernel; each block's activation records are built by the warp
// from x (fused_records).  Every warp works alone (no CTA-wide barrier): warp
// u of the grid takes run u.
// ---------------------------------------------------------------------------
__device__ __forceinline__ DecWarp& decode_prologue(uint8_t* smem_raw, int warp, int lane) {
    DecSmem& S = *reinterpret_cast<DecSmem*>(smem_raw);
    DecWarp& W = S.w[warp];
    // the next kernel in the stream may launch now: it waits (griddepcontrol)
    // for this grid before it touches memory this kernel uses
    pdl_launch_dependents();
    if (lane == 0) {
        for (int s = 0; s < DEC_SLOTS; ++s) mbar_init(&W.full[s], 1);
        fence_mbar_init();
    }
    if (lane < 2) W.zero32[lane] = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
    return W;
}

// Registers: at most 112 for one token group (four CTAs per SM then leave
// room in the register file for the next launch's prologue CTAs to become
// resident early); more token groups hold more accumulators and fragments
// (three CTAs per SM).
template <int G>
struct DecRegs { static constexpr int value = G == 1 ? DEC_MAX_REGS : 168; };

// W16: built with the 16-bit passthrough path (for layers flagged to have
// 16-bit blocks; the others take the smaller code).
template <int G, bool FUSED_X = false, bool W16 = false>
__global__ void __maxnreg__(DecRegs<G>::value) k_decode(DecodeParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    DecWarp& W = decode_prologue(smem_raw, warp, lane);
    decode_warp<G, FUSED_X, W16>(p, W, (int)blockIdx.x * DEC_WARPS + warp, lane);
}

// Several layers that share x in one launch (one token, fused activation
// records): the runs of layer l are warps unit_begin[l] .. unit_begin[l+1]-1.
constexpr int DEC_GROUP_MAX = 8;
struct DecodeGroup {
    DecodeParams layer[DEC_GROUP_MAX];
    int unit_begin[DEC_GROUP_MAX + 1];
    int n;
};

template <bool W16 = false>
__global__ void __maxnreg__(DEC_MAX_REGS) k_decode_group(const __grid_constant__ DecodeGroup gp) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    DecWarp& W = decode_prologue(smem_raw, warp, lane);
    const int v = (int)blockIdx.x * DEC_WARPS + warp;
    if (v >= gp.unit_begin[gp.n]) return;
    int l = 0;
    while (l + 1 < gp.n && v >= gp.unit_begin[l + 1]) ++l;
    decode_warp<1, true, W16>(gp.layer[l], W, v - gp.unit_begin[l], lane);
}

}  // namespace mpq
