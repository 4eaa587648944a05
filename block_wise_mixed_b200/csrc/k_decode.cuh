// k_decode.cuh -- memory-bound mixed-precision GEMV/GEMM for small M.
//
// y'[m][i] = sum_kb s[i,kb] * sum_{j in kb} x'[m][j] * (q[i][j] - z[i,kb])
// (the blocks' RTN dequantization, ScaleBITS summary "Approach" / "Key
// results"; 0-bit blocks are skipped -- they hold no bytes), then
// y[m][row_perm[i]] = y'[m][i].
//
// Work split.  At pack time the blocks are cut into `n_units` row-major runs
// of about equal estimated cost (bytes moved plus decode work per bit
// width); each run is one warp's work.  A unit descriptor of 128 bytes holds
// everything the warp needs to start: its run [t0, t1), the offsets of its
// first block of every width in the code segments and in the scale/zero
// arrays, the bit widths of its first 64 blocks, and where the partial sums
// of its first and last block rows go.  One coalesced load of it is the only
// dependent fetch before the first payload copy is issued.
//
// Each warp streams its non-zero blocks through a private ring of shared
// memory with 1-D bulk async copies (payload + 64 scales + 64 zeros + the
// activation slice in the column order of the block's low piece + F),
// several blocks ahead of the one it computes.  Codes become exact fp16
// subnormal pairs (q - z) * 2^-24 in registers (an AND or byte permute and
// one HFMA2 per pair; the high piece of a split code is added in before the
// multiply) and are multiplied on the tensor cores (mma.m16n8k16, fp32
// accumulation).  Per block and output row: acc += s * F * c.  Forming
// q - z per element keeps every product exact, so the fp32 rounding stays
// relative to sum |x * w_hat| even when most codes equal the zero point.
//
// A block row that lies inside one run is written straight to y.  A block
// row shared by several runs (the first and last row of a run) is finished
// by the last warp to arrive (a per-row arrival counter): it adds the
// contributors' partial sums -- a contiguous range of slots -- in run order,
// so results are deterministic.
//
// Every wait is bounded: after ~2 s it records MPQ_ERR_TIMEOUT and the warp
// stops computing (its arithmetic is skipped, its bookkeeping still runs).
#pragma once
#include "common.cuh"
#include "k_xprep.cuh"   // XQD_*

namespace mpq {

constexpr uint64_t DEC_WAIT_NS = 2000000000ull;

// Unit descriptor: 32 words.
enum DescWord {
    DW_T0 = 0, DW_T1 = 1, DW_SZ = 2,
    DW_CODE = 3,           // 3..9: code offset of the run's first block of width 1,2,3,4,5,6,8
    DW_A_SLOT = 10,        // first block row of the run: first partial slot of the row,
    DW_A_NC = 11,          //   number of runs that meet the row, this run's index among them
    DW_A_IDX = 12,
    DW_B_SLOT = 13,        // last block row of the run: the same three
    DW_B_NC = 14,
    DW_B_IDX = 15,
    DW_BITS = 16,          // 16..31: bit widths of the run's first 64 blocks (bytes)
    DESC_WORDS = 32
};
constexpr int DESC_INLINE_BITS = 64;

struct DecodeParams {
    const uint8_t* codes;
    const uint32_t* desc;     // [n_units][32]
    const uint8_t* bits8;     // [NB*KB] bit width per block (runs longer than 64 blocks)
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
constexpr int DEC_RING = 12288;      // bytes of ring per warp (>= largest stage)
constexpr int DEC_SLOTS = 8;         // stages in flight per warp
constexpr int DEC_MAX_TOKENS = 8;

struct DecWarp {
    uint8_t ring[DEC_RING];
    int32_t rows[64];         // output index of each row of the current block row
    __half xw[128];           // fused path: the block's x' slice, column order
    uint64_t full[DEC_SLOTS];
    uint4 zero16[4];          // zero B fragments for lanes beyond the token count
};
struct DecSmem {
    DecWarp w[DEC_WARPS];
};

// DEC_CTAS_PER_SM x (smem + 1 KB reserved) must fit the SM's 228 KB
static_assert(DEC_CTAS_PER_SM * (sizeof(DecSmem) + 1024) <= 228 * 1024, "decode smem too large");
// largest stage: an 8-bit payload
static_assert(DEC_RING >= 8 * 1024 + 256 + DEC_MAX_TOKENS * XQD_VAR, "ring too small");

__host__ __device__ constexpr int lo_width(int b) { return (b == 3) ? 2 : (b == 5 || b == 6) ? 4 : b; }
__host__ __device__ constexpr int hi_width(int b) { return (b == 3 || b == 5) ? 1 : (b == 6) ? 2 : 0; }
__host__ __device__ constexpr int variant_of(int p) { return p == 1 ? 0 : p == 2 ? 1 : p == 4 ? 2 : 3; }
// index of width b in the descriptor's code offsets (1,2,3,4,5,6,8 -> 0..6)
__host__ __device__ constexpr int width_index(int b) { return b == 8 ? 6 : b - 1; }

// ---------------------------------------------------------------------------
// Code extraction.  For one row and the lane's 32 columns, a[pi] becomes the
// fp16 pair ((q_a - z) * 2^-24, (q_b - z) * 2^-24) of pair pi (column order
// of k_xprep.cuh) -- exact subnormals.  An AND (or byte permute) leaves a
// code at bit `pos` of each half, i.e. the value q * 2^(pos-24); one HFMA2
// with 2^-pos and zc = -z * 2^-24 gives (q - z) * 2^-24.  A split code adds
// its high piece the same way, times 2^(low width), before the mma.
// ---------------------------------------------------------------------------
__device__ __forceinline__ constexpr uint32_t h2pow(int k) {      // (2^k, 2^k) fp16 bits
    return (uint32_t)((15 + k) << 10) * 0x10001u;
}
__device__ __forceinline__ uint32_t hadd2_bits(uint32_t a, uint32_t b) {
    return h2_bits(__hadd2(bits_h2(a), bits_h2(b)));
}

template <int P>
__device__ __forceinline__ void extract_lo(const uint32_t (&w)[P], uint32_t zc, uint32_t (&a)[16]) {
    if (P == 1) {
        const uint32_t u = w[0], v = w[0] >> 8;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            a[s] = hfma2_bits(u & (0x00010001u << s), h2pow(-s), zc);
            a[8 + s] = hfma2_bits(v & (0x00010001u << s), h2pow(-s), zc);
        }
    } else if (P == 2) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t u = w[i], v = w[i] >> 8;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                a[8 * i + s] = hfma2_bits(u & (0x00030003u << (2 * s)), h2pow(-2 * s), zc);
                a[8 * i + 4 + s] = hfma2_bits(v & (0x00030003u << (2 * s)), h2pow(-2 * s), zc);
            }
        }
    } else if (P == 4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t u = w[i], v = w[i] >> 8;
            a[4 * i + 0] = hadd2_bits(u & 0x000F000Fu, zc);
            a[4 * i + 1] = hfma2_bits(u & 0x00F000F0u, h2pow(-4), zc);
            a[4 * i + 2] = hadd2_bits(v & 0x000F000Fu, zc);
            a[4 * i + 3] = hfma2_bits(v & 0x00F000F0u, h2pow(-4), zc);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            a[2 * i + 0] = hadd2_bits(__byte_perm(w[i], 0u, 0x4240), zc);
            a[2 * i + 1] = hadd2_bits(__byte_perm(w[i], 0u, 0x4341), zc);
        }
    }
}

// High piece of a split code added onto the low pairs: a[pi] += 2^w * hi.
// B = 3: low 2-bit, high 1-bit (w = 2); B = 5: 4 + 1 (w = 4); B = 6: 4 + 2.
template <int B>
__device__ __forceinline__ void add_hi(const uint32_t (&h)[B == 6 ? 2 : 1], uint32_t (&a)[16]) {
    if (B == 3) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            // bytes 2i, 2i+1 hold the high bits of columns 16i..16i+7, 16i+8..16i+15
            const uint32_t pb = __byte_perm(h[0], 0u, (2 * i) | (4 << 4) | ((2 * i + 1) << 8) | (4 << 12));
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                a[8 * i + s] = hfma2_bits(pb & (0x00010001u << s), h2pow(2 - s), a[8 * i + s]);
                a[8 * i + 4 + s] = hfma2_bits(pb & (0x00010001u << (4 + s)), h2pow(-2 - s), a[8 * i + 4 + s]);
            }
        }
    } else if (B == 5) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // byte i holds the high bits of columns 8i..8i+7, in both halves
            const uint32_t pb = __byte_perm(h[0], 0u, i | (4 << 4) | (i << 8) | (4 << 12));
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                // column 8i+r at bit r (low half), 8i+r+4 at bit r+4 (high half)
                const uint32_t m = (uint32_t)((15 + 4 - r) << 10) | ((uint32_t)((15 - r) << 10) << 16);
                a[4 * i + r] = hfma2_bits(pb & ((1u << r) | (1u << (20 + r))), m, a[4 * i + r]);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int b0 = 2 * (i & 1);
            const uint32_t pb = __byte_perm(h[i >> 1], 0u, b0 | (4 << 4) | ((b0 + 1) << 8) | (4 << 12));
#pragma unroll
            for (int r = 0; r < 4; ++r)
                a[4 * i + r] = hfma2_bits(pb & (0x00030003u << (2 * r)), h2pow(4 - 2 * r), a[4 * i + r]);
        }
    }
}

template <int P>
__device__ __forceinline__ void load_words(const uint8_t* p, uint32_t (&w)[P]) {
    if (P == 1) {
        w[0] = *reinterpret_cast<const uint32_t*>(p);
    } else if (P == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        w[0] = v.x; w[1] = v.y;
    } else if (P == 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
        const uint4 v0 = reinterpret_cast<const uint4*>(p)[0];
        const uint4 v1 = reinterpret_cast<const uint4*>(p)[1];
        w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
        w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    }
}

// One row's 16 pairs for width B (stage = payload; lane offset t).
template <int B>
__device__ __forceinline__ void row_pairs(const uint8_t* stage, int r, int t, uint32_t zc,
                                          uint32_t (&a)[16]) {
    constexpr int P0 = lo_width(B), P1 = hi_width(B);
    uint32_t w[P0];
    load_words<P0>(stage + r * 16 * P0 + t * 4 * P0, w);
    extract_lo<P0>(w, zc, a);
    if (P1) {
        uint32_t h[B == 6 ? 2 : 1];
        const uint8_t* hp = stage + 64 * 16 * P0 + r * 16 * P1 + t * 4 * P1;
        if (B == 6) {
            const uint2 v = *reinterpret_cast<const uint2*>(hp);
            h[0] = v.x; h[B == 6 ? 1 : 0] = v.y;
        } else {
            h[0] = *reinterpret_cast<const uint32_t*>(hp);
        }
        add_hi<B>(h, a);
    }
}

// One 16-row tile rt of a block of width B, added into acc:
//   c = 2^-24 * sum over the block's 128 columns of (q - z) * x'
//   acc[rt][*] += s_row * F_tok * c        (C-fragment order: rows 16rt+g,
//   16rt+g+8 x tokens 2t, 2t+1).
// The caller loops over rt at run time, so each width's code is one tile's
// worth (small enough to stay in the instruction cache); the tile's eight
// k-steps alternate between two accumulators to halve the mma chain.
template <int B, bool ONE_TOKEN>
__device__ __forceinline__ void tile_accumulate(const uint8_t* stage, const uint32_t (&b)[16], int rt,
                                                int g, int t, float Fa, float Fb, float (&acc)[4][4]) {
    const uint16_t* sc16 = reinterpret_cast<const uint16_t*>(stage + 1024 * B);
    const int r0 = 16 * rt + g, r1 = r0 + 8;
    // -z * 2^-24 in both halves (z is an fp16 integer; 0x8001 = -2^-24)
    const uint32_t zc0 = h2_bits(__hmul2(bits_h2(__byte_perm((uint32_t)sc16[64 + r0], 0u, 0x1010)),
                                         bits_h2(0x80018001u)));
    const uint32_t zc1 = h2_bits(__hmul2(bits_h2(__byte_perm((uint32_t)sc16[64 + r1], 0u, 0x1010)),
                                         bits_h2(0x80018001u)));
    uint32_t a0[16], a1[16];
    row_pairs<B>(stage, r0, t, zc0, a0);
    row_pairs<B>(stage, r1, t, zc1, a1);
    float c[4] = {0.f, 0.f, 0.f, 0.f}, d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ks += 2) {
        mma_16816(c, a0[2 * ks], a1[2 * ks], a0[2 * ks + 1], a1[2 * ks + 1], b[2 * ks], b[2 * ks + 1]);
        mma_16816(d, a0[2 * ks + 2], a1[2 * ks + 2], a0[2 * ks + 3], a1[2 * ks + 3], b[2 * ks + 2],
                  b[2 * ks + 3]);
    }
    const float s0 = __half2float(__ushort_as_half(sc16[r0]));
    const float s1 = __half2float(__ushort_as_half(sc16[r1]));
    const float v0 = s0 * (Fa * (c[0] + d[0]));
    const float v2 = s1 * (Fa * (c[2] + d[2]));
    const float v1 = ONE_TOKEN ? 0.f : s0 * (Fb * (c[1] + d[1]));
    const float v3 = ONE_TOKEN ? 0.f : s1 * (Fb * (c[3] + d[3]));
#pragma unroll
    for (int k = 0; k < 4; ++k) {   // acc[rt] without run-time register indexing
        if (k == rt) {
            acc[k][0] += v0;
            acc[k][2] += v2;
            if (!ONE_TOKEN) { acc[k][1] += v1; acc[k][3] += v3; }
        }
    }
}

template <int B, bool ONE_TOKEN>
__device__ __forceinline__ void block_accumulate(const uint8_t* stage, const uint32_t (&b)[16], int g,
                                                 int t, float Fa, float Fb, float (&acc)[4][4]) {
#pragma unroll 1
    for (int rt = 0; rt < 4; ++rt) tile_accumulate<B, ONE_TOKEN>(stage, b, rt, g, t, Fa, Fb, acc);
}

__device__ __forceinline__ void load_bfrag(const uint8_t* src, uint32_t (&b)[16]) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 v = s4[i];
        b[4 * i] = v.x; b[4 * i + 1] = v.y; b[4 * i + 2] = v.z; b[4 * i + 3] = v.w;
    }
}

// Stage layout in the ring (all parts 16-byte multiples):
//   payload 1024*b | scales 128 | zeros 128 | x' variant of the low piece,
//   272 bytes per token (fragments, then F)
__device__ __forceinline__ uint32_t stage_bytes(uint32_t b, uint32_t Mg) {
    return 1024u * b + 256u + XQD_VAR * Mg;
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
// Fused activation record (one token, no prologue kernel): the record that
// k_xprep_decode would write for block column kb and piece-width variant vv,
// built by the warp into `rec` (shared memory, XQD_VAR bytes): the slice
// x[m][col_perm[128kb + c]], c = 0..127, scaled by its power of two 2^e and
// converted to fp16, paired in the variant's column order, then
// F = 2^(24 - e) -- the same arithmetic as k_xprep_decode.  cp holds the
// column indices 128kb + 4 lane .. +3 (after col_perm).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int4 fused_cols(const DecodeParams& p, uint32_t kb, int lane) {
    const int c0 = (int)kb * 128 + 4 * lane;
    if (!p.col_perm) return make_int4(c0, c0 + 1, c0 + 2, c0 + 3);
    return __ldg(reinterpret_cast<const int4*>(p.col_perm + c0));
}

__device__ __forceinline__ void fused_record(const DecodeParams& p, int4 cp, int vv, uint8_t* rec,
                                             __half* xw, int lane) {
    const uint16_t* xr = p.x + (size_t)p.m0 * p.K;
    float v[4];
    v[0] = __uint_as_float((uint32_t)xr[cp.x] << 16);
    v[1] = __uint_as_float((uint32_t)xr[cp.y] << 16);
    v[2] = __uint_as_float((uint32_t)xr[cp.z] << 16);
    v[3] = __uint_as_float((uint32_t)xr[cp.w] << 16);
    float amax = 0.f;
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
        const float a = fabsf(v[e4]);
        amax = (a > amax || a != a) ? a : amax;   // NaN-propagating max
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, amax, off);
        amax = (o > amax || o != o) ? o : amax;
    }
    int e = 0;
    if (amax > 0.f && isfinite(amax)) e = min(max(14 - ilogbf(amax), -103), 126);
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) xw[4 * lane + e4] = __float2half_rn(ldexpf(v[e4], e));
    __syncwarp();
    // lane -> quad lane tq = lane / 8, pairs 2 (lane % 8), +1
    const int tq = lane >> 3, pi0 = 2 * (lane & 7);
    uint32_t o[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        int ca, cb;
        xqd_pair_cols(vv, pi0 + i, ca, cb);
        o[i] = h2_bits(__halves2half2(xw[32 * tq + ca], xw[32 * tq + cb]));
    }
    *reinterpret_cast<uint2*>(rec + tq * 64 + pi0 * 4) = make_uint2(o[0], o[1]);
    if (lane == 0) *reinterpret_cast<float*>(rec + 256) = ldexpf(1.f, 24 - e);
    // generic writes into the ring, later overwritten by bulk copies
    fence_proxy_async_smem();
    __syncwarp();
}

// ---------------------------------------------------------------------------
// One warp's run u of the layer p (the body of the decode kernels below).
// ---------------------------------------------------------------------------
template <bool ONE_TOKEN, bool FUSED_X>
__device__ __forceinline__ void decode_warp(const DecodeParams& p, DecWarp& W, int u, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const uint32_t KB = (uint32_t)p.KB;
    const uint32_t lt_mask = (1u << lane) - 1u;
    if (u >= p.n_units) return;

    // ---- the unit descriptor: lane i holds word i ----
    const uint32_t dw = __ldg(p.desc + (size_t)u * DESC_WORDS + lane);
    const uint32_t t0 = __shfl_sync(0xffffffffu, dw, DW_T0);
    const uint32_t t1 = __shfl_sync(0xffffffffu, dw, DW_T1);
    uint32_t sz_base = __shfl_sync(0xffffffffu, dw, DW_SZ);
    // lanes DW_CODE..DW_CODE+6 keep the running code offset of their width
    uint32_t code_run = dw;


    const uint32_t Mg = (uint32_t)p.Mg;
    // xq offsets fit 32 bits: KB * M * XQD_REC < 2^32 (the host checks it)
    const uint32_t rec_bytes = (uint32_t)p.M_total * XQD_REC;
    const uint32_t var_bytes = (uint32_t)p.M_total * XQD_VAR;
    const uint32_t x_tok_off = (uint32_t)p.m0 * XQD_VAR;
    const uint32_t x_bytes = XQD_VAR * Mg;

    // ---- chunk state: lane l describes block t0 + 32*chunk + l ----
    uint32_t chunk = 0;
    uint32_t c_bits = 0, c_code = 0, c_sz = 0, c_x = 0;
    uint32_t pending = 0;            // non-zero blocks of the chunk not yet issued
    bool scan_done = false;
    uint32_t bits_pref = 0;          // prefetched widths of the next chunk (beyond the inline 64)

    bool aborted = false;            // a bounded wait ran out: stop computing
    auto load_chunk = [&]() {
        const uint32_t j = 32u * chunk + (uint32_t)lane;
        const bool in = t0 + j < t1;
        // widths of the first 64 blocks are inline in the descriptor
        const uint32_t jw = min(j, (uint32_t)DESC_INLINE_BITS - 1u);
        const uint32_t word = __shfl_sync(0xffffffffu, dw, DW_BITS + (int)(jw >> 2));
        uint32_t b = (j < (uint32_t)DESC_INLINE_BITS) ? (word >> (8 * (j & 3))) & 0xFFu : bits_pref;
        b = in ? b : 0u;
        // prefetch the next chunk's widths when they are not inline
        const uint32_t jn = j + 32u;
        if (jn >= (uint32_t)DESC_INLINE_BITS && t0 + jn < t1) bits_pref = __ldg(p.bits8 + t0 + jn);
        c_bits = b;
        // this block's activation variant for the launch's tokens, as a byte
        // offset into xq (one division per chunk instead of one per stage)
        c_x = ((t0 + j) % KB) * rec_bytes + (uint32_t)variant_of(lo_width(b == 0 ? 1 : (int)b)) * var_bytes +
              x_tok_off;
        // rank among the chunk's blocks of the same width -> code offset
        const uint32_t same = __match_any_sync(0xffffffffu, b);
        const uint32_t rank = __popc(same & lt_mask);
        const uint32_t base = __shfl_sync(0xffffffffu, code_run, DW_CODE + width_index(b == 0 ? 1 : (int)b));
        c_code = base + rank * 1024u * b;
        const uint32_t nz = __ballot_sync(0xffffffffu, b != 0u);
        c_sz = sz_base + 64u * __popc(nz & lt_mask);
        sz_base += 64u * __popc(nz);
        pending = nz;
    };
    // advance the running code offsets past the chunk (lane DW_CODE + i owns width i)
    auto advance_codes = [&]() {
        uint32_t add = 0;
#pragma unroll
        for (int i = 0; i < 7; ++i) {
            const uint32_t wb = (i == 6) ? 8u : (uint32_t)(i + 1);
            const uint32_t cnt = __popc(__ballot_sync(0xffffffffu, c_bits == wb));
            if (lane == DW_CODE + i) add = cnt * 1024u * wb;
        }
        code_run += add;
    };

    load_chunk();
    advance_codes();

    // ---- stage queue: entry k lives in lane k % DEC_SLOTS ----
    uint32_t q_head = 0, q_tail = 0;     // consumed / issued stages
    uint32_t r_head = 0, r_tail = 0;     // ring bytes issued / freed (monotone)
    uint32_t r_pos = 0;                  // physical ring offset of r_head
    uint32_t qe_t = 0, qe_bits = 0, qe_off = 0, qe_end = 0, qe_x = 0;
    bool xq_ready = false;               // x' is written by the prologue kernel
    auto issue_more = [&]() {
        while (q_tail - q_head < (uint32_t)DEC_SLOTS && !scan_done) {
            if (aborted) { scan_done = true; break; }
            if (pending == 0u) {
                if (t0 + 32u * (chunk + 1) >= t1) { scan_done = true; break; }
                ++chunk;
                load_chunk();
                advance_codes();
                continue;
            }
            if (q_head == q_tail) { r_head = 0; r_tail = 0; r_pos = 0; }   // empty ring: restart at 0
            const int l = __ffs(pending) - 1;
            const uint32_t b = __shfl_sync(0xffffffffu, c_bits, l);
            const uint32_t coff = __shfl_sync(0xffffffffu, c_code, l);
            const uint32_t szo = __shfl_sync(0xffffffffu, c_sz, l);
            const uint32_t xo = __shfl_sync(0xffffffffu, c_x, l);
            const uint32_t size = 1024u * b + 256u + x_bytes;   // stage_bytes(b, Mg)
            // a stage never wraps: when the ring's tail end is too short, skip to 0
            const bool skip = r_pos + size > (uint32_t)DEC_RING;
            const uint32_t start = skip ? r_head + ((uint32_t)DEC_RING - r_pos) : r_head;
            if (start + size - r_tail > (uint32_t)DEC_RING) break;   // ring full: compute first
            const uint32_t tt = t0 + 32u * chunk + (uint32_t)l;
            const uint32_t slot = q_tail % DEC_SLOTS;
            const uint32_t off = skip ? 0u : r_pos;
            if (lane == 0) {
                fence_proxy_async_smem();
                uint64_t* bar = &W.full[slot];
                // the fused path builds the activation record itself
                mbar_arrive_expect_tx(bar, FUSED_X ? size - x_bytes : size);
                uint8_t* dst = W.ring + off;
                bulk_g2s(dst, p.codes + coff, 1024u * b, bar);
                bulk_g2s(dst + 1024u * b, p.scales + szo, 128u, bar);
                bulk_g2s(dst + 1024u * b + 128u, p.zeros + szo, 128u, bar);
                if (!FUSED_X && xq_ready) bulk_g2s(dst + 1024u * b + 256u, p.xq + xo, x_bytes, bar);
            }
            if (lane == (int)slot) { qe_t = tt; qe_bits = b; qe_off = off; qe_end = start + size; qe_x = xo; }
            r_head = start + size;
            r_pos = off + size;
            ++q_tail;
            pending &= pending - 1u;
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
        cp_kb = __shfl_sync(0xffffffffu, qe_t, q_head % DEC_SLOTS) % KB;
        cp_pref = fused_cols(p, cp_kb, lane);
    }
    pdl_wait();
    xq_ready = true;
    if (!FUSED_X) {
        for (uint32_t k = q_head; k < q_tail; ++k) {
            const uint32_t slot = k % DEC_SLOTS;
            const uint32_t kbits = __shfl_sync(0xffffffffu, qe_bits, slot);
            const uint32_t ko = __shfl_sync(0xffffffffu, qe_off, slot);
            const uint32_t kx = __shfl_sync(0xffffffffu, qe_x, slot);
            if (lane == 0) bulk_g2s(W.ring + ko + 1024u * kbits + 256u, p.xq + kx, x_bytes, &W.full[slot]);
        }
    }

    const uint32_t nb_first = t0 / KB, nb_last = (t1 - 1) / KB;
    for (uint32_t nb = nb_first; nb <= nb_last; ++nb) {
        const uint32_t row_end = min(t1, (nb + 1) * KB);
        // output rows of this lane: 16rt+g (+8); their permuted indices, early
        int rp[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int i = (int)nb * 64 + 8 * q + g;   // q = 2rt + h -> row 16rt + 8h + g
            rp[q] = p.row_perm ? __ldg(p.row_perm + i) : i;
        }
        float acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;

        while (true) {
            issue_more();
            if (q_head == q_tail) break;    // nothing left for this warp at all
            const uint32_t slot = q_head % DEC_SLOTS;
            const uint32_t ft = __shfl_sync(0xffffffffu, qe_t, slot);
            if (ft >= row_end) break;       // the next block is in a later row
            const uint32_t fb = __shfl_sync(0xffffffffu, qe_bits, slot);
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
                const uint8_t* xs = stage + 1024u * fb + 256u;
                if (FUSED_X) {
                    const uint32_t kb = ft % KB;
                    const int4 cp = (kb == cp_kb) ? cp_pref : fused_cols(p, kb, lane);
                    fused_record(p, cp, variant_of(lo_width((int)fb)), W.ring + foff + 1024u * fb + 256u,
                                 W.xw, lane);
                }
                // this lane's B fragments: token g, quad lane t; zeros beyond Mg
                uint32_t bf[16];
                load_bfrag((uint32_t)g < Mg ? xs + g * XQD_VAR + t * 64
                                            : reinterpret_cast<const uint8_t*>(W.zero16), bf);
                const float Fa = (2u * t < Mg) ? *reinterpret_cast<const float*>(xs + (2 * t) * XQD_VAR + 256) : 0.f;
                const float Fb = (!ONE_TOKEN && 2u * t + 1u < Mg)
                                     ? *reinterpret_cast<const float*>(xs + (2 * t + 1) * XQD_VAR + 256) : 0.f;
                switch (fb) {
                    case 1: block_accumulate<1, ONE_TOKEN>(stage, bf, g, t, Fa, Fb, acc); break;
                    case 2: block_accumulate<2, ONE_TOKEN>(stage, bf, g, t, Fa, Fb, acc); break;
                    case 3: block_accumulate<3, ONE_TOKEN>(stage, bf, g, t, Fa, Fb, acc); break;
                    case 4: block_accumulate<4, ONE_TOKEN>(stage, bf, g, t, Fa, Fb, acc); break;
                    case 5: block_accumulate<5, ONE_TOKEN>(stage, bf, g, t, Fa, Fb, acc); break;
                    case 6: block_accumulate<6, ONE_TOKEN>(stage, bf, g, t, Fa, Fb, acc); break;
                    default: block_accumulate<8, ONE_TOKEN>(stage, bf, g, t, Fa, Fb, acc); break;
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
        // tokens 2t, 2t+1 of rows 16rt+g, 16rt+g+8
        const int tok_a = 2 * t, tok_b = 2 * t + 1;
        const bool wa = (uint32_t)tok_a < Mg, wb = !ONE_TOKEN && (uint32_t)tok_b < Mg;
        if (nc == 1u) {
#pragma unroll
            for (int rt = 0; rt < 4; ++rt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int n = rp[2 * rt + h];
                    if (wa) p.y[(size_t)(p.m0 + tok_a) * p.N + n] = acc[rt][2 * h];
                    if (wb) p.y[(size_t)(p.m0 + tok_b) * p.N + n] = acc[rt][2 * h + 1];
                }
            continue;
        }
        // shared row: deposit this run's partial sums, then count the arrival
        {
            float* part = p.partial + (size_t)(slot_base + idx) * Mg * 64;
#pragma unroll
            for (int rt = 0; rt < 4; ++rt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = 16 * rt + 8 * h + g;
                    if (wa) part[tok_a * 64 + r] = acc[rt][2 * h];
                    if (wb) part[tok_b * 64 + r] = acc[rt][2 * h + 1];
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
        if (t == 0) {   // the row's output indices, for the lanes that write y below
#pragma unroll
            for (int q = 0; q < 8; ++q) W.rows[8 * q + g] = rp[q];
        }
        __syncwarp();
        finish_shared_row(p.partial + (size_t)slot_base * Mg * 64, Mg, nc, p.y + (size_t)p.m0 * p.N,
                          p.N, W.rows, lane);
        if (lane == 0) p.counters[nb] = 0u;   // ready for the next launch
    }
}


// ---------------------------------------------------------------------------
// The kernels.  ONE_TOKEN: the launch has Mg == 1 (only C-fragment column 0
// carries data, so the per-block epilogue handles half the elements).
// FUSED_X (with ONE_TOKEN): no prologue kernel; each block's activation
// record is built by the warp from x (fused_record).  Every warp works
// alone (no CTA-wide barrier): warp u of the grid takes run u.
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
    if (lane < 4) W.zero16[lane] = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
    return W;
}

template <bool ONE_TOKEN, bool FUSED_X = false>
// At most 112 registers: four CTAs then leave room in the register file for
// the next launch's activation-prologue CTAs to become resident early.
__global__ void __maxnreg__(DEC_MAX_REGS) k_decode(DecodeParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    DecWarp& W = decode_prologue(smem_raw, warp, lane);
    decode_warp<ONE_TOKEN, FUSED_X>(p, W, (int)blockIdx.x * DEC_WARPS + warp, lane);
}

// Several layers that share x in one launch (one token, fused activation
// records): the runs of layer l are warps unit_begin[l] .. unit_begin[l+1]-1.
constexpr int DEC_GROUP_MAX = 8;
struct DecodeGroup {
    DecodeParams layer[DEC_GROUP_MAX];
    int unit_begin[DEC_GROUP_MAX + 1];
    int n;
};

__global__ void __maxnreg__(DEC_MAX_REGS) k_decode_group(const __grid_constant__ DecodeGroup gp) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    DecWarp& W = decode_prologue(smem_raw, warp, lane);
    const int v = (int)blockIdx.x * DEC_WARPS + warp;
    if (v >= gp.unit_begin[gp.n]) return;
    int l = 0;
    while (l + 1 < gp.n && v >= gp.unit_begin[l + 1]) ++l;
    decode_warp<true, true>(gp.layer[l], W, v - gp.unit_begin[l], lane);
}

}  // namespace mpq
