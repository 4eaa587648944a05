// k_decode.cuh -- memory-bound mixed-precision GEMV/GEMM for small M.
//
// y'[m][i] = sum_kb s[i,kb] * sum_{j in kb} x'[m][j] * (q[i][j] - z[i,kb])
// (the blocks' RTN dequantization, ScaleBITS summary "Approach" / "Key
// results"; 0-bit blocks are skipped -- they hold no bytes), then
// y[m][row_perm[i]] = y'[m][i] * tok_scale[m].
//
// Work split.  The table's blocks are cut, at pack time, into `n_units`
// row-major runs of about equal code bytes (sched); one CTA per run.  A CTA
// is 4 warps; the non-zero blocks of its run are dealt round-robin to the
// warps, and each warp streams its own blocks through a private ring of
// shared memory with 1-D bulk async copies (payload + 64 scales + 64 zeros +
// this block column's x' slice), several blocks ahead of the one it is
// computing.  A warp computes a whole 64x128 block: codes are turned into
// exact fp16 (q - z) pairs in registers (magic-number OR, then one HFMA2) and
// multiplied on the tensor cores with mma.m16n8k16 (fp32 accumulation, one
// group = 8 MMAs per 16 rows); the group result is scaled by s in fp32.
// At the end of each block row the 4 warps' partial sums are added in a fixed
// order.  A block row that is split between CTAs is finished by the last CTA
// to arrive (a per-row counter), which adds the CTAs' partials in unit order,
// so results are deterministic.
//
// Every wait is bounded: after ~2 s a wait records MPQ_ERR_TIMEOUT, sets a
// CTA-wide abort flag and the kernel winds down through the same barriers.
#pragma once
#include "common.cuh"

namespace mpq {

struct DecodeParams {
    const uint8_t* codes;
    const mpq_block* table;
    const uint32_t* sched;
    const uint16_t* scales;
    const uint16_t* zeros;
    const int32_t* row_perm;
    const uint8_t* xq;        // XP_DECODE layout, M_total tokens
    const float* tok_scale;   // [M_total]
    float* y;                 // [M_total][N]
    float* partial;           // [2*n_units][64][8]
    uint32_t* counters;       // [NB]
    uint32_t* err;
    int N, K, NB, KB;
    int M_total;              // tokens in xq / y
    int m0, Mg;               // this launch's token group [m0, m0+Mg), Mg <= 8
    int n_units;
};

constexpr int DEC_WARPS = 4;
constexpr int DEC_THREADS = DEC_WARPS * 32;
constexpr int DEC_RING = 16384;      // bytes of ring per warp
constexpr int DEC_SLOTS = 8;         // stages in flight per warp
constexpr uint32_t DEC_MAGIC = 0x64006400u;   // fp16 1024.0 in both halves
constexpr uint64_t DEC_WAIT_NS = 2000000000ull;

struct DecSmem {
    uint8_t ring[DEC_WARPS][DEC_RING];
    float red[DEC_WARPS][64][8];
    uint64_t full[DEC_WARPS][DEC_SLOTS];
    volatile int abort_flag;
    volatile int last_flag;
};

__device__ __forceinline__ uint32_t h2c(float lo, float hi) {
    return h2_bits(__halves2half2(__float2half_rn(lo), __float2half_rn(hi)));
}

// ---------------------------------------------------------------------------
// Code extraction.  For one row, one 8-code group i of this lane's 32 columns
// and j = 0..3, out[j] = fp16 pair (q[8i+j] - z, q[8i+j+4] - z), exact.
// ---------------------------------------------------------------------------

// p = 4: word i holds codes 8i..8i+7 as nibbles.
__device__ __forceinline__ void ext4(uint32_t w, uint32_t c1, uint32_t c16, uint32_t (&o)[4]) {
    const uint32_t k116 = 0x2C002C00u;  // 1/16
    const uint32_t w8 = w >> 8;
    o[0] = h2_bits(__hsub2(bits_h2(lop_and_or(w, 0x000F000Fu, DEC_MAGIC)), bits_h2(c1)));
    o[1] = hfma2_bits(lop_and_or(w, 0x00F000F0u, DEC_MAGIC), k116, c16);
    o[2] = h2_bits(__hsub2(bits_h2(lop_and_or(w8, 0x000F000Fu, DEC_MAGIC)), bits_h2(c1)));
    o[3] = hfma2_bits(lop_and_or(w8, 0x00F000F0u, DEC_MAGIC), k116, c16);
}

// p = 2: bytes 2i, 2i+1 of the lane's 8 bytes hold codes 8i..8i+7.
// c[j] = -(1024/4^j + z) in both halves.
__device__ __forceinline__ void ext2(uint32_t v, int sel, const uint32_t (&c)[4], uint32_t (&o)[4]) {
    const uint32_t P = __byte_perm(v, 0u, sel);
    o[0] = h2_bits(__hadd2(bits_h2(lop_and_or(P, 0x00030003u, DEC_MAGIC)), bits_h2(c[0])));
    o[1] = hfma2_bits(lop_and_or(P, 0x000C000Cu, DEC_MAGIC), 0x34003400u, c[1]);  // 1/4
    o[2] = hfma2_bits(lop_and_or(P, 0x00300030u, DEC_MAGIC), 0x2C002C00u, c[2]);  // 1/16
    o[3] = hfma2_bits(lop_and_or(P, 0x00C000C0u, DEC_MAGIC), 0x24002400u, c[3]);  // 1/64
}

// p = 1: byte i of the lane's word holds codes 8i..8i+7 (bit k = code 8i+k).
// c[j] = (-(1024/2^j + z), -(1024/2^(j+4) + z)).
__device__ __forceinline__ void ext1(uint32_t u, int sel, const uint32_t (&c)[4], uint32_t (&o)[4]) {
    const uint32_t P = __byte_perm(u, 0u, sel);
    // low half scaled by 2^-j, high half by 2^-(j+4)
    o[0] = hfma2_bits(lop_and_or(P, 0x00100001u, DEC_MAGIC), 0x2C003C00u, c[0]);
    o[1] = hfma2_bits(lop_and_or(P, 0x00200002u, DEC_MAGIC), 0x28003800u, c[1]);
    o[2] = hfma2_bits(lop_and_or(P, 0x00400004u, DEC_MAGIC), 0x24003400u, c[2]);
    o[3] = hfma2_bits(lop_and_or(P, 0x00800008u, DEC_MAGIC), 0x20003000u, c[3]);
}

// p = 8: words 2i and 2i+1 hold codes 8i..8i+3 and 8i+4..8i+7 as bytes.
__device__ __forceinline__ void ext8(uint32_t xa, uint32_t xb, uint32_t c1, uint32_t (&o)[4]) {
    const uint32_t T0 = __byte_perm(xa, xb, 0x5140);
    const uint32_t T1 = __byte_perm(xa, xb, 0x7362);
    o[0] = h2_bits(__hsub2(bits_h2(__byte_perm(T0, 0x64646464u, 0x4140)), bits_h2(c1)));
    o[1] = h2_bits(__hsub2(bits_h2(__byte_perm(T0, 0x64646464u, 0x4342)), bits_h2(c1)));
    o[2] = h2_bits(__hsub2(bits_h2(__byte_perm(T1, 0x64646464u, 0x4140)), bits_h2(c1)));
    o[3] = h2_bits(__hsub2(bits_h2(__byte_perm(T1, 0x64646464u, 0x4342)), bits_h2(c1)));
}

// High piece of a split code, already multiplied by 2^w (w = low width):
// the exact values 2^w * hi, no zero point.
// p = 1 (w = 2 or 4): scale (2^w/2^j, 2^w/2^(j+4)), offset -(1024 * that).
template <int W>
__device__ __forceinline__ void ext1_hi(uint32_t u, int sel, uint32_t (&o)[4]) {
    const uint32_t P = __byte_perm(u, 0u, sel);
    const uint32_t msk[4] = {0x00100001u, 0x00200002u, 0x00400004u, 0x00800008u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float lo = (float)(1 << W) / (float)(1 << j);
        const float hi = (float)(1 << W) / (float)(1 << (j + 4));
        o[j] = hfma2_bits(lop_and_or(P, msk[j], DEC_MAGIC), h2c(lo, hi), h2c(-1024.f * lo, -1024.f * hi));
    }
}
// p = 2 (w = 4): scale 16/4^j, offset -16384/4^j.
__device__ __forceinline__ void ext2_hi(uint32_t v, int sel, uint32_t (&o)[4]) {
    const uint32_t P = __byte_perm(v, 0u, sel);
    const uint32_t msk[4] = {0x00030003u, 0x000C000Cu, 0x00300030u, 0x00C000C0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float sc = 16.f / (float)(1 << (2 * j));
        o[j] = hfma2_bits(lop_and_or(P, msk[j], DEC_MAGIC), h2c(sc, sc), h2c(-1024.f * sc, -1024.f * sc));
    }
}

// Zero-point constants for a row with zero point z (an fp16 integer).
__device__ __forceinline__ uint32_t zc(float base, float z) { return h2c(-(base + z), -(base + z)); }

// ---------------------------------------------------------------------------
// One 64x128 block of width B: acc[rt][*] += s_row * sum_k x * (q - z).
// stage: payload (1024*B bytes) | scales (64 fp16) | zeros (64 fp16) | x'.
// ---------------------------------------------------------------------------
template <int B>
__device__ __forceinline__ void block_mma(const uint8_t* stage, const uint32_t (&bx)[16],
                                          float (&acc)[4][4], int g, int t) {
    const __half* sc = reinterpret_cast<const __half*>(stage + 1024 * B);
    const __half* zr = sc + 64;
    constexpr int P0 = (B == 3) ? 2 : (B == 5 || B == 6) ? 4 : B;   // low piece width
    constexpr int P1 = (B == 3 || B == 5) ? 1 : (B == 6) ? 2 : 0;   // high piece width
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) {
        const int r0 = 16 * rt + g, r1 = r0 + 8;
        const float s0 = __half2float(sc[r0]), s1 = __half2float(sc[r1]);
        const float z0 = __half2float(zr[r0]), z1 = __half2float(zr[r1]);
        // low-piece data (4*P0 bytes per row for this lane)
        uint32_t d0[P0], d1[P0];
        {
            const uint8_t* b0 = stage + r0 * 16 * P0 + t * 4 * P0;
            const uint8_t* b1 = stage + r1 * 16 * P0 + t * 4 * P0;
            if (P0 == 1) {
                d0[0] = *reinterpret_cast<const uint32_t*>(b0);
                d1[0] = *reinterpret_cast<const uint32_t*>(b1);
            } else if (P0 == 2) {
                uint2 a = *reinterpret_cast<const uint2*>(b0), c = *reinterpret_cast<const uint2*>(b1);
                d0[0] = a.x; d0[1] = a.y; d1[0] = c.x; d1[1] = c.y;
            } else {
#pragma unroll
                for (int q = 0; q < P0 / 4; ++q) {
                    uint4 a = reinterpret_cast<const uint4*>(b0)[q], c = reinterpret_cast<const uint4*>(b1)[q];
                    d0[4 * q + 0] = a.x; d0[4 * q + 1] = a.y; d0[4 * q + 2] = a.z; d0[4 * q + 3] = a.w;
                    d1[4 * q + 0] = c.x; d1[4 * q + 1] = c.y; d1[4 * q + 2] = c.z; d1[4 * q + 3] = c.w;
                }
            }
        }
        uint32_t e0[P1 > 0 ? P1 : 1], e1[P1 > 0 ? P1 : 1];
        if (P1 > 0) {
            const uint8_t* hb = stage + 64 * 16 * P0;
            const uint8_t* h0 = hb + r0 * 16 * P1 + t * 4 * P1;
            const uint8_t* h1 = hb + r1 * 16 * P1 + t * 4 * P1;
            if (P1 == 1) {
                e0[0] = *reinterpret_cast<const uint32_t*>(h0);
                e1[0] = *reinterpret_cast<const uint32_t*>(h1);
            } else {
                uint2 a = *reinterpret_cast<const uint2*>(h0), c = *reinterpret_cast<const uint2*>(h1);
                e0[0] = a.x; e0[1] = a.y; e1[0] = c.x; e1[1] = c.y;
            }
        }
        // zero-point constants of the low piece
        uint32_t k0[4], k1[4];
        if (P0 == 4) {
            k0[0] = h2_bits(__floats2half2_rn(1024.f + z0, 1024.f + z0)); k0[1] = zc(64.f, z0);
            k1[0] = h2_bits(__floats2half2_rn(1024.f + z1, 1024.f + z1)); k1[1] = zc(64.f, z1);
        } else if (P0 == 8) {
            k0[0] = h2_bits(__floats2half2_rn(1024.f + z0, 1024.f + z0));
            k1[0] = h2_bits(__floats2half2_rn(1024.f + z1, 1024.f + z1));
        } else if (P0 == 2) {
            k0[0] = zc(1024.f, z0); k0[1] = zc(256.f, z0); k0[2] = zc(64.f, z0); k0[3] = zc(16.f, z0);
            k1[0] = zc(1024.f, z1); k1[1] = zc(256.f, z1); k1[2] = zc(64.f, z1); k1[3] = zc(16.f, z1);
        } else {  // P0 == 1
            k0[0] = h2c(-(1024.f + z0), -(64.f + z0)); k0[1] = h2c(-(512.f + z0), -(32.f + z0));
            k0[2] = h2c(-(256.f + z0), -(16.f + z0));  k0[3] = h2c(-(128.f + z0), -(8.f + z0));
            k1[0] = h2c(-(1024.f + z1), -(64.f + z1)); k1[1] = h2c(-(512.f + z1), -(32.f + z1));
            k1[2] = h2c(-(256.f + z1), -(16.f + z1));  k1[3] = h2c(-(128.f + z1), -(8.f + z1));
        }
        float cg[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t a0[4], a1[4];
            if (P0 == 4) {
                ext4(d0[i], k0[0], k0[1], a0);
                ext4(d1[i], k1[0], k1[1], a1);
            } else if (P0 == 8) {
                ext8(d0[2 * i], d0[2 * i + 1], k0[0], a0);
                ext8(d1[2 * i], d1[2 * i + 1], k1[0], a1);
            } else if (P0 == 2) {
                const int sel = (i & 1) ? 0x4342 : 0x4140;
                ext2(d0[i >> 1], sel, k0, a0);
                ext2(d1[i >> 1], sel, k1, a1);
            } else {
                const int sel = i | (4 << 4) | (i << 8) | (4 << 12);
                ext1(d0[0], sel, k0, a0);
                ext1(d1[0], sel, k1, a1);
            }
            mma_16816(cg, a0[0], a1[0], a0[1], a1[1], bx[4 * i], bx[4 * i + 1]);
            mma_16816(cg, a0[2], a1[2], a0[3], a1[3], bx[4 * i + 2], bx[4 * i + 3]);
            if (P1 > 0) {
                uint32_t h0[4], h1[4];
                if (P1 == 1) {
                    const int sel = i | (4 << 4) | (i << 8) | (4 << 12);
                    ext1_hi<P0>(e0[0], sel, h0);
                    ext1_hi<P0>(e1[0], sel, h1);
                } else {
                    const int sel = (i & 1) ? 0x4342 : 0x4140;
                    ext2_hi(e0[i >> 1], sel, h0);
                    ext2_hi(e1[i >> 1], sel, h1);
                }
                mma_16816(cg, h0[0], h1[0], h0[1], h1[1], bx[4 * i], bx[4 * i + 1]);
                mma_16816(cg, h0[2], h1[2], h0[3], h1[3], bx[4 * i + 2], bx[4 * i + 3]);
            }
        }
        acc[rt][0] = fmaf(s0, cg[0], acc[rt][0]);
        acc[rt][1] = fmaf(s0, cg[1], acc[rt][1]);
        acc[rt][2] = fmaf(s1, cg[2], acc[rt][2]);
        acc[rt][3] = fmaf(s1, cg[3], acc[rt][3]);
    }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(DEC_THREADS, 3) k_decode(DecodeParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    DecSmem& S = *reinterpret_cast<DecSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int u = blockIdx.x;
    const int KB = p.KB;

    if (tid == 0) {
        for (int w = 0; w < DEC_WARPS; ++w)
            for (int s = 0; s < DEC_SLOTS; ++s) mbar_init(&S.full[w][s], 1);
        S.abort_flag = 0;
        fence_mbar_init();
    }
    const uint32_t t0 = p.sched[u], t1 = p.sched[u + 1];
    __syncthreads();
    // x', tok_scale, counters and y belong to the prologue kernel / earlier work
    pdl_wait();
    if (t0 >= t1) return;

    const int Mg = p.Mg;
    const uint32_t xslice = 256u * (uint32_t)Mg;
    uint8_t* ring = S.ring[warp];

    // ---- per-warp stream state (uniform across the warp) ----
    uint32_t tab_base = t0 & ~31u;          // table chunk start
    uint32_t nz_before = 0;                 // non-zero blocks of this unit before the chunk
    mpq_block ent;                          // this lane's entry of the chunk
    auto load_chunk = [&]() {
        const uint32_t tt = tab_base + lane;
        if (tt >= t0 && tt < t1) ent = p.table[tt];
        else ent = mpq_block{0u, 0u, 0u, 0u};
    };
    load_chunk();
    uint32_t scan_t = t0;
    uint32_t q_head = 0, q_tail = 0;         // consumed / issued stages
    uint32_t r_head = 0, r_tail = 0;         // ring bytes issued / freed
    // queue entry k lives in lane k % DEC_SLOTS
    uint32_t qe_t = 0, qe_bits = 0, qe_off = 0, qe_end = 0;

    auto issue_more = [&]() {
        while (q_tail - q_head < (uint32_t)DEC_SLOTS && scan_t < t1) {
            if (q_head == q_tail) { r_head = 0; r_tail = 0; }   // empty ring: restart at 0
            if (scan_t >= tab_base + 32) {
                const uint32_t nzm = __ballot_sync(0xffffffffu, ent.bits != 0u);
                nz_before += __popc(nzm);
                tab_base += 32;
                load_chunk();
                continue;
            }
            const uint32_t nzm = __ballot_sync(0xffffffffu, ent.bits != 0u);
            const uint32_t rank = nz_before + __popc(nzm & ((1u << lane) - 1u));
            const bool mine = (ent.bits != 0u) && ((rank & (DEC_WARPS - 1)) == (uint32_t)warp) &&
                              (tab_base + lane >= scan_t);
            const uint32_t cand = __ballot_sync(0xffffffffu, mine);
            if (cand == 0u) {
                scan_t = tab_base + 32;
                continue;
            }
            const int l = __ffs(cand) - 1;
            const uint32_t b = __shfl_sync(0xffffffffu, ent.bits, l);
            const uint32_t coff = __shfl_sync(0xffffffffu, ent.code_off, l);
            const uint32_t szo = __shfl_sync(0xffffffffu, ent.sz_off, l);
            const uint32_t tt = tab_base + l;
            const uint32_t size = 1024u * b + 256u + xslice;
            uint32_t start = r_head;
            const uint32_t pos = r_head % DEC_RING;
            if (pos + size > DEC_RING) start = r_head + (DEC_RING - pos);
            if (start + size - r_tail > DEC_RING) break;   // ring full: compute first
            const uint32_t slot = q_tail % DEC_SLOTS;
            const uint32_t off = start % DEC_RING;
            if (lane == 0) {
                fence_proxy_async_smem();
                uint64_t* bar = &S.full[warp][slot];
                mbar_arrive_expect_tx(bar, size);
                uint8_t* dst = ring + off;
                const uint32_t kb = tt % KB;
                bulk_g2s(dst, p.codes + coff, 1024u * b, bar);
                bulk_g2s(dst + 1024u * b, p.scales + szo, 128u, bar);
                bulk_g2s(dst + 1024u * b + 128u, p.zeros + szo, 128u, bar);
                bulk_g2s(dst + 1024u * b + 256u,
                         p.xq + ((size_t)kb * p.M_total + p.m0) * 256u, xslice, bar);
            }
            if (lane == (int)slot) { qe_t = tt; qe_bits = b; qe_off = off; qe_end = start + size; }
            r_head = start + size;
            ++q_tail;
            scan_t = tt + 1;
        }
    };

    float* red = &S.red[0][0][0];
    const uint32_t nb_first = t0 / KB, nb_last = (t1 - 1) / KB;
    for (uint32_t nb = nb_first; nb <= nb_last; ++nb) {
        const uint32_t row_end = min(t1, (nb + 1) * (uint32_t)KB);
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
            if (ft >= row_end) break;       // next block of mine is in a later row
            const uint32_t fb = __shfl_sync(0xffffffffu, qe_bits, slot);
            const uint32_t foff = __shfl_sync(0xffffffffu, qe_off, slot);
            const uint32_t fend = __shfl_sync(0xffffffffu, qe_end, slot);
            bool ok = true;
            if (!S.abort_flag) ok = mbar_wait_bounded(&S.full[warp][slot], (q_head / DEC_SLOTS) & 1u, DEC_WAIT_NS);
            if (!ok) {
                if (lane == 0) { set_error(p.err, MPQ_ERR_TIMEOUT); S.abort_flag = 1; }
            }
            __syncwarp();
            if (!S.abort_flag) {
                const uint8_t* stage = ring + foff;
                uint32_t bx[16];
                if (g < Mg) {
                    const uint4* xs = reinterpret_cast<const uint4*>(stage + 1024u * fb + 256u + g * 256 + t * 64);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 v = xs[q];
                        bx[4 * q] = v.x; bx[4 * q + 1] = v.y; bx[4 * q + 2] = v.z; bx[4 * q + 3] = v.w;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) bx[q] = 0u;
                }
                switch (fb) {
                    case 1: block_mma<1>(stage, bx, acc, g, t); break;
                    case 2: block_mma<2>(stage, bx, acc, g, t); break;
                    case 3: block_mma<3>(stage, bx, acc, g, t); break;
                    case 4: block_mma<4>(stage, bx, acc, g, t); break;
                    case 5: block_mma<5>(stage, bx, acc, g, t); break;
                    case 6: block_mma<6>(stage, bx, acc, g, t); break;
                    default: block_mma<8>(stage, bx, acc, g, t); break;
                }
            }
            __syncwarp();
            ++q_head;
            r_tail = fend;
        }

        // ---- end of block row nb: add the 4 warps' partials in a fixed order ----
#pragma unroll
        for (int rt = 0; rt < 4; ++rt) {
            float* rw = red + ((size_t)warp * 64 + 16 * rt + g) * 8;
            rw[2 * t] = acc[rt][0];
            rw[2 * t + 1] = acc[rt][1];
            rw[8 * 8 + 2 * t] = acc[rt][2];
            rw[8 * 8 + 2 * t + 1] = acc[rt][3];
        }
        named_bar_sync(1, DEC_THREADS);
        const bool complete = (nb * (uint32_t)KB >= t0) && ((nb + 1) * (uint32_t)KB <= t1);
        float sums[4];
        int rows[4], toks[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int idx = lane + 32 * q;           // 16 rows x 8 tokens per warp
            rows[q] = 16 * warp + (idx >> 3);
            toks[q] = idx & 7;
            const size_t o = (size_t)rows[q] * 8 + toks[q];
            sums[q] = ((red[o] + red[64 * 8 + o]) + red[2 * 64 * 8 + o]) + red[3 * 64 * 8 + o];
        }
        if (complete) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (toks[q] < Mg) {
                    const int i = (int)nb * 64 + rows[q];
                    const int n = p.row_perm ? p.row_perm[i] : i;
                    const int m = p.m0 + toks[q];
                    p.y[(size_t)m * p.N + n] = sums[q] * p.tok_scale[m];
                }
            }
        } else {
            const uint32_t first_row = t0 / KB;
            const uint32_t slot_id = 2u * (uint32_t)u + (nb == first_row ? 0u : 1u);
            float* part = p.partial + (size_t)slot_id * 64 * 8;
#pragma unroll
            for (int q = 0; q < 4; ++q) part[rows[q] * 8 + toks[q]] = sums[q];
            __threadfence();
            named_bar_sync(1, DEC_THREADS);
            if (tid == 0) {
                const uint32_t lo = max(t0, nb * (uint32_t)KB);
                const uint32_t cnt = row_end - lo;
                const uint32_t old = atomicAdd(&p.counters[nb], cnt);
                S.last_flag = (old + cnt == (uint32_t)KB);
            }
            named_bar_sync(1, DEC_THREADS);
            if (S.last_flag) {
                __threadfence();
                // contributors: the units whose runs meet block row nb
                uint32_t c_first = (uint32_t)u, c_last = (uint32_t)u;
                while (p.sched[c_first] > nb * (uint32_t)KB) --c_first;
                while (p.sched[c_last + 1] < (nb + 1) * (uint32_t)KB) ++c_last;
                float tot[4] = {0.f, 0.f, 0.f, 0.f};
                for (uint32_t c = c_first; c <= c_last; ++c) {
                    const uint32_t cs = p.sched[c], ce = p.sched[c + 1];
                    if (cs >= ce) continue;
                    const uint32_t sid = 2u * c + ((cs / KB) == nb ? 0u : 1u);
                    const float* pc = p.partial + (size_t)sid * 64 * 8;
#pragma unroll
                    for (int q = 0; q < 4; ++q) tot[q] += __ldcg(pc + rows[q] * 8 + toks[q]);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (toks[q] < Mg) {
                        const int i = (int)nb * 64 + rows[q];
                        const int n = p.row_perm ? p.row_perm[i] : i;
                        const int m = p.m0 + toks[q];
                        p.y[(size_t)m * p.N + n] = tot[q] * p.tok_scale[m];
                    }
                }
                if (tid == 0) p.counters[nb] = 0u;   // ready for the next launch
            }
        }
        named_bar_sync(1, DEC_THREADS);   // red[] is reused by the next row
    }
}

}  // namespace mpq
