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
#include "k_xprep.cuh"   // XQD_SLICE

namespace mpq {

struct DecodeParams {
    const uint8_t* codes;
    const mpq_block* table;
    const uint32_t* sched;
    const uint16_t* scales;
    const uint16_t* zeros;
    const int32_t* row_perm;
    const uint8_t* xq;        // k_xprep_decode layout: [KB][M_total][272 B]
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
constexpr int DEC_RING = 10752;      // bytes of ring per warp (>= largest stage)
constexpr int DEC_SLOTS = 8;         // stages in flight per warp
constexpr uint32_t DEC_MAGIC = 0x64006400u;   // fp16 1024.0 in both halves
constexpr uint64_t DEC_WAIT_NS = 2000000000ull;

struct DecSmem {
    uint8_t ring[DEC_WARPS][DEC_RING];
    float red[DEC_WARPS][64][8];
    uint64_t full[DEC_WARPS][DEC_SLOTS];
    mpq_block tab[DEC_WARPS][2][32];   // per-warp table chunks (current, next)
    uint4 zero16[4];          // zero B fragments for lanes beyond the token count
    volatile int abort_flag;
    volatile int last_flag;
};

// 4 CTAs per SM: 4 x (smem + 1 KB reserved) must fit the SM's 228 KB
static_assert(4 * (sizeof(DecSmem) + 1024) <= 228 * 1024, "decode smem too large for 4 CTAs/SM");
static_assert(DEC_RING >= 8 * 1024 + 256 + 272 * 8, "ring must hold the largest stage");

__device__ __forceinline__ uint32_t h2c(float lo, float hi) {
    return h2_bits(__halves2half2(__float2half_rn(lo), __float2half_rn(hi)));
}

// ---------------------------------------------------------------------------
// Code extraction.  For one row, one 8-code group i of this lane's 32 columns
// and j = 0..3, out[j] = fp16 pair (q[8i+j] - z, q[8i+j+4] - z), exact.
// ---------------------------------------------------------------------------

// p = 4: word i holds codes 8i..8i+7 as nibbles.  c1 = -(1024 + z), c16 = -(64 + z).
__device__ __forceinline__ void ext4(uint32_t w, uint32_t c1, uint32_t c16, uint32_t (&o)[4]) {
    const uint32_t k116 = 0x2C002C00u;  // 1/16
    const uint32_t w8 = w >> 8;
    o[0] = h2_bits(__hadd2(bits_h2(lop_and_or(w, 0x000F000Fu, DEC_MAGIC)), bits_h2(c1)));
    o[1] = hfma2_bits(lop_and_or(w, 0x00F000F0u, DEC_MAGIC), k116, c16);
    o[2] = h2_bits(__hadd2(bits_h2(lop_and_or(w8, 0x000F000Fu, DEC_MAGIC)), bits_h2(c1)));
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
// c1 = -(1024 + z).
__device__ __forceinline__ void ext8(uint32_t xa, uint32_t xb, uint32_t c1, uint32_t (&o)[4]) {
    const uint32_t T0 = __byte_perm(xa, xb, 0x5140);
    const uint32_t T1 = __byte_perm(xa, xb, 0x7362);
    o[0] = h2_bits(__hadd2(bits_h2(__byte_perm(T0, 0x64646464u, 0x4140)), bits_h2(c1)));
    o[1] = h2_bits(__hadd2(bits_h2(__byte_perm(T0, 0x64646464u, 0x4342)), bits_h2(c1)));
    o[2] = h2_bits(__hadd2(bits_h2(__byte_perm(T1, 0x64646464u, 0x4140)), bits_h2(c1)));
    o[3] = h2_bits(__hadd2(bits_h2(__byte_perm(T1, 0x64646464u, 0x4342)), bits_h2(c1)));
}

// High piece of a split code, already multiplied by 2^w (w = low width):
// the exact values 2^w * hi, no zero point.  Magic-number pairs carry
// multipliers m (low half) / m' (high half); an HFMA2 with scale 2^w/m and
// offset -1024*2^w/m removes the magic.  The constants are fp16 bit patterns
// (low half in bits 0-15).
// p = 1: m = 2^j, m' = 2^(j+4).
template <int W>
__device__ __forceinline__ void ext1_hi(uint32_t u, int sel, uint32_t (&o)[4]) {
    const uint32_t P = __byte_perm(u, 0u, sel);
    // W = 2: scale (4/2^j, 4/2^(j+4)); W = 4: scale (16/2^j, 16/2^(j+4))
    constexpr uint32_t sc2[4] = {0x34004400u, 0x30004000u, 0x2C003C00u, 0x28003800u};
    constexpr uint32_t of2[4] = {0xDC00EC00u, 0xD800E800u, 0xD400E400u, 0xD000E000u};
    constexpr uint32_t sc4[4] = {0x3C004C00u, 0x38004800u, 0x34004400u, 0x30004000u};
    constexpr uint32_t of4[4] = {0xE400F400u, 0xE000F000u, 0xDC00EC00u, 0xD800E800u};
    const uint32_t msk[4] = {0x00100001u, 0x00200002u, 0x00400004u, 0x00800008u};
#pragma unroll
    for (int j = 0; j < 4; ++j)
        o[j] = hfma2_bits(lop_and_or(P, msk[j], DEC_MAGIC), W == 2 ? sc2[j] : sc4[j],
                          W == 2 ? of2[j] : of4[j]);
}
// p = 2 (w = 4): m = m' = 4^j: scale 16/4^j, offset -16384/4^j.
__device__ __forceinline__ void ext2_hi(uint32_t v, int sel, uint32_t (&o)[4]) {
    const uint32_t P = __byte_perm(v, 0u, sel);
    constexpr uint32_t sc[4] = {0x4C004C00u, 0x44004400u, 0x3C003C00u, 0x34003400u};
    constexpr uint32_t of[4] = {0xF400F400u, 0xEC00EC00u, 0xE400E400u, 0xDC00DC00u};
    const uint32_t msk[4] = {0x00030003u, 0x000C000Cu, 0x00300030u, 0x00C000C0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = hfma2_bits(lop_and_or(P, msk[j], DEC_MAGIC), sc[j], of[j]);
}

// Zero-point constants for a row with zero point z (an fp16 integer).
__device__ __forceinline__ uint32_t zc(float base, float z) { return h2c(-(base + z), -(base + z)); }

// The same constants from z as (z, z) fp16 pair bits: -(base + z) = z*(-1) - base,
// exact in fp16 (base + z <= 1279).
__device__ __forceinline__ uint32_t zc2(uint32_t z2, uint32_t neg_base2) {
    return hfma2_bits(z2, 0xBC00BC00u, neg_base2);
}

// Low-piece zero-point constants for a row (see the ext* functions).
template <int P0>
__device__ __forceinline__ void zero_consts(uint32_t z2, uint32_t (&k)[4]) {
    if (P0 == 4) {
        k[0] = zc2(z2, 0xE400E400u);        // -(1024 + z)
        k[1] = zc2(z2, 0xD400D400u);        // -(64 + z)
    } else if (P0 == 8) {
        k[0] = zc2(z2, 0xE400E400u);
    } else if (P0 == 2) {
        k[0] = zc2(z2, 0xE400E400u);        // -(1024 + z)
        k[1] = zc2(z2, 0xDC00DC00u);        // -(256 + z)
        k[2] = zc2(z2, 0xD400D400u);        // -(64 + z)
        k[3] = zc2(z2, 0xCC00CC00u);        // -(16 + z)
    } else {
        k[0] = zc2(z2, 0xD400E400u);        // (-(1024 + z), -(64 + z))
        k[1] = zc2(z2, 0xD000E000u);        // (-(512 + z),  -(32 + z))
        k[2] = zc2(z2, 0xCC00DC00u);        // (-(256 + z),  -(16 + z))
        k[3] = zc2(z2, 0xC800D800u);        // (-(128 + z),  -(8 + z))
    }
}

// ---------------------------------------------------------------------------
// One 64x128 block of width B.  The lane owns rows 16rt+g and 16rt+g+8 of the
// four 16-row tiles rt and, in each row, the 32 columns of quad lane t.
// acc[rt][*] += s_row * 2^-e_tok * sum_k x * (q - z)  (fp32, C-fragment order).
// The loop over the 4 code groups i is rolled (small code: all 7 widths stay
// in the instruction cache); inside it the 4 row tiles are independent mma
// chains.  stage: payload (1024*B) | scales (64 fp16) | zeros (64 fp16) | x'.
// ---------------------------------------------------------------------------
template <int B>
__device__ __forceinline__ void block_mma(const uint8_t* stage, const uint8_t* xs_lane,
                                          float f0, float f1, float (&acc)[4][4], int g, int t) {
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(stage + 1024 * B);
    const uint16_t* zr = sc + 64;
    constexpr int P0 = (B == 3) ? 2 : (B == 5 || B == 6) ? 4 : B;   // low piece width
    constexpr int P1 = (B == 3 || B == 5) ? 1 : (B == 6) ? 2 : 0;   // high piece width
    constexpr int NK = (P0 == 1 || P0 == 2) ? 4 : (P0 == 4 ? 2 : 1);
    // per-row zero-point constants; rows 16rt+g (index 2rt) and +8 (2rt+1)
    uint32_t k[8][NK];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int r = 8 * q + g;   // q = 2rt + h  ->  row 16rt + 8h + g
        uint32_t kk[4];
        zero_consts<P0>(__byte_perm((uint32_t)zr[r], 0u, 0x1010), kk);
#pragma unroll
        for (int c = 0; c < NK; ++c) k[q][c] = kk[c];
    }
    float cg[4][4];
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
        for (int c = 0; c < 4; ++c) cg[rt][c] = 0.f;
    const uint8_t* lo_base = stage + t * 4 * P0;
    const uint8_t* hi_base = stage + 64 * 16 * P0 + t * 4 * P1;
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
        const uint4 bv = *reinterpret_cast<const uint4*>(xs_lane + 16 * i);   // B regs 4i..4i+3
        const int sel2 = (i & 1) ? 0x4342 : 0x4140;
        const int sel1 = i | (4 << 4) | (i << 8) | (4 << 12);
#pragma unroll
        for (int rt = 0; rt < 4; ++rt) {
            uint32_t a[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = 16 * rt + 8 * h + g;
                const uint32_t* kq = k[2 * rt + h];
                const uint8_t* rowp = lo_base + r * 16 * P0;
                if (P0 == 4) {
                    const uint32_t w = reinterpret_cast<const uint32_t*>(rowp)[i];
                    ext4(w, kq[0], kq[1], a[h]);
                } else if (P0 == 8) {
                    const uint2 w = reinterpret_cast<const uint2*>(rowp)[i];
                    ext8(w.x, w.y, kq[0], a[h]);
                } else if (P0 == 2) {
                    const uint32_t w = reinterpret_cast<const uint32_t*>(rowp)[i >> 1];
                    uint32_t kk[4] = {kq[0], kq[1], kq[2], kq[3]};
                    ext2(w, sel2, kk, a[h]);
                } else {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(rowp);
                    uint32_t kk[4] = {kq[0], kq[1], kq[2], kq[3]};
                    ext1(w, sel1, kk, a[h]);
                }
                if (P1 > 0) {   // (lo - z) + 2^w * hi, exact small integers
                    const uint8_t* hrow = hi_base + r * 16 * P1;
                    uint32_t hv[4];
                    if (P1 == 1) ext1_hi<P0>(*reinterpret_cast<const uint32_t*>(hrow), sel1, hv);
                    else ext2_hi(reinterpret_cast<const uint32_t*>(hrow)[i >> 1], sel2, hv);
#pragma unroll
                    for (int j = 0; j < 4; ++j) a[h][j] = h2_bits(__hadd2(bits_h2(a[h][j]), bits_h2(hv[j])));
                }
            }
            mma_16816(cg[rt], a[0][0], a[1][0], a[0][1], a[1][1], bv.x, bv.y);
            mma_16816(cg[rt], a[0][2], a[1][2], a[0][3], a[1][3], bv.z, bv.w);
        }
    }
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) {
        const float s0 = __half2float(__ushort_as_half(sc[16 * rt + g]));
        const float s1 = __half2float(__ushort_as_half(sc[16 * rt + 8 + g]));
        acc[rt][0] = fmaf(s0 * f0, cg[rt][0], acc[rt][0]);
        acc[rt][1] = fmaf(s0 * f1, cg[rt][1], acc[rt][1]);
        acc[rt][2] = fmaf(s1 * f0, cg[rt][2], acc[rt][2]);
        acc[rt][3] = fmaf(s1 * f1, cg[rt][3], acc[rt][3]);
    }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(DEC_THREADS, 4) k_decode(DecodeParams p) {
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
        for (int q = 0; q < 4; ++q) S.zero16[q] = make_uint4(0u, 0u, 0u, 0u);
        fence_mbar_init();
    }
    const uint32_t t0 = p.sched[u], t1 = p.sched[u + 1];
    __syncthreads();

    const int Mg = p.Mg;
    const uint32_t xslice = (uint32_t)XQD_SLICE * (uint32_t)Mg;
    uint8_t* ring = S.ring[warp];

    // ---- per-warp stream state (uniform across the warp) ----
    // Table chunks of 32 entries, the next one loaded a chunk ahead.  For the
    // current chunk, `mine` has a bit for every lane whose block is non-zero
    // and dealt to this warp (the unit's non-zero blocks go round-robin).
    uint32_t tab_base = t0 & ~31u;
    uint32_t nz_before = 0;          // non-zero blocks of this unit before the chunk
    int tb = 0;                      // which of the two chunk buffers is current
    // each lane copies its entry of the chunk at `base` (zeros outside [t0, t1))
    auto fetch = [&](uint32_t base, int buf) {
        const uint32_t tt = base + lane;
        const bool in = tt >= t0 && tt < t1;
        cp_async16(&S.tab[warp][buf][lane], p.table + (in ? tt : t0), in ? 16u : 0u);
        cp_async_commit();
    };
    fetch(tab_base, 0);
    fetch(tab_base + 32, 1);
    cp_async_wait_all();
    __syncwarp();
    auto mine_of = [&]() -> uint32_t {
        const uint32_t bits = S.tab[warp][tb][lane].bits;
        const uint32_t nzm = __ballot_sync(0xffffffffu, bits != 0u);
        const uint32_t rank = nz_before + __popc(nzm & ((1u << lane) - 1u));
        const uint32_t m = __ballot_sync(0xffffffffu, bits != 0u &&
                                                          (rank & (DEC_WARPS - 1)) == (uint32_t)warp);
        nz_before += __popc(nzm);
        return m;
    };
    uint32_t mine = mine_of();
    bool scan_done = false;
    uint32_t q_head = 0, q_tail = 0;     // consumed / issued stages
    uint32_t r_head = 0, r_tail = 0;     // ring bytes issued / freed
    // queue entry k lives in lane k % DEC_SLOTS
    uint32_t qe_t = 0, qe_bits = 0, qe_off = 0, qe_end = 0;
    bool xq_ready = false;               // x' is written by the prologue kernel

    auto issue_xq = [&](uint32_t tt, uint32_t b, uint32_t off, uint32_t slot) {
        const uint32_t kb = tt % KB;
        bulk_g2s(ring + off + 1024u * b + 256u,
                 p.xq + ((size_t)kb * p.M_total + p.m0) * XQD_SLICE, xslice, &S.full[warp][slot]);
    };
    auto issue_more = [&]() {
        while (q_tail - q_head < (uint32_t)DEC_SLOTS && !scan_done) {
            if (mine == 0u) {
                if (tab_base + 32 >= t1) { scan_done = true; break; }
                tab_base += 32;
                cp_async_wait_all();     // the next chunk landed long ago
                __syncwarp();
                tb ^= 1;
                fetch(tab_base + 32, tb ^ 1);   // refill the buffer just retired
                mine = mine_of();
                continue;
            }
            if (q_head == q_tail) { r_head = 0; r_tail = 0; }   // empty ring: restart at 0
            const int l = __ffs(mine) - 1;
            const mpq_block& en = S.tab[warp][tb][l];
            const uint32_t b = en.bits;
            const uint32_t size = 1024u * b + 256u + xslice;
            uint32_t start = r_head;
            const uint32_t pos = r_head % DEC_RING;
            if (pos + size > DEC_RING) start = r_head + (DEC_RING - pos);
            if (start + size - r_tail > DEC_RING) break;   // ring full: compute first
            const uint32_t coff = en.code_off;
            const uint32_t szo = en.sz_off;
            const uint32_t tt = tab_base + l;
            const uint32_t slot = q_tail % DEC_SLOTS;
            const uint32_t off = start % DEC_RING;
            if (lane == 0) {
                fence_proxy_async_smem();
                uint64_t* bar = &S.full[warp][slot];
                mbar_arrive_expect_tx(bar, size);
                uint8_t* dst = ring + off;
                bulk_g2s(dst, p.codes + coff, 1024u * b, bar);
                bulk_g2s(dst + 1024u * b, p.scales + szo, 128u, bar);
                bulk_g2s(dst + 1024u * b + 128u, p.zeros + szo, 128u, bar);
                if (xq_ready) issue_xq(tt, b, off, slot);
            }
            if (lane == (int)slot) { qe_t = tt; qe_bits = b; qe_off = off; qe_end = start + size; }
            r_head = start + size;
            ++q_tail;
            mine &= mine - 1u;
        }
    };

    // Weights do not depend on the prologue kernel: start streaming them, then
    // wait for x' (programmatic dependent launch) and add its copies.
    if (t0 < t1) issue_more();
    pdl_wait();
    if (t0 >= t1) return;
    xq_ready = true;
    for (uint32_t k = q_head; k < q_tail; ++k) {
        const uint32_t slot = k % DEC_SLOTS;
        const uint32_t kt = __shfl_sync(0xffffffffu, qe_t, slot);
        const uint32_t kb_ = __shfl_sync(0xffffffffu, qe_bits, slot);
        const uint32_t ko = __shfl_sync(0xffffffffu, qe_off, slot);
        if (lane == 0) issue_xq(kt, kb_, ko, slot);
    }

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
                const uint8_t* xs = stage + 1024u * fb + 256u;
                // this lane's B fragments (token g, quad lane t); zeros beyond Mg
                const uint8_t* xs_lane = (g < Mg) ? xs + g * XQD_SLICE + t * 64 : reinterpret_cast<const uint8_t*>(S.zero16);
                // 2^-e of the tokens 2t and 2t+1 (the C-fragment columns)
                const float f0 = (2 * t < Mg) ? *reinterpret_cast<const float*>(xs + (2 * t) * XQD_SLICE + 256) : 0.f;
                const float f1 = (2 * t + 1 < Mg) ? *reinterpret_cast<const float*>(xs + (2 * t + 1) * XQD_SLICE + 256) : 0.f;
                switch (fb) {
                    case 1: block_mma<1>(stage, xs_lane, f0, f1, acc, g, t); break;
                    case 2: block_mma<2>(stage, xs_lane, f0, f1, acc, g, t); break;
                    case 3: block_mma<3>(stage, xs_lane, f0, f1, acc, g, t); break;
                    case 4: block_mma<4>(stage, xs_lane, f0, f1, acc, g, t); break;
                    case 5: block_mma<5>(stage, xs_lane, f0, f1, acc, g, t); break;
                    case 6: block_mma<6>(stage, xs_lane, f0, f1, acc, g, t); break;
                    default: block_mma<8>(stage, xs_lane, f0, f1, acc, g, t); break;
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
            *reinterpret_cast<float2*>(rw + 2 * t) = make_float2(acc[rt][0], acc[rt][1]);
            *reinterpret_cast<float2*>(rw + 64 + 2 * t) = make_float2(acc[rt][2], acc[rt][3]);
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
                    p.y[(size_t)(p.m0 + toks[q]) * p.N + n] = sums[q];
                }
            }
        } else {
            const uint32_t first_row = t0 / KB;
            const uint32_t slot_id = 2u * (uint32_t)u + (nb == first_row ? 0u : 1u);
            float* part = p.partial + (size_t)slot_id * 64 * 8;
#pragma unroll
            for (int q = 0; q < 4; ++q) part[rows[q] * 8 + toks[q]] = sums[q];
            // the CTA barrier orders every thread's partial before thread 0's
            // release; the acquire side is thread 0's atomic + the barrier
            named_bar_sync(1, DEC_THREADS);
            if (tid == 0) {
                const uint32_t lo = max(t0, nb * (uint32_t)KB);
                const uint32_t cnt = row_end - lo;
                const uint32_t old = atomic_add_acq_rel_gpu(&p.counters[nb], cnt);
                S.last_flag = (old + cnt == (uint32_t)KB);
            }
            named_bar_sync(1, DEC_THREADS);
            if (S.last_flag) {
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
                        p.y[(size_t)(p.m0 + toks[q]) * p.N + n] = tot[q];
                    }
                }
                if (tid == 0) p.counters[nb] = 0u;   // ready for the next launch
            }
        }
        named_bar_sync(1, DEC_THREADS);   // red[] is reused by the next row
    }
}

}  // namespace mpq
