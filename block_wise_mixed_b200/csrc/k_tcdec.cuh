// k_tcdec.cuh -- mixed-precision GEMM for mid-size batches (9..16 tokens)
// on the integer tensor cores (tcgen05.mma kind::i8).
//
// The decode formulation (k_decode.cuh) carried to tcgen05: codes are used
// as unsigned bytes and each 128-column activation slice as integers X =
// rne(x' 2^e) split into three s8 digits, so every product and sum on the
// tensor core is exact and the zero point is removed exactly per block row.
// Per 128-wide k block of a 128-row tile (two 64-row block rows):
//   A = the tile's codes expanded to bytes in natural column order (written
//       by the worker warps into the K-major 128B-swizzled operand),
//   B = the three digits of every token's slice (N = 3 MP rows, digit-major,
//       written in the same layout by k_xprep_tcdec and fetched whole),
//   D = C_d[row][token] (s32, in TMEM; two buffers).
// The worker warps (WPQ per TMEM lane quadrant; thread = weight row; each
// warp 1/WPQ of the row's codes and of the tokens) expand k block a and then
// read k block a-1's accumulator:
//   E_d = C_d - z T_d,  V = E_0 + 256 E_1 + 65536 E_2 = sum (q - z) X,
//   acc[m] += s * F_m * V          (fp32, k blocks in order).
// Every weight is read once for all tokens (TileQuant abstract: compact
// buffers reused by native integer computation with local accumulation;
// the RTN blocks of the ScaleBITS summary, "Approach" / "Key results").
//
// Roles: warp 0 copies the codes (1-D bulk copies into code stages), the
// last warp the activation records (one bulk copy per k block, after the
// prologue kernel), warp 1 allocates TMEM and issues the MMAs (one thread),
// the warps in between expand and accumulate.  Measured on B200: faster
// than the dequantizing fp16 kernel up to 16 tokens (the 70B gate
// projection at 16 tokens 99 vs 130 us), slower above, where k_prefill
// stays in use.  16-bit passthrough blocks are not handled here (layers
// flagged MPQ_LAYER_16BIT take k_prefill).  All waits are bounded
// (MPQ_ERR_TIMEOUT), with a bounded drain of copies and MMAs in flight
// before TMEM is freed.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "k_decode.cuh"    // DEC_WAIT_NS, kWaitTest
#include "k_prefill.cuh"   // tcgen05 / TMEM helpers, PF_C_BYTES, sw128 layout
#include "k_xprep.cuh"     // xqd_integerize, xqd_digit

namespace mpq {

constexpr int TC_A_BYTES = 128 * 128;   // 128 rows x 128 codes (u8)
constexpr int TC_MP = 16;               // token columns (9..16 tokens)

// WPQ worker warps per TMEM lane quadrant: 4 with one CTA per SM (grids of
// at most one wave), 2 with two CTAs per SM (larger grids: one wave).
template <int MP, int WPQ>
struct TcCfg {
    static constexpr int CPW = 8 / WPQ;                        // 16-code chunks of a row per worker
    static constexpr int WORKERS = 4 * WPQ;                    // warps 2 .. WORKERS + 1
    static constexpr int WARPS = WORKERS + 3;
    static constexpr int THREADS = WARPS * 32;
    static constexpr int TQ = MP / WPQ;                        // tokens per worker warp
    static constexpr int NP = 3 * MP;                          // B rows: digit-major (d, token)
    static constexpr int REC = NP * 128 + MP * 16;             // record of one k block
    static constexpr int B_STRIDE = (REC + 1023) / 1024 * 1024;
    static constexpr int CTAS_PER_SM = WPQ == 2 ? 2 : 1;
    static constexpr int B_STAGES = WPQ == 2 ? 3 : 4;
    static constexpr int C_STAGES = WPQ == 2 ? 3 : 9;
    static constexpr uint32_t TMEM_COLS = 2 * NP <= 128 ? 128 : 2 * NP <= 256 ? 256 : 512;
};

template <int MP, int WPQ>
struct TcSmem {
    using Cfg = TcCfg<MP, WPQ>;
    uint8_t a[2][TC_A_BYTES];                               // 1024-aligned (offset 0)
    uint8_t b[Cfg::B_STAGES][Cfg::B_STRIDE];
    uint8_t c[Cfg::C_STAGES][PF_C_BYTES];
    uint64_t full_a[2], empty_a[2];
    uint64_t full_b[Cfg::B_STAGES], empty_b[Cfg::B_STAGES];
    uint64_t full_c[Cfg::C_STAGES], empty_c[Cfg::C_STAGES];
    uint64_t d_full[2], d_empty[2];
    uint32_t tmem_base;
    volatile int abort_flag;
    // followed by the widths of the tile's blocks: [2][KB] bytes
};

struct TcParams {
    const uint8_t* codes;
    const mpq_block* table;
    const uint16_t* scales;
    const uint16_t* zeros;
    const int32_t* row_perm;
    const uint8_t* rec;       // [KB] records of TcCfg::REC bytes (k_xprep_tcdec)
    float* y;                 // [M][N]
    uint32_t* err;
    int N, K, NB, KB, M;
};

// kind::i8 instruction descriptor: D = S32, A = U8, B = S8, both K-major.
__device__ __forceinline__ constexpr uint32_t umma_idesc_i8(int M, int N) {
    return (2u << 4) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 16 consecutive 32-bit columns of this warp's TMEM lanes (no wait).
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Codes of one 16-code chunk (codes 16c .. 16c+15 of a row) as four words of
// bytes in natural order, from the row's p-bit piece words w[] (code j of
// the row in word j / (32/p) at bit (j % (32/p)) p).
// ---------------------------------------------------------------------------
template <int P>
__device__ __forceinline__ void expand_chunk(const uint32_t* w, int c, uint32_t (&o)[4]) {
    if (P == 1) {
        // word c/2 holds codes 32(c/2) .. +31; nibble i = codes 4i .. 4i+3
        const uint32_t x = w[c >> 1] >> (16 * (c & 1));
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = (((x >> (4 * i)) & 0xFu) * 0x00204081u) & 0x01010101u;
    } else if (P == 2) {
        // word c holds codes 16c .. +15; a_s byte k = code 4k + s
        const uint32_t x = w[c];
        const uint32_t a0 = x & 0x03030303u, a1 = (x >> 2) & 0x03030303u;
        const uint32_t a2 = (x >> 4) & 0x03030303u, a3 = (x >> 6) & 0x03030303u;
        const uint32_t A = __byte_perm(a0, a1, 0x5140), B = __byte_perm(a2, a3, 0x5140);
        const uint32_t A2 = __byte_perm(a0, a1, 0x7362), B2 = __byte_perm(a2, a3, 0x7362);
        o[0] = __byte_perm(A, B, 0x5410);
        o[1] = __byte_perm(A, B, 0x7632);
        o[2] = __byte_perm(A2, B2, 0x5410);
        o[3] = __byte_perm(A2, B2, 0x7632);
    } else if (P == 4) {
        // words 2c, 2c+1 hold codes 16c .. +15 as nibbles
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t x = w[2 * c + h];
            const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;
            o[2 * h] = __byte_perm(lo, hi, 0x5140);
            o[2 * h + 1] = __byte_perm(lo, hi, 0x7362);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = w[4 * c + i];
    }
}

// Codes 16 CPW sub .. of row rr of a block of width B (payload in shared
// memory) into row r of the A tile: code bytes in natural column order,
// chunks CPW sub .. CPW sub + CPW - 1 at their 128B-swizzle positions.
template <int B, int TC_CPW>
__device__ __forceinline__ void expand_row(const uint8_t* payload, int rr, int sub, uint8_t* a_tile, int r) {
    constexpr int P0 = (B == 3) ? 2 : (B == 5 || B == 6) ? 4 : B;
    constexpr int P1 = (B == 3 || B == 5) ? 1 : (B == 6) ? 2 : 0;
    constexpr int WL = (TC_CPW * P0 + 1) / 2;          // piece words of the part (P = 1, CPW = 2: one)
    constexpr int WH = P1 ? (TC_CPW * P1 + 1) / 2 : 1;
    uint32_t wl[WL], wh[WH];
    {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(payload + rr * 16 * P0) + WL * sub;
#pragma unroll
        for (int i = 0; i < WL; ++i) wl[i] = src[i];
    }
    if (P1) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(payload + 64 * 16 * P0 + rr * 16 * P1) + WH * sub;
#pragma unroll
        for (int i = 0; i < WH; ++i) wh[i] = src[i];
    }
    uint8_t* row = a_tile + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
    for (int c = 0; c < TC_CPW; ++c) {
        uint32_t o[4];
        expand_chunk<P0>(wl, c, o);
        if (P1) {
            uint32_t hh[4];
            expand_chunk<P1>(wh, c, hh);
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] += hh[i] << P0;   // q = lo | hi << width(lo), bytewise
        }
        *reinterpret_cast<uint4*>(row + (((TC_CPW * sub + c) ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

template <int TC_CPW>
__device__ __forceinline__ void zero_row(uint8_t* a_tile, int r, int sub) {
    uint8_t* row = a_tile + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
    for (int c = 0; c < TC_CPW; ++c)
        *reinterpret_cast<uint4*>(row + (((TC_CPW * sub + c) ^ (r & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
}

// N consecutive 32-bit columns (N = 4, 8, 16 or 32) of this warp's TMEM
// lanes (no wait).
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 4 || N == 8 || N == 16 || N == 32, "TMEM load width");
    if constexpr (N == 32) {
        uint32_t lo[16], hi[16];
        tmem_ld16_nowait(taddr, lo);
        tmem_ld16_nowait(taddr + 16u, hi);
#pragma unroll
        for (int i = 0; i < 16; ++i) { r[i] = lo[i]; r[16 + i] = hi[i]; }
    } else if constexpr (N == 16) {
        tmem_ld16_nowait(taddr, r);
    } else if constexpr (N == 8) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                       "=r"(r[7])
                     : "r"(taddr));
    } else {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                     : "r"(taddr));
    }
}

// ---------------------------------------------------------------------------
// Activation records: record kb = [NP rows][128] s8 digits (row d MP + m =
// digit d of token m's slice kb, natural column order, 128B swizzle), then
// per token (T_0, T_1, T_2, F) -- zeros for the padding tokens m >= M.
// One warp per (k block, token); the lane holds columns 4 lane .. +3.
// ---------------------------------------------------------------------------
struct XprepTcParams {
    const uint16_t* x;        // bf16 bits, M x K
    const int32_t* col_perm;  // [K] or null
    uint8_t* rec;
    int M, K, MP, NP, REC;
};

__global__ void __launch_bounds__(XPREP_THREADS) k_xprep_tcdec(XprepTcParams p) {
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int KB = p.K / 128;
    const int item = blockIdx.x * (XPREP_THREADS / 32) + (threadIdx.x >> 5);   // = kb * MP + m
    if (item >= KB * p.MP) {
        pdl_wait();
        return;
    }
    const int kb = item / p.MP, m = item % p.MP;
    const int c0 = kb * 128 + 4 * lane;
    int4 cp = make_int4(c0, c0 + 1, c0 + 2, c0 + 3);
    if (p.col_perm) cp = *reinterpret_cast<const int4*>(p.col_perm + c0);
    pdl_wait();   // the kernel before may still read the records or write x
    int X[4] = {0, 0, 0, 0}, T[3] = {0, 0, 0};
    float F = 0.f;
    if (m < p.M) {
        const uint16_t* xr = p.x + (size_t)m * p.K;
        const int cs[4] = {cp.x, cp.y, cp.z, cp.w};
        float v[4];
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) v[e4] = __uint_as_float(((uint32_t)xr[cs[e4]]) << 16);
        xqd_integerize(v, X, T, F);
    }
    uint8_t* rec = p.rec + (size_t)kb * p.REC;
    // column 4 lane + e4: chunk lane / 4, byte 4 (lane % 4) + e4 of the row
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        const int n = d * p.MP + m;
        uint32_t word = 0;
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) word |= ((uint32_t)xqd_digit(X[e4], d) & 0xFFu) << (8 * e4);
        uint8_t* row = rec + (n >> 3) * 1024 + (n & 7) * 128;
        *reinterpret_cast<uint32_t*>(row + (((lane >> 2) ^ (n & 7)) << 4) + 4 * (lane & 3)) = word;
    }
    if (lane == 0)
        *reinterpret_cast<uint4*>(rec + p.NP * 128 + 16 * m) =
            make_uint4((uint32_t)T[0], (uint32_t)T[1], (uint32_t)T[2], __float_as_uint(F));
}

// ---------------------------------------------------------------------------
// The kernel: one CTA per 128-row tile, all k blocks.
// ---------------------------------------------------------------------------
template <int MP, int WPQ>
__global__ void __launch_bounds__(TcCfg<MP, WPQ>::THREADS, TcCfg<MP, WPQ>::CTAS_PER_SM)
k_tcdec(TcParams p) {
    using Cfg = TcCfg<MP, WPQ>;
    constexpr int TC_WORKERS = Cfg::WORKERS, TC_WARPS = Cfg::WARPS, TC_THREADS = Cfg::THREADS;
    constexpr int TC_CPW = Cfg::CPW;
    constexpr int NP = Cfg::NP, BS = Cfg::B_STAGES, CS = Cfg::C_STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    pdl_launch_dependents();
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    TcSmem<MP, WPQ>& S = *reinterpret_cast<TcSmem<MP, WPQ>*>(base);
    uint8_t* tbits = base + sizeof(TcSmem<MP, WPQ>);   // [2][KB] block widths

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nb0 = 2 * (int)blockIdx.x;
    const int KB = p.KB;
    for (int i = tid; i < 2 * KB; i += TC_THREADS) {
        const int h = i / KB, kb = i % KB;
        tbits[i] = nb0 + h < p.NB ? (uint8_t)p.table[(size_t)(nb0 + h) * KB + kb].bits : (uint8_t)0;
    }
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&S.full_a[s], TC_WORKERS);
            mbar_init(&S.empty_a[s], 1);     // MMA commit
            mbar_init(&S.d_full[s], 1);      // MMA commit
            mbar_init(&S.d_empty[s], TC_WORKERS);
        }
        for (int s = 0; s < BS; ++s) {
            mbar_init(&S.full_b[s], 1);
            mbar_init(&S.empty_b[s], TC_WORKERS);
        }
        for (int s = 0; s < CS; ++s) {
            mbar_init(&S.full_c[s], 1);
            mbar_init(&S.empty_c[s], TC_WORKERS);
        }
        S.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&S.tmem_base)),
                     "r"(Cfg::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = S.tmem_base;

    auto timed_out = [&]() {
        set_error(p.err, MPQ_ERR_TIMEOUT);
        S.abort_flag = 1;
    };
    auto bits_of = [&](int h, int kb) -> uint32_t { return tbits[h * KB + kb]; };
    int c_armed = 0, b_armed = 0;   // stages armed by the copy producers (lane 0)
    int mma_units = 0;              // units whose MMAs were issued (MMA thread)

    if (warp == 0) {
        // ------------------------------ codes ---------------------------------
        if (lane == 0) {
            int a = 0;
            for (int kb = 0; kb < KB && !S.abort_flag; ++kb) {
                const uint32_t b0 = bits_of(0, kb), b1 = bits_of(1, kb);
                if ((b0 | b1) == 0) continue;
                if (b0 > 8 || b1 > 8) {   // a 16-bit block: this kernel is not built for them
                    set_error(p.err, MPQ_ERR_BITS);
                    S.abort_flag = 1;
                    break;
                }
                const int sc = a % CS;
                if (!mbar_wait_bounded(&S.empty_c[sc], ((uint32_t)(a / CS) & 1u) ^ 1u, DEC_WAIT_NS)) {
                    timed_out();
                    break;
                }
                const uint32_t bytes = (b0 ? 1024u * b0 + 256u : 0u) + (b1 ? 1024u * b1 + 256u : 0u);
                mbar_arrive_expect_tx(&S.full_c[sc], bytes);
                c_armed = a + 1;
                if (kWaitTest) break;   // wait-test build: armed, no copy
                uint8_t* cst = S.c[sc];
                for (int h = 0; h < 2; ++h) {
                    const uint32_t b = h ? b1 : b0;
                    if (!b) continue;
                    const mpq_block e = p.table[(size_t)(nb0 + h) * KB + kb];
                    bulk_g2s(cst + h * 8192, p.codes + e.code_off, 1024u * b, &S.full_c[sc]);
                    bulk_g2s(cst + 16384 + h * 256, p.scales + e.sz_off, 128u, &S.full_c[sc]);
                    bulk_g2s(cst + 16384 + h * 256 + 128, p.zeros + e.sz_off, 128u, &S.full_c[sc]);
                }
                ++a;
            }
        }
        __syncwarp();
    } else if (warp == TC_WARPS - 1) {
        // --------------------------- activation records ------------------------
        pdl_wait();   // the records come from the prologue kernel
        if (lane == 0 && !kWaitTest) {
            int a = 0;
            for (int kb = 0; kb < KB && !S.abort_flag; ++kb) {
                if ((bits_of(0, kb) | bits_of(1, kb)) == 0) continue;
                const int sb = a % BS;
                if (!mbar_wait_bounded(&S.empty_b[sb], ((uint32_t)(a / BS) & 1u) ^ 1u, DEC_WAIT_NS)) {
                    timed_out();
                    break;
                }
                mbar_arrive_expect_tx(&S.full_b[sb], (uint32_t)Cfg::REC);
                b_armed = a + 1;
                bulk_g2s(S.b[sb], p.rec + (size_t)kb * Cfg::REC, (uint32_t)Cfg::REC, &S.full_b[sb]);
                ++a;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ----------------------------
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_i8(128, NP);
            int a = 0;
            for (int kb = 0; kb < KB && !S.abort_flag; ++kb) {
                if ((bits_of(0, kb) | bits_of(1, kb)) == 0) continue;
                const int s2 = a & 1, sb = a % BS;
                const uint32_t ph2 = (uint32_t)(a >> 1) & 1u;
                bool ok = mbar_wait_bounded(&S.full_a[s2], ph2, DEC_WAIT_NS);
                ok = ok && mbar_wait_bounded(&S.full_b[sb], (uint32_t)(a / BS) & 1u, DEC_WAIT_NS);
                ok = ok && mbar_wait_bounded(&S.d_empty[s2], ph2 ^ 1u, DEC_WAIT_NS);
                if (!ok) { timed_out(); break; }
                tc_fence_after();
                const uint32_t a_base = smem_u32(S.a[s2]), b_base = smem_u32(S.b[sb]);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)   // K = 32 bytes per MMA
                    umma_i8_ss(tmem_d + (uint32_t)(s2 * NP), umma_smem_desc_sw128(a_base + (uint32_t)(kk * 32)),
                               umma_smem_desc_sw128(b_base + (uint32_t)(kk * 32)), idesc, kk > 0 ? 1u : 0u);
                umma_commit(&S.empty_a[s2]);
                umma_commit(&S.d_full[s2]);
                ++a;
                mma_units = a;
            }
        }
        __syncwarp();
    } else {
        // --------------------- workers: expand, then accumulate ------------------
        const int quad = warp & 3;               // TMEM lane quadrant
        const int sub = (warp - 2) >> 2;         // which part: codes 16 CPW sub .., tokens TQ sub ..
        constexpr int TQ = Cfg::TQ;
        const int m0 = sub * TQ;
        const int r = quad * 32 + lane;          // tile row = TMEM lane
        const int h = r >> 6, rr = r & 63;
        float acc[TQ];
#pragma unroll
        for (int j = 0; j < TQ; ++j) acc[j] = 0.f;
        float s_prev = 0.f;
        int z_prev = 0, a = 0, kb_prev = -1;
        bool ok = true;
        // accumulator of unit `u` (its k block's records in B stage u % BS),
        // tokens m0 .. m0 + TQ - 1
        auto accumulate = [&](int u, float s, int z) {
            const int s2 = u & 1, sb = u % BS;
            // the MMA's completion, and the records' arrival (the digit sums
            // and F are read from the same stage)
            bool w = !S.abort_flag && mbar_wait_bounded(&S.d_full[s2], (uint32_t)(u >> 1) & 1u, DEC_WAIT_NS);
            w = w && mbar_wait_bounded(&S.full_b[sb], (uint32_t)(u / BS) & 1u, DEC_WAIT_NS);
            w = __all_sync(0xffffffffu, w);   // tcgen05.ld is .sync.aligned
            if (!w) {
                if (lane == 0 && !S.abort_flag) timed_out();
                return false;
            }
            if (m0 < p.M) {
                tc_fence_after();
                const uint8_t* tf = S.b[sb] + NP * 128;
                const uint32_t tbase = tmem_d + ((uint32_t)(quad * 32) << 16) + (uint32_t)(s2 * NP + m0);
                uint32_t c0[TQ], c1[TQ], c2[TQ];
                tmem_ld_cols<TQ>(tbase, c0);
                tmem_ld_cols<TQ>(tbase + (uint32_t)MP, c1);
                tmem_ld_cols<TQ>(tbase + (uint32_t)(2 * MP), c2);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < TQ; ++j) {
                    const int4 t4 = *reinterpret_cast<const int4*>(tf + 16 * (m0 + j));
                    const int e0 = (int)c0[j] - z * t4.x, e1 = (int)c1[j] - z * t4.y, e2 = (int)c2[j] - z * t4.z;
                    const float v = fmaf(65536.f, (float)e2, (float)(e0 + 256 * e1));
                    acc[j] = fmaf(s * __int_as_float(t4.w), v, acc[j]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&S.d_empty[s2]);
                mbar_arrive(&S.empty_b[sb]);
            }
            return true;
        };
        for (int kb = 0; kb < KB && ok; ++kb) {
            const uint32_t b0 = bits_of(0, kb), b1 = bits_of(1, kb);
            if ((b0 | b1) == 0) continue;
            if (S.abort_flag) { ok = false; break; }
            const int sc = a % CS, s2 = a & 1;
            bool w = mbar_wait_bounded(&S.full_c[sc], (uint32_t)(a / CS) & 1u, DEC_WAIT_NS);
            w = w && mbar_wait_bounded(&S.empty_a[s2], ((uint32_t)(a >> 1) & 1u) ^ 1u, DEC_WAIT_NS);
            if (!__all_sync(0xffffffffu, w)) { if (lane == 0) timed_out(); ok = false; break; }
            const uint32_t b = h ? b1 : b0;
            const uint8_t* cst = S.c[sc];
            uint8_t* a_tile = S.a[s2];
            float s_cur = 0.f;
            int z_cur = 0;
            if (b == 0 || b > 8) {
                zero_row<TC_CPW>(a_tile, r, sub);
            } else {
                const __half* scz = reinterpret_cast<const __half*>(cst + 16384 + h * 256);
                s_cur = __half2float(scz[rr]);
                z_cur = (int)__half2float(scz[64 + rr]);
                const uint8_t* pay = cst + h * 8192;
                switch (b) {
                    case 1: expand_row<1, TC_CPW>(pay, rr, sub, a_tile, r); break;
                    case 2: expand_row<2, TC_CPW>(pay, rr, sub, a_tile, r); break;
                    case 3: expand_row<3, TC_CPW>(pay, rr, sub, a_tile, r); break;
                    case 4: expand_row<4, TC_CPW>(pay, rr, sub, a_tile, r); break;
                    case 5: expand_row<5, TC_CPW>(pay, rr, sub, a_tile, r); break;
                    case 6: expand_row<6, TC_CPW>(pay, rr, sub, a_tile, r); break;
                    default: expand_row<8, TC_CPW>(pay, rr, sub, a_tile, r); break;
                }
            }
            fence_proxy_async_smem();   // generic-proxy writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&S.full_a[s2]);
                mbar_arrive(&S.empty_c[sc]);
            }
            if (kb_prev >= 0 && !accumulate(a - 1, s_prev, z_prev)) { ok = false; break; }
            s_prev = s_cur;
            z_prev = z_cur;
            kb_prev = kb;
            ++a;
        }
        if (ok && kb_prev >= 0) ok = accumulate(a - 1, s_prev, z_prev);
        // y[m][row_perm[i]] = acc
        const int i = nb0 * 64 + r;
        if (ok && i < p.N) {
            const int n = p.row_perm ? p.row_perm[i] : i;
#pragma unroll
            for (int j = 0; j < TQ; ++j)
                if (m0 + j < p.M) p.y[(size_t)(m0 + j) * p.N + n] = acc[j];
        }
    }
    // after an abort, copies and MMAs may still be in flight into this CTA's
    // shared memory and TMEM: wait for them (bounded) before the TMEM is freed
    __syncthreads();
    if (S.abort_flag && lane == 0) {
        if (warp == 0)
            for (int i = max(0, c_armed - CS); i < c_armed; ++i)
                mbar_wait_bounded(&S.full_c[i % CS], (uint32_t)(i / CS) & 1u, DEC_WAIT_NS);
        if (warp == TC_WARPS - 1)
            for (int i = max(0, b_armed - BS); i < b_armed; ++i)
                mbar_wait_bounded(&S.full_b[i % BS], (uint32_t)(i / BS) & 1u, DEC_WAIT_NS);
        if (warp == 1 && mma_units > 0)   // the last commit covers every MMA issued
            mbar_wait_bounded(&S.d_full[(mma_units - 1) & 1], (uint32_t)((mma_units - 1) >> 1) & 1u, DEC_WAIT_NS);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d),
                     "r"(Cfg::TMEM_COLS)
                     : "memory");
    }
}

}  // namespace mpq
