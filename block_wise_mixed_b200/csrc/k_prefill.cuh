// k_prefill.cuh -- tensor-core (tcgen05 / TMEM) mixed-precision GEMM for
// larger token counts.
//
// D[i][m] = sum_k w_hat'[i][k] * x'[m][k] for a tile of 128 weight rows
// (two 64-row block rows) and BN = 128 or 256 tokens, over all k blocks or
// one split of them; y[m][row_perm[i]] = D * tok_scale[m] (the splits summed
// and the rows reordered by k_finish_rows).
// The blocks' dequantization is the RTN of the ScaleBITS summary ("Approach",
// "Key results"); TileQuant's abstract describes the same split -- compact
// per-tile buffers expanded next to the 16-bit tensor-core computation.
//
// Roles (19 warps):
//   warp 0     producer of the codes: 1-D bulk copies of the two blocks'
//              payloads and scales/zeros per 128-wide k block, as far ahead as
//              the code stages allow.
//   warp 18    producer of the activations: the x' tile of each k block (TMA
//              tensor copy, 128B swizzle) into its own stages.
//   warp 1     allocates TMEM and issues tcgen05.mma (one elected thread).
//   warps 2-17 dequantize: each thread expands a quarter of one weight row's
//              128 codes into fp16 w_hat = (q - z) * s, written straight
//              into the K-major 128B-swizzled shared-memory A operand (four
//              warps per TMEM lane quadrant keep the schedulers busy); after
//              the last k block they read the fp32 accumulator out of TMEM
//              and write y' in W' row order (or the split's partial sums).
// A k block whose two blocks are both 0-bit is skipped by every role (no
// bytes, no MMA); a 0-bit block next to a non-zero one contributes zero rows.
// The operands are fp16 (A = dequantized weights, B = x' scaled per token by a
// power of two); accumulation is fp32 in TMEM.
//
// The x' layout (written by k_xprep, XP_PREFILL) permutes each 128-column
// group so that MMA k = 2*(4i+j)+h holds column 8i+j+4h: the extraction emits
// the pair (8i+j, 8i+j+4) in one register, so a group of 8 codes becomes one
// 16-byte chunk of A.
//
// All waits are bounded (MPQ_ERR_TIMEOUT); the kernel then winds down.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "dequant_magic.cuh"
#include "k_decode.cuh"       // DEC_WAIT_NS

namespace mpq {

constexpr int PF_DQ_WARPS = 16;                  // warps 2 .. 17
constexpr int PF_WARPS = PF_DQ_WARPS + 3;
constexpr int PF_THREADS = PF_WARPS * 32;
constexpr int PF_BM = 128;       // weight rows per tile (2 block rows)
constexpr int PF_A_BYTES = PF_BM * 256;           // 128 rows x 128 fp16
constexpr int PF_C_BYTES = 2 * 8192 + 4 * 128;    // two payloads + 2 x (scales, zeros)

// Tokens per tile: 128, or 256 for large batches (each dequantized weight
// tile then feeds twice the tensor-core work).  Activation stages hold half
// a k block (64 columns) so that both fit in shared memory.
//
// With 256 tokens a k block's MMAs take about as long as its dequantization,
// so three weight stages keep the dequantizing warps one k block further
// ahead (two code stages make the room).
template <int BN>
struct PfCfg {
    static constexpr int A_STAGES = BN == 256 ? 3 : 2;   // dequantized weight tiles
    static constexpr int B_STAGES = BN == 256 ? 3 : 4;   // half-k-block activation stages (from L2)
    static constexpr int B_BYTES = BN * 128;              // BN tokens x 64 fp16
    static constexpr int C_STAGES = BN == 256 ? 2 : 5;   // packed codes (from HBM)
    static constexpr uint32_t TMEM_COLS = BN;             // fp32 accumulator columns
};

template <int BN>
struct PrefillSmem {
    uint8_t a[PfCfg<BN>::A_STAGES][PF_A_BYTES];    // 1024-aligned (offset 0)
    uint8_t b[PfCfg<BN>::B_STAGES][PfCfg<BN>::B_BYTES];
    uint8_t c[PfCfg<BN>::C_STAGES][PF_C_BYTES];
    uint64_t full_a[PfCfg<BN>::A_STAGES];
    uint64_t empty_a[PfCfg<BN>::A_STAGES];
    uint64_t full_b[PfCfg<BN>::B_STAGES];
    uint64_t empty_b[PfCfg<BN>::B_STAGES];
    uint64_t full_c[PfCfg<BN>::C_STAGES];
    uint64_t empty_c[PfCfg<BN>::C_STAGES];
    uint64_t d_full;
    uint32_t tmem_base;
    volatile int abort_flag;
    // followed by the widths of the tile's blocks: [2][KB] bytes
};

struct PrefillParams {
    const uint8_t* codes;
    const mpq_block* table;
    const uint16_t* scales;
    const uint16_t* zeros;
    const int32_t* row_perm;
    const float* tok_scale;   // [M]
    float* out;               // output base (see out_scatter)
    int out_scatter;          // 1: out = y, rows scattered through row_perm;
                              // 0: out = [split][M][N] in W' row order (k_finish_rows
                              //    adds the splits and applies row_perm)
    uint32_t* err;
    int N, K, NB, KB, M;
    int tiles_n;              // ceil(NB / 2)
    int tiles_m;              // ceil(M / BN)
    int kb_per_split;         // k blocks per CTA (split-K when < KB)
};

__device__ __forceinline__ uint64_t umma_smem_desc_sw128(uint32_t saddr) {
    // K-major, 128-byte swizzle: 8-row groups 1024 B apart (SBO), LBO unused
    // (1), descriptor version 1, layout type 2 = SWIZZLE_128B.
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// kind::f16 instruction descriptor: D = F32, A = B = F16, both K-major.
__device__ __forceinline__ constexpr uint32_t umma_idesc_f16(int M, int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// 32 consecutive fp32 columns of this warp's TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Offset of the 16-byte chunk holding K elements 8*kc..8*kc+7 of row r in a
// 128-row x 128-K tile stored K-major with 128B swizzle (two 64-K halves).
__device__ __forceinline__ uint32_t sw128_chunk(int r, int kc) {
    return (uint32_t)((kc >> 3) * (PF_BM * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                      (((kc & 7) ^ (r & 7)) << 4));
}

// A 16-bit passthrough block (TileQuant abstract: the highest-scoring tiles
// stay at 16 bits): groups [g0, g0+4) of row rr, read straight from the
// block's bf16 payload in global memory (16 bytes per group), converted to
// fp16 (exact for |w| in the fp16 normal range; the pack limits |w| to
// 65504) and stored in the tile's column order.
__device__ __forceinline__ void passthrough_row_part(const uint8_t* blk, int rr, int g0, uint8_t* a_tile, int r) {
    const int sw = (g0 & 8) ? 2 : 0;
    uint4 v[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi)
        v[gi] = __ldg(reinterpret_cast<const uint4*>(blk + rr * 256 + 16 * (g0 + (gi ^ sw))));
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
        const uint32_t u[4] = {v[gi].x, v[gi].y, v[gi].z, v[gi].w};
        float f[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            f[2 * c] = __uint_as_float(u[c] << 16);
            f[2 * c + 1] = __uint_as_float(u[c] & 0xFFFF0000u);
        }
        // position pair j of the chunk holds columns (j, j + 4)
        uint4 w;
        w.x = h2_bits(__floats2half2_rn(f[0], f[4]));
        w.y = h2_bits(__floats2half2_rn(f[1], f[5]));
        w.z = h2_bits(__floats2half2_rn(f[2], f[6]));
        w.w = h2_bits(__floats2half2_rn(f[3], f[7]));
        *reinterpret_cast<uint4*>(a_tile + sw128_chunk(r, g0 + (gi ^ sw))) = w;
    }
}

// Dequantizes groups [g0, g0+4) (8 codes each) of row rr of one block of
// width B into the A tile row r: w_hat = (q - z) * s in fp16.  A warp covers
// 8 whole rows (lane = row * 4 + quarter), so the lanes' code bytes are one
// contiguous run of shared memory (one conflict-free vector load each).  The
// quarters 2 and 3 take their groups in the order 2, 3, 0, 1: chunks kc and
// kc + 8 of a row share a bank group under the 128B swizzle, and with this
// order the 8 lanes of each store phase (two rows x four quarters) hit 8
// different bank groups.
template <int P>
__device__ __forceinline__ void load_part(const uint8_t* p, uint32_t (&w)[P]) {
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

template <int B>
__device__ __forceinline__ void dequant_row_part(const uint8_t* payload, const __half* scz, int rr,
                                                 int g0, uint8_t* a_tile, int r) {
    constexpr int P0 = (B == 3) ? 2 : (B == 5 || B == 6) ? 4 : B;
    constexpr int P1 = (B == 3 || B == 5) ? 1 : (B == 6) ? 2 : 0;
    const __half sh = scz[rr];
    const uint32_t z2 = __byte_perm((uint32_t)__half_as_ushort(scz[64 + rr]), 0u, 0x1010);
    const __half2 s2 = __half2half2(sh);
    uint32_t k[4];
    zero_consts<P0>(z2, k);
    // the part's 32 codes: 4*P0 bytes of the low piece, 4*P1 of the high one
    uint32_t d[P0];
    load_part<P0>(payload + rr * 16 * P0 + g0 * P0, d);
    uint32_t e[P1 > 0 ? P1 : 1];
    if (P1 == 1) e[0] = *reinterpret_cast<const uint32_t*>(payload + 64 * 16 * P0 + rr * 16 + g0);
    if (P1 == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(payload + 64 * 16 * P0 + rr * 32 + 2 * g0);
        e[0] = v.x; e[P1 > 1 ? 1 : 0] = v.y;
    }
    // group order: step gi takes group gi ^ sw (sw = 2 for quarters 2, 3)
    const int sw = (g0 & 8) ? 2 : 0;
    if (P0 == 4 || P0 == 8) {
        constexpr int H = P0 / 2;   // words of two groups
#pragma unroll
        for (int i = 0; i < H; ++i) {
            const uint32_t lo = d[i], hi = d[i + H];
            d[i] = sw ? hi : lo;
            d[i + H] = sw ? lo : hi;
        }
    } else if (P0 == 2) {
        const uint32_t lo = d[0], hi = d[P0 > 1 ? 1 : 0];
        d[0] = sw ? hi : lo;
        d[P0 > 1 ? 1 : 0] = sw ? lo : hi;
    }
    if (P1 == 2) {
        const uint32_t lo = e[0], hi = e[P1 > 1 ? 1 : 0];
        e[0] = sw ? hi : lo;
        e[P1 > 1 ? 1 : 0] = sw ? lo : hi;
    }
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
        const int g = gi ^ sw;   // the group this step takes
        uint32_t o[4];
        if (P0 == 4) {
            ext4(d[gi], k[0], k[1], o);
        } else if (P0 == 8) {
            ext8(d[2 * gi], d[2 * gi + 1], k[0], o);
        } else if (P0 == 2) {
            ext2(d[gi >> 1], (gi & 1) ? 0x4342 : 0x4140, k, o);
        } else {
            ext1(d[0], g | (4 << 4) | (g << 8) | (4 << 12), k, o);
        }
        if (P1 > 0) {
            uint32_t h[4];
            if (P1 == 1) ext1_hi<P0>(e[0], g | (4 << 4) | (g << 8) | (4 << 12), h);
            else ext2_hi(e[gi >> 1], (gi & 1) ? 0x4342 : 0x4140, h);
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = h2_bits(__hadd2(bits_h2(o[j]), bits_h2(h[j])));
        }
        uint4 w;
        w.x = h2_bits(__hmul2(bits_h2(o[0]), s2));
        w.y = h2_bits(__hmul2(bits_h2(o[1]), s2));
        w.z = h2_bits(__hmul2(bits_h2(o[2]), s2));
        w.w = h2_bits(__hmul2(bits_h2(o[3]), s2));
        *reinterpret_cast<uint4*>(a_tile + sw128_chunk(r, g0 + g)) = w;
    }
}

template <int BN>
__global__ void __launch_bounds__(PF_THREADS, 1)
k_prefill(PrefillParams p, const __grid_constant__ CUtensorMap tmap_x) {
    using Cfg = PfCfg<BN>;
    constexpr int PF_A_STAGES = Cfg::A_STAGES;
    constexpr int PF_C_STAGES = Cfg::C_STAGES;
    constexpr int PF_B_STAGES = Cfg::B_STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the next kernel may launch once every CTA of this grid has started; it
    // waits (griddepcontrol.wait) for this grid before touching its memory
    pdl_launch_dependents();
    // the operand tiles need 1024-byte alignment (128B swizzle atoms); pointer
    // arithmetic on smem_raw keeps the shared address space for the compiler
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    PrefillSmem<BN>& S = *reinterpret_cast<PrefillSmem<BN>*>(base);
    uint8_t* tbits = base + sizeof(PrefillSmem<BN>);   // [2][KB] block widths

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tiles = p.tiles_n * p.tiles_m;
    const int split = blockIdx.x / tiles;
    const int tile_n = (blockIdx.x % tiles) % p.tiles_n;
    const int tile_m = (blockIdx.x % tiles) / p.tiles_n;
    const int nb0 = 2 * tile_n;
    const int m0 = tile_m * BN;
    // this CTA's k blocks: [kb0, kb0 + KB) of the layer's p.KB
    const int kb0 = split * p.kb_per_split;
    const int KB = max(0, min(p.KB, kb0 + p.kb_per_split) - kb0);

    // stage the widths of this CTA's blocks: tbits[h*KB + kb]
    for (int i = tid; i < 2 * KB; i += PF_THREADS) {
        const int h = i / KB, kb = i % KB;
        const int nb = nb0 + h;
        tbits[i] = nb < p.NB ? (uint8_t)p.table[(size_t)nb * p.KB + kb0 + kb].bits : (uint8_t)0;
    }
    if (tid == 0) {
        for (int s = 0; s < PF_A_STAGES; ++s) {
            mbar_init(&S.full_a[s], PF_DQ_WARPS);
            mbar_init(&S.empty_a[s], 1);
        }
        for (int s = 0; s < PF_B_STAGES; ++s) {
            mbar_init(&S.full_b[s], 1);
            mbar_init(&S.empty_b[s], 1);
        }
        for (int s = 0; s < PF_C_STAGES; ++s) {
            mbar_init(&S.full_c[s], 1);
            mbar_init(&S.empty_c[s], PF_DQ_WARPS);
        }
        mbar_init(&S.d_full, 1);
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

    // stages armed by the two copy producers (lane 0), for the drain after an abort
    int c_armed = 0, b_armed = 0;
    if (warp == 0) {
        // -------------------- producer of the packed codes --------------------
        // runs as far ahead as the code stages allow (the weights do not
        // depend on the prologue kernel); the code and scale offsets of 32 k
        // blocks are read from the table at a time, one k block per lane
        int a = 0;
        bool stop = false;
        for (int kbb = 0; kbb < KB && !stop; kbb += 32) {
            uint32_t co0 = 0, so0 = 0, co1 = 0, so1 = 0;
            if (kbb + lane < KB) {
                const size_t e = (size_t)nb0 * p.KB + kb0 + kbb + lane;
                co0 = p.table[e].code_off; so0 = p.table[e].sz_off;
                if (nb0 + 1 < p.NB) { co1 = p.table[e + p.KB].code_off; so1 = p.table[e + p.KB].sz_off; }
            }
            const int n = min(32, KB - kbb);
            for (int j = 0; j < n; ++j) {
                const int kb = kbb + j;
                const uint32_t b0 = bits_of(0, kb), b1 = bits_of(1, kb);
                if ((b0 | b1) == 0) continue;
                const uint32_t c0 = __shfl_sync(0xffffffffu, co0, j), s0 = __shfl_sync(0xffffffffu, so0, j);
                const uint32_t c1 = __shfl_sync(0xffffffffu, co1, j), s1 = __shfl_sync(0xffffffffu, so1, j);
                bool ok = true;
                if (lane == 0) {
                    const int sc = a % PF_C_STAGES;
                    const uint32_t pc = (uint32_t)(a / PF_C_STAGES) & 1u;
                    ok = !S.abort_flag && mbar_wait_bounded(&S.empty_c[sc], pc ^ 1u, DEC_WAIT_NS);
                    if (ok) {
                        // 16-bit blocks are read by the dequantizing warps
                        // themselves: the stage carries their payload offsets
                        const uint32_t q0 = (b0 && b0 != 16) ? b0 : 0u, q1 = (b1 && b1 != 16) ? b1 : 0u;
                        const uint32_t bytes = (q0 ? 1024u * q0 + 256u : 0u) + (q1 ? 1024u * q1 + 256u : 0u);
                        uint8_t* cst = S.c[sc];
                        if (b0 == 16) *reinterpret_cast<uint32_t*>(cst + 16384) = c0;
                        if (b1 == 16) *reinterpret_cast<uint32_t*>(cst + 16384 + 256) = c1;
                        // those generic writes, and the ones of the stage's earlier
                        // uses, come before this use's bulk copies
                        fence_proxy_async_smem();
                        mbar_arrive_expect_tx(&S.full_c[sc], bytes);
                        c_armed = a + 1;
                        if (kWaitTest) {
                            // wait-test build: armed, no copy; the consumers' waits run out
                        } else if (q0) {
                            bulk_g2s(cst, p.codes + c0, 1024u * b0, &S.full_c[sc]);
                            bulk_g2s(cst + 16384, p.scales + s0, 128u, &S.full_c[sc]);
                            bulk_g2s(cst + 16384 + 128, p.zeros + s0, 128u, &S.full_c[sc]);
                        }
                        if (q1 && !kWaitTest) {
                            bulk_g2s(cst + 8192, p.codes + c1, 1024u * b1, &S.full_c[sc]);
                            bulk_g2s(cst + 16384 + 256, p.scales + s1, 128u, &S.full_c[sc]);
                            bulk_g2s(cst + 16384 + 384, p.zeros + s1, 128u, &S.full_c[sc]);
                        }
                    } else if (!S.abort_flag) {
                        timed_out();
                    }
                }
                if (!__shfl_sync(0xffffffffu, ok, 0) || kWaitTest) { stop = true; break; }
                ++a;
            }
        }
        __syncwarp();
    } else if (warp == PF_WARPS - 1) {
        // ------------------- producer of the activation tiles -----------------
        pdl_wait();   // x' comes from the prologue kernel
        if (lane == 0 && !kWaitTest) {
            int bq = 0;   // half-k-block activation tiles issued
            for (int kb = 0; kb < KB && !S.abort_flag; ++kb) {
                if ((bits_of(0, kb) | bits_of(1, kb)) == 0) continue;
                for (int hh = 0; hh < 2; ++hh, ++bq) {
                    const int s = bq % PF_B_STAGES;
                    const uint32_t ps = (uint32_t)(bq / PF_B_STAGES) & 1u;
                    if (!mbar_wait_bounded(&S.empty_b[s], ps ^ 1u, DEC_WAIT_NS)) { timed_out(); break; }
                    mbar_arrive_expect_tx(&S.full_b[s], (uint32_t)Cfg::B_BYTES);
                    b_armed = bq + 1;
                    tma_load_2d(S.b[s], &tmap_x, (kb0 + kb) * 128 + 64 * hh, m0, &S.full_b[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ----------------------------
        const uint32_t idesc = umma_idesc_f16(PF_BM, BN);
        int a = 0;
        if (lane == 0) {
            bool stop = false;
            for (int kb = 0; kb < KB && !S.abort_flag && !stop; ++kb) {
                if ((bits_of(0, kb) | bits_of(1, kb)) == 0) continue;
                const int sa = a % PF_A_STAGES;
                const uint32_t pa = (uint32_t)(a / PF_A_STAGES) & 1u;
                if (!mbar_wait_bounded(&S.full_a[sa], pa, DEC_WAIT_NS)) { timed_out(); break; }
                const uint32_t a_base = smem_u32(S.a[sa]);
                for (int hh = 0; hh < 2; ++hh) {
                    const int bq = 2 * a + hh;
                    const int sb = bq % PF_B_STAGES;
                    const uint32_t pb = (uint32_t)(bq / PF_B_STAGES) & 1u;
                    if (!mbar_wait_bounded(&S.full_b[sb], pb, DEC_WAIT_NS)) { timed_out(); stop = true; break; }
                    tc_fence_after();
                    const uint32_t b_base = smem_u32(S.b[sb]);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        // A: the 64-column half hh of the k block; B: this half's stage
                        const uint32_t off = (uint32_t)(hh * (PF_BM * 128) + kk * 32);
                        umma_f16_ss(tmem_d, umma_smem_desc_sw128(a_base + off),
                                    umma_smem_desc_sw128(b_base + (uint32_t)(kk * 32)), idesc,
                                    (a > 0 || hh > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&S.empty_b[sb]);
                }
                if (stop) break;
                umma_commit(&S.empty_a[sa]);
                ++a;
            }
            if (a > 0) umma_commit(&S.d_full);
            else mbar_arrive(&S.d_full);
        }
        __syncwarp();
    } else {
        // ---------------------- dequantize, then epilogue ----------------------
        const int dw = warp - 2;                 // 0..15
        // dequantization: rows 8*dw .. 8*dw+7, lane = row * 4 + quarter
        const int r = 8 * dw + (lane >> 2);
        const int h = r >> 6, rr = r & 63;
        const int g0 = 4 * (lane & 3);           // the quarter's first group of 8 codes
        // epilogue: TMEM lane quadrant of this warp, and which 32 tokens it takes
        const int quad = warp & 3;
        const int part = dw >> 2;
        int a = 0;
        bool any = false;
        for (int kb = 0; kb < KB; ++kb) {
            const uint32_t b0 = bits_of(0, kb), b1 = bits_of(1, kb);
            if ((b0 | b1) == 0) continue;
            any = true;
            if (S.abort_flag) break;
            const int sc = a % PF_C_STAGES;
            const uint32_t pc = (uint32_t)(a / PF_C_STAGES) & 1u;
            const int s = a % PF_A_STAGES;
            const uint32_t ps = (uint32_t)(a / PF_A_STAGES) & 1u;
            bool ok = mbar_wait_bounded(&S.full_c[sc], pc, DEC_WAIT_NS);
            ok = ok && mbar_wait_bounded(&S.empty_a[s], ps ^ 1u, DEC_WAIT_NS);
            if (!__all_sync(0xffffffffu, ok)) { if (lane == 0) timed_out(); break; }
            const uint32_t b = h ? b1 : b0;
            uint8_t* a_tile = S.a[s];
            const uint8_t* cst = S.c[sc];
            const __half* scz = reinterpret_cast<const __half*>(cst + 16384 + h * 256);
            switch (b) {
                case 0: {
                    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int gi = 0; gi < 4; ++gi)
                        *reinterpret_cast<uint4*>(a_tile + sw128_chunk(r, g0 + gi)) = zero;
                    break;
                }
                case 16:
                    passthrough_row_part(p.codes + *reinterpret_cast<const uint32_t*>(cst + 16384 + h * 256), rr, g0,
                                         a_tile, r);
                    break;
                case 1: dequant_row_part<1>(cst + h * 8192, scz, rr, g0, a_tile, r); break;
                case 2: dequant_row_part<2>(cst + h * 8192, scz, rr, g0, a_tile, r); break;
                case 3: dequant_row_part<3>(cst + h * 8192, scz, rr, g0, a_tile, r); break;
                case 4: dequant_row_part<4>(cst + h * 8192, scz, rr, g0, a_tile, r); break;
                case 5: dequant_row_part<5>(cst + h * 8192, scz, rr, g0, a_tile, r); break;
                case 6: dequant_row_part<6>(cst + h * 8192, scz, rr, g0, a_tile, r); break;
                default: dequant_row_part<8>(cst + h * 8192, scz, rr, g0, a_tile, r); break;
            }
            fence_proxy_async_smem();   // generic-proxy writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&S.full_a[s]);
                mbar_arrive(&S.empty_c[sc]);
            }
            ++a;
        }
        // epilogue: this warp's 32 rows x its BN/4 tokens
        pdl_wait();   // tok_scale comes from the prologue kernel
        bool ok = S.abort_flag ? false : mbar_wait_bounded(&S.d_full, 0u, DEC_WAIT_NS);
        ok = __all_sync(0xffffffffu, ok);   // warp-uniform: tcgen05.ld is .sync.aligned
        if (!ok && !S.abort_flag && lane == 0) timed_out();
        tc_fence_after();
        const int re = quad * 32 + lane;         // TMEM lane = weight row of the tile
        const int i = nb0 * 64 + re;
        const bool row_ok = i < p.N;
        // in W' row order the 32 lanes write 32 consecutive floats (one 128-byte
        // line); through row_perm every value would be a separate scattered store
        const int n = row_ok ? ((p.row_perm && p.out_scatter) ? p.row_perm[i] : i) : 0;
        float* out = p.out + (p.out_scatter ? 0 : (size_t)split * p.M * p.N);
        for (int cc = 0; cc < BN / 128; ++cc) {
            const int col0 = part * (BN / 4) + cc * 32;
            float v[32];
            if (any && ok) {
                tmem_ld32(tmem_d + ((uint32_t)(quad * 32) << 16) + (uint32_t)col0, v);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = 0.f;
            }
            if (row_ok) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int m = m0 + col0 + j;
                    if (m < p.M) out[(size_t)m * p.N + n] = v[j] * p.tok_scale[m];
                }
            }
        }
    }
    // after an abort, copies and tensor-core work may still be in flight into
    // this CTA's shared memory and TMEM: wait for them (bounded) before the
    // TMEM is freed and the CTA leaves.  A stage's last arm is the only one
    // that can be pending (a stage is re-armed only after it was consumed).
    __syncthreads();
    if (S.abort_flag && lane == 0) {
        if (warp == 0)
            for (int i = max(0, c_armed - PF_C_STAGES); i < c_armed; ++i)
                mbar_wait_bounded(&S.full_c[i % PF_C_STAGES], (uint32_t)(i / PF_C_STAGES) & 1u, DEC_WAIT_NS);
        if (warp == PF_WARPS - 1)
            for (int i = max(0, b_armed - PF_B_STAGES); i < b_armed; ++i)
                mbar_wait_bounded(&S.full_b[i % PF_B_STAGES], (uint32_t)(i / PF_B_STAGES) & 1u, DEC_WAIT_NS);
        if (warp == 1) mbar_wait_bounded(&S.d_full, 0u, DEC_WAIT_NS);   // all issued MMAs
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

// ---------------------------------------------------------------------------
// After the tensor-core kernel: y[m][row_perm[i]] = sum over the k splits (in
// split order) of part[split][m][i].  One CTA per token row: the splits' rows
// are read coalesced and their sum scattered into shared memory through
// row_perm, then the row is written back coalesced.  part may be y itself
// (one split: the reordering is then in place; every thread reads before any
// writes, after the barrier).  (SFMP abstract: the reordering costs only a
// small step.)
// ---------------------------------------------------------------------------
constexpr int FINISH_THREADS = 512;

__device__ __forceinline__ void f4_acc(float4& a, const float4 b) {
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
}

// The sum over the splits of four consecutive values of a row, stored at
// their own columns (mode 0) or into shared memory through row_perm (mode 1).
__device__ __forceinline__ void finish_put4(float* yr, float* srow, const int32_t* row_perm, int i4,
                                            float4 v, int mode) {
    if (mode == 0) {
        reinterpret_cast<float4*>(yr)[i4] = v;
        return;
    }
    const int4 r = reinterpret_cast<const int4*>(row_perm)[i4];
    srow[r.x] = v.x; srow[r.y] = v.y; srow[r.z] = v.z; srow[r.w] = v.w;
}

__global__ void __launch_bounds__(FINISH_THREADS) k_finish_rows(float* y, const float* part, int splits,
                                                               size_t split_stride, const int32_t* row_perm,
                                                               int N, int mode) {
    // mode 0: no row order; 1: reorder through shared memory (N floats)
    extern __shared__ __align__(16) float srow[];
    pdl_launch_dependents();
    pdl_wait();   // the partial sums come from the kernel before
    const size_t row = (size_t)blockIdx.x * N;
    float* yr = y + row;
    const float* pr = part + row;
    const bool vec = (N % 4 == 0) && (split_stride % 4 == 0) &&
                     (((uintptr_t)yr | (uintptr_t)pr | (uintptr_t)row_perm) & 15) == 0;
    if (vec) {
        // 16-byte loads, two of them in flight per thread and split
        const int n4 = N / 4;
        for (int i0 = threadIdx.x; i0 < n4; i0 += 2 * FINISH_THREADS) {
            const int i1 = i0 + FINISH_THREADS;
            const bool two = i1 < n4;
            float4 a = reinterpret_cast<const float4*>(pr)[i0];
            float4 b = two ? reinterpret_cast<const float4*>(pr)[i1] : make_float4(0.f, 0.f, 0.f, 0.f);
            for (int sp = 1; sp < splits; ++sp) {
                const float4* ps = reinterpret_cast<const float4*>(pr + (size_t)sp * split_stride);
                f4_acc(a, ps[i0]);
                if (two) f4_acc(b, ps[i1]);
            }
            finish_put4(yr, srow, row_perm, i0, a, mode);
            if (two) finish_put4(yr, srow, row_perm, i1, b, mode);
        }
    } else {
        for (int i = threadIdx.x; i < N; i += FINISH_THREADS) {
            float v = pr[i];
            for (int sp = 1; sp < splits; ++sp) v += pr[(size_t)sp * split_stride + i];
            if (mode == 0) yr[i] = v;
            else srow[row_perm[i]] = v;
        }
    }
    if (mode != 1) return;
    __syncthreads();
    if (vec) {
        for (int i4 = threadIdx.x; i4 < N / 4; i4 += FINISH_THREADS)
            reinterpret_cast<float4*>(yr)[i4] = reinterpret_cast<const float4*>(srow)[i4];
    } else {
        for (int n = threadIdx.x; n < N; n += FINISH_THREADS) yr[n] = srow[n];
    }
}

}  // namespace mpq
