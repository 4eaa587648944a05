// k_pack.cuh -- RTN quantize + bit-split pack kernel (format v1).
//
// Method: ScaleBITS summary, "Approach" (64x128 blocks with one bit width
// each, after bi-directional channel reordering) and "Key results" /
// "Limitations" (scalar RTN with group size 128); TileQuant abstract (the
// precision map guides compact weight buffers).
//
// One CTA walks a range of rows of the reordered matrix W'.  For each row it
// stages the whole source row W[row_perm[i]] in shared memory with one bulk
// copy (double-buffered, so the next row streams in while this one is
// quantized), then every warp takes groups (blocks kb of this row): gathers
// the 128 columns through col_perm from shared memory, finds the range,
// picks the fp16 scale and zero in fp64, rounds each weight in fp32 (the
// exhaustive check in the test suite shows fp32 and exact rounding agree for
// every bf16 weight and fp16 scale), and writes the codes as bit-split pieces.
#pragma once
#include "common.cuh"

namespace mpq {

struct PackParams {
    const uint16_t* W;         // bf16 bits, N x K, original order
    const mpq_block* table;    // [NB*KB]
    const int32_t* row_perm;   // [N] or null
    const int32_t* col_perm;   // [K] or null
    uint8_t* codes;
    uint16_t* scales;
    uint16_t* zeros;
    uint32_t* err;
    int N, K, KB;
    int rows_per_cta;
};

constexpr int PACK_THREADS = 256;

__device__ __forceinline__ double f16_to_f64(uint16_t h) {
    return (double)__half2float(__ushort_as_half(h));
}

// Smallest positive finite fp16 pattern h with value(h)*qmax >= d (d > 0).
// Returns 0 when none exists.  value(h)*qmax is exact in fp64.
__device__ __forceinline__ uint32_t min_scale_bits(double d, double qmax) {
    double r = d / qmax;
    uint32_t h;
    if (r > 65504.0) {
        h = 0x7BFF;
    } else {
        h = __half_as_ushort(__double2half(r));  // round to nearest
        if (h == 0) h = 1;
        if (h > 0x7BFF) h = 0x7BFF;
    }
    // step up until it covers d, then down while the previous one still does
    while (h <= 0x7BFF && f16_to_f64((uint16_t)h) * qmax < d) ++h;
    if (h > 0x7BFF) return 0;
    while (h > 1 && f16_to_f64((uint16_t)(h - 1)) * qmax >= d) --h;
    return h;
}

__device__ __forceinline__ uint32_t f16_bits_small_int(int v) {
    return __half_as_ushort(__int2half_rn(v));  // exact for 0..2048
}

// STAGED: the source row and the column order are staged in shared memory
// (about 6 K bytes); rows too long for that (K beyond ~38 K) are read from
// global memory directly (the row is L1/L2-resident while its groups are
// quantized).
template <bool STAGED>
__global__ void __launch_bounds__(PACK_THREADS)
k_pack(PackParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int K = p.K, KB = p.KB;
    const uint32_t row_bytes = (uint32_t)K * 2u;
    // layout: [row buffer 0][row buffer 1][col_perm as uint16][2 mbarriers]
    uint16_t* rowbuf0 = reinterpret_cast<uint16_t*>(smem);
    uint16_t* rowbuf1 = reinterpret_cast<uint16_t*>(smem + row_bytes);
    uint16_t* cperm = reinterpret_cast<uint16_t*>(smem + 2 * row_bytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * row_bytes +
                                                 ((row_bytes + 15u) & ~15u));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int i_begin = blockIdx.x * p.rows_per_cta;
    const int i_end = min(p.N, i_begin + p.rows_per_cta);
    if (i_begin >= i_end) return;

    if (STAGED && p.col_perm)
        for (int j = tid; j < K; j += PACK_THREADS) cperm[j] = (uint16_t)p.col_perm[j];
    if (STAGED && tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto src_row = [&](int i) -> const uint16_t* {
        int s = p.row_perm ? p.row_perm[i] : i;
        return p.W + (size_t)s * K;
    };
    // column c of the reordered row (through col_perm when given)
    auto col = [&](int c) -> int {
        if (!p.col_perm) return c;
        return STAGED ? (int)cperm[c] : __ldg(p.col_perm + c);
    };
    if (STAGED && tid == 0) {
        mbar_arrive_expect_tx(&bars[0], row_bytes);
        bulk_g2s(rowbuf0, src_row(i_begin), row_bytes, &bars[0]);
    }

    int it = 0;
    for (int i = i_begin; i < i_end; ++i, ++it) {
        const int buf = it & 1;
        const uint16_t* row = STAGED ? (buf ? rowbuf1 : rowbuf0) : src_row(i);
        if (STAGED) {
            // prefetch the next row into the other buffer (its previous contents
            // were released by the __syncthreads at the end of the last iteration)
            if (tid == 0 && i + 1 < i_end) {
                uint16_t* nrow = buf ? rowbuf0 : rowbuf1;
                mbar_arrive_expect_tx(&bars[buf ^ 1], row_bytes);
                bulk_g2s(nrow, src_row(i + 1), row_bytes, &bars[buf ^ 1]);
            }
            if (!mbar_wait_bounded(&bars[buf], (uint32_t)((it >> 1) & 1), 2000000000ull)) {
                if (tid == 0) set_error(p.err, MPQ_ERR_TIMEOUT);
                return;  // a copy that never lands: stop this CTA
            }
        }

        const int nb = i >> 6, r = i & 63;
        for (int kb = warp; kb < KB; kb += PACK_THREADS / 32) {
            const mpq_block e = p.table[(size_t)nb * KB + kb];
            const int b = (int)e.bits;
            if (b == 0) continue;
            if (b == 16) {
                // passthrough (TileQuant abstract: the highest-scoring tiles
                // stay at 16 bits): the row's bf16 weights, scale 1, zero 0;
                // finite and within the fp16 range (the tensor-core path)
                const int c0 = kb * 128 + 4 * lane;
                uint16_t wb[4];
                bool finite = true, in_range = true;
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    wb[e4] = row[col(c0 + e4)];
                    const float v = __uint_as_float(((uint32_t)wb[e4]) << 16);
                    finite &= isfinite(v);
                    in_range &= fabsf(v) <= 65504.f;
                }
                if (!__all_sync(0xffffffffu, finite)) {
                    if (lane == 0) set_error(p.err, MPQ_ERR_NONFINITE);
                    continue;
                }
                if (!__all_sync(0xffffffffu, in_range)) {
                    if (lane == 0) set_error(p.err, MPQ_ERR_RANGE);
                    continue;
                }
                *reinterpret_cast<uint2*>(p.codes + e.code_off + (uint32_t)r * 256u + 8u * lane) =
                    make_uint2((uint32_t)wb[0] | ((uint32_t)wb[1] << 16), (uint32_t)wb[2] | ((uint32_t)wb[3] << 16));
                if (lane == 0) {
                    p.scales[e.sz_off + r] = 0x3C00u;
                    p.zeros[e.sz_off + r] = 0u;
                }
                continue;
            }
            // gather this lane's 4 contiguous columns j = 4*lane .. 4*lane+3
            float w[4];
            const int c0 = kb * 128 + 4 * lane;
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
                w[e4] = __uint_as_float(((uint32_t)row[col(c0 + e4)]) << 16);
            }
            bool finite = true;
            float lo = 0.f, hi = 0.f;
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
                finite &= isfinite(w[e4]);
                lo = fminf(lo, w[e4]);
                hi = fmaxf(hi, w[e4]);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
            }
            if (!__all_sync(0xffffffffu, finite)) {
                if (lane == 0) set_error(p.err, MPQ_ERR_NONFINITE);
                continue;
            }
            const double qmax = (double)((1 << b) - 1);
            const double d = (double)hi - (double)lo;  // exact
            uint32_t s_bits, z_int;
            if (d == 0.0) {
                s_bits = 0x3C00u;
                z_int = 0;
            } else {
                s_bits = min_scale_bits(d, qmax);
                if (s_bits == 0 || f16_to_f64((uint16_t)s_bits) * qmax > 65504.0) {
                    if (lane == 0) set_error(p.err, MPQ_ERR_RANGE);
                    continue;
                }
                z_int = (uint32_t)rint(-(double)lo / f16_to_f64((uint16_t)s_bits));
            }
            const float s_f = __half2float(__ushort_as_half((uint16_t)s_bits));
            const int qmaxi = (1 << b) - 1;
            uint32_t q[4];
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
                int v = (d == 0.0) ? 0 : (int)rintf(__fdiv_rn(w[e4], s_f)) + (int)z_int;
                q[e4] = (uint32_t)min(max(v, 0), qmaxi);
            }
            if (lane == 0) {
                p.scales[e.sz_off + r] = (uint16_t)s_bits;
                p.zeros[e.sz_off + r] = (uint16_t)f16_bits_small_int((int)z_int);
            }
            // bit-split pieces, low piece first
            int pw[2], np;
            switch (b) {
                case 3: pw[0] = 2; pw[1] = 1; np = 2; break;
                case 5: pw[0] = 4; pw[1] = 1; np = 2; break;
                case 6: pw[0] = 4; pw[1] = 2; np = 2; break;
                default: pw[0] = b; np = 1; break;
            }
            uint8_t* payload = p.codes + e.code_off;
            uint32_t piece_base = 0, shift = 0;
            for (int pi = 0; pi < np; ++pi) {
                const int pb = pw[pi];
                const uint32_t m = (1u << pb) - 1u;
                uint32_t f = 0;
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) f |= ((q[e4] >> shift) & m) << (e4 * pb);
                // 8/pb consecutive lanes share one 32-bit word
                const int n = 8 / pb;
                uint32_t x = f << ((lane % n) * 4 * pb);
                for (int off = 1; off < n; off <<= 1) x |= __shfl_xor_sync(0xffffffffu, x, off);
                if (lane % n == 0) {
                    uint32_t* rowp = reinterpret_cast<uint32_t*>(payload + piece_base +
                                                                 (uint32_t)r * 16u * pb);
                    rowp[lane / n] = x;
                }
                piece_base += 64u * 16u * pb;
                shift += pb;
            }
        }
        __syncthreads();  // everyone is done with `row` before it is refilled
    }
}

}  // namespace mpq
