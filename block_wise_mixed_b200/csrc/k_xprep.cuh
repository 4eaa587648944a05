// k_xprep.cuh -- activation prologue: x'[m][j] = x[m][col_perm[j]].
//
// SFMP abstract: row-column reordering costs "a small activation reordering
// overhead during inference" -- this kernel is that step.  It also converts
// bf16 -> fp16 for the tensor-core operands.  To keep every bf16 value exact
// in fp16 (8 significant bits fit in 11) and away from fp16 overflow, token m
// is scaled by an exact power of two 2^e_m chosen from its largest magnitude
// (e_m = 14 - floor(log2(amax_m)), so amax*2^e lies in [2^14, 2^15)); the
// GEMM epilogues multiply by tok_scale[m] = 2^-e_m, which is exact.
//
// Layouts written:
//   XP_DECODE : [KB][M][4][16] half2 -- for block column kb, token m and quad
//               lane t, register r = 4i+j holds the columns (32t+8i+j,
//               32t+8i+j+4) of that block column: exactly the B fragment of
//               mma.m16n8k16 that the decode kernel pairs with its code
//               extraction order.
//   XP_PREFILL: [M][K] half, K contiguous, each 128-column group permuted so
//               that position 2*(4i+j)+h holds column 8i+j+4h -- the order in
//               which the tensor-core kernel's dequantization emits weights.
// Block 0 also clears the decode kernel's per-block-row counters (when given).
//
// k_xprep_decode (below) is the small-batch variant; its layout is described
// there.
#pragma once
#include "common.cuh"

namespace mpq {

enum XprepLayout { XP_DECODE = 0, XP_PREFILL = 1 };

struct XprepParams {
    const uint16_t* x;         // bf16 bits, M x K
    const int32_t* col_perm;   // [K] or null
    __half* xq;                // output (layout above)
    float* tok_scale;          // [M] = 2^-e_m
    uint32_t* counters;        // [n_counters] cleared by block 0 (may be null)
    int n_counters;
    int M, K;
};

constexpr int XPREP_THREADS = 256;

template <int LAYOUT>
__global__ void __launch_bounds__(XPREP_THREADS) k_xprep(XprepParams p) {
    // let the GEMM kernel that follows start its prologue early, then wait
    // for the kernel before (x and the workspace may still be in use there)
    pdl_launch_dependents();
    pdl_wait();
    __shared__ float red[XPREP_THREADS / 32];
    const int m = blockIdx.x, tid = threadIdx.x, K = p.K;
    if (m == 0) {
        if (p.counters)
            for (int i = tid; i < p.n_counters; i += XPREP_THREADS) p.counters[i] = 0u;
    }
    const uint16_t* xr = p.x + (size_t)m * K;
    // 1. amax over the row (order-free, so read it unpermuted, 8 values per load)
    float amax = 0.f;
    const uint4* xv = reinterpret_cast<const uint4*>(xr);
    for (int c = tid; c < K / 8; c += XPREP_THREADS) {
        uint4 v = xv[c];
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            float a = fabsf(__uint_as_float(w[h] << 16));
            float b = fabsf(__uint_as_float(w[h] & 0xffff0000u));
            // NaN-propagating max: fmaxf would drop NaN
            amax = (a > amax || a != a) ? a : amax;
            amax = (b > amax || b != b) ? b : amax;
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        float o = __shfl_xor_sync(0xffffffffu, amax, off);
        amax = (o > amax || o != o) ? o : amax;
    }
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    if (tid == 0) {
        float a = red[0];
        for (int i = 1; i < XPREP_THREADS / 32; ++i) a = (red[i] > a || red[i] != red[i]) ? red[i] : a;
        red[0] = a;
    }
    __syncthreads();
    amax = red[0];
    int e = 0;
    if (amax > 0.f && isfinite(amax)) e = min(max(14 - ilogbf(amax), -126), 126);
    if (tid == 0) p.tok_scale[m] = ldexpf(1.f, -e);

    auto load = [&](int j) -> float {
        int c = p.col_perm ? p.col_perm[j] : j;
        return ldexpf(__uint_as_float(((uint32_t)xr[c]) << 16), e);
    };
    if (LAYOUT == XP_DECODE) {
        const int KB = K / 128;
        __half2* out = reinterpret_cast<__half2*>(p.xq);
        for (int idx = tid; idx < K / 2; idx += XPREP_THREADS) {
            const int kb = idx >> 6, rem = idx & 63;
            const int t = rem >> 4, r = rem & 15, i = r >> 2, j = r & 3;
            const int col = kb * 128 + 32 * t + 8 * i + j;
            __half2 v = __halves2half2(__float2half_rn(load(col)), __float2half_rn(load(col + 4)));
            out[((size_t)kb * p.M + m) * 64 + rem] = v;
        }
        (void)KB;
    } else {
        __half2* out = reinterpret_cast<__half2*>(p.xq + (size_t)m * K);
        for (int c2 = tid; c2 < K / 2; c2 += XPREP_THREADS) {
            const int kb = c2 >> 6, r = c2 & 63, i = r >> 2, j = r & 3;
            const int col = kb * 128 + 8 * i + j;
            out[c2] = __halves2half2(__float2half_rn(load(col)), __float2half_rn(load(col + 4)));
        }
    }
}

// ---------------------------------------------------------------------------
// Small-batch activation records (k_xprep_decode).
//
// The decode kernel turns a pair of packed codes into the fp16 pair
// ((q_a - z) * 2^-24, (q_b - z) * 2^-24) -- exact subnormals -- with one AND
// (or byte permute) and one HFMA2 per pair.  Which two columns share a pair
// follows from where a p-bit piece puts its codes in a 32-bit word (the two
// 16-bit halves), so each piece width p = 1, 2, 4, 8 pairs the columns in its
// own order, and the activation slice is stored once per order ("variant").
// For quad lane t of the mma, pair index pi (0..15) of a row's 32 columns
// 32t..32t+31 holds the columns (colA, colB):
//   p = 1: cols (s + 8*(pi/8), s + 8*(pi/8) + 16),  s = pi % 8
//   p = 2: cols (16i + 4h + s, 16i + 4h + s + 8),   i = pi/8, h = (pi/4)%2, s = pi%4
//   p = 4: cols (8i + r, 8i + r + 4),               i = pi/4, r = pi % 4
//   p = 8: cols (4i + r, 4i + r + 2),               i = pi/2, r = pi % 2
// and register pi of the mma B fragment is (x'[colA], x'[colB]).
//
// Each 128-column slice (block column kb) of token m is scaled by its own
// power of two 2^e (amax * 2^e in [2^14, 2^15), e >= -103), so that bf16
// values are exact in fp16.  The tensor cores then accumulate
// c_r = 2^-24 * sum_j (q_j - z_r) x'_j, and the block adds s_r * F * c_r to
// output row r, with F = 2^(24 - e).
//
// Record of block column kb (XQD_REC * M bytes, 16-byte aligned): for each
// variant v = 0..3 (p = 1, 2, 4, 8) and token m, XQD_VAR = 272 bytes:
//   [t = 0..3][pi = 0..15] half2 (256 B), then F as float4 (F, 0, 0, 0)
// so one variant of a token group is one contiguous run of 272*Mg bytes.
// Block 0 also clears the decode kernel's per-block-row counters.
// ---------------------------------------------------------------------------
constexpr int XQD_VAR = 272;                 // one variant of one token: fragments + F
constexpr int XQD_REC = 4 * XQD_VAR;

__device__ __forceinline__ void xqd_pair_cols(int v, int pi, int& ca, int& cb) {
    if (v == 0) {
        ca = (pi & 7) + 8 * (pi >> 3); cb = ca + 16;
    } else if (v == 1) {
        ca = 16 * (pi >> 3) + 4 * ((pi >> 2) & 1) + (pi & 3); cb = ca + 8;
    } else if (v == 2) {
        ca = 8 * (pi >> 2) + (pi & 3); cb = ca + 4;
    } else {
        ca = 4 * (pi >> 1) + (pi & 1); cb = ca + 2;
    }
}

constexpr int XPREP_DEC_WARPS = XPREP_THREADS / 32;

__global__ void __launch_bounds__(XPREP_THREADS) k_xprep_decode(XprepParams p) {
    pdl_launch_dependents();
    __shared__ float xs[XPREP_DEC_WARPS][64];   // 128 fp16 per warp
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int KB = p.K / 128;
    const int item = blockIdx.x * XPREP_DEC_WARPS + warp;   // = kb * M + m
    const bool active = item < KB * p.M;
    const int kb = active ? item / p.M : 0, m = active ? item % p.M : 0;
    // lane holds columns 4*lane .. 4*lane+3 of the slice; the column order is
    // static, so it is read before waiting for the kernel that writes x
    const int c0 = kb * 128 + 4 * lane;
    int4 cp = make_int4(c0, c0 + 1, c0 + 2, c0 + 3);
    if (p.col_perm && active) cp = *reinterpret_cast<const int4*>(p.col_perm + c0);
    pdl_wait();   // the kernel before may still read the workspace or write x
    if (blockIdx.x == 0) {
        if (p.counters)
            for (int i = tid; i < p.n_counters; i += XPREP_THREADS) p.counters[i] = 0u;
    }
    if (!active) return;
    const uint16_t* xr = p.x + (size_t)m * p.K;
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
    // x' = fp16(x * 2^e) (exact for bf16 inputs in range)
    __half* xw = reinterpret_cast<__half*>(xs[warp]);
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) xw[4 * lane + e4] = __float2half_rn(ldexpf(v[e4], e));
    __syncwarp();
    // lane -> variant vv = lane / 8, quad lane tq = (lane / 2) % 4, pairs 8*(lane % 2) .. +7
    const int vv = lane >> 3, tq = (lane >> 1) & 3, pi0 = 8 * (lane & 1);
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int ca, cb;
        xqd_pair_cols(vv, pi0 + i, ca, cb);
        o[i] = h2_bits(__halves2half2(xw[32 * tq + ca], xw[32 * tq + cb]));
    }
    uint8_t* rec = reinterpret_cast<uint8_t*>(p.xq) + (size_t)kb * p.M * XQD_REC;
    uint4* dst = reinterpret_cast<uint4*>(rec + (size_t)vv * p.M * XQD_VAR + (size_t)m * XQD_VAR +
                                          tq * 64 + pi0 * 4);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    if ((lane & 7) == 0)   // one lane per variant writes F after the fragments
        *reinterpret_cast<float4*>(rec + (size_t)vv * p.M * XQD_VAR + (size_t)m * XQD_VAR + 256) =
            make_float4(ldexpf(1.f, 24 - e), 0.f, 0.f, 0.f);
}

}  // namespace mpq
