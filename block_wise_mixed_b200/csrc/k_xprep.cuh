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
// Layout written (XP_PREFILL): [M][K] half, K contiguous, each 128-column
// group permuted so that position 2*(4i+j)+h holds column 8i+j+4h -- the
// order in which the tensor-core kernel's dequantization emits weights.
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
    // CTA (m, y) converts the y-th of gridDim.y column ranges of token m
    // (every CTA of the token finds the row maximum itself)
    const int m = blockIdx.x, tid = threadIdx.x, K = p.K;
    if (m == 0 && blockIdx.y == 0) {
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
    if (tid == 0 && blockIdx.y == 0) p.tok_scale[m] = ldexpf(1.f, -e);

    auto load = [&](int j) -> float {
        int c = p.col_perm ? p.col_perm[j] : j;
        return ldexpf(__uint_as_float(((uint32_t)xr[c]) << 16), e);
    };
    {
        __half2* out = reinterpret_cast<__half2*>(p.xq + (size_t)m * K);
        const int per = (K / 2 + gridDim.y - 1) / gridDim.y;
        const int c_end = min(K / 2, ((int)blockIdx.y + 1) * per);
        for (int c2 = (int)blockIdx.y * per + tid; c2 < c_end; c2 += XPREP_THREADS) {
            const int kb = c2 >> 6, r = c2 & 63, i = r >> 2, j = r & 3;
            const int col = kb * 128 + 8 * i + j;
            out[c2] = __halves2half2(__float2half_rn(load(col)), __float2half_rn(load(col + 4)));
        }
    }
}

// ---------------------------------------------------------------------------
// Small-batch activation records (k_xprep_decode).
//
// The decode kernel multiplies packed codes by activations on the integer
// tensor cores (mma.m16n8k32, u8 codes x s8 activations, s32 accumulation),
// so every product and every sum is exact.  Each 128-column slice (block
// column kb) of token m is turned into integers by its own power of two:
//   e = 22 - floor(log2 amax)  (one less if amax * 2^e would exceed XQD_XMAX),
//   X_c = rne(x'_c * 2^e),  |X_c| <= XQD_XMAX < 2^23,
// which is exact for every element within a factor 2^15 of the slice maximum
// (bf16 carries 8 significant bits) and otherwise off by at most half a unit
// (2^-23 of the slice maximum).  X = d0 + 256 d1 + 65536 d2 with every digit
// in [-128, 127]: three s8 "digits", three columns of the mma's B operand.
// With T_d = sum_c d_d(X_c) (exact), the decode kernel forms per output row
//   E_d = sum_c (q_c - z) d_d(X_c) = C_d - z T_d                (int32, exact)
//   V   = E_0 + 256 E_1 + 65536 E_2 = sum_c (q_c - z) X_c
// and adds s * F * V with F = 2^-e (a non-finite slice gives F = NaN, so
// non-finite x gives non-finite y).
//
// The kernel unpacks four codes of one 32-bit code word into the four bytes
// of a register with one AND (a "plane" of the word), so the column order
// of the A operand depends on the piece width p that the codes come from.
// For k-tile j (32 columns of the A operand), register half hf (mma
// registers a0/a1 vs a2/a3), quad lane t and byte b, the operand column
// kappa = 32j + 16hf + 4t + b holds the code of slice column
//   p = 1:  32t + 8b + 2j + hf
//   p = 2:  32t + 16(j/2) + 4b + 2(j%2) + hf
//   p = 4:  32t + 8j + 2b + hf
//   p = 8:  32t + 8j + 4hf + b
// (xqd_col below), and each width has its own copy ("variant") of the slice.
//
// Record of block column kb (XQD_REC * M bytes, 16-byte aligned): for each
// variant v = 0..3 (p = 1, 2, 4, 8) and token m, XQD_VAR = 400 bytes:
//   [d = 0..2][t = 0..3][j = 0..3][hf = 0, 1][b = 0..3] s8: digit d of X at
//   column kappa -- for quad lane t and mma column d, the 32 bytes are its
//   B-fragment registers of the four k-tiles in order;
//   then T_0, T_1, T_2 (int32) and F (float);
// and variant 4, for 16-bit passthrough blocks: the slice's 128 bf16 values
// in column order (the first 256 of its 400 bytes).  One variant of a token
// group is one contiguous run of 400*Mg bytes.
// Block 0 also clears the decode kernel's per-block-row counters.
// ---------------------------------------------------------------------------
constexpr int XQD_DIGITS = 3;
constexpr int XQD_VAR = XQD_DIGITS * 128 + 16;   // one variant of one token: digits, T_d, F
constexpr int XQD_VARIANTS = 5;                  // p = 1, 2, 4, 8, and the bf16 slice
constexpr int XQD_REC = XQD_VARIANTS * XQD_VAR;
constexpr float XQD_XMAX = 8355711.f;            // 127 * (1 + 256 + 65536): three s8 digits

__host__ __device__ __forceinline__ int xqd_col(int v, int kappa) {
    const int j = kappa >> 5, hf = (kappa >> 4) & 1, t = (kappa >> 2) & 3, b = kappa & 3;
    if (v == 0) return 32 * t + 8 * b + 2 * j + hf;
    if (v == 1) return 32 * t + 16 * (j >> 1) + 4 * b + 2 * (j & 1) + hf;
    if (v == 2) return 32 * t + 8 * j + 2 * b + hf;
    return 32 * t + 8 * j + 4 * hf + b;
}

// Balanced base-256 digit d of X (|X| <= XQD_XMAX).
__device__ __forceinline__ int xqd_digit(int X, int d) {
    const int d0 = ((X + 128) & 255) - 128;
    if (d == 0) return d0;
    const int X1 = (X - d0) >> 8;
    const int d1 = ((X1 + 128) & 255) - 128;
    if (d == 1) return d1;
    return (X1 - d1) >> 8;
}

// Byte position of slice column c within a digit row of variant v: the
// inverse of xqd_col (kappa = 32j + 16hf + 4t + b is stored at 32t + 8j +
// 4hf + b).
__host__ __device__ __forceinline__ int xqd_pos(int v, int c) {
    const int t = c >> 5, r = c & 31;
    int j, hf, b;
    if (v == 0) { b = r >> 3; j = (r & 7) >> 1; hf = r & 1; }
    else if (v == 1) { j = 2 * (r >> 4) + ((r & 3) >> 1); b = (r & 15) >> 2; hf = r & 1; }
    else if (v == 2) { j = r >> 3; b = (r & 7) >> 1; hf = r & 1; }
    else { j = r >> 3; hf = (r & 7) >> 2; b = r & 3; }
    return 32 * t + 8 * j + 4 * hf + b;
}

// Slice exponent e from the slice's largest magnitude (NaN-propagating max).
__device__ __forceinline__ int xqd_exponent(float amax) {
    int e = 0;
    if (amax > 0.f && isfinite(amax)) {
        e = 22 - ilogbf(amax);
        if (ldexpf(amax, e) > XQD_XMAX) e -= 1;
        e = min(e, 126);
    }
    return e;
}

// The slice's integers: the warp's lane holds slice columns 4 lane .. +3
// (values v[]); X[] receives their integers and T[0..2] the digit sums of
// the whole slice (every lane); F is 2^-e, or NaN for a non-finite slice.
__device__ __forceinline__ void xqd_integerize(const float (&v)[4], int (&X)[4], int (&T)[3], float& F) {
    float amax = 0.f;
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
        const float a = fabsf(v[e4]);
        amax = (a > amax || a != a) ? a : amax;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, amax, off);
        amax = (o > amax || o != o) ? o : amax;
    }
    const int e = xqd_exponent(amax);
    T[0] = T[1] = T[2] = 0;
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
        const float sv = ldexpf(v[e4], e);
        X[e4] = isfinite(sv) ? __float2int_rn(sv) : 0;
#pragma unroll
        for (int d = 0; d < 3; ++d) T[d] += xqd_digit(X[e4], d);
    }
#pragma unroll
    for (int d = 0; d < 3; ++d)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) T[d] += __shfl_xor_sync(0xffffffffu, T[d], off);
    F = isfinite(amax) ? ldexpf(1.f, -e) : __int_as_float(0x7fc00000);
}

// One variant's record into rec (shared memory, XQD_VAR bytes): each lane
// stores the three digits of its four columns at their positions, then lane
// 0 the digit sums and F.
__device__ __forceinline__ void xqd_scatter_variant(const int (&X)[4], const int (&T)[3], float F, int vv,
                                                    uint8_t* rec, int lane) {
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
        const int pos = xqd_pos(vv, 4 * lane + e4);
#pragma unroll
        for (int d = 0; d < 3; ++d) rec[d * 128 + pos] = (uint8_t)xqd_digit(X[e4], d);
    }
    if (lane == 0)
        *reinterpret_cast<uint4*>(rec + XQD_DIGITS * 128) =
            make_uint4((uint32_t)T[0], (uint32_t)T[1], (uint32_t)T[2], __float_as_uint(F));
}

constexpr int XPREP_DEC_WARPS = XPREP_THREADS / 32;

__global__ void __launch_bounds__(XPREP_THREADS, 8) k_xprep_decode(XprepParams p) {
    pdl_launch_dependents();
    // one variant at a time per warp (small, so that the CTAs fit beside the
    // decode kernel's on an SM; few CTAs, so that they keep few SMs from
    // taking the next decode launch's CTAs while they wait for the kernel
    // before)
    __shared__ __align__(16) uint8_t recs[XPREP_DEC_WARPS][XQD_VAR];
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
    int X[4], T[3];
    float F;
    xqd_integerize(v, X, T, F);
    uint8_t* rs = recs[warp];
    // variant vv of token m of block column kb
    uint8_t* rec = reinterpret_cast<uint8_t*>(p.xq) + (size_t)kb * p.M * XQD_REC + (size_t)m * XQD_VAR;
#pragma unroll 1
    for (int vv = 0; vv < 4; ++vv) {
        xqd_scatter_variant(X, T, F, vv, rs, lane);
        __syncwarp();
        if (lane < XQD_VAR / 16)
            reinterpret_cast<uint4*>(rec + (size_t)vv * p.M * XQD_VAR)[lane] =
                reinterpret_cast<const uint4*>(rs)[lane];
        __syncwarp();
    }
    // variant 4: the bf16 slice in column order
    *reinterpret_cast<uint2*>(rec + (size_t)4 * p.M * XQD_VAR + 8 * lane) =
        make_uint2((uint32_t)xr[cp.x] | ((uint32_t)xr[cp.y] << 16), (uint32_t)xr[cp.z] | ((uint32_t)xr[cp.w] << 16));
}

}  // namespace mpq
