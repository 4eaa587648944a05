// k_alloc.cuh -- budgeted per-block bit allocation (the step that produces
// the bit map the pack consumes).
//
// "ScaleBITS: Scalable Bitwidth Search for Hardware-Aligned Mixed-Precision
// LLMs" -- abstract: global bitwidth allocation under a memory budget as a
// constrained optimization, solved by "a scalable approximation to the greedy
// algorithm"; summary page, "Approach": a batched approximation to greedy
// knapsack allocation per 64x128 block under a global budget; "Key results":
// 16-36 search iterations against about 3e6 for classic greedy.
//
// Reading (the pages give no formulas): each block t has a loss L[t][b] per
// allowed width b (a sensitivity surrogate).  With a price lam per bit, every
// block independently takes w_t(lam) = argmin_b L[t][b] + lam * b (ties to
// the smaller width); the total S(lam) does not grow with lam.  The price is
// found by bisection until S fits the budget B; the leftover is then filled
// in the classic greedy order (loss saved per bit, descending; block index,
// ascending), a round at a time.  On losses convex in the width this is the
// classic greedy's result.  All arithmetic is fp64 with explicit rounding
// (product, then sum), so the result is a deterministic function of the
// inputs.
//
// One CTA of ALLOC_THREADS threads runs the whole search: each bisection
// step is one pass over the blocks with a block-wide sum; a fill round finds
// the exact prefix of the ordered upgrades with a radix select over the
// 96-bit keys (gain bits, inverted block index), 8 bits per pass, on
// histograms of the upgrades' bit increments in shared memory.
#pragma once
#include "common.cuh"

namespace mpq {

constexpr int ALLOC_THREADS = 1024;
constexpr int ALLOC_MAX_STEPS = 64;

struct AllocParams {
    const float* loss;         // [n][8]: widths 0,1,2,3,4,5,6,8
    uint8_t* bits;             // [n] out
    uint32_t* info;            // [4] out: iterations, total bits (low, high word), status
    unsigned long long* gkey;  // [n] workspace: gain bits of the qualifying upgrade (0: none)
    uint8_t* ginc;             // [n] workspace: its bit increment
    long long n;
    unsigned long long budget;
    uint32_t mask;             // bit b set: width b allowed
};

__device__ __forceinline__ int alloc_col(int b) { return b == 8 ? 7 : b; }

// w_t(lam): argmin over the allowed widths of L + lam * b (product rounded
// first), ties to the smaller width.
__device__ __forceinline__ int alloc_width_at(const float* L, uint32_t mask, double lam) {
    int best_b = -1;
    double best = 0.0;
#pragma unroll
    for (int b = 0; b <= 8; ++b) {
        if (!((mask >> b) & 1u)) continue;
        const double c = __dadd_rn((double)L[alloc_col(b)], __dmul_rn(lam, (double)b));
        if (best_b < 0 || c < best) { best = c; best_b = b; }
    }
    return best_b;
}

__device__ __forceinline__ int alloc_next(uint32_t mask, int b) {
    for (int n = b + 1; n <= 8; ++n)
        if ((mask >> n) & 1u) return n;
    return -1;
}

// Block-wide sum / max of one value per thread (all threads call).
__device__ __forceinline__ unsigned long long block_sum_u64(unsigned long long v, unsigned long long* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    unsigned long long s = 0;
    for (int i = 0; i < ALLOC_THREADS / 32; ++i) s += red[i];
    return s;
}

__device__ __forceinline__ double block_max_f64(double v, double* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, off));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double m = red[0];
    for (int i = 1; i < ALLOC_THREADS / 32; ++i) m = fmax(m, red[i]);
    return m;
}

__global__ void __launch_bounds__(ALLOC_THREADS, 1) k_allocate_bits(AllocParams p) {
    __shared__ unsigned long long red_u[ALLOC_THREADS / 32];
    __shared__ double red_d[ALLOC_THREADS / 32];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t sh_digit;
    __shared__ unsigned long long sh_acc;
    const long long n = p.n;
    const int tid = threadIdx.x;
    const int bmin = __ffs(p.mask) - 1;
    const unsigned long long B = p.budget;

    // ---- pass 0: S(0), non-finite losses, and hi = the largest per-bit saving over bmin
    unsigned long long s0 = 0, bad = 0;
    double hi_t = 0.0;
    for (long long t = tid; t < n; t += ALLOC_THREADS) {
        const float* L = p.loss + t * 8;
        for (int b = 0; b <= 8; ++b)
            if (((p.mask >> b) & 1u) && !isfinite(L[alloc_col(b)])) bad = 1;
        s0 += (unsigned long long)alloc_width_at(L, p.mask, 0.0);
        const double l0 = (double)L[alloc_col(bmin)];
        for (int b = bmin + 1; b <= 8; ++b) {
            if (!((p.mask >> b) & 1u)) continue;
            hi_t = fmax(hi_t, __ddiv_rn(__dsub_rn(l0, (double)L[alloc_col(b)]), (double)(b - bmin)));
        }
    }
    bad = block_sum_u64(bad, red_u);
    if (bad) {
        if (tid == 0) p.info[3] = MPQ_ERR_NONFINITE;
        return;
    }
    const unsigned long long S0 = block_sum_u64(s0, red_u);
    double hi = block_max_f64(hi_t, red_d);
    uint32_t iters = 1;
    double lam = 0.0;
    unsigned long long S_hi = S0;
    if (S0 > B) {
        auto total_at = [&](double l) -> unsigned long long {
            unsigned long long s = 0;
            for (long long t = tid; t < n; t += ALLOC_THREADS)
                s += (unsigned long long)alloc_width_at(p.loss + t * 8, p.mask, l);
            return block_sum_u64(s, red_u);
        };
        double lo = 0.0;
        S_hi = total_at(hi);
        int steps = 0;
        while (S_hi > B && steps < ALLOC_MAX_STEPS) {   // rounding at the bracket's edge
            hi = __dmul_rn(hi, 2.0);
            S_hi = total_at(hi);
            ++steps;
        }
        while (S_hi != B && steps < ALLOC_MAX_STEPS && __dsub_rn(hi, lo) > __dmul_rn(hi, 0x1p-20)) {
            const double mid = __dmul_rn(__dadd_rn(lo, hi), 0.5);
            if (mid == lo || mid == hi) break;
            const unsigned long long S = total_at(mid);
            ++steps;
            if (S <= B) { hi = mid; S_hi = S; } else { lo = mid; }
        }
        iters += (uint32_t)steps;
        lam = hi;
    }
    // ---- widths at the price
    for (long long t = tid; t < n; t += ALLOC_THREADS)
        p.bits[t] = (uint8_t)alloc_width_at(p.loss + t * 8, p.mask, lam);
    unsigned long long total = S_hi;
    __syncthreads();

    // ---- fill rounds: the longest prefix, in (gain desc, index asc) order, of
    // the qualifying next-width upgrades whose increments fit R
    while (lam != 0.0 || S0 > B) {
        const unsigned long long R = B - total;
        unsigned long long any = 0;
        for (long long t = tid; t < n; t += ALLOC_THREADS) {
            const float* L = p.loss + t * 8;
            const int w = p.bits[t];
            const int nx = alloc_next(p.mask, w);
            unsigned long long key = 0;
            uint8_t inc = 0;
            if (nx >= 0 && (unsigned long long)(nx - w) <= R) {
                const double g = __ddiv_rn(__dsub_rn((double)L[alloc_col(w)], (double)L[alloc_col(nx)]),
                                           (double)(nx - w));
                if (g > 0.0) { key = (unsigned long long)__double_as_longlong(g); inc = (uint8_t)(nx - w); }
            }
            p.gkey[t] = key;
            p.ginc[t] = inc;
            any |= key;
        }
        if (block_sum_u64(any != 0 ? 1ull : 0ull, red_u) == 0) break;
        // radix select over the 96-bit key (gain bits, ~index), most significant
        // digit first.  Digits 11..4 are the gain's bytes, 3..0 the inverted
        // index's.  acc = increments of the keys already known to be in the
        // prefix; the fixed high digits are those of the bucket holding the
        // first key that does not fit.  If every bucket at a level fits, all
        // keys whose fixed digits are >= the prefix are taken (dstop = that
        // level); after all 12 levels the prefix is that first key itself.
        unsigned long long prefix_hi = 0;   // gain digits fixed so far
        uint32_t prefix_lo = 0;             // index digits fixed so far
        unsigned long long acc = 0;
        int dstop = -1;
        for (int d = 11; d >= 0; --d) {
            for (int i = tid; i < 256; i += ALLOC_THREADS) hist[i] = 0u;
            __syncthreads();
            for (long long t = tid; t < n; t += ALLOC_THREADS) {
                const unsigned long long g = p.gkey[t];
                if (!g) continue;
                const uint32_t il = ~(uint32_t)t;
                bool match;
                uint32_t digit;
                if (d >= 4) {
                    const int sh = 8 * (d - 4);
                    match = (d == 11) || ((g >> (sh + 8)) == prefix_hi);
                    digit = (uint32_t)(g >> sh) & 0xFFu;
                } else {
                    const int sh = 8 * d;
                    match = (g == prefix_hi) && ((d == 3) || ((il >> (sh + 8)) == prefix_lo));
                    digit = (il >> sh) & 0xFFu;
                }
                if (match) atomicAdd(&hist[digit], (uint32_t)p.ginc[t]);
            }
            __syncthreads();
            if (tid == 0) {
                unsigned long long a2 = acc;
                uint32_t split = 256u;
                for (int v = 255; v >= 0; --v) {
                    if (a2 + hist[v] <= R) { a2 += hist[v]; continue; }
                    split = (uint32_t)v;
                    break;
                }
                sh_acc = a2;
                sh_digit = split;
            }
            __syncthreads();
            const uint32_t split = sh_digit;
            acc = sh_acc;
            __syncthreads();
            if (split == 256u) { dstop = d; break; }
            if (d >= 4) prefix_hi = (prefix_hi << 8) | split;
            else prefix_lo = (prefix_lo << 8) | split;
        }
        // take the prefix
        unsigned long long taken = 0;
        for (long long t = tid; t < n; t += ALLOC_THREADS) {
            const unsigned long long g = p.gkey[t];
            if (!g) continue;
            const uint32_t il = ~(uint32_t)t;
            bool in;
            if (dstop >= 4)
                in = (dstop == 11) || ((g >> (8 * (dstop - 3))) >= prefix_hi);
            else if (dstop >= 0)
                in = (g > prefix_hi) || (g == prefix_hi && ((dstop == 3) || ((il >> (8 * (dstop + 1))) >= prefix_lo)));
            else
                in = (g > prefix_hi) || (g == prefix_hi && il > prefix_lo);
            if (in) {
                p.bits[t] = (uint8_t)(p.bits[t] + p.ginc[t]);
                taken += p.ginc[t];
            }
        }
        taken = block_sum_u64(taken, red_u);
        if (taken == 0) break;
        total += taken;
        ++iters;
        __syncthreads();
    }
    if (tid == 0) {
        p.info[0] = iters;
        p.info[1] = (uint32_t)total;
        p.info[2] = (uint32_t)(total >> 32);
        p.info[3] = MPQ_OK;
    }
}

}  // namespace mpq
