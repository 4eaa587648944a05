// mpq_api.cu -- the C ABI of libmpq (declared in include/mpq.h): host-side
// validation, the plan (segment offsets, block table, decode schedule) and
// the kernel launches.  The library allocates no device memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <vector>

#include "../../include/mpq.h"
#include "common.cuh"
#include "k_alloc.cuh"
#include "k_decode.cuh"
#include "k_pack.cuh"
#include "k_prefill.cuh"
#include "k_tcdec.cuh"
#include "k_xprep.cuh"
#include "k_ycast.cuh"

using namespace mpq;

namespace {

constexpr int kMaxUnits = 148 * DEC_CTAS_PER_SM * DEC_WARPS;   // one run per resident decode warp
constexpr uint64_t kMinUnitCost = 4096; // cost units (bytes) per run, at least
constexpr int kMaxDecodeTokens = DEC_MAX_TOKENS;   // tokens per decode launch
// Larger batches take the tensor-core kernel: it streams every weight tile
// once for any M <= 256 and its time hardly grows with M up to 128, while a
// decode launch (<= 8 tokens) costs about as much as the whole tensor-core
// call at M = 8 and twice as much at M = 16 (measured on the 14336 x 4096 and
// 28672 x 8192 layers).
constexpr int kDecodeMaxM = 8;
// 9..16 tokens on layers of at least 100 tiles of 128 rows: the integer
// tensor-core kernel (k_tcdec; one CTA per tile, all k blocks); smaller
// layers, and layers with 16-bit blocks, take k_prefill, which splits k
// across CTAs (measured: the 8192-row q projection at 16 tokens 68 us with
// 64 k_tcdec CTAs against 38 us split)
constexpr int kTcDecMaxM = 16;
constexpr int kTcDecMinTiles = 100;
constexpr int kPackRowsPerCta = 1;
constexpr size_t kPackStagedMaxSmem = 227 * 1024;   // the sm_100 maximum per CTA

inline size_t round256(size_t v) { return (v + 255) & ~size_t(255); }

inline bool bits_ok(int b) {
    return b == 0 || b == 1 || b == 2 || b == 3 || b == 4 || b == 5 || b == 6 || b == 8 || b == 16;
}

// Estimated cost of one block for the decode schedule, in bytes: what it
// streams (payload, scales/zeros, one activation variant) plus a stand-in
// for its decode work (code extraction and tensor-core passes).  Split
// widths (3, 5, 6) make two passes.  Zero-bit blocks only cost bookkeeping.
inline uint64_t block_cost(int b) {
    static const uint32_t work[9] = {0, 2048, 2048, 4096, 2304, 4352, 4352, 0, 2560};
    if (b == 16) return 16384u + 256u + 272u + 2048u;   // two halves, bf16 mma
    return b == 0 ? 32u : 1024u * (uint64_t)b + 256u + 272u + work[b];
}

inline uint64_t sched_words_of(int64_t n_units, uint64_t n_stages) {
    return (uint64_t)n_units * DESC_WORDS + (uint64_t)STAGE_WORDS * n_stages;
}

// Layout of the plan for (N, K, bits) -- the same arithmetic as mpq_plan.
// sched (optional) receives the decode schedule: n_units run descriptors of
// DESC_WORDS words (see k_decode.cuh), then one STAGE_WORDS-word stage
// descriptor per non-zero block, in block order.
mpq_status make_plan(int32_t N, int32_t K, const uint8_t* bits, mpq_layout* L,
                     std::vector<mpq_block>* table, std::vector<uint32_t>* sched) {
    if (N <= 0 || K <= 0 || N % 64 != 0 || K % 128 != 0) return MPQ_ERR_SHAPE;
    const int NB = N / 64, KB = K / 128;
    const int64_t T = (int64_t)NB * KB;
    std::memset(L, 0, sizeof *L);
    L->N = N; L->K = K; L->NB = NB; L->KB = KB;
    uint64_t count[17] = {0};
    for (int64_t t = 0; t < T; ++t) {
        if (!bits_ok(bits[t])) return MPQ_ERR_BITS;
        ++count[bits[t]];
    }
    static const int order[8] = {1, 2, 3, 4, 5, 6, 8, 16};
    uint64_t off = 0;
    for (int b : order) {
        L->seg_off[b] = off;
        L->seg_bytes[b] = count[b] * 1024u * (uint64_t)b;
        off += L->seg_bytes[b];
    }
    L->codes_bytes = off;
    if (off >= (1ull << 32)) return MPQ_ERR_SHAPE;
    uint64_t nz = 0, total = 0, n16 = 0;
    for (int64_t t = 0; t < T; ++t) total += bits[t], nz += bits[t] != 0, n16 += bits[t] == 16;
    L->n_sz = 64u * nz;
    L->bit_total = total;
    const uint64_t n_stages = nz + n16;   // a 16-bit block streams as two halves

    // decode runs: cut the cost prefix into about equal parts, drop empty runs
    std::vector<uint64_t> pre((size_t)T + 1, 0);
    for (int64_t t = 0; t < T; ++t) pre[(size_t)t + 1] = pre[(size_t)t] + block_cost(bits[t]);
    const uint64_t cost = pre[(size_t)T];
    int64_t want = (int64_t)((cost + kMinUnitCost - 1) / kMinUnitCost);
    want = std::max<int64_t>(1, std::min<int64_t>(want, std::min<int64_t>(kMaxUnits, T)));
    std::vector<uint32_t> bounds;
    bounds.reserve((size_t)want + 1);
    bounds.push_back(0u);
    if ((uint64_t)want >= nz) {
        // at least as many runs as non-zero blocks (a small layer): one
        // non-zero block per run, so that no warp gets two -- zero-bit blocks
        // join the run before them
        bool seen_nz = false;
        for (int64_t t = 0; t < T; ++t) {
            if (!bits[t]) continue;
            if (seen_nz) bounds.push_back((uint32_t)t);
            seen_nz = true;
        }
    } else {
        for (int64_t u = 1; u < want; ++u) {
            // run u starts at the first block whose cost prefix reaches u*cost/want
            const uint64_t target = (uint64_t)((unsigned __int128)u * cost / (uint64_t)want);
            const uint32_t tb = (uint32_t)(std::lower_bound(pre.begin(), pre.begin() + T, target) - pre.begin());
            if (tb > bounds.back() && tb < (uint32_t)T) bounds.push_back(tb);
        }
    }
    bounds.push_back((uint32_t)T);
    const int64_t units = (int64_t)bounds.size() - 1;
    L->n_units = (int32_t)units;
    if (sched_words_of(units, n_stages) >= (1ull << 31)) return MPQ_ERR_SHAPE;
    L->sched_words = (int32_t)sched_words_of(units, n_stages);

    if (table) {
        table->assign((size_t)T, mpq_block{0, 0, 0, 0});
        uint64_t seen[17] = {0}, k = 0, bp = 0;
        for (int64_t t = 0; t < T; ++t) {
            const int b = bits[t];
            mpq_block& e = (*table)[(size_t)t];
            e.bit_prefix = (uint32_t)bp;
            if (b) {
                e.code_off = (uint32_t)(L->seg_off[b] + seen[b] * 1024u * (uint64_t)b);
                e.sz_off = (uint32_t)(64u * k);
                e.bits = (uint32_t)b;
                ++seen[b];
                ++k;
            }
            bp += (uint64_t)b;
        }
    }
    if (sched) {
        sched->assign((size_t)L->sched_words, 0u);
        // runs meeting each block row, and the first partial slot of shared rows
        std::vector<uint32_t> row_first((size_t)NB, 0u), row_last((size_t)NB, 0u), row_slot((size_t)NB, 0u);
        for (int64_t u = units - 1; u >= 0; --u)
            for (uint32_t nb = bounds[(size_t)u] / KB; nb <= (bounds[(size_t)u + 1] - 1) / KB; ++nb)
                row_first[nb] = (uint32_t)u;
        for (int64_t u = 0; u < units; ++u)
            for (uint32_t nb = bounds[(size_t)u] / KB; nb <= (bounds[(size_t)u + 1] - 1) / KB; ++nb)
                row_last[nb] = (uint32_t)u;
        uint64_t slots = 0;
        for (int nb = 0; nb < NB; ++nb) {
            const uint32_t nc = row_last[nb] - row_first[nb] + 1;
            row_slot[nb] = (uint32_t)slots;
            if (nc > 1) slots += nc;
        }
        // stage descriptors: every non-zero block in block order (a 16-bit
        // block twice: rows 0..31, then rows 32..63)
        uint32_t* st = sched->data() + (size_t)units * DESC_WORDS;
        uint64_t seen[17] = {0}, k = 0, si = 0;
        for (int64_t t = 0; t < T; ++t) {
            const int b = bits[t];
            if (!b) continue;
            const uint32_t code = (uint32_t)(L->seg_off[b] + seen[b] * 1024u * (uint64_t)b);
            for (uint32_t half = 0; half < (b == 16 ? 2u : 1u); ++half) {
                uint32_t* e = st + (size_t)si * STAGE_WORDS;
                e[SW_CODE] = code + half * 8192u;
                e[SW_SZ] = (uint32_t)(64u * k);
                e[SW_KB_BITS] = (uint32_t)(t % KB) | ((uint32_t)b << 16) | (half << 24);
                e[SW_NB] = (uint32_t)(t / KB);
                ++si;
            }
            ++seen[b];
            ++k;
        }
        auto stages_of = [&](int b) -> uint64_t { return b == 0 ? 0u : b == 16 ? 2u : 1u; };
        uint64_t stage = 0;
        int64_t t = 0;
        for (int64_t u = 0; u < units; ++u) {
            const uint32_t t0 = bounds[(size_t)u], t1 = bounds[(size_t)u + 1];
            uint32_t* d = sched->data() + (size_t)u * DESC_WORDS;
            for (; t < t0; ++t) stage += stages_of(bits[t]);
            uint64_t ns = 0;
            for (uint32_t j = t0; j < t1; ++j) ns += stages_of(bits[j]);
            d[DW_T0] = t0;
            d[DW_T1] = t1;
            d[DW_S0] = (uint32_t)stage;
            d[DW_NS] = (uint32_t)ns;
            const uint32_t ra = t0 / KB, rb = (t1 - 1) / KB;
            d[DW_A_SLOT] = row_slot[ra];
            d[DW_A_NC] = row_last[ra] - row_first[ra] + 1u;
            d[DW_A_IDX] = (uint32_t)u - row_first[ra];
            d[DW_B_SLOT] = row_slot[rb];
            d[DW_B_NC] = row_last[rb] - row_first[rb] + 1u;
            d[DW_B_IDX] = (uint32_t)u - row_first[rb];
        }
    }
    return MPQ_OK;
}

bool perm_ok(const int32_t* p, int n) {
    std::vector<char> seen((size_t)n, 0);
    for (int i = 0; i < n; ++i) {
        if (p[i] < 0 || p[i] >= n || seen[(size_t)p[i]]) return false;
        seen[(size_t)p[i]] = 1;
    }
    return true;
}

inline mpq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MPQ_OK : MPQ_ERR_CUDA; }

constexpr size_t kUnpermMaxBytes = 200 * 1024;   // one row of y in shared memory

// Tensor-core launch shape: 256-token tiles beyond one 128-token tile, and
// the k blocks split across CTAs (partial sums reduced by k_finish_rows)
// while the grid stays within one wave of 148 SMs.  A split grid has at most
// 74 tiles of 128 rows, so a row of y then always fits in shared memory.
struct PrefillShape {
    int BN, tiles_n, tiles_m, splits, kb_per_split;
};
PrefillShape prefill_shape(int N, int K, int M) {
    PrefillShape ps{};
    const int NB = N / 64, KB = K / 128;
    ps.BN = M > 128 ? 256 : 128;
    // 256-token stages leave shared memory for the widths of up to ~440 k blocks
    if (ps.BN == 256 && sizeof(PrefillSmem<256>) + 1024 + (size_t)2 * KB > (size_t)227 * 1024) ps.BN = 128;
    ps.tiles_n = (NB + 1) / 2;
    ps.tiles_m = (M + ps.BN - 1) / ps.BN;
    const int ctas = ps.tiles_n * ps.tiles_m;
    int splits = 1;
    while (splits < 8 && ctas * splits * 2 <= 148 && KB / (splits * 2) >= 4 &&
           (size_t)N * 4 <= kUnpermMaxBytes)
        splits *= 2;
    ps.kb_per_split = (KB + splits - 1) / splits;
    ps.splits = (KB + ps.kb_per_split - 1) / ps.kb_per_split;
    return ps;
}

// Workspace carve-up of mpq_linear.
struct LinearWs {
    uint32_t* err;
    uint32_t* counters;
    float* tok_scale;
    __half* xq;
    float* partial;
    size_t bytes;
};

LinearWs carve_linear(void* ws, const mpq_layer* layer, int32_t M) {
    LinearWs w{};
    const int NB = layer->N / 64;
    size_t off = 256;
    uint8_t* base = static_cast<uint8_t*>(ws);
    w.err = reinterpret_cast<uint32_t*>(base);
    w.counters = reinterpret_cast<uint32_t*>(base + off);
    off += round256((size_t)NB * 4);
    w.tok_scale = reinterpret_cast<float*>(base + off);
    off += round256((size_t)M * 4);
    w.xq = reinterpret_cast<__half*>(base + off);
    // decode: [KB][XQD_REC * M]; tensor-core path: [M][K] fp16 (smaller)
    off += round256((size_t)(layer->K / 128) * M * XQD_REC);
    // partial sums of shared block rows: at most n_units + NB slots of
    // 64 rows x (tokens per launch)
    w.partial = reinterpret_cast<float*>(base + off);
    if (M > kDecodeMaxM) {
        // tensor-core path: [splits][M][N] fp32 partial sums when k is split
        const PrefillShape ps = prefill_shape(layer->N, layer->K, M);
        off += round256(ps.splits > 1 ? (size_t)ps.splits * M * layer->N * 4 : 0);
    } else {
        off += round256((size_t)(layer->n_units + NB) * 64 * std::min(M, kMaxDecodeTokens) * 4);
    }
    w.bytes = off;
    return w;
}

// The kernels read the layer's buffers with 16-byte vector loads and bulk
// copies, which need 16-byte aligned addresses.
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool layer_aligned(const mpq_layer* L) {
    return aligned16(L->codes) && aligned16(L->table) && aligned16(L->sched) && aligned16(L->scales) &&
           aligned16(L->zeros) && aligned16(L->row_perm) && aligned16(L->col_perm);
}

mpq_status check_layer(const mpq_layer* L) {
    if (!L) return MPQ_ERR_ARG;
    if (L->N <= 0 || L->K <= 0 || L->N % 64 || L->K % 128) return MPQ_ERR_SHAPE;
    if (!L->table || !L->sched || L->n_units <= 0) return MPQ_ERR_ARG;
    if (!layer_aligned(L)) return MPQ_ERR_ARG;
    return MPQ_OK;
}

// Raises a kernel's dynamic shared-memory limit once per device.
template <typename F>
cudaError_t ensure_smem_attr(F* kernel, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}
std::atomic<uint64_t> g_decode_attr{0};
std::atomic<uint64_t> g_decode_attr8{0};
std::atomic<uint64_t> g_decode_attr16{0};
std::atomic<uint64_t> g_decode_attr_w{0};
std::atomic<uint64_t> g_decode_attr8_w{0};
std::atomic<uint64_t> g_decode_attr16_w{0};
std::atomic<uint64_t> g_decode_attr_f_w{0};
std::atomic<uint64_t> g_decode_attr_g_w{0};
std::atomic<uint64_t> g_decode_attr_f{0};
std::atomic<uint64_t> g_decode_attr_g{0};
std::atomic<uint64_t> g_prefill_attr{0};
std::atomic<uint64_t> g_prefill_attr256{0};
std::atomic<uint64_t> g_unperm_attr{0};
std::atomic<uint64_t> g_pack_attr{0};

// cuTensorMapEncodeTiled from the driver, looked up through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// 2-D fp16 [rows][K] tensor, 64 x box_rows boxes, 128-byte swizzle.
bool make_tmap_fp16(CUtensorMap* map, const void* ptr, int K, int rows, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int BN>
size_t prefill_smem_bytes(int KB) {
    return sizeof(PrefillSmem<BN>) + 1024 + (size_t)2 * KB;
}


}  // namespace

extern "C" {

mpq_status mpq_plan(int32_t N, int32_t K, const uint8_t* bits_host, mpq_layout* out) {
    if (!out || !bits_host) return MPQ_ERR_ARG;
    return make_plan(N, K, bits_host, out, nullptr, nullptr);
}

mpq_status mpq_plan_schedule(const mpq_layout* L, const uint8_t* bits_host, uint32_t* sched_host) {
    if (!L || !bits_host || !sched_host) return MPQ_ERR_ARG;
    mpq_layout chk;
    std::vector<uint32_t> sched;
    mpq_status st = make_plan(L->N, L->K, bits_host, &chk, nullptr, &sched);
    if (st != MPQ_OK) return st;
    if (chk.n_units != L->n_units || chk.sched_words != L->sched_words) return MPQ_ERR_ARG;
    std::memcpy(sched_host, sched.data(), sched.size() * 4);
    return MPQ_OK;
}

size_t mpq_pack_workspace_size(const mpq_layout*) { return 256; }

mpq_status mpq_pack(const mpq_layout* L, const void* W_dev, const uint8_t* bits_host,
                    const int32_t* row_perm_host, const int32_t* col_perm_host,
                    const mpq_layer* out, void* ws, size_t ws_bytes, void* stream) {
    return mpq_pack_timed(L, W_dev, bits_host, row_perm_host, col_perm_host, out, ws, ws_bytes,
                          stream, nullptr, nullptr);
}

mpq_status mpq_pack_timed(const mpq_layout* L, const void* W_dev, const uint8_t* bits_host,
                          const int32_t* row_perm_host, const int32_t* col_perm_host,
                          const mpq_layer* out, void* ws, size_t ws_bytes, void* stream,
                          void* ev_begin, void* ev_end) {
    if (!L || !W_dev || !bits_host || !out) return MPQ_ERR_ARG;
    mpq_layout chk;
    std::vector<mpq_block> table;
    std::vector<uint32_t> sched;
    mpq_status st = make_plan(L->N, L->K, bits_host, &chk, &table, &sched);
    if (st != MPQ_OK) return st;
    if (chk.codes_bytes != L->codes_bytes || chk.n_sz != L->n_sz || chk.n_units != L->n_units ||
        chk.sched_words != L->sched_words)
        return MPQ_ERR_ARG;
    if (out->N != L->N || out->K != L->K || out->n_units != L->n_units) return MPQ_ERR_ARG;
    if (row_perm_host && !perm_ok(row_perm_host, L->N)) return MPQ_ERR_PERM;
    if (col_perm_host && !perm_ok(col_perm_host, L->K)) return MPQ_ERR_PERM;
    if (col_perm_host && L->K > 65536) return MPQ_ERR_SHAPE;
    if ((row_perm_host != nullptr) != (out->row_perm != nullptr) ||
        (col_perm_host != nullptr) != (out->col_perm != nullptr))
        return MPQ_ERR_ARG;
    if (!out->table || !out->sched || (L->codes_bytes && !out->codes) ||
        (L->n_sz && (!out->scales || !out->zeros)))
        return MPQ_ERR_ARG;
    if (!layer_aligned(out) || !aligned16(W_dev)) return MPQ_ERR_ARG;
    if (!ws || ws_bytes < mpq_pack_workspace_size(L)) return MPQ_ERR_WORKSPACE;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t T = table.size();
    cudaError_t e = cudaMemcpyAsync(const_cast<mpq_block*>(out->table), table.data(),
                                    T * sizeof(mpq_block), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(const_cast<uint32_t*>(out->sched), sched.data(),
                            sched.size() * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && row_perm_host)
        e = cudaMemcpyAsync(const_cast<int32_t*>(out->row_perm), row_perm_host,
                            (size_t)L->N * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && col_perm_host)
        e = cudaMemcpyAsync(const_cast<int32_t*>(out->col_perm), col_perm_host,
                            (size_t)L->K * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, 4, s);
    if (e != cudaSuccess) return MPQ_ERR_CUDA;
    if (ev_begin && cudaEventRecord(static_cast<cudaEvent_t>(ev_begin), s) != cudaSuccess)
        return MPQ_ERR_CUDA;
    if (L->bit_total == 0) {   // nothing to quantize
        if (ev_end && cudaEventRecord(static_cast<cudaEvent_t>(ev_end), s) != cudaSuccess)
            return MPQ_ERR_CUDA;
        return MPQ_OK;
    }

    PackParams p{};
    p.W = static_cast<const uint16_t*>(W_dev);
    p.table = out->table;
    p.row_perm = out->row_perm;
    p.col_perm = out->col_perm;
    p.codes = static_cast<uint8_t*>(const_cast<void*>(out->codes));
    p.scales = const_cast<uint16_t*>(out->scales);
    p.zeros = const_cast<uint16_t*>(out->zeros);
    p.err = static_cast<uint32_t*>(ws);
    p.N = L->N;
    p.K = L->K;
    p.KB = L->KB;
    p.rows_per_cta = kPackRowsPerCta;
    // two row buffers, the column order as uint16, two mbarriers; rows longer
    // than that allows are read from global memory by the unstaged kernel
    const size_t row_bytes = (size_t)L->K * 2;
    const size_t smem = 2 * row_bytes + ((row_bytes + 15) & ~size_t(15)) + 64;
    const bool staged = smem <= kPackStagedMaxSmem;
    if (staged) {
        e = ensure_smem_attr(k_pack<true>, (int)kPackStagedMaxSmem, g_pack_attr);
        if (e != cudaSuccess) return MPQ_ERR_CUDA;
    }
    const int grid = (L->N + kPackRowsPerCta - 1) / kPackRowsPerCta;
    if (staged) k_pack<true><<<grid, PACK_THREADS, smem, s>>>(p);
    else k_pack<false><<<grid, PACK_THREADS, 0, s>>>(p);
    e = cudaGetLastError();
    if (e == cudaSuccess && ev_end) e = cudaEventRecord(static_cast<cudaEvent_t>(ev_end), s);
    return cuda_status(e);
}

size_t mpq_linear_workspace_size(const mpq_layer* layer, int32_t M) {
    if (!layer || M < 0) return 0;
    return carve_linear(nullptr, layer, M).bytes;
}

mpq_status mpq_linear(const mpq_layer* layer, const void* x_dev, int32_t M, float* y_dev,
                      void* ws, size_t ws_bytes, void* stream) {
    return mpq_linear_timed(layer, x_dev, M, y_dev, ws, ws_bytes, stream, nullptr, nullptr);
}

size_t mpq_linear_typed_workspace_size(const mpq_layer* layer, int32_t M, mpq_ydtype ydt) {
    if (!layer || M < 0) return 0;
    const size_t base = round256(carve_linear(nullptr, layer, M).bytes);
    // bf16: the fp32 product is kept in the workspace before rounding
    return ydt == MPQ_Y_BF16 ? base + (size_t)M * layer->N * 4 : base;
}

mpq_status mpq_linear_typed(const mpq_layer* layer, const void* x_dev, int32_t M, void* y_dev,
                            mpq_ydtype ydt, void* ws, size_t ws_bytes, void* stream) {
    if (ydt == MPQ_Y_F32)
        return mpq_linear(layer, x_dev, M, static_cast<float*>(y_dev), ws, ws_bytes, stream);
    if (ydt != MPQ_Y_BF16) return MPQ_ERR_ARG;
    mpq_status st = check_layer(layer);
    if (st != MPQ_OK) return st;
    if (M < 0) return MPQ_ERR_SHAPE;
    if (M == 0) return MPQ_OK;
    if (!x_dev || !y_dev || !aligned16(x_dev)) return MPQ_ERR_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return MPQ_ERR_WORKSPACE;
    const size_t base = round256(carve_linear(nullptr, layer, M).bytes);
    const size_t n = (size_t)M * layer->N;
    if (ws_bytes < base + n * 4) return MPQ_ERR_WORKSPACE;
    float* y32 = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + base);
    st = mpq_linear(layer, x_dev, M, y32, ws, base, stream);
    if (st != MPQ_OK) return st;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t c{};
    c.gridDim = dim3((unsigned)std::min<size_t>((n / 4 + YCAST_THREADS - 1) / YCAST_THREADS + 1, 148 * 8));
    c.blockDim = dim3(YCAST_THREADS);
    c.stream = static_cast<cudaStream_t>(stream);
    c.attrs = pdl;
    c.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&c, k_y_to_bf16, (const float*)y32,
                                          static_cast<uint16_t*>(y_dev), n));
}

}  // extern "C"

namespace {

// One token on a layer whose runs hold at most two blocks on average: the
// decode kernel builds its activation records itself (no prologue kernel, one
// launch boundary less on this latency-bound path).
bool fused_one_token(const mpq_layer* layer, int32_t M) {
    const size_t blocks = (size_t)(layer->N / 64) * (layer->K / 128);
    return M == 1 && blocks <= 2 * (size_t)layer->n_units;
}

// Decode-kernel arguments of one layer (the token group is set by the caller).
DecodeParams decode_params(const mpq_layer* layer, const void* x_dev, int32_t M, float* y_dev,
                           const LinearWs& w) {
    DecodeParams dp{};
    dp.codes = static_cast<const uint8_t*>(layer->codes);
    dp.desc = layer->sched;
    dp.stages = reinterpret_cast<const uint4*>(layer->sched + (size_t)layer->n_units * DESC_WORDS);
    dp.scales = layer->scales;
    dp.zeros = layer->zeros;
    dp.row_perm = layer->row_perm;
    dp.xq = reinterpret_cast<const uint8_t*>(w.xq);
    dp.x = static_cast<const uint16_t*>(x_dev);
    dp.col_perm = layer->col_perm;
    dp.y = y_dev;
    dp.partial = w.partial;
    dp.counters = w.counters;
    dp.err = w.err;
    dp.N = layer->N;
    dp.K = layer->K;
    dp.NB = layer->N / 64;
    dp.KB = layer->K / 128;
    dp.M_total = M;
    dp.n_units = layer->n_units;
    dp.m0 = 0;
    dp.Mg = 1;
    return dp;
}

std::atomic<uint64_t> g_tcdec_attr1{0};
std::atomic<uint64_t> g_tcdec_attr2{0};

template <int WPQ>
size_t tcdec_smem_bytes(int KB) {
    return sizeof(TcSmem<TC_MP, WPQ>) + 1024 + (size_t)2 * KB;
}

template <int WPQ>
mpq_status tcdec_launch(const TcParams& tp, int tiles, cudaStream_t s, cudaLaunchAttribute* pdl,
                        std::atomic<uint64_t>& attr) {
    const size_t smem = tcdec_smem_bytes<WPQ>(tp.KB);
    const size_t cap = WPQ == 2 ? 113 * 1024 : 227 * 1024;   // two CTAs per SM, or one
    if (smem > cap) return MPQ_ERR_SHAPE;
    cudaError_t e = ensure_smem_attr(k_tcdec<TC_MP, WPQ>, (int)cap, attr);
    if (e != cudaSuccess) return MPQ_ERR_CUDA;
    cudaLaunchConfig_t c{};
    c.gridDim = dim3((unsigned)tiles);
    c.blockDim = dim3(TcCfg<TC_MP, WPQ>::THREADS);
    c.dynamicSmemBytes = smem;
    c.stream = s;
    c.attrs = pdl;
    c.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&c, k_tcdec<TC_MP, WPQ>, tp));
}

// 9..16 tokens on a layer without 16-bit blocks: activation records
// (k_xprep_tcdec), then the integer tensor-core kernel, chained by
// programmatic dependent launch.  Grids of at most one wave take the
// variant with one CTA per SM and more worker warps; larger grids the
// one with two CTAs per SM (one wave instead of two).
mpq_status tcdec_run(const mpq_layer* layer, const void* x_dev, int32_t M, float* y_dev, const LinearWs& w,
                     cudaStream_t s, cudaLaunchConfig_t xc, void* ev_begin, void* ev_end) {
    const int KB = layer->K / 128, NB = layer->N / 64;
    const int tiles = (NB + 1) / 2;
    XprepTcParams xt{};
    xt.x = static_cast<const uint16_t*>(x_dev);
    xt.col_perm = layer->col_perm;
    xt.rec = reinterpret_cast<uint8_t*>(w.xq);
    xt.M = M;
    xt.K = layer->K;
    xt.MP = TC_MP;
    xt.NP = 3 * TC_MP;
    xt.REC = TcCfg<TC_MP, 2>::REC;
    const int items = KB * TC_MP, per = XPREP_THREADS / 32;
    xc.gridDim = dim3((unsigned)((items + per - 1) / per));
    cudaError_t e = cudaLaunchKernelEx(&xc, k_xprep_tcdec, xt);
    if (e != cudaSuccess) return MPQ_ERR_CUDA;
    TcParams tp{};
    tp.codes = static_cast<const uint8_t*>(layer->codes);
    tp.table = layer->table;
    tp.scales = layer->scales;
    tp.zeros = layer->zeros;
    tp.row_perm = layer->row_perm;
    tp.rec = xt.rec;
    tp.y = y_dev;
    tp.err = w.err;
    tp.N = layer->N;
    tp.K = layer->K;
    tp.NB = NB;
    tp.KB = KB;
    tp.M = M;
    if (ev_begin && cudaEventRecord(static_cast<cudaEvent_t>(ev_begin), s) != cudaSuccess) return MPQ_ERR_CUDA;
    cudaLaunchAttribute* pdl = const_cast<cudaLaunchAttribute*>(xc.attrs);
    const mpq_status st = tiles <= 148 ? tcdec_launch<4>(tp, tiles, s, pdl, g_tcdec_attr1)
                                       : tcdec_launch<2>(tp, tiles, s, pdl, g_tcdec_attr2);
    if (st != MPQ_OK) return st;
    if (ev_end && cudaEventRecord(static_cast<cudaEvent_t>(ev_end), s) != cudaSuccess) return MPQ_ERR_CUDA;
    return MPQ_OK;
}

// mpq_linear on a carved workspace (arguments already checked).
mpq_status linear_run(const mpq_layer* layer, const void* x_dev, int32_t M, float* y_dev,
                      const LinearWs& w, cudaStream_t s, void* ev_begin, void* ev_end) {
    const int NB = layer->N / 64, KB = layer->K / 128;
    const bool use_tc = M > kDecodeMaxM;
    const bool use_tcdec = use_tc && M <= kTcDecMaxM && (layer->flags & MPQ_LAYER_16BIT) == 0 &&
                           (NB + 1) / 2 >= kTcDecMinTiles;
    if (!use_tc && (uint64_t)KB * (uint64_t)M * XQD_REC >= (1ull << 32)) return MPQ_ERR_SHAPE;
    const bool fused = !use_tc && fused_one_token(layer, M);
    XprepParams xp{};
    xp.x = static_cast<const uint16_t*>(x_dev);
    xp.col_perm = layer->col_perm;
    xp.xq = w.xq;
    xp.tok_scale = w.tok_scale;
    xp.counters = w.counters;
    xp.n_counters = NB;
    xp.M = M;
    xp.K = layer->K;
    // Every launch may overlap the end of the kernel before it (programmatic
    // dependent launch): each kernel waits (griddepcontrol.wait) for its
    // predecessor before it touches memory the predecessor uses.
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t xc{};
    xc.blockDim = dim3(XPREP_THREADS);
    xc.stream = s;
    xc.attrs = pdl;
    xc.numAttrs = 1;
    cudaError_t e;
    if (use_tcdec)
        return tcdec_run(layer, x_dev, M, y_dev, w, s, xc, ev_begin, ev_end);
    if (use_tc) {
        xp.counters = nullptr;
        // few tokens: several CTAs per token, about two waves in all
        const int per_token = std::max(1, std::min(layer->K / 1024, (2 * 148 + M - 1) / M));
        xc.gridDim = dim3((unsigned)M, (unsigned)per_token);
        e = cudaLaunchKernelEx(&xc, k_xprep<XP_PREFILL>, xp);
    } else if (!fused) {
        const int items = KB * M, per = XPREP_THREADS / 32;
        xc.gridDim = dim3((unsigned)((items + per - 1) / per));
        e = cudaLaunchKernelEx(&xc, k_xprep_decode, xp);
    } else {
        e = cudaSuccess;
    }
    if (e != cudaSuccess) return MPQ_ERR_CUDA;

    if (use_tc) {
        const PrefillShape shape = prefill_shape(layer->N, layer->K, M);
        const bool wide = shape.BN == 256;
        const int BN = shape.BN;
        const size_t smem = wide ? prefill_smem_bytes<256>(KB) : prefill_smem_bytes<128>(KB);
        if (smem > 227 * 1024) return MPQ_ERR_SHAPE;
        e = wide ? ensure_smem_attr(k_prefill<256>, 227 * 1024, g_prefill_attr256)   // the sm_100 maximum
                 : ensure_smem_attr(k_prefill<128>, 227 * 1024, g_prefill_attr);
        if (e != cudaSuccess) return MPQ_ERR_CUDA;
        CUtensorMap tmap;
        if (!make_tmap_fp16(&tmap, w.xq, layer->K, M, BN)) return MPQ_ERR_CUDA;
        PrefillParams pp{};
        pp.codes = static_cast<const uint8_t*>(layer->codes);
        pp.table = layer->table;
        pp.scales = layer->scales;
        pp.zeros = layer->zeros;
        pp.row_perm = layer->row_perm;
        pp.tok_scale = w.tok_scale;
        pp.tiles_m = shape.tiles_m;
        pp.kb_per_split = shape.kb_per_split;
        pp.err = w.err;
        pp.N = layer->N;
        pp.K = layer->K;
        pp.NB = NB;
        pp.KB = KB;
        pp.M = M;
        pp.tiles_n = (NB + 1) / 2;
        // Output: split partials, or y in W' row order reordered in place, go
        // through k_finish_rows (coalesced stores); the epilogue scatters
        // through row_perm itself only when a row of y does not fit in shared
        // memory (and k is not split).
        const bool row_fits = (size_t)layer->N * 4 <= kUnpermMaxBytes;
        const bool finish = shape.splits > 1 || (layer->row_perm && row_fits);
        pp.out_scatter = finish ? 0 : 1;
        pp.out = shape.splits > 1 ? w.partial : y_dev;
        if (finish) {
            e = ensure_smem_attr(k_finish_rows, (int)kUnpermMaxBytes, g_unperm_attr);
            if (e != cudaSuccess) return MPQ_ERR_CUDA;
        }
        const int tiles_m = shape.tiles_m;
        cudaLaunchConfig_t pc{};
        pc.gridDim = dim3((unsigned)(pp.tiles_n * tiles_m * shape.splits));
        pc.blockDim = dim3(PF_THREADS);
        pc.dynamicSmemBytes = smem;
        pc.stream = s;
        pc.attrs = pdl;
        pc.numAttrs = 1;
        if (ev_begin && cudaEventRecord(static_cast<cudaEvent_t>(ev_begin), s) != cudaSuccess)
            return MPQ_ERR_CUDA;
        e = wide ? cudaLaunchKernelEx(&pc, k_prefill<256>, pp, tmap)
                 : cudaLaunchKernelEx(&pc, k_prefill<128>, pp, tmap);
        if (e != cudaSuccess) return MPQ_ERR_CUDA;
        if (finish) {
            cudaLaunchConfig_t uc{};
            uc.gridDim = dim3((unsigned)M);
            uc.blockDim = dim3(FINISH_THREADS);
            // 0: no row order, 1: reorder through shared memory
            const int mode = layer->row_perm ? 1 : 0;
            uc.dynamicSmemBytes = mode == 1 ? (size_t)layer->N * 4 : 0;
            uc.stream = s;
            uc.attrs = pdl;
            uc.numAttrs = 1;
            e = cudaLaunchKernelEx(&uc, k_finish_rows, y_dev, (const float*)pp.out, shape.splits,
                                   (size_t)M * layer->N, layer->row_perm, layer->N, mode);
            if (e != cudaSuccess) return MPQ_ERR_CUDA;
        }
        if (ev_end && cudaEventRecord(static_cast<cudaEvent_t>(ev_end), s) != cudaSuccess)
            return MPQ_ERR_CUDA;
        return MPQ_OK;
    }

    const bool w16 = (layer->flags & MPQ_LAYER_16BIT) != 0;
    e = w16 ? ensure_smem_attr(k_decode<1, false, true>, (int)sizeof(DecSmem), g_decode_attr_w)
            : ensure_smem_attr(k_decode<1>, (int)sizeof(DecSmem), g_decode_attr);
    if (e == cudaSuccess)
        e = w16 ? ensure_smem_attr(k_decode<2, false, true>, (int)sizeof(DecSmem), g_decode_attr8_w)
                : ensure_smem_attr(k_decode<2>, (int)sizeof(DecSmem), g_decode_attr8);
    if (e == cudaSuccess)
        e = w16 ? ensure_smem_attr(k_decode<4, false, true>, (int)sizeof(DecSmem), g_decode_attr16_w)
                : ensure_smem_attr(k_decode<4>, (int)sizeof(DecSmem), g_decode_attr16);
    if (e == cudaSuccess)
        e = w16 ? ensure_smem_attr(k_decode<1, true, true>, (int)sizeof(DecSmem), g_decode_attr_f_w)
                : ensure_smem_attr(k_decode<1, true>, (int)sizeof(DecSmem), g_decode_attr_f);
    if (e != cudaSuccess) return MPQ_ERR_CUDA;
    DecodeParams dp = decode_params(layer, x_dev, M, y_dev, w);

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((layer->n_units + DEC_WARPS - 1) / DEC_WARPS));
    cfg.blockDim = dim3(DEC_THREADS);
    cfg.dynamicSmemBytes = sizeof(DecSmem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (ev_begin && cudaEventRecord(static_cast<cudaEvent_t>(ev_begin), s) != cudaSuccess)
        return MPQ_ERR_CUDA;
    for (int m0 = 0; m0 < M; m0 += kMaxDecodeTokens) {
        dp.m0 = m0;
        dp.Mg = std::min(kMaxDecodeTokens, M - m0);
        // token groups of two: one for up to 2 tokens, two for 4, four for 8
        if (w16)
            e = fused ? cudaLaunchKernelEx(&cfg, k_decode<1, true, true>, dp)
                : dp.Mg <= 2 ? cudaLaunchKernelEx(&cfg, k_decode<1, false, true>, dp)
                : dp.Mg <= 4 ? cudaLaunchKernelEx(&cfg, k_decode<2, false, true>, dp)
                             : cudaLaunchKernelEx(&cfg, k_decode<4, false, true>, dp);
        else
            e = fused ? cudaLaunchKernelEx(&cfg, k_decode<1, true>, dp)
                : dp.Mg <= 2 ? cudaLaunchKernelEx(&cfg, k_decode<1>, dp)
                : dp.Mg <= 4 ? cudaLaunchKernelEx(&cfg, k_decode<2>, dp)
                             : cudaLaunchKernelEx(&cfg, k_decode<4>, dp);
        if (e != cudaSuccess) return MPQ_ERR_CUDA;
    }
    if (ev_end && cudaEventRecord(static_cast<cudaEvent_t>(ev_end), s) != cudaSuccess)
        return MPQ_ERR_CUDA;
    return MPQ_OK;
}

}  // namespace

extern "C" {

mpq_status mpq_linear_timed(const mpq_layer* layer, const void* x_dev, int32_t M, float* y_dev,
                            void* ws, size_t ws_bytes, void* stream, void* ev_begin,
                            void* ev_end) {
    mpq_status st = check_layer(layer);
    if (st != MPQ_OK) return st;
    if (M < 0) return MPQ_ERR_SHAPE;
    if (M == 0) return MPQ_OK;
    if (!x_dev || !y_dev || !aligned16(x_dev)) return MPQ_ERR_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return MPQ_ERR_WORKSPACE;
    LinearWs w = carve_linear(ws, layer, M);
    if (ws_bytes < w.bytes) return MPQ_ERR_WORKSPACE;
    return linear_run(layer, x_dev, M, y_dev, w, static_cast<cudaStream_t>(stream), ev_begin, ev_end);
}

size_t mpq_linear_group_workspace_size(const mpq_layer* layers, int32_t n, int32_t M) {
    if (!layers || n < 1 || n > MPQ_GROUP_MAX || M < 0) return 0;
    size_t total = 0;
    for (int i = 0; i < n; ++i) total += round256(carve_linear(nullptr, &layers[i], M).bytes);
    return total;
}

mpq_status mpq_linear_group(const mpq_layer* layers, int32_t n, const void* x_dev, int32_t M,
                            float* const* y_devs, void* ws, size_t ws_bytes, void* stream) {
    if (!layers || !y_devs || n < 1 || n > MPQ_GROUP_MAX) return MPQ_ERR_ARG;
    for (int i = 0; i < n; ++i) {
        const mpq_status st = check_layer(&layers[i]);
        if (st != MPQ_OK) return st;
        if (layers[i].K != layers[0].K) return MPQ_ERR_SHAPE;
        if (!y_devs[i]) return MPQ_ERR_ARG;
    }
    if (M < 0) return MPQ_ERR_SHAPE;
    if (M == 0) return MPQ_OK;
    if (!x_dev || !aligned16(x_dev)) return MPQ_ERR_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return MPQ_ERR_WORKSPACE;
    if (ws_bytes < mpq_linear_group_workspace_size(layers, n, M)) return MPQ_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // each layer's part of the workspace; one error word (the first) for all
    static_assert(MPQ_GROUP_MAX == DEC_GROUP_MAX, "group size of the C ABI and the kernel");
    LinearWs w[MPQ_GROUP_MAX];
    size_t off = 0;
    bool all_fused = true;
    for (int i = 0; i < n; ++i) {
        w[i] = carve_linear(static_cast<uint8_t*>(ws) + off, &layers[i], M);
        w[i].err = static_cast<uint32_t*>(ws);
        off += round256(w[i].bytes);
        all_fused = all_fused && fused_one_token(&layers[i], M);
    }
    if (!all_fused) {
        for (int i = 0; i < n; ++i) {
            const mpq_status st = linear_run(&layers[i], x_dev, M, y_devs[i], w[i], s, nullptr, nullptr);
            if (st != MPQ_OK) return st;
        }
        return MPQ_OK;
    }
    // one launch over all the layers' runs
    bool w16 = false;
    for (int i = 0; i < n; ++i) w16 = w16 || (layers[i].flags & MPQ_LAYER_16BIT) != 0;
    cudaError_t e = w16 ? ensure_smem_attr(k_decode_group<true>, (int)sizeof(DecSmem), g_decode_attr_g_w)
                        : ensure_smem_attr(k_decode_group<false>, (int)sizeof(DecSmem), g_decode_attr_g);
    if (e != cudaSuccess) return MPQ_ERR_CUDA;
    DecodeGroup gp{};
    gp.n = n;
    gp.unit_begin[0] = 0;
    for (int i = 0; i < n; ++i) {
        gp.layer[i] = decode_params(&layers[i], x_dev, M, y_devs[i], w[i]);
        gp.unit_begin[i + 1] = gp.unit_begin[i] + layers[i].n_units;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((gp.unit_begin[n] + DEC_WARPS - 1) / DEC_WARPS));
    cfg.blockDim = dim3(DEC_THREADS);
    cfg.dynamicSmemBytes = sizeof(DecSmem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(w16 ? cudaLaunchKernelEx(&cfg, k_decode_group<true>, gp)
                           : cudaLaunchKernelEx(&cfg, k_decode_group<false>, gp));
}

size_t mpq_linear_host_workspace_size(const mpq_layer* layer, int32_t M) {
    if (!layer || M < 0) return 0;
    return mpq_linear_workspace_size(layer, M) + round256((size_t)M * layer->K * 2) +
           round256((size_t)M * layer->N * 4);
}

mpq_status mpq_linear_host(const mpq_layer* layer, const void* x_host, int32_t M, float* y_host,
                           void* ws, size_t ws_bytes, void* stream) {
    mpq_status st = check_layer(layer);
    if (st != MPQ_OK) return st;
    if (M < 0) return MPQ_ERR_SHAPE;
    if (M == 0) return MPQ_OK;
    if (!x_host || !y_host) return MPQ_ERR_ARG;
    if (!ws || ws_bytes < mpq_linear_host_workspace_size(layer, M)) return MPQ_ERR_WORKSPACE;
    const size_t inner = mpq_linear_workspace_size(layer, M);
    uint8_t* xb = static_cast<uint8_t*>(ws) + inner;
    float* yb = reinterpret_cast<float*>(xb + round256((size_t)M * layer->K * 2));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(xb, x_host, (size_t)M * layer->K * 2, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return MPQ_ERR_CUDA;
    st = mpq_linear(layer, xb, M, yb, ws, inner, stream);
    if (st != MPQ_OK) return st;
    if (cudaMemcpyAsync(y_host, yb, (size_t)M * layer->N * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MPQ_ERR_CUDA;
    return MPQ_OK;
}

size_t mpq_allocate_bits_workspace_size(int64_t n_blocks) {
    if (n_blocks <= 0) return 0;
    return round256((size_t)n_blocks * 8) + round256((size_t)n_blocks);
}

mpq_status mpq_allocate_bits(int64_t n_blocks, const float* loss_dev, uint32_t allowed,
                             uint64_t budget, uint8_t* bits_dev, uint32_t* info_dev, void* ws,
                             size_t ws_bytes, void* stream) {
    if (n_blocks <= 0 || n_blocks > (1ll << 24) || !loss_dev || !bits_dev || !info_dev) return MPQ_ERR_ARG;
    if (allowed == 0u || (allowed & ~0x17Fu)) return MPQ_ERR_ARG;   // widths 0..6 and 8
    const int bmin = __builtin_ctz(allowed);
    if (budget < (uint64_t)bmin * (uint64_t)n_blocks) return MPQ_ERR_ARG;
    if (!ws || ws_bytes < mpq_allocate_bits_workspace_size(n_blocks) ||
        (reinterpret_cast<uintptr_t>(ws) & 255))
        return MPQ_ERR_WORKSPACE;
    AllocParams p{};
    p.loss = loss_dev;
    p.bits = bits_dev;
    p.info = info_dev;
    p.gkey = static_cast<unsigned long long*>(ws);
    p.ginc = static_cast<uint8_t*>(ws) + round256((size_t)n_blocks * 8);
    p.n = n_blocks;
    p.budget = budget;
    p.mask = allowed;
    k_allocate_bits<<<1, ALLOC_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return cuda_status(cudaGetLastError());
}

mpq_status mpq_fold_orders(int32_t n, const int32_t* row_perm_a, const int32_t* col_perm_b,
                           int32_t* out) {
    if (n <= 0 || !out) return MPQ_ERR_ARG;
    if ((row_perm_a && !perm_ok(row_perm_a, n)) || (col_perm_b && !perm_ok(col_perm_b, n)))
        return MPQ_ERR_PERM;
    std::vector<int32_t> inv((size_t)n);
    for (int32_t i = 0; i < n; ++i) inv[(size_t)(row_perm_a ? row_perm_a[i] : i)] = i;
    for (int32_t j = 0; j < n; ++j) out[j] = inv[(size_t)(col_perm_b ? col_perm_b[j] : j)];
    return MPQ_OK;
}

mpq_status mpq_check(const void* ws, void* stream) {
    if (!ws) return MPQ_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t err = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MPQ_ERR_CUDA;
    if (cudaMemcpy(&err, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MPQ_ERR_CUDA;
    // reported: clear it for the calls that follow
    if (err != 0u && cudaMemset(const_cast<void*>(ws), 0, 4) != cudaSuccess) return MPQ_ERR_CUDA;
    return static_cast<mpq_status>(err);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// mpq_linear_noalloc: mpq_linear for callers that cannot allocate device
// memory.  Its scratch is this fixed array, which every device that loads the
// library holds until the process exits.  Host code must not hand the
// array's name to a kernel (in host code it is only a stand-in for the
// symbol); the device address is looked up with cudaGetSymbolAddress, with
// the calling device current, on every call (the lookup allocates nothing,
// and a fresh lookup stays right after the device's context is recreated).
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[MPQ_NOALLOC_SCRATCH_BYTES];

namespace {
mpq_status noalloc_scratch(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MPQ_ERR_CUDA;
    *out = p;
    return MPQ_OK;
}
}  // namespace

extern "C" {

mpq_status mpq_linear_noalloc(const mpq_layer* layer, const void* x_dev, int32_t M,
                              float* y_dev, void* stream) {
    mpq_status st = check_layer(layer);
    if (st != MPQ_OK) return st;
    if (M < 0) return MPQ_ERR_SHAPE;
    if (M == 0) return MPQ_OK;
    if (mpq_linear_workspace_size(layer, M) > (size_t)MPQ_NOALLOC_SCRATCH_BYTES)
        return MPQ_ERR_WORKSPACE;
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != MPQ_OK) return st;
    // The scratch starts zeroed (static storage) and every call that ends
    // without a device error leaves its counters at zero; the error word
    // keeps the first device error until mpq_noalloc_check reads it.
    return mpq_linear(layer, x_dev, M, y_dev, scratch, (size_t)MPQ_NOALLOC_SCRATCH_BYTES, stream);
}

mpq_status mpq_noalloc_check(void* stream) {
    void* scratch = nullptr;
    mpq_status st = noalloc_scratch(&scratch);
    if (st != MPQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t err = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MPQ_ERR_CUDA;
    if (cudaMemcpy(&err, scratch, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MPQ_ERR_CUDA;
    // A call that stopped on a device error may have left arrival counters
    // set: clear the whole array, back to its state at load time.
    if (err != 0u && cudaMemset(scratch, 0, (size_t)MPQ_NOALLOC_SCRATCH_BYTES) != cudaSuccess)
        return MPQ_ERR_CUDA;
    return static_cast<mpq_status>(err);
}

const char* mpq_status_string(mpq_status s) {
    switch (s) {
        case MPQ_OK: return "MPQ_OK";
        case MPQ_ERR_ARG: return "MPQ_ERR_ARG";
        case MPQ_ERR_SHAPE: return "MPQ_ERR_SHAPE";
        case MPQ_ERR_BITS: return "MPQ_ERR_BITS";
        case MPQ_ERR_PERM: return "MPQ_ERR_PERM";
        case MPQ_ERR_NONFINITE: return "MPQ_ERR_NONFINITE";
        case MPQ_ERR_RANGE: return "MPQ_ERR_RANGE";
        case MPQ_ERR_WORKSPACE: return "MPQ_ERR_WORKSPACE";
        case MPQ_ERR_CUDA: return "MPQ_ERR_CUDA";
        case MPQ_ERR_TIMEOUT: return "MPQ_ERR_TIMEOUT";
    }
    return "MPQ_ERR_UNKNOWN";
}

}  // extern "C"
