// Host side of the C ABI declared in include/tp_reconcile.h: plan set-up,
// argument checks, TMA descriptors and kernel launches. No device memory is
// allocated here and nothing synchronises the caller's stream except
// tp_device_error_flags, which says so.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>

#include "tp_kernels_exact.cuh"
#include "tp_kernels_tc.cuh"
#include "tp_kernels_tc2.cuh"
#include "tp_kernels_mx.cuh"
#include "tp_kernels_ring.cuh"
#include "tp_reconcile.h"

// Fixed scratch for tp_rowlinear_reconcile_noalloc: fold counters and the
// staged partials of callers that cannot allocate device memory. Every GPU
// that loads this library holds it until the process exits. Its first
// kNoAllocCounterBytes hold the counters of every plan (zero-initialised,
// left zero by each call), the rest the partials.
constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB
constexpr size_t kNoAllocCounterBytes = 8192;       // 2 x 1024 H tiles: H <= 131072
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

struct tp_plan {
    int n_ranks;
    int64_t max_tokens, k, hidden, ks, hc;
    int device;
    int sm_count;
    int smem_optin;
    int variant;
    int staged;
    void* noalloc_scratch;  // device address of g_noalloc_scratch on this plan's device
};

namespace {

thread_local int t_last_cuda_error = 0;

// Device address of the no-alloc scratch array on the current device. In host
// code the array's name is only a host-side stand-in, never a device address:
// cudaGetSymbolAddress, with the device current, gives the address kernels
// use. It is looked up again at every plan creation (a cheap query), so a
// plan made after cudaDeviceReset gets the array of the new context.
cudaError_t noalloc_scratch_current(void** out) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = ptr;
    return cudaSuccess;
}

tp_status cuda_fail(cudaError_t e) {
    t_last_cuda_error = static_cast<int>(e);
    return TP_ERR_CUDA;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        else if (g_encode_err == cudaSuccess)
            g_encode_err = cudaErrorSymbolNotFound;
    });
    return g_encode;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
    if (!a || !b || an == 0 || bn == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + bn && b0 < a0 + an;
}

tp_status check_device(const tp_plan* p) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    return dev == p->device ? TP_OK : TP_ERR_INVALID;
}

// --------------------------------------------------------- exact variant --

struct ExactConfig {
    int mt, bh, grid_x, grid_y, stages, threads;
    size_t smem;
    uint32_t w_stage, x_stage;
};

constexpr size_t kSmemBudgetShared = 110 * 1024;   // two CTAs per SM
constexpr size_t kSmemBudgetAlone = 200 * 1024;

ExactConfig exact_config(const tp_plan* p, int64_t tokens) {
    ExactConfig c{};
    c.mt = tokens <= 1 ? 1 : tokens <= 2 ? 2 : tokens <= 4 ? 4 : 8;
    const int n = p->n_ranks;
    const int64_t mtiles = (tokens + c.mt - 1) / c.mt;
    int64_t htiles = std::max<int64_t>(1, p->sm_count / std::max<int64_t>(1, mtiles));
    int64_t bh = (p->hidden + htiles - 1) / htiles;
    const int64_t bh_cap = std::min<int64_t>(256, tpr::kMaxExactChains / n);
    bh = std::max<int64_t>(1, std::min<int64_t>(bh, std::min<int64_t>(bh_cap, p->hidden)));
    c.bh = static_cast<int>(bh);
    c.grid_x = static_cast<int>((p->hidden + bh - 1) / bh);
    c.grid_y = static_cast<int>(mtiles);
    const int chains = n * c.bh;
    c.threads = ((chains + 31) / 32 + 1) * 32;
    c.w_stage = static_cast<uint32_t>(((static_cast<size_t>(chains) * 128 + 1023) / 1024) * 1024);
    c.x_stage = static_cast<uint32_t>(static_cast<size_t>(n) * c.mt * 128);
    const size_t fixed = 2 * tpr::kMaxStages * sizeof(uint64_t) +
                         static_cast<size_t>(chains) * c.mt * sizeof(uint16_t) + 1024;
    const size_t stage = c.w_stage + c.x_stage;
    size_t budget = stage <= 16 * 1024 ? kSmemBudgetShared : kSmemBudgetAlone;
    budget = std::min<size_t>(budget, static_cast<size_t>(p->smem_optin));
    int stages = budget > fixed ? static_cast<int>((budget - fixed) / stage) : 0;
    c.stages = std::min(stages, tpr::kMaxStages);
    c.smem = fixed + static_cast<size_t>(c.stages) * stage;
    return c;
}

tp_status encode_maps(const tp_plan* p, const ExactConfig& c, const void* x, const void* w,
                      int64_t tokens, CUtensorMap* mw, CUtensorMap* mx) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return cuda_fail(g_encode_err);
    const cuuint32_t estr[3] = {1, 1, 1};
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p->ks),
                                    static_cast<cuuint64_t>(p->hidden),
                                    static_cast<cuuint64_t>(p->n_ranks)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p->ks) * 2,
                                       static_cast<cuuint64_t>(p->hidden * p->ks) * 2};
        const cuuint32_t box[3] = {static_cast<cuuint32_t>(tpr::kKBlock),
                                   static_cast<cuuint32_t>(c.bh),
                                   static_cast<cuuint32_t>(p->n_ranks)};
        CUresult r = enc(mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    }
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p->ks),
                                    static_cast<cuuint64_t>(p->n_ranks),
                                    static_cast<cuuint64_t>(tokens)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p->ks) * 2,
                                       static_cast<cuuint64_t>(p->k) * 2};
        const cuuint32_t box[3] = {static_cast<cuuint32_t>(tpr::kKBlock),
                                   static_cast<cuuint32_t>(p->n_ranks),
                                   static_cast<cuuint32_t>(c.mt)};
        CUresult r = enc(mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    }
    return TP_OK;
}

// Launch with programmatic dependent launch; cluster_x > 1 also groups the
// CTAs in clusters of cluster_x (the grid is a multiple of it).
template <typename Kern, typename... Args>
cudaError_t launch_pdl_cluster(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                               int cluster_x, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int na = 1;
    if (cluster_x > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        na = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
    return launch_pdl_cluster(kernel, grid, block, smem, stream, 1, args...);
}

tp_status launch_exact(const tp_plan* p, const void* x, const void* w, const void* residual,
                       void* out, void* partials, int64_t tokens, bool fused,
                       cudaStream_t stream) {
    const ExactConfig c = exact_config(p, tokens);
    if (c.stages < 2) return TP_ERR_UNSUPPORTED;
    CUtensorMap mw, mx;
    tp_status st = encode_maps(p, c, x, w, tokens, &mw, &mx);
    if (st != TP_OK) return st;
    tpr::ExactParams prm{};
    prm.n_ranks = p->n_ranks;
    prm.bh = c.bh;
    prm.ks = static_cast<int>(p->ks);
    prm.hidden = static_cast<int>(p->hidden);
    prm.hc = static_cast<int>(p->hc);
    prm.tokens = static_cast<int>(tokens);
    prm.stages = c.stages;
    prm.fused = fused ? 1 : 0;
    prm.w_stage_bytes = c.w_stage;
    prm.x_stage_bytes = c.x_stage;
    prm.w_box_bytes = static_cast<uint32_t>(tpr::kKBlock * c.bh * p->n_ranks * 2);
    prm.x_box_bytes = static_cast<uint32_t>(tpr::kKBlock * p->n_ranks * c.mt * 2);
    prm.residual = static_cast<const uint16_t*>(residual);
    prm.out = static_cast<uint16_t*>(out);
    prm.partials = static_cast<uint16_t*>(partials);
    const dim3 grid(c.grid_x, c.grid_y), block(c.threads);
    cudaError_t e;
    switch (c.mt) {
        case 1: e = launch_pdl(tpr::exact_partial_kernel<1>, grid, block, c.smem, stream, mw, mx, prm); break;
        case 2: e = launch_pdl(tpr::exact_partial_kernel<2>, grid, block, c.smem, stream, mw, mx, prm); break;
        case 4: e = launch_pdl(tpr::exact_partial_kernel<4>, grid, block, c.smem, stream, mw, mx, prm); break;
        default: e = launch_pdl(tpr::exact_partial_kernel<8>, grid, block, c.smem, stream, mw, mx, prm); break;
    }
    return e == cudaSuccess ? TP_OK : cuda_fail(e);
}

// -------------------------------------------------------- tensor variant --

struct TcConfig {
    int fmt;   // the kernel's form (tpr::kFmt*): MXFP8 for at most 8 tokens is block-scaled
    int bn, stages, grid, units, h_tiles, m_tiles, splits, x_rows;
    bool cluster_fold;   // the N ranks of a tile on one cluster, folded on chip
    bool splits_allowed; // a reconciliation call (the kernel may fold; K may be split)
    size_t smem;
};

constexpr int64_t kTensorMinTokens = 1;      // AUTO uses the tensor cores from here

int tc_token_tile(int64_t tokens) {
    return tokens <= 32 ? 32 : tokens <= 64 ? 64 : tokens <= 128 ? 128 : 256;
}

// allow_split: the call folds (S2-S4) in this library, so K may be split
// across CTAs when there are fewer units than SMs; calls with a token tile of
// at most 128 whose N ranks x K parts make at most 8 CTAs (at most 4 parts)
// fold on chip in clusters of those CTAs.
TcConfig tc_config(const tp_plan* p, int64_t tokens, bool allow_split, int fmt = tpr::kFmtBf16) {
    TcConfig c{};
    c.splits_allowed = allow_split;
    // MXFP8 for at most 8 tokens: the codes go to the block-scaled MMA as
    // stored and the activations are split into two E4M3 terms on chip
    if (fmt == tpr::kFmtMxfp8 && tokens <= 8) fmt = tpr::kFmtMxfp8Bs;
    c.fmt = fmt;
    c.bn = tc_token_tile(tokens);
    // quantised forms: token tiles up to 128 (their converted slots share
    // tensor memory with the accumulators)
    if (fmt != tpr::kFmtBf16) c.bn = std::min(c.bn, 128);
    c.h_tiles = static_cast<int>((p->hidden + tpr::kTcRows - 1) / tpr::kTcRows);
    c.m_tiles = static_cast<int>((tokens + c.bn - 1) / c.bn);
    const int base_units = p->n_ranks * c.h_tiles * c.m_tiles;
    // Small token tiles stream weights: two CTAs per SM (about 100 KB each,
    // tensor memory 2 x 2*BN columns). Large tiles: one CTA per SM, deep ring.
    const bool two_per_sm = c.bn <= 64;
    const int slots = p->sm_count * (two_per_sm ? 2 : 1);
    // Fewer units than SMs: split K so every SM streams weights.
    const int kblock = tpr::fmt_k_block(fmt);
    const int nkb = static_cast<int>((p->ks + kblock - 1) / kblock);
    c.splits = 1;
    if (allow_split && base_units > 0 && base_units < p->sm_count)
        c.splits = std::max(1, std::min({slots / base_units, nkb, tpr::kMaxSplits}));
    // cluster fold (the CLUSTER variant): the N ranks x K parts of a tile in
    // one portable cluster
    c.cluster_fold = allow_split && p->variant == TP_VARIANT_CLUSTER && base_units > 0 &&
                     c.bn <= 128 && c.splits <= 4 && p->n_ranks * c.splits <= 8;
    // Quantised weights: a stage holds codes, scales and activations (the
    // converted bf16 tiles live in tensor memory).
    // At most 8 tokens: one 8-row atom of x a block instead of the BN-row tile
    c.x_rows = tokens <= 8 && c.m_tiles == 1 ? 8 : c.bn;
    const size_t stage = tpr::fmt_code_tile(fmt) + tpr::fmt_scale_tile(fmt) + tpr::fmt_b_tile(fmt, c.x_rows);
    // the cluster fold's tile in shared memory: the tile's tokens x 128 rows,
    // bf16 partials or fp32 part sums
    const size_t part_tile = c.cluster_fold ? static_cast<size_t>(std::min<int64_t>(c.bn, tokens)) *
                                                  tpr::kTcRows * (c.splits > 1 ? 4 : 2)
                                            : 0;
    const size_t fixed = (4 * tpr::kTcMaxStages + 7 + 2 * tpr::kCvtSlotsMax) * sizeof(uint64_t) + 16 + 128 +
                         1024 + part_tile;
    const size_t budget = std::min<size_t>(two_per_sm ? 110 * 1024 : 200 * 1024,
                                           static_cast<size_t>(p->smem_optin));
    c.stages = budget > fixed
                   ? static_cast<int>(std::min<size_t>(tpr::kTcMaxStages, (budget - fixed) / stage))
                   : 0;
    c.smem = fixed + static_cast<size_t>(c.stages) * stage;
    c.units = base_units * c.splits;
    if (c.cluster_fold) {
        // clusters of N * splits CTAs, one per (H tile, token tile) at a time
        const int tiles = c.h_tiles * c.m_tiles;
        const int cl = p->n_ranks * c.splits;
        c.grid = cl * std::max(1, std::min(tiles, slots / cl));
    } else {
        c.grid = std::min(c.units, slots);
    }
    return c;
}

// x_box_tokens: token rows of one activation box (the 1-SM kernel's BN, or
// the half tile a CTA of a pair stages).
tp_status encode_tc_maps(const tp_plan* p, int x_box_tokens, const void* x, const void* w,
                         int64_t tokens, CUtensorMap* mw, CUtensorMap* mx, bool x_block_scaled = false) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return cuda_fail(g_encode_err);
    const cuuint32_t estr[3] = {1, 1, 1};
    {
        // Packed weights [N][H][Ks]: {Ks, H, N}, 128 rows x 64 columns per box.
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p->ks), static_cast<cuuint64_t>(p->hidden),
                                    static_cast<cuuint64_t>(p->n_ranks)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p->ks) * 2,
                                       static_cast<cuuint64_t>(p->hidden * p->ks) * 2};
        const cuuint32_t box[3] = {tpr::kTcKBlock, tpr::kTcRows, 1};
        CUresult r = enc(mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    }
    {
        // Activations [M][N][Ks]: {Ks, N, M}, BN token rows x 64 columns of one
        // rank (128-byte swizzle, the MMA's B tiles), or for the block-scaled
        // form 8 token rows x 128 columns unswizzled (the splitting warps' input).
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p->ks), static_cast<cuuint64_t>(p->n_ranks),
                                    static_cast<cuuint64_t>(tokens)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p->ks) * 2,
                                       static_cast<cuuint64_t>(p->k) * 2};
        const cuuint32_t box[3] = {x_block_scaled ? static_cast<cuuint32_t>(tpr::kMxChunkCols)
                                                  : static_cast<cuuint32_t>(tpr::kTcKBlock),
                                   1, static_cast<cuuint32_t>(x_box_tokens)};
        CUresult r = enc(mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         x_block_scaled ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    }
    return TP_OK;
}

// The tensor-core partials: bf16 [N][M][H] when the units are not split, or
// fp32 k-part sums [splits][N][M][H] (allow_split) for the ring kernel to add.
size_t tc_partial_bytes(const tp_plan* p, const TcConfig& c, int64_t tokens) {
    // the counter fold (a reconciliation of one or two tokens) stores its
    // parts with their call's tag: 8 bytes a part
    const bool tagged = c.splits_allowed && tokens <= 2 && !c.cluster_fold;
    const size_t elem = tagged ? 8u * c.splits : c.splits > 1 ? 4u * c.splits : 2u;
    return static_cast<size_t>(p->n_ranks) * static_cast<size_t>(tokens) * static_cast<size_t>(p->hidden) * elem;
}

// Calls that run on CTA pairs: bf16 shards, prefill-sized token tiles, no
// k-split, not the cluster fold.
bool tc2_path(const tp_plan* p, const TcConfig& c, int fmt) {
    return fmt == tpr::kFmtBf16 && c.bn == tpr::kTc2Tokens && c.splits == 1 && !c.cluster_fold &&
           p->sm_count >= 2;
}

// The partials [N][M][H] of a prefill-sized call on CTA pairs: units of
// (rank, 256 rows of H, 256 tokens), two CTAs per unit, one per SM.
tp_status launch_tc2(const tp_plan* p, const void* x, const void* w, void* partials, int64_t tokens,
                     cudaStream_t stream, bool fold = false, unsigned int* counters = nullptr,
                     const void* residual = nullptr, void* out = nullptr) {
    const int h_pairs = static_cast<int>((p->hidden + 2 * tpr::kTcRows - 1) / (2 * tpr::kTcRows));
    const int m_tiles = static_cast<int>((tokens + tpr::kTc2Tokens - 1) / tpr::kTc2Tokens);
    const int units = p->n_ranks * h_pairs * m_tiles;
    const size_t fixed = (2 * tpr::kTc2MaxStages + 5) * sizeof(uint64_t) + 16 + 1024;
    const size_t budget = std::min<size_t>(200 * 1024, static_cast<size_t>(p->smem_optin));
    const int stages = static_cast<int>(std::min<size_t>(tpr::kTc2MaxStages, (budget - fixed) / tpr::kTc2Stage));
    if (stages < 2) return TP_ERR_UNSUPPORTED;
    const size_t smem = fixed + static_cast<size_t>(stages) * tpr::kTc2Stage;
    const int pairs = std::min(units, p->sm_count / 2);
    CUtensorMap mw, mx;
    tp_status st = encode_tc_maps(p, tpr::kTc2HalfTokens, x, w, tokens, &mw, &mx);
    if (st != TP_OK) return st;
    tpr::Tc2Params prm{};
    prm.n_ranks = p->n_ranks;
    prm.ks = static_cast<int>(p->ks);
    prm.hidden = static_cast<int>(p->hidden);
    prm.tokens = static_cast<int>(tokens);
    prm.h_pairs = h_pairs;
    prm.m_tiles = m_tiles;
    prm.units = units;
    prm.stages = stages;
    prm.partials = static_cast<uint16_t*>(partials);
    prm.fold = fold ? 1 : 0;
    prm.hc = static_cast<int>(p->hc);
    prm.counters = fold ? counters : nullptr;
    prm.residual = static_cast<const uint16_t*>(residual);
    prm.out = static_cast<uint16_t*>(out);
    cudaError_t e = launch_pdl(tpr::tc2_partial_kernel, dim3(static_cast<unsigned>(2 * pairs)),
                               dim3(tpr::kTcThreads), smem, stream, mw, mx, prm);
    return e == cudaSuccess ? TP_OK : cuda_fail(e);
}

// NVFP4 block-scale bytes (H*K/16); the second-level exponent g (int32)
// follows them in the same buffer.
size_t nv_scale_bytes(const tp_plan* p) {
    return static_cast<size_t>(p->hidden) * static_cast<size_t>(p->k) / 16;
}

// Weights of a tensor-core call: packed bf16 shards, or MXFP8 codes with
// their scales.
struct TcWeights {
    const void* w;        // [N][H][Ks] bf16; MXFP8 E4M3 codes; NVFP4 E2M1 code pairs
    const void* scales;   // MXFP8 [N][H/128][Ks/128][512] E8M0 chunks; NVFP4 [N][Ks/64][H][4] E4M3 + g
    int fmt;              // tpr::kFmt*
};

// MXFP8 codes [N][H][Ks] bytes, 128 rows per box: 64 codes with the 64-byte
// swizzle for the converters (their reads and swizzled writes are then free
// of bank conflicts), or 128 codes with the 128-byte swizzle the block-scaled
// MMA reads. (The scales travel by plain bulk copies of their chunks.)
tp_status encode_mx_maps(const tp_plan* p, const void* q, bool block_scaled, CUtensorMap* mq) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return cuda_fail(g_encode_err);
    const cuuint32_t estr[3] = {1, 1, 1};
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p->ks), static_cast<cuuint64_t>(p->hidden),
                                static_cast<cuuint64_t>(p->n_ranks)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p->ks), static_cast<cuuint64_t>(p->hidden * p->ks)};
    const cuuint32_t box[3] = {block_scaled ? static_cast<cuuint32_t>(tpr::kMxChunkCols)
                                            : static_cast<cuuint32_t>(tpr::kTcKBlock),
                               tpr::kTcRows, 1};
    CUresult r = enc(mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(q), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     block_scaled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? TP_OK : cuda_fail(cudaErrorInvalidValue);
}

// NVFP4 code pairs [N][H][Ks/2] bytes, 128 rows x 32 bytes per box, and the
// block scales [N][Ks/64][H][4] as 32-bit words, 128 words per box.
tp_status encode_nv_maps(const tp_plan* p, const void* q, const void* scales, CUtensorMap* mq,
                         CUtensorMap* ms) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return cuda_fail(g_encode_err);
    const cuuint32_t estr[3] = {1, 1, 1};
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p->ks / 2), static_cast<cuuint64_t>(p->hidden),
                                    static_cast<cuuint64_t>(p->n_ranks)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p->ks / 2),
                                       static_cast<cuuint64_t>(p->hidden * p->ks / 2)};
        const cuuint32_t box[3] = {tpr::kTcKBlock / 2, tpr::kTcRows, 1};
        // 32-byte swizzle, for the converters' banks (as for MXFP8)
        CUresult r = enc(mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(q), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    }
    {
        const int64_t nkb = p->ks / tpr::kTcKBlock;
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p->hidden), static_cast<cuuint64_t>(nkb),
                                    static_cast<cuuint64_t>(p->n_ranks)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(4 * p->hidden),
                                       static_cast<cuuint64_t>(4 * p->hidden * nkb)};
        const cuuint32_t box[3] = {tpr::kTcRows, 1, 1};
        CUresult r = enc(ms, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(scales), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    }
    return TP_OK;
}

template <int BN, int MODE, int FMT>
cudaError_t launch_tc_kernel(dim3 grid, size_t smem, cudaStream_t stream, int cluster_x,
                             const CUtensorMap& mw, const CUtensorMap& mx, const CUtensorMap& ms,
                             const tpr::TcParams& prm) {
    return launch_pdl_cluster(tpr::tc_partial_kernel<BN, MODE, FMT>, grid,
                              dim3(FMT != tpr::kFmtBf16 ? tpr::kTcMxThreads : tpr::kTcThreads), smem,
                              stream, cluster_x, mw, mx, ms, prm);
}

// The block-scaled MXFP8 form (at most 8 tokens, one 32-column tile) for an
// epilogue mode.
cudaError_t dispatch_tc_bs(int mode, dim3 grid, size_t smem, cudaStream_t st, int cl, const CUtensorMap& mw,
                           const CUtensorMap& mx, const CUtensorMap& ms, const tpr::TcParams& prm) {
    using namespace tpr;
    if (mode == kTcClusterFold)
        return launch_tc_kernel<32, kTcClusterFold, kFmtMxfp8Bs>(grid, smem, st, cl, mw, mx, ms, prm);
    if (mode == kTcCounterFold)
        return launch_tc_kernel<32, kTcCounterFold, kFmtMxfp8Bs>(grid, smem, st, 1, mw, mx, ms, prm);
    return launch_tc_kernel<32, kTcStore, kFmtMxfp8Bs>(grid, smem, st, 1, mw, mx, ms, prm);
}

// The instantiation for a token tile and an epilogue mode.
template <int MX>
cudaError_t dispatch_tc(int bn, int mode, dim3 grid, size_t smem, cudaStream_t st, int cl,
                        const CUtensorMap& mw, const CUtensorMap& mx, const CUtensorMap& ms,
                        const tpr::TcParams& prm) {
    using namespace tpr;
    if (mode == kTcClusterFold) {
        if (bn == 32) return launch_tc_kernel<32, kTcClusterFold, MX>(grid, smem, st, cl, mw, mx, ms, prm);
        if (bn == 64) return launch_tc_kernel<64, kTcClusterFold, MX>(grid, smem, st, cl, mw, mx, ms, prm);
        return launch_tc_kernel<128, kTcClusterFold, MX>(grid, smem, st, cl, mw, mx, ms, prm);
    }
    if (mode == kTcCounterFold)   // at most two tokens: a 32-token tile
        return launch_tc_kernel<32, kTcCounterFold, MX>(grid, smem, st, 1, mw, mx, ms, prm);
    if (bn == 32) return launch_tc_kernel<32, kTcStore, MX>(grid, smem, st, 1, mw, mx, ms, prm);
    if (bn == 64) return launch_tc_kernel<64, kTcStore, MX>(grid, smem, st, 1, mw, mx, ms, prm);
    if constexpr (MX != kFmtBf16) {   // quantised forms: token tiles up to 128
        return launch_tc_kernel<128, kTcStore, MX>(grid, smem, st, 1, mw, mx, ms, prm);
    } else {
        if (bn == 128) return launch_tc_kernel<128, kTcStore, MX>(grid, smem, st, 1, mw, mx, ms, prm);
        return launch_tc_kernel<256, kTcStore, MX>(grid, smem, st, 1, mw, mx, ms, prm);
    }
}

// allow_split (a reconciliation call): the kernel also runs S2-S4 (residual,
// out) on chip when the configuration folds in clusters, or for few tokens
// with `fold`, counting stored parts per H tile in `counters` (zero on entry,
// zero on return); else a ring kernel must follow.
tp_status launch_tc(const tp_plan* p, const void* x, const TcWeights& wt, void* partials,
                    int64_t tokens, bool allow_split, bool fold, unsigned int* counters,
                    const void* residual, void* out, cudaStream_t stream) {
    const TcConfig c = tc_config(p, tokens, allow_split, wt.fmt);
    if (c.stages < 2) return TP_ERR_UNSUPPORTED;
    if (c.cluster_fold) fold = false;
    // Prefill-sized bf16 tiles without a k-split run on CTA pairs (2-SM MMA),
    // which fold in their epilogue with `fold`.
    if (tc2_path(p, c, c.fmt))
        return launch_tc2(p, x, wt.w, partials, tokens, stream, fold,
                          counters ? counters + 2 * c.h_tiles : nullptr,   // after the counter fold's words
                          residual, out);
    if (fold && (c.m_tiles != 1 || tokens > 2)) return TP_ERR_UNSUPPORTED;  // the kernel folds <= 2 rows
    CUtensorMap mw, mx, ms;
    tp_status st = encode_tc_maps(p, c.x_rows, x, wt.w, tokens, &mw, &mx, c.fmt == tpr::kFmtMxfp8Bs);
    if (st != TP_OK) return st;
    if (c.fmt == tpr::kFmtMxfp8 || c.fmt == tpr::kFmtMxfp8Bs) {
        if ((st = encode_mx_maps(p, wt.w, c.fmt == tpr::kFmtMxfp8Bs, &mw)) != TP_OK) return st;
        ms = mw;   // not read
    } else if (wt.fmt == tpr::kFmtNvfp4) {
        if ((st = encode_nv_maps(p, wt.w, wt.scales, &mw, &ms)) != TP_OK) return st;
    } else {
        ms = mw;   // not read
    }
    tpr::TcParams prm{};
    prm.n_ranks = p->n_ranks;
    prm.ks = static_cast<int>(p->ks);
    prm.hidden = static_cast<int>(p->hidden);
    prm.tokens = static_cast<int>(tokens);
    prm.h_tiles = c.h_tiles;
    prm.m_tiles = c.m_tiles;
    prm.splits = c.splits;
    prm.units = c.units;
    prm.stages = c.stages;
    prm.x_rows = c.x_rows;
    prm.partials = static_cast<uint16_t*>(partials);
    prm.partials_f32 = static_cast<float*>(partials);
    prm.hc = static_cast<int>(p->hc);
    prm.counters = fold ? counters : nullptr;
    prm.residual = static_cast<const uint16_t*>(residual);
    prm.out = static_cast<uint16_t*>(out);
    prm.x = static_cast<const uint16_t*>(x);
    prm.k = p->k;
    prm.mx_scales = wt.fmt == tpr::kFmtMxfp8 ? static_cast<const uint8_t*>(wt.scales) : nullptr;
    prm.mx_kg = static_cast<int>((p->ks + tpr::kMxChunkCols - 1) / tpr::kMxChunkCols);
    prm.nv_gexp = wt.fmt == tpr::kFmtNvfp4
                      ? reinterpret_cast<const int*>(static_cast<const uint8_t*>(wt.scales) + nv_scale_bytes(p))
                      : nullptr;
    const int mode = c.cluster_fold ? tpr::kTcClusterFold : fold ? tpr::kTcCounterFold : tpr::kTcStore;
    const int cl = c.cluster_fold ? p->n_ranks * c.splits : 1;
    const dim3 grid(c.grid);
    const cudaError_t e =
        c.fmt == tpr::kFmtMxfp8Bs  ? dispatch_tc_bs(mode, grid, c.smem, stream, cl, mw, mx, ms, prm)
        : c.fmt == tpr::kFmtMxfp8  ? dispatch_tc<tpr::kFmtMxfp8>(c.bn, mode, grid, c.smem, stream, cl, mw, mx, ms, prm)
        : c.fmt == tpr::kFmtNvfp4  ? dispatch_tc<tpr::kFmtNvfp4>(c.bn, mode, grid, c.smem, stream, cl, mw, mx, ms, prm)
                                   : dispatch_tc<tpr::kFmtBf16>(c.bn, mode, grid, c.smem, stream, cl, mw, mx, ms, prm);
    return e == cudaSuccess ? TP_OK : cuda_fail(e);
}

tp_status launch_ring_splits(const tp_plan* p, const void* parts, int splits, const void* residual,
                             void* out, int64_t tokens, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>((p->hidden + 255) / 256),
                    static_cast<unsigned>(std::min<int64_t>(tokens, 65535)));
    cudaError_t e = launch_pdl(tpr::ring_reduce_splits_kernel, grid, dim3(256), 0, stream,
                               static_cast<const float*>(parts), splits,
                               static_cast<const uint16_t*>(residual), static_cast<uint16_t*>(out),
                               p->n_ranks, tokens, static_cast<int>(p->hidden), static_cast<int>(p->hc));
    return e == cudaSuccess ? TP_OK : cuda_fail(e);
}

tp_status launch_ring(const tp_plan* p, const void* partials, const void* residual, void* out,
                      int64_t tokens, cudaStream_t stream) {
    const int64_t total = tokens * (p->hidden / 8);
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(p->sm_count) * 8);
    cudaError_t e = launch_pdl(tpr::ring_reduce_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                               stream, static_cast<const uint16_t*>(partials),
                               static_cast<const uint16_t*>(residual), static_cast<uint16_t*>(out),
                               p->n_ranks, tokens, static_cast<int>(p->hidden),
                               static_cast<int>(p->hc));
    return e == cudaSuccess ? TP_OK : cuda_fail(e);
}

#define TC_KERNELS(MX)                                                                   \
    reinterpret_cast<const void*>(tpr::tc_partial_kernel<32, tpr::kTcStore, MX>),          \
        reinterpret_cast<const void*>(tpr::tc_partial_kernel<64, tpr::kTcStore, MX>),      \
        reinterpret_cast<const void*>(tpr::tc_partial_kernel<128, tpr::kTcStore, MX>),     \
        reinterpret_cast<const void*>(tpr::tc_partial_kernel<32, tpr::kTcCounterFold, MX>), \
        reinterpret_cast<const void*>(tpr::tc_partial_kernel<32, tpr::kTcClusterFold, MX>), \
        reinterpret_cast<const void*>(tpr::tc_partial_kernel<64, tpr::kTcClusterFold, MX>), \
        reinterpret_cast<const void*>(tpr::tc_partial_kernel<128, tpr::kTcClusterFold, MX>)

// Lets every exact kernel use the device's opt-in shared memory less its own
// static shared memory; returns the smallest such dynamic allowance.
cudaError_t set_kernel_attrs(int smem_optin, int* dyn_max) {
    const void* kernels[] = {
        reinterpret_cast<const void*>(tpr::exact_partial_kernel<1>),
        reinterpret_cast<const void*>(tpr::exact_partial_kernel<2>),
        reinterpret_cast<const void*>(tpr::exact_partial_kernel<4>),
        reinterpret_cast<const void*>(tpr::exact_partial_kernel<8>),
        TC_KERNELS(tpr::kFmtBf16), TC_KERNELS(tpr::kFmtMxfp8), TC_KERNELS(tpr::kFmtNvfp4),
        reinterpret_cast<const void*>(tpr::tc_partial_kernel<32, tpr::kTcStore, tpr::kFmtMxfp8Bs>),
        reinterpret_cast<const void*>(tpr::tc_partial_kernel<32, tpr::kTcCounterFold, tpr::kFmtMxfp8Bs>),
        reinterpret_cast<const void*>(tpr::tc_partial_kernel<32, tpr::kTcClusterFold, tpr::kFmtMxfp8Bs>),
        reinterpret_cast<const void*>(tpr::tc_partial_kernel<256, tpr::kTcStore, tpr::kFmtBf16>),
        reinterpret_cast<const void*>(tpr::tc2_partial_kernel)};
    int lowest = smem_optin;
    for (const void* k : kernels) {
        cudaFuncAttributes fa{};
        cudaError_t e = cudaFuncGetAttributes(&fa, k);
        if (e != cudaSuccess) return e;
        const int dyn = smem_optin - static_cast<int>(fa.sharedSizeBytes);
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
        if (e != cudaSuccess) return e;
        lowest = std::min(lowest, dyn);
    }
    *dyn_max = lowest;
    return cudaSuccess;
}

}  // namespace

extern "C" {

tp_status tp_plan_create(tp_plan** out, int n_ranks, int64_t max_tokens, int64_t k, int64_t hidden,
                         int dtype) {
    if (!out) return TP_ERR_INVALID;
    *out = nullptr;
    if (dtype != TP_BF16) return TP_ERR_UNSUPPORTED;
    if (n_ranks < 1 || n_ranks > 8 || max_tokens < 0 || k <= 0 || hidden <= 0) return TP_ERR_INVALID;
    if (k % n_ranks != 0 || hidden % n_ranks != 0) return TP_ERR_INVALID;
    if ((k / n_ranks) % 8 != 0 || (hidden / n_ranks) % 8 != 0) return TP_ERR_INVALID;
    if (hidden > INT32_MAX || k > INT32_MAX || max_tokens > INT32_MAX) return TP_ERR_UNSUPPORTED;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    int sms = 0, optin = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
        return cuda_fail(e);
    int dyn_max = 0;
    if ((e = set_kernel_attrs(optin, &dyn_max)) != cudaSuccess) return cuda_fail(e);
    void* scratch = nullptr;
    if ((e = noalloc_scratch_current(&scratch)) != cudaSuccess) return cuda_fail(e);
    tp_plan* p = new (std::nothrow) tp_plan{};
    if (!p) return TP_ERR_INVALID;
    p->n_ranks = n_ranks;
    p->max_tokens = max_tokens;
    p->k = k;
    p->hidden = hidden;
    p->ks = k / n_ranks;
    p->hc = hidden / n_ranks;
    p->device = dev;
    p->sm_count = sms;
    p->smem_optin = dyn_max;
    p->variant = TP_VARIANT_AUTO;
    p->staged = 0;
    p->noalloc_scratch = scratch;
    *out = p;
    return TP_OK;
}

tp_status tp_plan_set_variant(tp_plan* plan, int variant, int staged) {
    if (!plan) return TP_ERR_INVALID;
    if (variant != TP_VARIANT_AUTO && variant != TP_VARIANT_EXACT && variant != TP_VARIANT_TENSOR &&
        variant != TP_VARIANT_CLUSTER)
        return TP_ERR_INVALID;
    if (staged != 0 && staged != 1) return TP_ERR_INVALID;
    plan->variant = variant;
    plan->staged = staged;
    return TP_OK;
}

// AUTO: the tensor cores with staged partials (fastest at every token count
// measured on B200, including single-token decode, where a 32-token tile is
// padded but the point is bound by the weight stream; in a chain of calls the
// staged form beats the cluster fold, whose CTAs hold their SMs until the
// whole cluster has folded). EXACT stays selectable: its partials are the
// k-ascending fp32 sums bit for bit.
static int effective_variant(const tp_plan* plan, int64_t tokens) {
    if (plan->variant == TP_VARIANT_AUTO)
        return tokens >= kTensorMinTokens ? TP_VARIANT_TENSOR : TP_VARIANT_EXACT;
    if (plan->variant == TP_VARIANT_CLUSTER) return TP_VARIANT_TENSOR;   // the same kernels
    return plan->variant;
}

int tp_plan_kernel_variant(const tp_plan* plan, int64_t tokens) {
    if (!plan || tokens < 1) return -1;
    return effective_variant(plan, tokens);
}

// The tensor path folds inside its partial kernel: in clusters of the N ranks
// x K parts of a tile (the CLUSTER variant), up to this many tokens by the
// CTA holding a tile's last ticket (counter fold), and on CTA pairs (bf16
// prefill) by the CTA storing a half tile's last rank; other calls stage
// their partials for a ring kernel.
constexpr int64_t kFoldMaxTokens = 2;

static bool tc_folds(const tp_plan* plan, int64_t tokens, int fmt = tpr::kFmtBf16) {
    if (tokens <= kFoldMaxTokens) return true;
    const TcConfig c = tc_config(plan, tokens, true, fmt);
    return c.cluster_fold || tc2_path(plan, c, fmt);
}

// Fold counter block at the start of every workspace: two uint32 per
// 128-row H tile (tickets taken, parts stored), 256-byte rounded, reserved
// on every staged path so that calls of other variants or token counts
// sharing the workspace leave the counters alone.
static size_t counter_tiles(const tp_plan* plan) {
    return static_cast<size_t>((plan->hidden + tpr::kTcRows - 1) / tpr::kTcRows);
}
static size_t counter_block_bytes(const tp_plan* plan) {
    // CTA pairs: one counter per half tile (128 rows x 256 tokens), after the
    // counter fold's tickets and fold counts
    const size_t pair_words = 2 * static_cast<size_t>((plan->hidden + 2 * tpr::kTcRows - 1) / (2 * tpr::kTcRows)) *
                              static_cast<size_t>((plan->max_tokens + tpr::kTc2Tokens - 1) / tpr::kTc2Tokens);
    return ((2 * counter_tiles(plan) + pair_words) * 4 + 255) / 256 * 256;
}

// Bytes of staged partials a call writes (0: none, the exact fused kernel).
static size_t partial_bytes(const tp_plan* plan, int64_t tokens) {
    if (effective_variant(plan, tokens) == TP_VARIANT_TENSOR) {
        const TcConfig c = tc_config(plan, tokens, true);
        return c.cluster_fold ? 0 : tc_partial_bytes(plan, c, tokens);
    }
    if (!plan->staged) return 0;
    return static_cast<size_t>(plan->n_ranks) * static_cast<size_t>(tokens) *
           static_cast<size_t>(plan->hidden) * 2;
}

size_t tp_plan_workspace_bytes(const tp_plan* plan, int64_t tokens) {
    if (!plan || tokens <= 0) return 0;
    const size_t pb = partial_bytes(plan, tokens);
    if (pb == 0) return 0;
    return (counter_block_bytes(plan) + pb + 255) / 256 * 256;
}

int tp_plan_launches(const tp_plan* plan, int64_t tokens) {
    if (!plan || tokens < 0) return -1;
    if (tokens == 0) return 0;
    if (effective_variant(plan, tokens) == TP_VARIANT_TENSOR) return tc_folds(plan, tokens) ? 1 : 2;
    return plan->staged ? 2 : 1;
}

size_t tp_plan_packed_bytes(const tp_plan* plan) {
    return plan ? static_cast<size_t>(plan->hidden) * static_cast<size_t>(plan->k) * 2 : 0;
}

tp_status tp_pack_weights(const tp_plan* plan, const void* w_hk, void* w_packed, void* stream) {
    if (!plan || !w_hk || !w_packed) return TP_ERR_INVALID;
    if (!aligned16(w_hk) || !aligned16(w_packed)) return TP_ERR_ALIGN;
    const size_t bytes = static_cast<size_t>(plan->hidden) * plan->k * 2;
    if (overlaps(w_hk, bytes, w_packed, bytes)) return TP_ERR_INVALID;
    tp_status st = check_device(plan);
    if (st != TP_OK) return st;
    const int64_t total = plan->hidden * (plan->k / 8);
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(plan->sm_count) * 16);
    tpr::pack_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint16_t*>(w_hk), static_cast<uint16_t*>(w_packed),
        static_cast<int>(plan->hidden), plan->k, plan->ks);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TP_OK : cuda_fail(e);
}

static tp_status check_point_args(const tp_plan* plan, const void* x, const void* w, int64_t tokens) {
    if (!plan) return TP_ERR_INVALID;
    if (tokens < 0 || tokens > plan->max_tokens) return TP_ERR_INVALID;
    if (tokens > 0 && (!x || !w)) return TP_ERR_INVALID;
    if (!aligned16(x) || !aligned16(w)) return TP_ERR_ALIGN;
    return TP_OK;
}

// Argument checks shared by both reconcile entry points (all but the workspace).
static tp_status check_reconcile_args(const tp_plan* plan, const void* x, const void* w_packed,
                                      const void* residual, const void* out, int64_t tokens) {
    tp_status st = check_point_args(plan, x, w_packed, tokens);
    if (st != TP_OK || tokens == 0) return st;
    if (!residual || !out) return TP_ERR_INVALID;
    if (!aligned16(residual) || !aligned16(out)) return TP_ERR_ALIGN;
    const size_t mh = static_cast<size_t>(tokens) * plan->hidden * 2;
    const size_t xb = static_cast<size_t>(tokens) * plan->k * 2;
    const size_t wb = static_cast<size_t>(plan->hidden) * plan->k * 2;
    if (overlaps(out, mh, x, xb) || overlaps(out, mh, w_packed, wb) || overlaps(out, mh, residual, mh))
        return TP_ERR_INVALID;
    return TP_OK;
}

// S1-S4 on the tensor cores: one kernel that folds on chip (cluster fold, or
// the counter fold for one or two tokens), else the partial kernel and a ring
// kernel over the staged parts.
static tp_status tensor_reconcile(const tp_plan* plan, const void* x, const TcWeights& wt,
                                  const void* residual, void* out, int64_t tokens,
                                  unsigned int* counters, void* partials, cudaStream_t s) {
    const bool fold = tc_folds(plan, tokens, wt.fmt);
    tp_status st = launch_tc(plan, x, wt, partials, tokens, true, fold, counters, residual, out, s);
    if (st != TP_OK || fold) return st;
    const int splits = tc_config(plan, tokens, true, wt.fmt).splits;
    if (splits > 1) return launch_ring_splits(plan, partials, splits, residual, out, tokens, s);
    return launch_ring(plan, partials, residual, out, tokens, s);
}

// S1-S4 with the fold counters and the staged partials given apart.
static tp_status reconcile_launch(const tp_plan* plan, const void* x, const void* w_packed,
                                  const void* residual, void* out, int64_t tokens,
                                  unsigned int* counters, void* partials, cudaStream_t s) {
    tp_status st = check_device(plan);
    if (st != TP_OK) return st;
    if (effective_variant(plan, tokens) == TP_VARIANT_TENSOR) {
        return tensor_reconcile(plan, x, TcWeights{w_packed, nullptr, tpr::kFmtBf16}, residual, out, tokens,
                                counters, partials, s);
    } else {
        if (!plan->staged)
            return launch_exact(plan, x, w_packed, residual, out, nullptr, tokens, true, s);
        st = launch_exact(plan, x, w_packed, nullptr, nullptr, partials, tokens, false, s);
        if (st != TP_OK) return st;
    }
    return launch_ring(plan, partials, residual, out, tokens, s);
}

tp_status tp_rowlinear_reconcile(const tp_plan* plan, const void* x, const void* w_packed,
                                 const void* residual, void* out, int64_t tokens, void* workspace,
                                 void* stream) {
    tp_status st = check_reconcile_args(plan, x, w_packed, residual, out, tokens);
    if (st != TP_OK || tokens == 0) return st;
    if (!aligned16(workspace)) return TP_ERR_ALIGN;
    const size_t ws = tp_plan_workspace_bytes(plan, tokens);
    if (overlaps(out, static_cast<size_t>(tokens) * plan->hidden * 2, workspace, ws)) return TP_ERR_INVALID;
    if (ws && !workspace) return TP_ERR_WORKSPACE;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    return reconcile_launch(plan, x, w_packed, residual, out, tokens,
                            reinterpret_cast<unsigned int*>(base),
                            ws ? base + counter_block_bytes(plan) : nullptr,
                            static_cast<cudaStream_t>(stream));
}

tp_status tp_rowlinear_reconcile_noalloc(const tp_plan* plan, const void* x, const void* w_packed,
                                         const void* residual, void* out, int64_t tokens,
                                         void* stream) {
    if (!plan) return TP_ERR_INVALID;
    if (tokens < 0 || tokens > plan->max_tokens) return TP_ERR_INVALID;
    if (tokens == 0) return TP_OK;   // nothing to launch, nothing staged
    // Refused before anything is touched when the scratch cannot hold it.
    if (counter_block_bytes(plan) > kNoAllocCounterBytes ||
        partial_bytes(plan, tokens) > kNoAllocScratchBytes - kNoAllocCounterBytes)
        return TP_ERR_WORKSPACE;
    tp_status st = check_reconcile_args(plan, x, w_packed, residual, out, tokens);
    if (st != TP_OK) return st;
    uint8_t* base = static_cast<uint8_t*>(plan->noalloc_scratch);
    return reconcile_launch(plan, x, w_packed, residual, out, tokens,
                            reinterpret_cast<unsigned int*>(base), base + kNoAllocCounterBytes,
                            static_cast<cudaStream_t>(stream));
}

tp_status tp_rowlinear_partials(const tp_plan* plan, const void* x, const void* w_packed,
                                void* partials, int64_t tokens, void* stream) {
    tp_status st = check_point_args(plan, x, w_packed, tokens);
    if (st != TP_OK) return st;
    if (tokens == 0) return TP_OK;
    if (!partials) return TP_ERR_INVALID;
    if (!aligned16(partials)) return TP_ERR_ALIGN;
    const size_t pb = static_cast<size_t>(plan->n_ranks) * tokens * plan->hidden * 2;
    if (overlaps(partials, pb, x, static_cast<size_t>(tokens) * plan->k * 2) ||
        overlaps(partials, pb, w_packed, static_cast<size_t>(plan->hidden) * plan->k * 2))
        return TP_ERR_INVALID;
    if ((st = check_device(plan)) != TP_OK) return st;
    const int variant = effective_variant(plan, tokens);
    if (variant == TP_VARIANT_TENSOR)
        return launch_tc(plan, x, TcWeights{w_packed, nullptr, tpr::kFmtBf16}, partials, tokens, false, false,
                         nullptr, nullptr,
                         nullptr, static_cast<cudaStream_t>(stream));
    return launch_exact(plan, x, w_packed, nullptr, nullptr, partials, tokens, false,
                        static_cast<cudaStream_t>(stream));
}

tp_status tp_ring_reduce(const tp_plan* plan, const void* partials, const void* residual, void* out,
                         int64_t tokens, void* stream) {
    if (!plan) return TP_ERR_INVALID;
    if (tokens < 0 || tokens > plan->max_tokens) return TP_ERR_INVALID;
    if (tokens == 0) return TP_OK;
    if (!partials || !residual || !out) return TP_ERR_INVALID;
    if (!aligned16(partials) || !aligned16(residual) || !aligned16(out)) return TP_ERR_ALIGN;
    const size_t mh = static_cast<size_t>(tokens) * plan->hidden * 2;
    if (overlaps(out, mh, partials, mh * plan->n_ranks) || overlaps(out, mh, residual, mh))
        return TP_ERR_INVALID;
    tp_status st = check_device(plan);
    if (st != TP_OK) return st;
    return launch_ring(plan, partials, residual, out, tokens, static_cast<cudaStream_t>(stream));
}

uint64_t tp_ring_bytes(int n_ranks, int64_t tokens, int64_t hidden, int elem_bytes, int64_t points) {
    if (n_ranks < 1 || tokens < 0 || hidden < 0 || elem_bytes < 0 || points < 0) return 0;
    const uint64_t payload = static_cast<uint64_t>(tokens) * static_cast<uint64_t>(hidden) *
                             static_cast<uint64_t>(elem_bytes) * static_cast<uint64_t>(points);
    return 2ull * static_cast<uint64_t>(n_ranks - 1) * payload / static_cast<uint64_t>(n_ranks);
}

// ---------------------------------------------------- MXFP8 weight shards --

// Scale bytes of an MXFP8 shard set: one 512-byte chunk per rank, 128-row
// tile and 128 columns of a rank slice.
size_t mx_scale_bytes(const tp_plan* p) {
    const int64_t h_tiles = (p->hidden + 127) / 128;
    const int64_t kg = (p->ks + tpr::kMxChunkCols - 1) / tpr::kMxChunkCols;
    return static_cast<size_t>(p->n_ranks) * h_tiles * kg * tpr::kMxChunk;
}

tp_status tp_plan_mxfp8_bytes(const tp_plan* plan, size_t* q_bytes, size_t* scale_bytes) {
    if (!plan || !q_bytes || !scale_bytes) return TP_ERR_INVALID;
    if (plan->ks % tpr::kMxPair != 0) return TP_ERR_UNSUPPORTED;
    *q_bytes = static_cast<size_t>(plan->hidden) * static_cast<size_t>(plan->k);
    *scale_bytes = mx_scale_bytes(plan);
    return TP_OK;
}

size_t tp_plan_mxfp8_workspace_bytes(const tp_plan* plan, int64_t tokens) {
    if (!plan || tokens <= 0) return 0;
    const TcConfig c = tc_config(plan, tokens, true, tpr::kFmtMxfp8);
    const size_t pb = c.cluster_fold ? 0 : tc_partial_bytes(plan, c, tokens);
    if (pb == 0) return 0;
    return (counter_block_bytes(plan) + pb + 255) / 256 * 256;
}

tp_status tp_pack_weights_mxfp8(const tp_plan* plan, const void* w_hk, void* w_q, void* w_scales,
                                void* stream) {
    if (!plan || !w_hk || !w_q || !w_scales) return TP_ERR_INVALID;
    if (plan->ks % tpr::kMxPair != 0) return TP_ERR_UNSUPPORTED;
    if (!aligned16(w_hk) || !aligned16(w_q) || !aligned16(w_scales)) return TP_ERR_ALIGN;
    const size_t wb = static_cast<size_t>(plan->hidden) * plan->k * 2;
    const size_t qb = wb / 2, sb = mx_scale_bytes(plan);
    if (overlaps(w_hk, wb, w_q, qb) || overlaps(w_hk, wb, w_scales, sb) || overlaps(w_q, qb, w_scales, sb))
        return TP_ERR_INVALID;
    tp_status st = check_device(plan);
    if (st != TP_OK) return st;
    // the chunks' padding (rows past H, runs past K/N) reads as scale 2^-127
    cudaError_t me = cudaMemsetAsync(w_scales, 0, sb, static_cast<cudaStream_t>(stream));
    if (me != cudaSuccess) return cuda_fail(me);
    const int64_t blocks_total = static_cast<int64_t>(plan->n_ranks) * plan->hidden * (plan->ks / tpr::kMxBlock);
    const int64_t grid = std::min<int64_t>((blocks_total + 255) / 256, static_cast<int64_t>(plan->sm_count) * 16);
    tpr::pack_weights_mx_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint16_t*>(w_hk), static_cast<uint8_t*>(w_q), static_cast<uint8_t*>(w_scales),
        plan->n_ranks, static_cast<int>(plan->hidden), plan->k, plan->ks);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TP_OK : cuda_fail(e);
}

tp_status tp_rowlinear_reconcile_mxfp8(const tp_plan* plan, const void* x, const void* w_q,
                                       const void* w_scales, const void* residual, void* out,
                                       int64_t tokens, void* workspace, void* stream) {
    if (!plan) return TP_ERR_INVALID;
    if (tokens < 0 || tokens > plan->max_tokens) return TP_ERR_INVALID;
    if (tokens == 0) return TP_OK;
    if (plan->ks % tpr::kMxPair != 0) return TP_ERR_UNSUPPORTED;
    if (!x || !w_q || !w_scales || !residual || !out) return TP_ERR_INVALID;
    if (!aligned16(x) || !aligned16(w_q) || !aligned16(w_scales) || !aligned16(residual) ||
        !aligned16(out) || !aligned16(workspace))
        return TP_ERR_ALIGN;
    const size_t mh = static_cast<size_t>(tokens) * plan->hidden * 2;
    const size_t xb = static_cast<size_t>(tokens) * plan->k * 2;
    const size_t qb = static_cast<size_t>(plan->hidden) * plan->k, sb = mx_scale_bytes(plan);
    const size_t ws = tp_plan_mxfp8_workspace_bytes(plan, tokens);
    if (overlaps(out, mh, x, xb) || overlaps(out, mh, w_q, qb) || overlaps(out, mh, w_scales, sb) ||
        overlaps(out, mh, residual, mh) || overlaps(out, mh, workspace, ws))
        return TP_ERR_INVALID;
    if (ws && !workspace) return TP_ERR_WORKSPACE;
    tp_status st = check_device(plan);
    if (st != TP_OK) return st;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    return tensor_reconcile(plan, x, TcWeights{w_q, w_scales, tpr::kFmtMxfp8}, residual, out, tokens,
                            reinterpret_cast<unsigned int*>(base),
                            ws ? base + counter_block_bytes(plan) : nullptr,
                            static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------- NVFP4 weight shards --

tp_status tp_plan_nvfp4_bytes(const tp_plan* plan, size_t* q_bytes, size_t* scale_bytes) {
    if (!plan || !q_bytes || !scale_bytes) return TP_ERR_INVALID;
    if (plan->ks % tpr::kTcKBlock != 0) return TP_ERR_UNSUPPORTED;
    *q_bytes = static_cast<size_t>(plan->hidden) * static_cast<size_t>(plan->k) / 2;
    *scale_bytes = nv_scale_bytes(plan) + 16;
    return TP_OK;
}

size_t tp_plan_nvfp4_workspace_bytes(const tp_plan* plan, int64_t tokens) {
    if (!plan || tokens <= 0) return 0;
    const TcConfig c = tc_config(plan, tokens, true, tpr::kFmtNvfp4);
    const size_t pb = c.cluster_fold ? 0 : tc_partial_bytes(plan, c, tokens);
    if (pb == 0) return 0;
    return (counter_block_bytes(plan) + pb + 255) / 256 * 256;
}

tp_status tp_pack_weights_nvfp4(const tp_plan* plan, const void* w_hk, void* w_q, void* w_scales,
                                void* stream) {
    if (!plan || !w_hk || !w_q || !w_scales) return TP_ERR_INVALID;
    if (plan->ks % tpr::kTcKBlock != 0) return TP_ERR_UNSUPPORTED;
    if (!aligned16(w_hk) || !aligned16(w_q) || !aligned16(w_scales)) return TP_ERR_ALIGN;
    const size_t wb = static_cast<size_t>(plan->hidden) * plan->k * 2;
    const size_t qb = wb / 4, sb = nv_scale_bytes(plan) + 16;
    if (overlaps(w_hk, wb, w_q, qb) || overlaps(w_hk, wb, w_scales, sb) || overlaps(w_q, qb, w_scales, sb))
        return TP_ERR_INVALID;
    tp_status st = check_device(plan);
    if (st != TP_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* trailer = static_cast<uint8_t*>(w_scales) + nv_scale_bytes(plan);
    cudaError_t e = cudaMemsetAsync(trailer, 0, 16, s);
    if (e != cudaSuccess) return cuda_fail(e);
    const int64_t nvec = plan->hidden * plan->k / 8;
    const int64_t g1 = std::min<int64_t>((nvec + 255) / 256, static_cast<int64_t>(plan->sm_count) * 8);
    tpr::nv_amax_kernel<<<static_cast<unsigned>(g1), 256, 0, s>>>(
        static_cast<const uint16_t*>(w_hk), nvec, reinterpret_cast<uint32_t*>(trailer + 4));
    const int64_t blocks_total = static_cast<int64_t>(plan->n_ranks) * plan->hidden * (plan->ks / 16);
    const int64_t g2 = std::min<int64_t>((blocks_total + 255) / 256, static_cast<int64_t>(plan->sm_count) * 16);
    tpr::pack_weights_nv_kernel<<<static_cast<unsigned>(g2), 256, 0, s>>>(
        static_cast<const uint16_t*>(w_hk), static_cast<uint8_t*>(w_q), static_cast<uint8_t*>(w_scales),
        reinterpret_cast<int*>(trailer), reinterpret_cast<const uint32_t*>(trailer + 4), plan->n_ranks,
        static_cast<int>(plan->hidden), plan->k, plan->ks);
    e = cudaGetLastError();
    return e == cudaSuccess ? TP_OK : cuda_fail(e);
}

tp_status tp_rowlinear_reconcile_nvfp4(const tp_plan* plan, const void* x, const void* w_q,
                                       const void* w_scales, const void* residual, void* out,
                                       int64_t tokens, void* workspace, void* stream) {
    if (!plan) return TP_ERR_INVALID;
    if (tokens < 0 || tokens > plan->max_tokens) return TP_ERR_INVALID;
    if (tokens == 0) return TP_OK;
    if (plan->ks % tpr::kTcKBlock != 0) return TP_ERR_UNSUPPORTED;
    if (!x || !w_q || !w_scales || !residual || !out) return TP_ERR_INVALID;
    if (!aligned16(x) || !aligned16(w_q) || !aligned16(w_scales) || !aligned16(residual) ||
        !aligned16(out) || !aligned16(workspace))
        return TP_ERR_ALIGN;
    const size_t mh = static_cast<size_t>(tokens) * plan->hidden * 2;
    const size_t xb = static_cast<size_t>(tokens) * plan->k * 2;
    const size_t qb = static_cast<size_t>(plan->hidden) * plan->k / 2, sb = nv_scale_bytes(plan) + 16;
    const size_t ws = tp_plan_nvfp4_workspace_bytes(plan, tokens);
    if (overlaps(out, mh, x, xb) || overlaps(out, mh, w_q, qb) || overlaps(out, mh, w_scales, sb) ||
        overlaps(out, mh, residual, mh) || overlaps(out, mh, workspace, ws))
        return TP_ERR_INVALID;
    if (ws && !workspace) return TP_ERR_WORKSPACE;
    tp_status st = check_device(plan);
    if (st != TP_OK) return st;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    return tensor_reconcile(plan, x, TcWeights{w_q, w_scales, tpr::kFmtNvfp4}, residual, out, tokens,
                            reinterpret_cast<unsigned int*>(base),
                            ws ? base + counter_block_bytes(plan) : nullptr,
                            static_cast<cudaStream_t>(stream));
}

// ------------------------------------------- ring protocol between ranks --

// CTAs per rank of the ring protocol: the same for every call of a plan (the
// step flags of a rank are one per CTA), and N of them fit on the device at once.
static int ring_ctas_per_rank(const tp_plan* plan) {
    return std::max(1, std::min(plan->sm_count / plan->n_ranks, 64));
}

static size_t ring_flag_bytes(const tp_plan* plan) {
    return (static_cast<size_t>(ring_ctas_per_rank(plan)) * 4 + 255) / 256 * 256;
}

size_t tp_ring_rank_workspace_bytes(const tp_plan* plan, int64_t tokens) {
    if (!plan || tokens < 0 || tokens > plan->max_tokens) return 0;
    const size_t mh = static_cast<size_t>(tokens) * static_cast<size_t>(plan->hidden) * 2;
    return ring_flag_bytes(plan) + 2 * ((mh + 255) / 256 * 256);
}

tp_status tp_ring_allreduce_ranks(const tp_plan* plan, const void* const* partials, const void* residual,
                                  void* const* outs, void* const* workspaces, int first_rank,
                                  int launch_ranks, int64_t tokens, uint64_t wait_limit_ns, void* stream) {
    if (!plan || !partials || !outs || !workspaces) return TP_ERR_INVALID;
    const int n = plan->n_ranks;
    if (tokens < 0 || tokens > plan->max_tokens) return TP_ERR_INVALID;
    if (first_rank < 0 || launch_ranks < 1 || first_rank + launch_ranks > n) return TP_ERR_INVALID;
    if (tokens == 0) return TP_OK;
    if (!residual) return TP_ERR_INVALID;
    if (!aligned16(residual)) return TP_ERR_ALIGN;
    const size_t mh = static_cast<size_t>(tokens) * static_cast<size_t>(plan->hidden) * 2;
    const size_t ws = tp_ring_rank_workspace_bytes(plan, tokens);
    for (int r = 0; r < n; ++r) {
        if (!partials[r] || !outs[r] || !workspaces[r]) return TP_ERR_INVALID;
        if (!aligned16(partials[r]) || !aligned16(outs[r]) || !aligned16(workspaces[r])) return TP_ERR_ALIGN;
        for (int q = 0; q < n; ++q)
            if (overlaps(outs[r], mh, partials[q], mh) || overlaps(outs[r], mh, workspaces[q], ws) ||
                (q != r && overlaps(outs[r], mh, outs[q], mh)) ||
                (q != r && overlaps(workspaces[r], ws, workspaces[q], ws)) ||
                overlaps(workspaces[r], ws, partials[q], mh))
                return TP_ERR_INVALID;
        if (overlaps(outs[r], mh, residual, mh)) return TP_ERR_INVALID;
    }
    tp_status st = check_device(plan);
    if (st != TP_OK) return st;
    tpr::RingRanks rk{};
    const size_t slot = (mh + 255) / 256 * 256;
    for (int r = 0; r < n; ++r) {
        uint8_t* w = static_cast<uint8_t*>(workspaces[r]);
        rk.partial[r] = static_cast<const uint16_t*>(partials[r]);
        rk.flags[r] = reinterpret_cast<uint32_t*>(w);
        rk.work[r] = reinterpret_cast<uint16_t*>(w + ring_flag_bytes(plan));
        rk.gather[r] = reinterpret_cast<uint16_t*>(w + ring_flag_bytes(plan) + slot);
        rk.out[r] = static_cast<uint16_t*>(outs[r]);
    }
    tpr::RingParams prm{};
    prm.n_ranks = n;
    prm.first_rank = first_rank;
    prm.ctas_per_rank = ring_ctas_per_rank(plan);
    prm.hidden = static_cast<int>(plan->hidden);
    prm.hc = static_cast<int>(plan->hc);
    prm.tokens = tokens;
    prm.residual = static_cast<const uint16_t*>(residual);
    prm.wait_limit_ns = wait_limit_ns ? wait_limit_ns : 1000000000ull;   // 1 s
    // One launch for the ranks it runs; cooperative, so all their CTAs are
    // resident together (a rank's CTAs wait on its predecessor's).
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(launch_ranks * prm.ctas_per_rank));
    cfg.blockDim = dim3(tpr::kRingThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, tpr::ring_protocol_kernel, rk, prm);
    return e == cudaSuccess ? TP_OK : cuda_fail(e);
}

uint64_t tp_allreduce_bytes(int scheme, int n_ranks, int64_t tokens, int64_t hidden, int elem_bytes,
                            int64_t points) {
    if (n_ranks < 2 || tokens < 0 || hidden < 0 || elem_bytes < 0 || points < 0) return 0;
    const uint64_t n = static_cast<uint64_t>(n_ranks);
    const uint64_t b = static_cast<uint64_t>(tokens) * static_cast<uint64_t>(hidden) *
                       static_cast<uint64_t>(elem_bytes) * static_cast<uint64_t>(points);
    switch (scheme) {
        case TP_ALLREDUCE_RING: return 2ull * (n - 1) * b / n;
        case TP_ALLREDUCE_NAIVE: return (n - 1) * b;
        case TP_ALLREDUCE_SWITCH: return b;
        default: return 0;
    }
}

uint64_t tp_moe_combine_bytes(int scheme, int n_ranks, int64_t tokens, int64_t hidden, int elem_bytes,
                              int64_t top_k, int local_accumulate) {
    if (top_k < 1 || (local_accumulate != 0 && local_accumulate != 1)) return 0;
    const uint64_t one = tp_allreduce_bytes(scheme, n_ranks, tokens, hidden, elem_bytes, 1);
    return local_accumulate ? one : static_cast<uint64_t>(top_k) * one;
}

void tp_plan_destroy(tp_plan* plan) { delete plan; }

const char* tp_status_string(tp_status status) {
    switch (status) {
        case TP_OK: return "ok";
        case TP_ERR_INVALID: return "invalid argument";
        case TP_ERR_ALIGN: return "pointer not 16-byte aligned";
        case TP_ERR_UNSUPPORTED: return "unsupported shape, dtype or variant";
        case TP_ERR_WORKSPACE: return "workspace missing or too small";
        case TP_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

int tp_last_cuda_error(void) { return t_last_cuda_error; }

tp_status tp_device_error_flags(const tp_plan* plan, uint32_t* flags, int reset) {
    if (!plan || !flags) return TP_ERR_INVALID;
    tp_status st = check_device(plan);
    if (st != TP_OK) return st;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e);
    uint32_t v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, tpr::g_device_error, sizeof v)) != cudaSuccess) return cuda_fail(e);
    if (reset) {
        const uint32_t zero = 0;
        if ((e = cudaMemcpyToSymbol(tpr::g_device_error, &zero, sizeof zero)) != cudaSuccess)
            return cuda_fail(e);
        // A call that ran out of a wait may have left fold counters of the
        // no-alloc scratch above zero and parts of any tag in it; clear it all
        // (device idle: synchronised above).
        if (v != 0 && (e = cudaMemset(plan->noalloc_scratch, 0, kNoAllocScratchBytes)) != cudaSuccess)
            return cuda_fail(e);
    }
    *flags = v;
    return TP_OK;
}

}  // extern "C"
