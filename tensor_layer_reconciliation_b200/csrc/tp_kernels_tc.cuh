// Partial kernel on the tensor cores (S1) for decode, and for any call with a
// k-split; prompts of more than 128 tokens without a split run on CTA pairs
// (tp_kernels_tc2.cuh).
//
// "Interconnects e clusters", 01 Conceito: each rank computes a partial
// result over its slice of the weight matrix; prefill runs every position
// of the prompt at once, which makes the partial a dense contraction.
//
// Work unit = (rank r, 128 rows of H, BN tokens, k-split s): the tile
//     P[r][m0 .. m0+BN)[h0 .. h0+128) = x_r[m0 ..][:] . W_r[h0 ..][:]^T
// computed as D = A * B^T on tcgen05 with A = the 128 x 64 weight block
// (rows of W_r, K-major) and B = the BN x 64 activation block (rows of x_r,
// K-major), both staged by TMA with the 128-byte swizzle, D in tensor memory
// as 128 lanes (h) x BN fp32 columns (m). Putting the weights on the
// 128-row side keeps BN free to be small, so decode batches of 32 or 64
// tokens use the tensor cores without padding the token dimension.
//
// Roles (persistent CTAs, units strided by the grid):
//   warp 0     TMA producer: a STAGES-deep ring of (A, B) blocks, "full"
//              mbarriers with transaction bytes, "empty" mbarriers released
//              by the MMA completion. Weight blocks of the first STAGES
//              iterations are issued before griddepcontrol.wait.
//   warp 1     allocates the tensor memory; one thread issues 4 MMAs
//              (K = 16 each) per 64-column block and commits; two
//              accumulator buffers let the epilogue of one unit overlap the
//              MMAs of the next.
//   warps 2-5  epilogue: tcgen05.ld of their 32-lane quarter, one
//              round-to-nearest-even to bf16 per partial, stores to the
//              partial buffer [N][M][H] (32 consecutive h per warp store).
// When there are fewer units than SMs (few ranks, small H) the K range of
// each unit is split in SPLITS contiguous parts handled by different CTAs;
// each part's fp32 sum is stored unrounded in [SPLITS][N][M][H] and the
// ring kernel adds the parts in split order before the one rounding to bf16.
// Units run token tile fastest, so CTAs working at the same time share each
// weight tile through L2 (a tile of weights serves every token tile of a call).
// Folding (S2-S4) inside this kernel, two ways:
//  * cluster fold (N * SPLITS <= 8): the C = N * SPLITS CTAs of a thread-block
//    cluster are the N ranks (and K parts) of one (H tile, token tile). Each
//    keeps its accumulator (a bf16 partial, or an fp32 part sum) in its own
//    shared memory; after an mbarrier handshake across the cluster each CTA
//    folds 1/C of the tile's outputs, reading the parts of every output through
//    the cluster's shared window in ring order, and adds the residual. The partials never leave the chip and the
//    fold work is spread over all N CTAs (CTAs of a cluster run at the same
//    time, so the waits between them always end).
//  * counter fold (one or two tokens with a k-split): the CTA that stores the
//    last of the N * SPLITS parts of an (H tile, token tile) -- found with a
//    per-tile counter in the workspace -- folds that tile, each epilogue
//    thread one row h.
// Otherwise (more tokens with a k-split) a ring kernel folds the stored parts.
// Quantised weights (FMT = MXFP8 or NVFP4): the producer stages code tiles
// (128 rows x 64 codes) and their scales instead of bf16 weight tiles; four
// more warps (6-9) turn each code tile into the bf16 tile the MMA reads
// (MXFP8: E4M3 * 2^s; NVFP4: E2M1 * E4M3 block scale * 2^g; exact in bf16
// for the shards the formats' definitions allow), each thread one row, into
// one of the converted slots in tensor memory beside the accumulators (a row
// a lane, two bf16 a column); the MMA reads A from there, waits for its slot
// and frees it (and the stage, whose activation tile it reads) when it is
// done. Everything after the MMA -- the three epilogues -- is the same.
// Accumulation order inside the tensor core is the hardware's; the partial
// is the fp32 sum rounded once to bf16, like the oracle's, but only equal to
// it where the two fp32 sums round to the same bf16 value.
#pragma once

#include "tp_kernels_mx.cuh"
#include "tp_tcgen05.cuh"

namespace tpr {

constexpr int kTcRows = 128;               // MMA M: weight rows per tile
constexpr int kTcKBlock = 64;              // bf16 columns per staged block
constexpr int kTcMaxStages = 16;
constexpr int kTcThreads = 192;            // producer, MMA and 4 epilogue warps
constexpr int kTcMxThreads = 320;          // quantised weights: + 4 converter warps
constexpr uint32_t kTcATile = kTcRows * kTcKBlock * 2;  // 16 KB
// Quantised forms: converted bf16 tiles in flight between the converters and
// the MMAs live in tensor memory beside the accumulators (k-block i goes to
// slot i % slots; at most kCvtSlotsMax slots).
constexpr int kCvtSlotsMax = 8;
constexpr uint32_t kMxCodeTile = kTcRows * kTcKBlock;   // 8 KB of E4M3 codes
constexpr uint32_t kMxScaleTile = kMxChunk;             // the scale chunk holding the block's scales
constexpr uint32_t kNvCodeTile = kTcRows * kTcKBlock / 2;  // 4 KB: two E2M1 codes a byte
constexpr uint32_t kNvScaleTile = kTcRows * 4;             // the 4 E4M3 block scales of each row

// Weight formats of the tensor-core kernel (a template parameter).
constexpr int kFmtBf16 = 0;    // packed bf16 shards, staged by TMA as the MMA's A tiles
constexpr int kFmtMxfp8 = 1;   // E4M3 codes + E8M0 scales per 32, widened on chip
constexpr int kFmtNvfp4 = 2;   // E2M1 codes + E4M3 scales per 16 (x 2^g), widened on chip
constexpr int kFmtMxfp8Bs = 3; // MXFP8 codes read by the block-scaled MMA (at most 8 tokens)

// Block-scaled MXFP8 form. The codes and their E8M0 scales go to the tensor
// cores as stored (tcgen05.mma kind::mxf8f6f4, one scale per 32 values of K
// on each side), 128 columns of K a stage. The bf16 activations are split on
// chip into two E4M3 terms with E8M0 scales of their own, one pair per 32
// values of K: x = 2^e1 q1 + 2^e2 q2, e1 = floor(log2 max|x|) - 7 (so the
// run's largest value over 2^e1 lies in [128, 256): nothing saturates), q1
// the E4M3 value nearest x / 2^e1, and q2 the same for the remainder
// x - 2^e1 q1 under its own maximum. A bf16 value has 8 significant bits; q1
// takes the leading 4 and the remainder fits the 4 of q2 whenever q1 is a
// normal E4M3 value, so every x at least 2^(e1 - 6) (about 2^-13 of its run's
// maximum) is split exactly; a smaller one is off by at most 2^(e1 - 14).
// The MMA's B operand holds q1 of token t in row t and q2 in row 8 + t; the
// epilogue adds accumulator columns t and 8 + t in fp32.
// A stage's activation slot first receives the bf16 block of x by TMA ([8
// tokens][128] bf16, 2 KB, no swizzle; a barrier of its own, x_full); the
// splitting warps read it into registers and then write the B tile and its
// scale chunk over it.
constexpr uint32_t kBsBRows = 16;                         // MMA N: 8 tokens x 2 terms
constexpr uint32_t kBsXTile = 8 * kMxChunkCols * 2;       // the bf16 activation block
constexpr uint32_t kBsSfbOff = kBsBRows * 128;            // B scale chunk after the B tile
constexpr uint32_t kBsBTile = 3 * 1024;                   // B tile + scale chunk, 1024-aligned
constexpr uint32_t kBsCodeTile = kTcRows * kMxChunkCols;  // 16 KB of E4M3 codes
// The four K = 32 steps of a stage alternate between this many accumulators
// (16 columns each, within the unit's 32), summed by the epilogue: MMAs into
// different accumulators do not wait on one another's results.
constexpr int kBsAccs = 2;

__host__ __device__ constexpr uint32_t fmt_code_tile(int fmt) {
    return fmt == kFmtMxfp8 ? kMxCodeTile
           : fmt == kFmtNvfp4 ? kNvCodeTile
           : fmt == kFmtMxfp8Bs ? kBsCodeTile
                                : kTcATile;
}
__host__ __device__ constexpr uint32_t fmt_scale_tile(int fmt) {
    return fmt == kFmtMxfp8 || fmt == kFmtMxfp8Bs ? kMxScaleTile : fmt == kFmtNvfp4 ? kNvScaleTile : 0;
}
// Columns of K one stage holds.
__host__ __device__ constexpr int fmt_k_block(int fmt) {
    return fmt == kFmtMxfp8Bs ? kMxChunkCols : kTcKBlock;
}
// Activation bytes of one stage: x_rows rows of the block, or (block-scaled
// form) the split B tile with its scale chunk.
__host__ __device__ constexpr uint32_t fmt_b_tile(int fmt, int x_rows) {
    return fmt == kFmtMxfp8Bs ? kBsBTile : static_cast<uint32_t>(x_rows) * kTcKBlock * 2;
}

// What the epilogue does with each accumulator (a template parameter, so each
// form compiles only its own epilogue):
constexpr int kTcStore = 0;         // store the partials (or fp32 k-parts) for a ring kernel
constexpr int kTcCounterFold = 1;   // store k-parts; the CTA that completes a tile folds it
constexpr int kTcClusterFold = 2;   // fold on chip across the cluster's N CTAs

struct TcParams {
    int n_ranks;   // N
    int ks;        // K / N
    int hidden;    // H
    int tokens;    // M
    int h_tiles;   // ceil(H / 128)
    int m_tiles;   // ceil(M / BN)
    int splits;    // k-splits per (rank, h tile, m tile)
    int units;     // N * h_tiles * m_tiles * splits
    int stages;    // 2 .. kTcMaxStages
    int x_rows;    // token rows of x staged per block: BN, or 8 (one swizzle atom) for at most 8 tokens
    uint16_t* partials;     // [N][M][H] bf16 (splits == 1)
    float* partials_f32;    // [splits][N][M][H] fp32 sums of each k part (splits > 1); the 64-bit tagged parts of the counter fold

    int hc;                       // H / N, the chunk each rank owns in the ring
    unsigned int* counters;       // [2][h_tiles * m_tiles]: tickets taken (zero between calls), folds done
    const uint16_t* x;            // [M][K] activations (for the L2 prefetch)
    int64_t k;                    // K
    const uint16_t* residual;     // [M][H]
    uint16_t* out;                // [M][H]
    const int* nv_gexp;           // NVFP4: the second-level exponent g
    const uint8_t* mx_scales;     // MXFP8: chunked E8M0 scales [N][h_tiles][mx_kg][512]
    int mx_kg;                    // MXFP8: ceil(K/N / 128), scale chunks per row tile
};

// Cluster fold of one (H tile, token tile). The cluster's C = N * SPLITS CTAs
// hold, in shared memory, the tile's partial of rank q / SPLITS over K part
// q % SPLITS (CTA q of the cluster): bf16 [T][128] when SPLITS == 1 (the
// partial itself), fp32 [T][128] sums of the part otherwise (T = the tile's
// tokens, at most BN). The tile's T x 16 vectors of 8 rows are shared out
// evenly; for each, rank r's partial is the fp32 sum of its parts in split
// (k-ascending) order rounded once to bf16, the N partials are added in ring
// order from the chunk's owner (all loads before the first add), then the
// residual, and the output is stored. et = epilogue thread, 0..127.
// Eight ring adds at once (a on the left): bf16 round-to-nearest-even each.
__device__ __forceinline__ uint4 bf16x8_add_tc(uint4 a, uint4 b) {
    return make_uint4(bf16x2_add(a.x, b.x), bf16x2_add(a.y, b.y), bf16x2_add(a.z, b.z),
                      bf16x2_add(a.w, b.w));
}

// The residual of this thread's first output vector of the cluster fold
// (zero if it has none), loaded while the cluster's partial tiles are being
// written, before the handshake.
__device__ __forceinline__ uint4 cluster_fold_first_residual(const TcParams& p, uint32_t crank, int csize,
                                                             int ht, int m0, int bn, int et) {
    const int t_tile = min(bn, p.tokens - m0);
    const int nv = t_tile * (kTcRows / 8);
    const int v = static_cast<int>(crank) * nv / csize + et;
    const int v1 = (static_cast<int>(crank) + 1) * nv / csize;
    const int h = ht * kTcRows + (v & 15) * 8;
    if (v >= v1 || h >= p.hidden) return make_uint4(0, 0, 0, 0);
    return ld_global_nc_v4(p.residual + static_cast<size_t>(m0 + (v >> 4)) * p.hidden + h);
}

template <int SPLITS>
__device__ __forceinline__ void cluster_fold_tile(const TcParams& p, const void* part_buf,
                                                  uint32_t crank, int csize, int ht, int m0,
                                                  int bn, int et, uint4 first_res) {
    const int n = p.n_ranks;
    const int t_tile = min(bn, p.tokens - m0);                      // tokens of this tile
    const int nv = t_tile * (kTcRows / 8);
    const int v0 = static_cast<int>(crank) * nv / csize, v1 = (static_cast<int>(crank) + 1) * nv / csize;
#pragma unroll 1
    for (int v = v0 + et; v < v1; v += 128) {
        const int tt = v >> 4;                                      // token in the tile
        const int hv = (v & 15) * 8;                                // row offset in the tile
        const int m = m0 + tt;
        const int h = ht * kTcRows + hv;
        if (h >= p.hidden) continue;
        const int c = h / p.hc;
        uint4 sum;
        if constexpr (SPLITS == 1) {
            const uint16_t* mine = static_cast<const uint16_t*>(part_buf) + tt * kTcRows + hv;
            uint4 pv[kMaxRanks];
#pragma unroll
            for (int i = 0; i < kMaxRanks; ++i) {
                if (i < n) {
                    int rr = c + i;   // ring order: the chunk's owner first
                    if (rr >= n) rr -= n;
                    pv[i] = ld_dsmem_v4(mapa_shared(mine, static_cast<uint32_t>(rr)));
                }
            }
            sum = pv[0];
#pragma unroll
            for (int i = 1; i < kMaxRanks; ++i)
                if (i < n) sum = bf16x8_add_tc(sum, pv[i]);
        } else {
            static_assert(SPLITS >= 2 && SPLITS <= 4, "cluster of at most 8 CTAs");
            // rank by rank in ring order (the parts of a rank loaded together)
            const float* mine = static_cast<const float*>(part_buf) + tt * kTcRows + hv;
#pragma unroll 1
            for (int i = 0; i < n; ++i) {
                int rr = c + i;
                if (rr >= n) rr -= n;
                uint4 a[SPLITS][2];
#pragma unroll
                for (int sp = 0; sp < SPLITS; ++sp) {
                    const uint32_t base = mapa_shared(mine, static_cast<uint32_t>(rr * SPLITS + sp));
                    a[sp][0] = ld_dsmem_v4(base);
                    a[sp][1] = ld_dsmem_v4(base + 16);
                }
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float((&a[0][e >> 2].x)[e & 3]);
#pragma unroll
                for (int sp = 1; sp < SPLITS; ++sp)
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        f[e] = __fadd_rn(f[e], __uint_as_float((&a[sp][e >> 2].x)[e & 3]));
                const uint4 pr = make_uint4(bf16x2_from_f32(f[0], f[1]), bf16x2_from_f32(f[2], f[3]),
                                            bf16x2_from_f32(f[4], f[5]), bf16x2_from_f32(f[6], f[7]));
                sum = i == 0 ? pr : bf16x8_add_tc(sum, pr);
            }
        }
        const size_t o = static_cast<size_t>(m) * p.hidden + h;
        const uint4 rv = v == v0 + et ? first_res : ld_global_nc_v4(p.residual + o);
        st_global_v4(p.out + o, bf16x8_add_tc(rv, sum));
    }
}

// Four E4M3 codes (one word, the earlier k in the low byte) times the scale
// pair (f, f) (two f32 in 64 bits) -> two bf16x2 words: each code widened to
// f16 (exact), then f32, multiplied (exact: 4 significant bits times a power
// of two) and rounded to bf16 (exact for every value bf16 holds).
__device__ __forceinline__ void e4m3x4_scaled_bf16(uint32_t w, uint64_t f2, uint32_t& o0, uint32_t& o1) {
    asm("{\n\t"
        ".reg .b16 c0, c1;\n\t.reg .b32 h, a, b;\n\t.reg .f16 h0, h1;\n\t.reg .b64 v;\n\t"
        "mov.b32 {c0, c1}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 h, c0;\n\t"
        "mov.b32 {h0, h1}, h;\n\t"
        "cvt.f32.f16 a, h0;\n\t"
        "cvt.f32.f16 b, h1;\n\t"
        "mov.b64 v, {a, b};\n\t"
        "mul.rn.f32x2 v, v, %3;\n\t"
        "mov.b64 {a, b}, v;\n\t"
        "cvt.rn.bf16x2.f32 %0, b, a;\n\t"
        "cvt.rn.f16x2.e4m3x2 h, c1;\n\t"
        "mov.b32 {h0, h1}, h;\n\t"
        "cvt.f32.f16 a, h0;\n\t"
        "cvt.f32.f16 b, h1;\n\t"
        "mov.b64 v, {a, b};\n\t"
        "mul.rn.f32x2 v, v, %3;\n\t"
        "mov.b64 {a, b}, v;\n\t"
        "cvt.rn.bf16x2.f32 %1, b, a;\n\t"
        "}"
        : "=r"(o0), "=r"(o1)
        : "r"(w), "l"(f2));
}

// Eight E2M1 codes (one word: byte i holds codes 2i (bits 0-3) and 2i+1)
// times (f, f) -> four bf16x2 words, as e4m3x4_scaled_bf16 (2 significant bits
// times a 4-bit block scale times a power of two: exact in f32).
__device__ __forceinline__ void e2m1x8_scaled_bf16(uint32_t w, uint64_t f2, uint32_t* o) {
    asm("{\n\t"
        ".reg .b8 c0, c1, c2, c3;\n\t.reg .b32 h, a, b;\n\t.reg .f16 h0, h1;\n\t.reg .b64 v;\n\t"
        "mov.b32 {c0, c1, c2, c3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 h, c0;\n\t"
        "mov.b32 {h0, h1}, h;\n\t"
        "cvt.f32.f16 a, h0;\n\t"
        "cvt.f32.f16 b, h1;\n\t"
        "mov.b64 v, {a, b};\n\t"
        "mul.rn.f32x2 v, v, %5;\n\t"
        "mov.b64 {a, b}, v;\n\t"
        "cvt.rn.bf16x2.f32 %0, b, a;\n\t"
        "cvt.rn.f16x2.e2m1x2 h, c1;\n\t"
        "mov.b32 {h0, h1}, h;\n\t"
        "cvt.f32.f16 a, h0;\n\t"
        "cvt.f32.f16 b, h1;\n\t"
        "mov.b64 v, {a, b};\n\t"
        "mul.rn.f32x2 v, v, %5;\n\t"
        "mov.b64 {a, b}, v;\n\t"
        "cvt.rn.bf16x2.f32 %1, b, a;\n\t"
        "cvt.rn.f16x2.e2m1x2 h, c2;\n\t"
        "mov.b32 {h0, h1}, h;\n\t"
        "cvt.f32.f16 a, h0;\n\t"
        "cvt.f32.f16 b, h1;\n\t"
        "mov.b64 v, {a, b};\n\t"
        "mul.rn.f32x2 v, v, %5;\n\t"
        "mov.b64 {a, b}, v;\n\t"
        "cvt.rn.bf16x2.f32 %2, b, a;\n\t"
        "cvt.rn.f16x2.e2m1x2 h, c3;\n\t"
        "mov.b32 {h0, h1}, h;\n\t"
        "cvt.f32.f16 a, h0;\n\t"
        "cvt.f32.f16 b, h1;\n\t"
        "mov.b64 v, {a, b};\n\t"
        "mul.rn.f32x2 v, v, %5;\n\t"
        "mov.b64 {a, b}, v;\n\t"
        "cvt.rn.bf16x2.f32 %3, b, a;\n\t"
        "}"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
        : "r"(w), "l"(f2));
}

// (f, f) as one 64-bit operand of the packed f32x2 multiply.
__device__ __forceinline__ uint64_t f32_pair(float f) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %1};" : "=l"(d) : "f"(f));
    return d;
}

// Widens row t of a staged E4M3 code tile (64 codes in a 64-byte row, placed
// by TMA with the 64-byte swizzle: 16-byte chunk c of row t at chunk
// c ^ ((t >> 1) & 3)), with its two E8M0 scales (codes 0-31, 32-63), into
// this thread's lane of a bf16 A tile in tensor memory: 32 columns from
// taddr, two values a column, k ascending. With the swizzle the eight rows a
// quarter-warp reads at once lie in eight different bank groups.
__device__ __forceinline__ void mx_convert_row(const uint8_t* code_row, const uint8_t* scale_row,
                                               uint32_t taddr, int t) {
    const uint32_t sb = *reinterpret_cast<const uint16_t*>(scale_row);
#pragma unroll
    for (int half = 0; half < 2; ++half) {                   // codes 32half .. 32half+31
        const uint64_t f = f32_pair(e8m0_to_f32(half ? sb >> 8 : sb & 0xFFu));
        uint32_t o[16];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * half + cc;                     // codes 16c .. 16c+15
            const uint4 q = *reinterpret_cast<const uint4*>(code_row + 16 * (c ^ ((t >> 1) & 3)));
            e4m3x4_scaled_bf16(q.x, f, o[8 * cc + 0], o[8 * cc + 1]);
            e4m3x4_scaled_bf16(q.y, f, o[8 * cc + 2], o[8 * cc + 3]);
            e4m3x4_scaled_bf16(q.z, f, o[8 * cc + 4], o[8 * cc + 5]);
            e4m3x4_scaled_bf16(q.w, f, o[8 * cc + 6], o[8 * cc + 7]);
        }
        tmem_st_16cols(taddr + 16 * half, o);
    }
}

// NVFP4 row: 32 bytes of codes (64 E2M1 values, the earlier k in the low
// nibble; TMA's 32-byte swizzle puts half c of row t at half c ^ ((t >> 2) & 1)),
// the row's four E4M3 block scales (one per 16 values) and the second-level
// factor 2^g -> this thread's lane of a bf16 A tile in tensor memory, as in
// mx_convert_row.
__device__ __forceinline__ void nv_convert_row(const uint8_t* code_row, const uint8_t* scale_row,
                                               float two_g, uint32_t taddr, int t) {
    const uint32_t sw = *reinterpret_cast<const uint32_t*>(scale_row);
    const uint32_t h01 = f16x2_from_e4m3x2(static_cast<uint16_t>(sw & 0xFFFFu));
    const uint32_t h23 = f16x2_from_e4m3x2(static_cast<uint16_t>(sw >> 16));
    const uint64_t f[4] = {f32_pair(f16_lo_to_f32(h01) * two_g), f32_pair(f16_hi_to_f32(h01) * two_g),
                           f32_pair(f16_lo_to_f32(h23) * two_g), f32_pair(f16_hi_to_f32(h23) * two_g)};
#pragma unroll
    for (int c = 0; c < 2; ++c) {                            // codes 32c .. 32c+31
        const uint4 q = *reinterpret_cast<const uint4*>(code_row + 16 * (c ^ ((t >> 2) & 1)));
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};        // 8 codes a word
        uint32_t o[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {                      // word i: codes 32c + 8i .. +7, block 2c + i/2
            uint32_t oo[4];
            e2m1x8_scaled_bf16(w[i], f[2 * c + (i >> 1)], oo);
            o[4 * i + 0] = oo[0];
            o[4 * i + 1] = oo[1];
            o[4 * i + 2] = oo[2];
            o[4 * i + 3] = oo[3];
        }
        tmem_st_16cols(taddr + 16 * c, o);
    }
}

// Counter fold: K parts carry the tag of their call (the tile's fold count
// + 1) in the same 64-bit word -- the fp32 part, or the bf16 partial when K is
// not split, in the low half, the tag in the high half -- so the CTA folding
// a tile reads them without waiting for a count: a part whose tag is not yet
// this call's is read again (bounded). Word-sized stores and loads are
// single-copy atomic, so a part is never seen half-written.
// A tagged part as it is now at gpu scope: a volatile relaxed load, so that
// a polling loop reads memory again on every pass (a plain load of an address
// the loop never writes may be hoisted out of it).
__device__ __forceinline__ uint64_t ld_cg_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
// The low half of a tagged part once its tag is `tag` (read again until then).
__device__ __forceinline__ bool tagged_part(const uint64_t* p, uint32_t tag, uint32_t& v) {
    uint64_t w = ld_cg_u64(p);
    if (static_cast<uint32_t>(w >> 32) != tag) {
        const uint64_t t0 = globaltimer_ns();
        while (static_cast<uint32_t>((w = ld_cg_u64(p)) >> 32) != tag)
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                atomicOr(&g_device_error, kErrWaitTimeout);
                return false;
            }
    }
    v = static_cast<uint32_t>(w);
    return true;
}

// S2-S3 of one output element from tagged parts: rank r's partial is the sum
// of its SPLITS fp32 parts in split (k) order rounded once to bf16 (or its
// bf16 partial when SPLITS == 1); the N partials are added in ring order
// from the chunk's owner c. All loads are issued before the first check
// (up to 16 of them at once; more go a rank at a time).
__device__ __forceinline__ bool fold_tagged(const TcParams& p, size_t plane, size_t off, int c, uint32_t tag,
                                            uint16_t& out) {
    const int n = p.n_ranks, splits = p.splits;
    bool ok = true;
    uint16_t s = 0;
    const uint64_t* parts = reinterpret_cast<const uint64_t*>(p.partials_f32);
    if (splits == 1) {   // bf16 partials
        uint64_t w[kMaxRanks];
#pragma unroll
        for (int i = 0; i < kMaxRanks; ++i)
            if (i < n) {
                int rr = c + i;
                if (rr >= n) rr -= n;
                w[i] = ld_cg_u64(parts + static_cast<size_t>(rr) * plane + off);
            }
#pragma unroll
        for (int i = 0; i < kMaxRanks; ++i)
            if (i < n) {
                uint32_t v = static_cast<uint32_t>(w[i]);
                if (static_cast<uint32_t>(w[i] >> 32) != tag) {
                    int rr = c + i;
                    if (rr >= n) rr -= n;
                    ok = tagged_part(parts + static_cast<size_t>(rr) * plane + off, tag, v) && ok;
                }
                s = i == 0 ? static_cast<uint16_t>(v) : bf16_add(s, static_cast<uint16_t>(v));
            }
        out = s;
        return ok;
    }
    if (n * splits <= 16) {
        uint64_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < n * splits) {
                const int i = j / splits, sp = j - i * splits;
                int rr = c + i;
                if (rr >= n) rr -= n;
                w[j] = ld_cg_u64(parts + (static_cast<size_t>(sp) * n + rr) * plane + off);
            }
        float f = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < n * splits) {
                const int i = j / splits, sp = j - i * splits;
                uint32_t vb = static_cast<uint32_t>(w[j]);
                if (static_cast<uint32_t>(w[j] >> 32) != tag) {
                    int rr = c + i;
                    if (rr >= n) rr -= n;
                    ok = tagged_part(parts + (static_cast<size_t>(sp) * n + rr) * plane + off, tag, vb) && ok;
                }
                const float v = __uint_as_float(vb);
                f = sp == 0 ? v : __fadd_rn(f, v);
                if (sp == splits - 1) {
                    const uint16_t pr = f32_to_bf16_rne(f);
                    s = i == 0 ? pr : bf16_add(s, pr);
                }
            }
        out = s;
        return ok;
    }
#pragma unroll 1
    for (int i = 0; i < n; ++i) {
        int rr = c + i;
        if (rr >= n) rr -= n;
        float f = 0.0f;
#pragma unroll 1
        for (int sp = 0; sp < splits; ++sp) {
            uint32_t vb = 0;
            ok = tagged_part(parts + (static_cast<size_t>(sp) * n + rr) * plane + off, tag, vb) && ok;
            const float v = __uint_as_float(vb);
            f = sp == 0 ? v : __fadd_rn(f, v);
        }
        const uint16_t pr = f32_to_bf16_rne(f);
        s = i == 0 ? pr : bf16_add(s, pr);
    }
    out = s;
    return ok;
}

// Token tiles up to 64 run two CTAs per SM: at most 168 registers a thread
// (96 with the converter warps).
// E8M0 exponent of a split term under run maximum a: floor(log2 a) - 7,
// at least -127 (a = 0 or below the f32 normal range gives -127).
__device__ __forceinline__ int split_exp(float a) {
    return max(-127, static_cast<int>((__float_as_uint(a) >> 23) & 0xFFu) - 134);
}

// Block-scaled form, one 32-value run of the activations: lane 4t + part of
// a converter warp holds x[t][8 part .. 8 part + 7] of the run (bf16 in v,
// zeros past the tokens or K/N); the four lanes of token t hold the whole
// run. Writes q1 to row t and q2 to row 8 + t of the B tile `bt` (rows of
// 128 bytes with the 128-byte swizzle: 16-byte chunk c of row n at chunk
// c ^ (n % 8)), columns 32 run + 8 part .. + 7, and the exponents' E8M0
// bytes to the scale chunk after the tile (row n, byte `run`).
__device__ __forceinline__ void x_split_run(uint4 v, uint8_t* bt, int t, int run, int part) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float y[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        y[2 * i] = bf16_lo(w[i]);
        y[2 * i + 1] = bf16_hi(w[i]);
    }
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(y[i]));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
    const int e1 = split_exp(a);
    const float inv1 = pow2_f32(-e1), sc1 = pow2_f32(e1);
    // q1, and the remainder (exact: both sides carry at most 8 significant
    // bits within a few binades of each other)
    uint32_t q1[2], q2[2];
    float rem[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint16_t c = e4m3x2_from_f32(y[2 * i] * inv1, y[2 * i + 1] * inv1);
        const uint32_t h = f16x2_from_e4m3x2(c);
        rem[2 * i] = y[2 * i] - f16_lo_to_f32(h) * sc1;
        rem[2 * i + 1] = y[2 * i + 1] - f16_hi_to_f32(h) * sc1;
        if (i & 1) q1[i >> 1] |= static_cast<uint32_t>(c) << 16;
        else q1[i >> 1] = c;
    }
    float b = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) b = fmaxf(b, fabsf(rem[i]));
    b = fmaxf(b, __shfl_xor_sync(0xFFFFFFFFu, b, 1));
    b = fmaxf(b, __shfl_xor_sync(0xFFFFFFFFu, b, 2));
    const int e2 = split_exp(b);
    const float inv2 = pow2_f32(-e2);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint16_t c = e4m3x2_from_f32(rem[2 * i] * inv2, rem[2 * i + 1] * inv2);
        if (i & 1) q2[i >> 1] |= static_cast<uint32_t>(c) << 16;
        else q2[i >> 1] = c;
    }
    const int chunk = 2 * run + (part >> 1);
    const int off = ((chunk ^ (t & 7)) << 4) + (part & 1) * 8;
    *reinterpret_cast<uint2*>(bt + t * 128 + off) = make_uint2(q1[0], q1[1]);
    *reinterpret_cast<uint2*>(bt + (8 + t) * 128 + off) = make_uint2(q2[0], q2[1]);
    if (part == 0) {
        bt[kBsSfbOff + t * 16 + run] = static_cast<uint8_t>(e1 + 127);
        bt[kBsSfbOff + (8 + t) * 16 + run] = static_cast<uint8_t>(e2 + 127);
    }
}

template <int BN, int MODE, int FMT>
__global__ void __launch_bounds__(FMT != kFmtBf16 ? kTcMxThreads : kTcThreads, BN <= 64 ? 2 : 1)
    tc_partial_kernel(const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_s, const TcParams p) {
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M = 128");
    // Activation rows staged per block: the whole BN-row tile, or, for at most
    // eight tokens, one 8-row swizzle atom that every 8-row group of the MMA's
    // B operand reads (descriptor stride 0): rows 8.. of the product repeat
    // rows 0..7 in accumulator columns nobody reads.
    constexpr bool BS = FMT == kFmtMxfp8Bs;                     // block-scaled MMA on the codes
    static_assert(!BS || BN == 32, "block-scaled form: a 32-column accumulator, at most 8 tokens");
    static_assert(!BS || (kBsAccs >= 1 && kBsAccs * 16 <= BN && 4 % kBsAccs == 0), "accumulators fit the unit's columns");
    const uint32_t kBTile = fmt_b_tile(FMT, p.x_rows);
    const bool x_atom = !BS && p.x_rows < BN;
    constexpr bool MX = FMT == kFmtMxfp8 || FMT == kFmtNvfp4;   // converted on chip
    constexpr int KB = fmt_k_block(FMT);                        // columns of K a stage holds
    constexpr uint32_t kWTile = fmt_code_tile(FMT);             // weight bytes staged per block
    constexpr uint32_t kSTile = fmt_scale_tile(FMT);            // scale bytes staged per block
    // Tensor memory: two accumulators of BN columns; the quantised forms add
    // their converted A slots (32 columns each: 128 rows x 64 bf16) after them,
    // within 256 columns a CTA when two share an SM.
    constexpr int kSlots = !MX ? 1 : BN <= 32 ? 6 : BN <= 64 ? 4 : 8;
    constexpr uint32_t kSlotCol0 = 2 * BN;
    // The block-scaled form adds, per stage, the A and B scales (4 columns
    // each) after them: a stage's copies never overwrite scales the previous
    // stages' MMAs may still read.
    constexpr uint32_t kTmemCols = MX ? (BN <= 64 ? 256u : 512u) : BS ? 256u : (2 * BN < 32 ? 32u : 2u * BN);
    static_assert(!MX || (BN <= 128 && kSlotCol0 + 32 * kSlots <= kTmemCols && kSlots <= kCvtSlotsMax),
                  "converted slots fit in tensor memory");
    constexpr uint32_t kSfaCol = 2 * BN, kSfbCol = 2 * BN + 4;   // + 8 per stage
    static_assert(!BS || kSfbCol + 8 * (kTcMaxStages - 1) + 4 <= kTmemCols, "block scales fit in tensor memory");
    constexpr uint32_t kIdesc = idesc_bf16_f32(kTcRows, BN);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int S = p.stages;
    uint8_t* a_ring = smem;                                              // weight tiles (TMA)
    uint8_t* b_ring = a_ring + static_cast<size_t>(S) * kWTile;         // activation tiles
    uint8_t* s_ring = b_ring + static_cast<size_t>(S) * kBTile;          // scale tiles
    uint64_t* full = reinterpret_cast<uint64_t*>(s_ring + static_cast<size_t>(S) * kSTile);
    uint64_t* empty = full + kTcMaxStages;
    uint64_t* acc_full = empty + kTcMaxStages;   // [2]
    uint64_t* acc_empty = acc_full + 2;          // [2]
    uint64_t* mma_done = acc_empty + 2;
    uint64_t* fold_ready = mma_done + 1;   // cluster fold: all N partial tiles written
    uint64_t* fold_freed = fold_ready + 1; // cluster fold: all N CTAs done reading mine
    uint64_t* cvt_full = fold_freed + 1;              // MX: [kSlots] converted tile ready (4 warps)
    uint64_t* cvt_empty = cvt_full + kCvtSlotsMax;    // MX: [kSlots] converted tile read by the MMAs
    // MX: [S] a stage's activation block landed (its codes and scales land on
    // full[s], so the converters need not wait for the dependency)
    uint64_t* full_x = cvt_empty + kCvtSlotsMax;
    // BS: full_x [S] a stage's split activations written (4 warps); x_full
    // [S] its bf16 activation block landed
    uint64_t* x_full = full_x + kTcMaxStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(x_full + kTcMaxStages);
    // cluster fold: this CTA's bf16 partial tile, [BN tokens][128 rows]
    uint16_t* part_buf = reinterpret_cast<uint16_t*>(
        (reinterpret_cast<uintptr_t>(tmem_slot + 4) + 127) & ~static_cast<uintptr_t>(127));
    __shared__ int abort_flag;
    __shared__ int fold_mine;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = (p.ks + KB - 1) / KB;
    // Cluster fold: cluster c takes tiles c, c + clusters, ...; its CTA of rank
    // r (in the cluster) computes rank r's partial of each.
    constexpr bool kCluster = MODE == kTcClusterFold;
    const int csize = kCluster ? p.n_ranks * p.splits : 1;
    const uint32_t crank = kCluster ? cluster_ctarank() : 0u;
    const int cid = static_cast<int>(blockIdx.x) / csize;
    const int n_clusters = static_cast<int>(gridDim.x) / csize;
    const int tiles = p.h_tiles * p.m_tiles;
    const int my_units =
        kCluster ? (tiles > cid ? (tiles - 1 - cid) / n_clusters + 1 : 0)
                       : (p.units > static_cast<int>(blockIdx.x)
                              ? (p.units - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                              : 0);
    // unit index -> (rank, h tile, m tile, split); token tile fastest
    auto unit_of = [&](int lu, int& r, int& ht, int& mt, int& sp) {
        if (kCluster) {   // CTA q of the cluster: rank q / SPLITS, K part q % SPLITS
            const int t = cid + lu * n_clusters;
            mt = t % p.m_tiles;
            ht = t / p.m_tiles;
            r = static_cast<int>(crank) / p.splits;
            sp = static_cast<int>(crank) - r * p.splits;
            return;
        }
        const int u = static_cast<int>(blockIdx.x) + lu * static_cast<int>(gridDim.x);
        mt = u % p.m_tiles;
        int t = u / p.m_tiles;
        sp = t % p.splits;
        t /= p.splits;
        ht = t % p.h_tiles;
        r = t / p.h_tiles;
    };
    // k-blocks [kb_lo, kb_hi) of split sp
    auto split_range = [&](int sp, int& kb_lo, int& kb_hi) {
        kb_lo = sp * nkb / p.splits;
        kb_hi = (sp + 1) * nkb / p.splits;
    };
    // quantised weights, one unit: the 4 epilogue warps also convert (8 converter warps)
    const bool cvt_helpers = MX && my_units == 1;
    // Store form, one unit: the epilogue stages the bf16 partial tile in the
    // stage ring (idle once the unit's last MMA is done) and stores whole
    // 16-byte vectors instead of one 2-byte value per token and row.
    const bool stage_tile = MODE == kTcStore && p.splits == 1 && my_units == 1 && p.tokens > 2 &&
                            static_cast<uint32_t>(BN) * kTcRows * 2 <= static_cast<uint32_t>(S) * (kWTile + kBTile);
    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_x[s], BS ? 4 : 1);       // BS: the four splitting warps
            mbar_init(&x_full[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(mma_done, 1);
        mbar_init(fold_ready, static_cast<uint32_t>(csize));
        mbar_init(fold_freed, static_cast<uint32_t>(csize));
        for (int j = 0; j < kSlots; ++j) {
            mbar_init(&cvt_full[j], 4);
            mbar_init(&cvt_empty[j], 1);
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (kCluster) cluster_sync_all();   // peers' barriers exist before any remote arrival
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    // Converters: a group of four warps, one per tensor-memory lane quarter;
    // thread `row` (its lane) widens row `row` of the staged code tiles in
    // issue order (k-block i into converted slot i % kSlots). With the helpers
    // (a CTA with one unit) the epilogue warps form a second group: group g
    // then takes the k-blocks with i % 2 == g.
    auto run_converters = [&](int group) {
        const int row = 32 * (warp & 3) + lane;
        if constexpr (MX) {
            const float two_g = FMT == kFmtNvfp4 ? ldexpf(1.0f, *p.nv_gexp) : 1.0f;
            int i = 0, s = 0, j = 0;
            uint32_t ph = 0, jph = 0;   // parities of full[s] and of slot j's use for k-block i
            bool ok = true;
            for (int lu = 0; lu < my_units && ok; ++lu) {
                int r, ht, mt, sp, kb_lo, kb_hi;
                unit_of(lu, r, ht, mt, sp);
                split_range(sp, kb_lo, kb_hi);
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!cvt_helpers || (i & 1) == group) {
                        ok = mbar_wait_bounded(&full[s], ph) && mbar_wait_bounded(&cvt_empty[j], jph ^ 1u);
                        if (!__all_sync(0xFFFFFFFFu, ok) ||
                            *reinterpret_cast<volatile int*>(&abort_flag) != 0) {
                            ok = false;
                            atomicExch(&abort_flag, 1);
                            break;
                        }
                        const uint8_t* srow = s_ring + static_cast<size_t>(s) * kSTile;
                        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * (warp & 3)) << 16) +
                                               kSlotCol0 + 32u * static_cast<uint32_t>(j);
                        if (FMT == kFmtMxfp8)
                            // row's two scales of this 64-column block in the chunk
                            mx_convert_row(a_ring + static_cast<size_t>(s) * kWTile + row * kTcKBlock,
                                           srow + (row & 31) * 16 + (row >> 5) * 4 + 2 * (kb & 1), taddr, row);
                        else
                            nv_convert_row(a_ring + static_cast<size_t>(s) * kWTile + row * (kTcKBlock / 2),
                                           srow + row * 4, two_g, taddr, row);
                        // the tensor-memory stores are done before the MMA may read them
                        tmem_st_wait();
                        tc_fence_before_sync();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&cvt_full[j]);
                    }
                    ++i;
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                    if (++j == kSlots) {
                        j = 0;
                        jph ^= 1u;
                    }
                }
            }
        }
    };

    // Block-scaled form: converter warp 6 + run splits run `run` (32 columns)
    // of every stage's 128 activation columns, for the (at most 8) tokens,
    // into the stage's B tile and its scale chunk: the bf16 block lands in
    // the stage's slot by TMA (x_full), each lane takes its 16 bytes into
    // registers, and once all four warps have theirs (one barrier, which also
    // makes the decision to give up common to them) the split overwrites it.
    auto run_x_split = [&]() {
        if constexpr (BS) {
            const int run = warp - 6;
            const int t = lane >> 2, part = lane & 3;
            // the scale chunks' bytes no split writes (rows 16.., columns 1..)
            // are never read by the MMA: zero them once all the same
            for (int s = 0; s < S; ++s)
                *reinterpret_cast<uint32_t*>(b_ring + static_cast<size_t>(s) * kBTile + kBsSfbOff +
                                             4 * (32 * run + lane)) = 0u;
            asm volatile("bar.sync 3, 128;" ::: "memory");   // zeroed before any split
            int s = 0;
            uint32_t ph = 0;   // parity of stage s's use
            bool ok = true;
            for (int lu = 0; lu < my_units && ok; ++lu) {
                int r, ht, mt, sp, kb_lo, kb_hi;
                unit_of(lu, r, ht, mt, sp);
                split_range(sp, kb_lo, kb_hi);
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    ok = mbar_wait_bounded(&x_full[s], ph);
                    uint8_t* bt = b_ring + static_cast<size_t>(s) * kBTile;
                    const uint4 v = *reinterpret_cast<const uint4*>(bt + t * (kMxChunkCols * 2) + (run * 32 + part * 8) * 2);
                    if (bar_sync_any(3, 128, !ok || *reinterpret_cast<volatile int*>(&abort_flag) != 0)) {
                        ok = false;
                        atomicExch(&abort_flag, 1);
                        break;
                    }
                    x_split_run(v, bt, t, run, part);
                    fence_proxy_async_smem();   // the tensor core reads them through the async proxy
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full_x[s]);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
        }
    };

    if (warp == 0) {
        // ---------------------------------------------------------- producer --
        if (lane == 0) {
            tma_prefetch_desc(&tmap_w);
            tma_prefetch_desc(&tmap_x);
            if (FMT == kFmtNvfp4) tma_prefetch_desc(&tmap_s);
            // bytes landing on full[s]: the whole stage, or (quantised) codes and
            // scales only, the activation block then counting on full_x[s]
            const uint32_t tx = (MX || BS) ? kWTile + kSTile : kWTile + kBTile + kSTile;
            // The weights of one k-block (and their scales) into stage st.
            // (NVFP4 code tiles hold two codes a byte: 32 bytes per 64-column block)
            constexpr int kWCols = FMT == kFmtNvfp4 ? kTcKBlock / 2 : KB;
            auto load_w = [&](int st, int kb_, int ht_, int r_) {
                tma_load_3d(a_ring + static_cast<size_t>(st) * kWTile, &tmap_w, &full[st],
                            kb_ * kWCols, ht_ * kTcRows, r_);
                if (FMT == kFmtNvfp4)   // 128 words from word ht*128
                    tma_load_3d(s_ring + static_cast<size_t>(st) * kSTile, &tmap_s, &full[st], ht_ * kTcRows,
                                kb_, r_);
                else if (FMT == kFmtMxfp8 || BS)   // the 512-byte chunk holding the block's scales
                    bulk_load(s_ring + static_cast<size_t>(st) * kSTile,
                              p.mx_scales + ((static_cast<int64_t>(r_) * p.h_tiles + ht_) * p.mx_kg +
                                             kb_ * KB / kMxChunkCols) * kMxChunk,
                              kMxChunk, &full[st]);
            };
            // Walk (unit, k-block) in issue order.
            struct Cursor {
                int lu, kb, kb_hi, r, ht, mt, sp;
            };
            auto enter_unit = [&](Cursor& c) {
                if (c.lu < my_units) {
                    unit_of(c.lu, c.r, c.ht, c.mt, c.sp);
                    split_range(c.sp, c.kb, c.kb_hi);
                }
            };
            auto advance = [&](Cursor& c) {
                if (++c.kb == c.kb_hi) {
                    ++c.lu;
                    enter_unit(c);
                }
            };
            Cursor cur{0, 0, 0, 0, 0, 0, 0};
            enter_unit(cur);
            int pre = 0;
            while (pre < S && cur.lu < my_units) {
                mbar_arrive_expect_tx(&full[pre], tx);
                load_w(pre, cur.kb, cur.ht, cur.r);
                ++pre;
                advance(cur);
            }
            // The activation rows of the first stages into L2 as well (the
            // first unit's tokens, the K range of those stages): coherent there
            // even if the previous kernel writes them, and close when the wait
            // returns.
            if (pre > 0) {
                Cursor c0{0, 0, 0, 0, 0, 0, 0};
                enter_unit(c0);
                const int64_t k_lo = static_cast<int64_t>(c0.kb) * KB;
                const int64_t k_hi = min(static_cast<int64_t>(min(c0.kb + pre, c0.kb_hi)) * KB,
                                         static_cast<int64_t>(p.ks));
                const int m_end = min(p.tokens, (c0.mt + 1) * BN);
                for (int m = c0.mt * BN; m < m_end; ++m)
                    bulk_prefetch_l2(p.x + m * p.k + static_cast<int64_t>(c0.r) * p.ks + k_lo,
                                     static_cast<uint32_t>((k_hi - k_lo) * 2));
            }
            pdl_wait();  // activations may be produced by the previous kernel
            if (BS) {   // the bf16 blocks the splitting warps take (own barrier)
                Cursor c0{0, 0, 0, 0, 0, 0, 0};
                enter_unit(c0);
                for (int i = 0; i < pre; ++i) {
                    mbar_arrive_expect_tx(&x_full[i], kBsXTile);
                    tma_load_3d(b_ring + static_cast<size_t>(i) * kBTile, &tmap_x, &x_full[i], c0.kb * KB, c0.r,
                                c0.mt * BN);
                    advance(c0);
                }
            } else {
                // the same first positions again, for their activation blocks
                Cursor c0{0, 0, 0, 0, 0, 0, 0};
                enter_unit(c0);
                for (int i = 0; i < pre; ++i) {
                    if (MX) mbar_arrive_expect_tx(&full_x[i], kBTile);
                    tma_load_3d(b_ring + static_cast<size_t>(i) * kBTile, &tmap_x, MX ? &full_x[i] : &full[i],
                                c0.kb * kTcKBlock, c0.r, c0.mt * BN);
                    advance(c0);
                }
            }
            int issued = pre;
            int s = pre % S;
            uint32_t phase = pre >= S ? 1u : 0u;   // parity of slot s's next fill
            while (cur.lu < my_units) {
                if (!mbar_wait_bounded(&empty[s], phase ^ 1u)) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                if (*reinterpret_cast<volatile int*>(&abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], tx);
                load_w(s, cur.kb, cur.ht, cur.r);
                if (BS) {
                    mbar_arrive_expect_tx(&x_full[s], kBsXTile);
                    tma_load_3d(b_ring + static_cast<size_t>(s) * kBTile, &tmap_x, &x_full[s], cur.kb * KB, cur.r,
                                cur.mt * BN);
                } else {
                    if (MX) mbar_arrive_expect_tx(&full_x[s], kBTile);
                    tma_load_3d(b_ring + static_cast<size_t>(s) * kBTile, &tmap_x, MX ? &full_x[s] : &full[s],
                                cur.kb * kTcKBlock, cur.r, cur.mt * BN);
                }
                ++issued;
                advance(cur);
                if (++s == S) {
                    s = 0;
                    phase ^= 1u;
                }
            }
            // Wait (bounded) for the copies still landing in this CTA's memory.
            // A wait that runs out has set the device error word; the launch's
            // results are then invalid and the context should be discarded.
            const int first = issued > S ? issued - S : 0;
            for (int i = first; i < issued; ++i)
                if (!mbar_wait_bounded(&full[i % S], static_cast<uint32_t>(i / S) & 1u) ||
                    (MX && !mbar_wait_bounded(&full_x[i % S], static_cast<uint32_t>(i / S) & 1u)) ||
                    (BS && !mbar_wait_bounded(&x_full[i % S], static_cast<uint32_t>(i / S) & 1u)))
                    break;
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issue --
        if (lane == 0) {
            int i = 0, s = 0, j = 0;
            uint32_t ph = 0, jph = 0;   // parities of full[s] and (MX) of converted slot j
            for (int lu = 0; lu < my_units; ++lu) {
                const int b = lu & 1;
                const uint32_t aph = static_cast<uint32_t>(lu >> 1) & 1u;
                if (!mbar_wait_bounded(&acc_empty[b], aph ^ 1u)) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d = tmem_base + static_cast<uint32_t>(b * BN);
                int r, ht, mt, sp, kb_lo, kb_hi;
                unit_of(lu, r, ht, mt, sp);
                split_range(sp, kb_lo, kb_hi);
                bool ok = true;
                for (int kb = kb_lo; kb < kb_hi; ++kb, ++i) {
                    // MX: the converters consumed the codes; the MMA needs the activations
                    // BS: the codes and scales, then the split activations
                    if (!mbar_wait_bounded(MX ? &full_x[s] : &full[s], ph) ||
                        (MX && !mbar_wait_bounded(&cvt_full[j], jph)) ||
                        (BS && !mbar_wait_bounded(&full_x[s], ph))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    uint64_t bd = smem_desc_k128(b_ring + static_cast<size_t>(s) * kBTile);
                    if (x_atom) bd &= ~(0x3FFFull << 32);   // stride between 8-row groups: 0
                    if constexpr (MX) {
                        // A: the converted tile in tensor memory, 8 columns per 16 of K
                        const uint32_t at = tmem_base + kSlotCol0 + 32u * static_cast<uint32_t>(j);
#pragma unroll
                        for (int kk = 0; kk < kTcKBlock / 16; ++kk)
                            umma_bf16_ta(d, at + 8u * kk, bd + 2ull * kk, kIdesc, (kb != kb_lo) || (kk != 0));
                    } else if constexpr (BS) {
                        // the stage's two scale chunks into its own tensor-memory
                        // columns (in issue order with the MMAs)
                        const uint32_t sfa = tmem_base + kSfaCol + 8u * static_cast<uint32_t>(s);
                        const uint32_t sfb = tmem_base + kSfbCol + 8u * static_cast<uint32_t>(s);
                        tmem_cp_32x128b_x4(sfa, smem_desc_rows16(s_ring + static_cast<size_t>(s) * kSTile));
                        tmem_cp_32x128b_x4(sfb, smem_desc_rows16(b_ring + static_cast<size_t>(s) * kBTile + kBsSfbOff));
                        const uint64_t ad = smem_desc_k128(a_ring + static_cast<size_t>(s) * kWTile);
                        // K = 32 a step (32 bytes of each row); step kk reads scale
                        // byte kk and goes to accumulator kk % kBsAccs
#pragma unroll
                        for (int kk = 0; kk < KB / 32; ++kk)
                            umma_mxf8(d + kBsBRows * static_cast<uint32_t>(kk % kBsAccs), ad + 2ull * kk, bd + 2ull * kk,
                                      idesc_mxf8_f32(kTcRows, kBsBRows, kk),
                                      (static_cast<uint32_t>(kk) << 30) | sfa, (static_cast<uint32_t>(kk) << 30) | sfb,
                                      (kb != kb_lo) || (kk >= kBsAccs));
                    } else {
                        const uint64_t ad = smem_desc_k128(a_ring + static_cast<size_t>(s) * kTcATile);
#pragma unroll
                        for (int kk = 0; kk < kTcKBlock / 16; ++kk)
                            umma_bf16(d, ad + 2ull * kk, bd + 2ull * kk, kIdesc, (kb != kb_lo) || (kk != 0));
                    }
                    umma_commit(&empty[s]);  // frees the stage when these MMAs finish
                    if (MX) umma_commit(&cvt_empty[j]);   // and the converted slot
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                    if (++j == kSlots) {
                        j = 0;
                        jph ^= 1u;
                    }
                }
                if (!ok) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                umma_commit(&acc_full[b]);
            }
            // Every MMA issued has finished before the tensor memory is freed.
            // A first wait that runs out (error word set) gets one more bound.
            umma_commit(mma_done);
            if (!mbar_wait_bounded(mma_done, 0)) (void)mbar_wait_bounded(mma_done, 0);
        }
    } else if ((MX || BS) && warp >= 6) {
        // ------------------------------------ converters (quantised weights) --
        if constexpr (BS) run_x_split();
        else run_converters(0);
    } else {
        // ---------------------------------------------------------- epilogue --
        // A CTA with one unit has nothing for these warps until its MMAs end:
        // they widen every other code tile meanwhile.
        if (MX && cvt_helpers) run_converters(1);
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        pdl_wait();  // the fold reads the residual and writes the output in stream order
        for (int lu = 0; lu < my_units; ++lu) {
            const int b = lu & 1;
            const uint32_t aph = static_cast<uint32_t>(lu >> 1) & 1u;
            int r, ht, mt, sp;
            unit_of(lu, r, ht, mt, sp);
            // Counter fold: this CTA's place among the parts of its tile, taken
            // before the accumulator is ready (the tags, not the tickets, say
            // which parts have landed: the ticket only elects the CTA that
            // folds), so the round trip overlaps the MMAs.
            unsigned int ticket = 0, tag = 0;
            if (MODE == kTcCounterFold) {
                if (threadIdx.x == 64) ticket = atomicAdd(p.counters + ht * p.m_tiles + mt, 1u);
                // this call's tag: the tile's folds so far + 1 (the previous
                // call's fold is complete: the epilogue waited for the dependency)
                tag = __ldcg(p.counters + p.h_tiles * p.m_tiles + ht * p.m_tiles + mt) + 1u;
            }
            bool ok = mbar_wait_bounded(&acc_full[b], aph);
            // cluster fold: the peers have read the previous unit's partial tile
            if (kCluster && lu > 0)
                ok = mbar_wait_cluster_bounded(fold_freed, static_cast<uint32_t>(lu - 1) & 1u) && ok;
            bool bad = !__all_sync(0xFFFFFFFFu, ok);
            if (bad) atomicExch(&abort_flag, 1);
            bad = bad || *reinterpret_cast<volatile int*>(&abort_flag) != 0;
            // The four epilogue warps leave together: one answer for all of them.
            if (bar_sync_any(2, 128, bad)) break;
            tc_fence_after_sync();
            const int h = ht * kTcRows + q * 32 + lane;
            const int m0 = mt * BN;
            const size_t plane = static_cast<size_t>(p.tokens) * p.hidden;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t v[32];
                tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(b * BN + c0),
                               v);
                if constexpr (BS) {   // token i's two activation terms in each accumulator
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float f = __fadd_rn(__uint_as_float(v[i]), __uint_as_float(v[i + 8]));
#pragma unroll
                        for (int a = 1; a < kBsAccs; ++a)
                            f = __fadd_rn(f, __fadd_rn(__uint_as_float(v[16 * a + i]), __uint_as_float(v[16 * a + i + 8])));
                        v[i] = __float_as_uint(f);
                    }
                }
                if (kCluster) {
                    // [token][row] in shared memory, the tile's tokens only: lanes
                    // write 32 consecutive rows; bf16 partials, or fp32 part sums
                    const int t_tile = min(BN, p.tokens - m0);
                    const int row = q * 32 + lane;
                    if (p.splits == 1) {
                        uint16_t* dst = part_buf + static_cast<size_t>(c0) * kTcRows + row;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (c0 + i < t_tile) dst[i * kTcRows] = f32_to_bf16_rne(__uint_as_float(v[i]));
                    } else {
                        float* dst = reinterpret_cast<float*>(part_buf) + static_cast<size_t>(c0) * kTcRows + row;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (c0 + i < t_tile) dst[i * kTcRows] = __uint_as_float(v[i]);
                    }
                } else if (stage_tile) {
                    // [token][128 rows] in the (now idle) stage ring: lanes write
                    // 32 consecutive rows of one token
                    uint16_t* dst = reinterpret_cast<uint16_t*>(a_ring) + static_cast<size_t>(c0) * kTcRows +
                                    q * 32 + lane;
#pragma unroll
                    for (int i = 0; i < 32; ++i) dst[i * kTcRows] = f32_to_bf16_rne(__uint_as_float(v[i]));
                } else if (MODE == kTcCounterFold) {
                    if (h < p.hidden) {
                        if (p.splits == 1) {   // (bf16, tag) words [N][M][H]
                            uint64_t* dst = reinterpret_cast<uint64_t*>(p.partials_f32) + static_cast<size_t>(r) * plane + h;
#pragma unroll
                            for (int i = 0; i < 2; ++i) {   // at most two tokens
                                const int m = m0 + c0 + i;
                                if (m < p.tokens)
                                    dst[static_cast<size_t>(m) * p.hidden] =
                                        (static_cast<uint64_t>(tag) << 32) | f32_to_bf16_rne(__uint_as_float(v[i]));
                            }
                        } else {               // (fp32, tag) words [splits][N][M][H]
                            uint64_t* dst = reinterpret_cast<uint64_t*>(p.partials_f32) +
                                            (static_cast<size_t>(sp) * p.n_ranks + r) * plane + h;
#pragma unroll
                            for (int i = 0; i < 2; ++i) {
                                const int m = m0 + c0 + i;
                                if (m < p.tokens)
                                    dst[static_cast<size_t>(m) * p.hidden] =
                                        (static_cast<uint64_t>(tag) << 32) | v[i];
                            }
                        }
                    }
                } else if (h < p.hidden) {
                    if (p.splits == 1) {
                        uint16_t* dst = p.partials + static_cast<size_t>(r) * plane + h;

#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int m = m0 + c0 + i;
                            if (m < p.tokens)
                                dst[static_cast<size_t>(m) * p.hidden] =
                                    f32_to_bf16_rne(__uint_as_float(v[i]));
                        }
                    } else {
                        float* dst = p.partials_f32 +
                                     (static_cast<size_t>(sp) * p.n_ranks + r) * plane + h;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int m = m0 + c0 + i;
                            if (m < p.tokens) dst[static_cast<size_t>(m) * p.hidden] = __uint_as_float(v[i]);
                        }
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
            if (stage_tile) {
                // the tile's token rows, 16 bytes a store
                asm volatile("bar.sync 2, 128;" ::: "memory");
                const int t_tile = min(BN, p.tokens - m0);
                const int et = static_cast<int>(threadIdx.x) - 64;
                const uint8_t* tile = a_ring;
                for (int idx = et; idx < t_tile * (kTcRows / 8); idx += 128) {
                    const int m = idx / (kTcRows / 8);
                    const int hh = ht * kTcRows + (idx % (kTcRows / 8)) * 8;
                    if (hh < p.hidden)
                        st_global_v4(p.partials + static_cast<size_t>(r) * plane +
                                         static_cast<size_t>(m0 + m) * p.hidden + hh,
                                     *reinterpret_cast<const uint4*>(tile + static_cast<size_t>(m) * kTcRows * 2 +
                                                                     (idx % (kTcRows / 8)) * 16));
                }
            }
            if (kCluster) {
                // Every CTA of the cluster has its partial tile in shared memory
                // once each has arrived on everyone's fold_ready.
                const uint4 res0 = cluster_fold_first_residual(p, crank, csize, ht, m0, BN,
                                                               static_cast<int>(threadIdx.x) - 64);
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (warp == 2 && lane == 0) {
                    fence_acq_rel_cluster();
                    for (int pr = 0; pr < csize; ++pr)
                        mbar_arrive_cluster(mapa_shared(fold_ready, static_cast<uint32_t>(pr)));
                }
                if (!mbar_wait_cluster_bounded(fold_ready, static_cast<uint32_t>(lu) & 1u))
                    atomicExch(&abort_flag, 1);
                else
                    // 1 .. 4 K parts, N * parts <= 8 (the host launches no other cluster fold)
                    if (p.splits == 1) cluster_fold_tile<1>(p, part_buf, crank, csize, ht, m0, BN, threadIdx.x - 64, res0);
                    else if (p.splits == 2) cluster_fold_tile<2>(p, part_buf, crank, csize, ht, m0, BN, threadIdx.x - 64, res0);
                    else if (p.splits == 3) cluster_fold_tile<3>(p, part_buf, crank, csize, ht, m0, BN, threadIdx.x - 64, res0);
                    else cluster_fold_tile<4>(p, part_buf, crank, csize, ht, m0, BN, threadIdx.x - 64, res0);
                // All reads of the peers' tiles are done: free them for the next unit.
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (warp == 2 && lane == 0) {
                    fence_acq_rel_cluster();
                    for (int pr = 0; pr < csize; ++pr)
                        mbar_arrive_cluster(mapa_shared(fold_freed, static_cast<uint32_t>(pr)));
                }
            }
            if (MODE == kTcCounterFold) {
                // The CTA holding the last ticket of this (H tile, token tile)
                // folds it: ring order, residual add. Its parts are read by tag,
                // so the other CTAs leave as soon as their parts are stored.
                uint16_t res[2] = {0, 0};   // this thread's residual, loaded meanwhile
                if (h < p.hidden)
                    for (int m = m0, i = 0; m < p.tokens && i < 2; ++m, ++i)
                        res[i] = p.residual[static_cast<size_t>(m) * p.hidden + h];
                unsigned int* tickets = p.counters + ht * p.m_tiles + mt;
                unsigned int* folds = tickets + p.h_tiles * p.m_tiles;
                if (threadIdx.x == 64) fold_mine = ticket == static_cast<unsigned int>(p.n_ranks * p.splits - 1);
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (fold_mine) {
                    bool ok = true;
                    if (h < p.hidden) {
                        const int c = h / p.hc;
                        // at most two tokens here (m_tiles == 1, tokens <= 2); this
                        // thread's own part it stored itself
                        for (int m = m0, i = 0; m < p.tokens && i < 2; ++m, ++i) {
                            const size_t off = static_cast<size_t>(m) * p.hidden + h;
                            uint16_t sum = 0;
                            ok = fold_tagged(p, plane, off, c, tag, sum) && ok;
                            p.out[off] = bf16_add(res[i], sum);
                        }
                    }
                    if (!ok) atomicExch(&abort_flag, 1);
                    if (threadIdx.x == 64) {   // for the next call
                        *folds = tag;
                        *tickets = 0u;
                    }
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    // Cluster fold: no CTA leaves while a peer may still read its shared
    // memory or arrive on its barriers (every wait above is bounded, so every
    // thread of the cluster gets here).
    if (kCluster) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace tpr
