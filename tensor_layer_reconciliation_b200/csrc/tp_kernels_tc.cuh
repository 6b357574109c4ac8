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
// Folding (S2-S4): for one or two tokens the CTA that stores the last of
// the N * SPLITS parts of an (H tile, token tile) -- found with a per-tile
// counter in the workspace -- folds that tile itself, each epilogue thread
// one row h, so a call is one kernel and the next call's kernel waits on one
// grid instead of two. For more tokens the fold stays a kernel of its own:
// there the CTA that completes a tile would read N * SPLITS * 128 * BN
// values behind its next accumulator (measured slower from 32 tokens up),
// while a separate kernel spreads that work over the whole GPU.
// Accumulation order inside the tensor core is the hardware's; the partial
// is the fp32 sum rounded once to bf16, like the oracle's, but only equal to
// it where the two fp32 sums round to the same bf16 value.
#pragma once

#include "tp_tcgen05.cuh"

namespace tpr {

constexpr int kTcRows = 128;               // MMA M: weight rows per tile
constexpr int kTcKBlock = 64;              // bf16 columns per staged block
constexpr int kTcMaxStages = 8;
constexpr int kTcThreads = 192;            // producer, MMA and 4 epilogue warps
constexpr uint32_t kTcATile = kTcRows * kTcKBlock * 2;  // 16 KB

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
    uint16_t* partials;     // [N][M][H] bf16 (splits == 1)
    float* partials_f32;    // [splits][N][M][H] fp32 sums of each k part (splits > 1)
    // In-kernel fold (S2-S4), few tokens only; fold == 0 leaves it to the ring kernel.
    int fold;
    int hc;                       // H / N, the chunk each rank owns in the ring
    unsigned int* counters;       // [h_tiles][m_tiles] parts stored so far; zero between calls
    const uint16_t* residual;     // [M][H]
    uint16_t* out;                // [M][H]
};

template <int BN>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_partial_kernel(const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_x, const TcParams p) {
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M = 128");
    constexpr uint32_t kBTile = BN * kTcKBlock * 2;
    constexpr uint32_t kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;  // two accumulators
    constexpr uint32_t kIdesc = idesc_bf16_f32(kTcRows, BN);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int S = p.stages;
    uint8_t* a_ring = smem;
    uint8_t* b_ring = a_ring + static_cast<size_t>(S) * kTcATile;
    uint64_t* full = reinterpret_cast<uint64_t*>(b_ring + static_cast<size_t>(S) * kBTile);
    uint64_t* empty = full + kTcMaxStages;
    uint64_t* acc_full = empty + kTcMaxStages;   // [2]
    uint64_t* acc_empty = acc_full + 2;          // [2]
    uint64_t* mma_done = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    __shared__ int abort_flag;
    __shared__ int fold_mine;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = (p.ks + kTcKBlock - 1) / kTcKBlock;
    const int my_units = p.units > static_cast<int>(blockIdx.x)
                             ? (p.units - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                             : 0;
    // unit index -> (rank, h tile, m tile, split); token tile fastest
    auto unit_of = [&](int lu, int& r, int& ht, int& mt, int& sp) {
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
    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------------------------------------------------- producer --
        if (lane == 0) {
            tma_prefetch_desc(&tmap_w);
            tma_prefetch_desc(&tmap_x);
            const uint32_t tx = kTcATile + kBTile;
            // Walk (unit, k-block) in issue order.
            int lu = 0, kb = 0, kb_hi = 0, r = 0, ht = 0, mt = 0, sp = 0;
            auto enter_unit = [&]() {
                if (lu < my_units) {
                    unit_of(lu, r, ht, mt, sp);
                    split_range(sp, kb, kb_hi);
                }
            };
            auto advance = [&]() {
                if (++kb == kb_hi) {
                    ++lu;
                    enter_unit();
                }
            };
            enter_unit();
            int pre_r[kTcMaxStages], pre_mt[kTcMaxStages], pre_kb[kTcMaxStages];
            int pre = 0;
            while (pre < S && lu < my_units) {
                mbar_arrive_expect_tx(&full[pre], tx);
                tma_load_3d(a_ring + static_cast<size_t>(pre) * kTcATile, &tmap_w, &full[pre],
                            kb * kTcKBlock, ht * kTcRows, r);
                pre_r[pre] = r;
                pre_mt[pre] = mt;
                pre_kb[pre] = kb;
                ++pre;
                advance();
            }
            pdl_wait();  // activations may be produced by the previous kernel
            for (int i = 0; i < pre; ++i)
                tma_load_3d(b_ring + static_cast<size_t>(i) * kBTile, &tmap_x, &full[i],
                            pre_kb[i] * kTcKBlock, pre_r[i], pre_mt[i] * BN);
            int issued = pre;
            int s = pre % S;
            uint32_t phase = pre >= S ? 1u : 0u;   // parity of slot s's next fill
            while (lu < my_units) {
                if (!mbar_wait_bounded(&empty[s], phase ^ 1u)) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                if (*reinterpret_cast<volatile int*>(&abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], tx);
                tma_load_3d(a_ring + static_cast<size_t>(s) * kTcATile, &tmap_w, &full[s],
                            kb * kTcKBlock, ht * kTcRows, r);
                tma_load_3d(b_ring + static_cast<size_t>(s) * kBTile, &tmap_x, &full[s],
                            kb * kTcKBlock, r, mt * BN);
                ++issued;
                advance();
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
                if (!mbar_wait_bounded(&full[i % S], static_cast<uint32_t>(i / S) & 1u)) break;
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issue --
        if (lane == 0) {
            int i = 0;
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
                    const int s = i % S;
                    if (!mbar_wait_bounded(&full[s], static_cast<uint32_t>(i / S) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t ad = smem_desc_k128(a_ring + static_cast<size_t>(s) * kTcATile);
                    const uint64_t bd = smem_desc_k128(b_ring + static_cast<size_t>(s) * kBTile);
#pragma unroll
                    for (int kk = 0; kk < kTcKBlock / 16; ++kk)
                        umma_bf16(d, ad + 2ull * kk, bd + 2ull * kk, kIdesc,
                                  (kb != kb_lo) || (kk != 0));
                    umma_commit(&empty[s]);  // frees the stage when these MMAs finish
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
    } else {
        // ---------------------------------------------------------- epilogue --
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        pdl_wait();  // the fold reads the residual and writes the output in stream order
        for (int lu = 0; lu < my_units; ++lu) {
            const int b = lu & 1;
            const uint32_t aph = static_cast<uint32_t>(lu >> 1) & 1u;
            bool bad = !__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&acc_full[b], aph));
            if (bad) atomicExch(&abort_flag, 1);
            bad = bad || *reinterpret_cast<volatile int*>(&abort_flag) != 0;
            // The four epilogue warps leave together: one answer for all of them.
            if (bar_sync_any(2, 128, bad)) break;
            tc_fence_after_sync();
            int r, ht, mt, sp;
            unit_of(lu, r, ht, mt, sp);
            const int h = ht * kTcRows + q * 32 + lane;
            const int m0 = mt * BN;
            const size_t plane = static_cast<size_t>(p.tokens) * p.hidden;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t v[32];
                tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(b * BN + c0),
                               v);
                if (h < p.hidden) {
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
            if (p.fold) {
                // The CTA that stores the last of the N * SPLITS parts of this
                // (H tile, token tile) folds the tile: ring order, residual add.
                // Residual of this thread's row, loaded while the count goes round.
                uint16_t res[2] = {0, 0};
                if (h < p.hidden)
                    for (int m = m0, i = 0; m < p.tokens && i < 2; ++m, ++i)
                        res[i] = p.residual[static_cast<size_t>(m) * p.hidden + h];
                __threadfence();  // this thread's parts are visible before the count
                asm volatile("bar.sync 2, 128;" ::: "memory");
                unsigned int* cnt = p.counters + ht * p.m_tiles + mt;
                if (warp == 2 && lane == 0)
                    fold_mine = atomicAdd(cnt, 1u) == static_cast<unsigned int>(p.n_ranks * p.splits - 1);
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (fold_mine) {
                    __threadfence();  // the other CTAs' parts, counted above, are read after it
                    if (h < p.hidden) {
                        const int c = h / p.hc;
                        // at most two tokens here (m_tiles == 1, tokens <= 2)
                        for (int m = m0, i = 0; m < p.tokens && i < 2; ++m, ++i) {
                            const size_t off = static_cast<size_t>(m) * p.hidden + h;
                            const uint16_t sum =
                                p.splits == 1
                                    ? ring_fold_bf16<true>(p.partials, p.n_ranks, plane, off, c)
                                : p.n_ranks * p.splits <= 16
                                    ? ring_fold_f32_parts16<true>(p.partials_f32, p.splits,
                                                                  p.n_ranks, plane, off, c)
                                    : ring_fold_f32_parts_by_rank<true>(p.partials_f32, p.splits,
                                                                        p.n_ranks, plane, off, c);
                            p.out[off] = bf16_add(res[i], sum);
                        }
                    }
                    if (warp == 2 && lane == 0) atomicExch(cnt, 0u);  // zero for the next call
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace tpr
