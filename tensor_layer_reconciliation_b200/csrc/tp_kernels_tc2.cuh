// Partial kernel on CTA pairs (S1) for prefill: the dense contraction of a
// long prompt, run as 2-SM tensor-core MMAs.
//
// "Interconnects e clusters", 01 Conceito: each rank computes a partial
// result over its slice of the weight matrix; prefill processes every
// position of the prompt at once, a dense contraction.
//
// Work unit = (rank r, 256 rows of H, 256 tokens), computed by a cluster of
// two CTAs on two SMs as D = A * B^T with one tcgen05.mma.cta_group::2 per
// 16 columns of K: A = the 256 x 64 weight block (CTA c of the pair holds
// rows 128c .. 128c+127), B = the 256 x 64 token block (CTA c holds tokens
// 128c .. 128c+127), both staged by TMA with the 128-byte swizzle at the
// same shared-memory offsets in the two CTAs; each CTA's tensor memory
// receives its 128 rows of D for all 256 tokens. Compared with one CTA per
// 128 x 256 tile, every SM stages half the token block, so a stage is 32 KB
// instead of 48 KB: fewer bytes through L2 and through shared memory per
// multiply, and more stages in flight.
//
// Roles (both CTAs run the same code; "leader" = cluster rank 0):
//   warp 0     TMA producer of this CTA's halves. The loads count their
//              bytes on the leader's "full" barrier of the stage, which the
//              leader's producer arms with the bytes of both CTAs. A stage
//              is reloaded after this CTA's own "empty" barrier fired (the
//              leader's MMA completion arrives on both CTAs' barriers).
//   warp 1     allocates the pair's tensor memory (both CTAs, same warp);
//              in the leader one thread issues the MMAs and commits stage
//              and accumulator completions to both CTAs.
//   warps 2-5  epilogue of this CTA's 128 rows: tcgen05.ld, one rounding to
//              bf16 per partial, stores to [N][M][H]; then an arrival on the
//              leader's "accumulator empty" barrier (8 arrivals: 4 warps x 2
//              CTAs) so the leader may reuse the accumulator. With `fold`,
//              the CTA that stores the last of the N ranks' partials of its
//              128 rows x 256 tokens (a counter per half tile) folds them
//              there (S2-S4: ring order, residual, output) while the leader
//              already multiplies the next unit.
// Units run token tile fastest (CTAs working at the same time share weight
// tiles through L2). Two accumulators of 256 fp32 columns fill the 512
// tensor-memory columns, so the epilogue of one unit overlaps the next
// unit's MMAs. Every wait is bounded; both CTAs meet at two cluster barriers
// (after set-up, before the tensor memory is freed) on every path.
#pragma once

#include "tp_kernels_tc.cuh"

namespace tpr {

constexpr int kTc2Tokens = 256;                      // MMA N: tokens per unit
constexpr int kTc2HalfTokens = kTc2Tokens / 2;       // tokens staged per CTA
constexpr uint32_t kTc2BTile = kTc2HalfTokens * kTcKBlock * 2;  // 16 KB
constexpr uint32_t kTc2Stage = kTcATile + kTc2BTile;            // 32 KB per CTA
constexpr int kTc2MaxStages = 8;

struct Tc2Params {
    int n_ranks;   // N
    int ks;        // K / N
    int hidden;    // H
    int tokens;    // M
    int h_pairs;   // ceil(H / 256)
    int m_tiles;   // ceil(M / 256)
    int units;     // N * h_pairs * m_tiles
    int stages;    // 2 .. kTc2MaxStages
    uint16_t* partials;  // [N][M][H] bf16
    int fold;                     // fold in the epilogue (else a ring kernel follows)
    int hc;                       // H / N
    unsigned int* counters;       // [h_pairs * m_tiles][2] parts stored per half tile; zero between calls
    const uint16_t* residual;     // [M][H]
    uint16_t* out;                // [M][H]
};

// S2-S4 of one half tile (128 rows from h0, tokens m0 .. m1-1) from the
// staged partials, by the 128 epilogue threads (et): 16-byte vectors of 8
// rows, V of them in flight per thread, each folded in ring order from its
// chunk's owner (all N <= NR loads before the first add), the residual added.
template <int V, int NR>
__device__ __forceinline__ void tc2_fold_half(const Tc2Params& p, int h0, int m0, int m1, int et) {
    const size_t plane = static_cast<size_t>(p.tokens) * p.hidden;
    const int total = (m1 - m0) * (kTcRows / 8);
    for (int v0 = et; v0 < total; v0 += V * 128) {
        uint4 pv[V][NR], rv[V];
        size_t off[V];
        int c[V];
        bool ok[V];
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const int v = v0 + j * 128;
            const int m = m0 + v / (kTcRows / 8);
            const int h = h0 + (v % (kTcRows / 8)) * 8;
            ok[j] = v < total && h < p.hidden;
            off[j] = static_cast<size_t>(m) * p.hidden + h;
            c[j] = h / p.hc;
            if (ok[j]) {
#pragma unroll
                for (int i = 0; i < NR; ++i)
                    if (i < p.n_ranks) {
                        int rr = c[j] + i;
                        if (rr >= p.n_ranks) rr -= p.n_ranks;
                        pv[j][i] = __ldcg(reinterpret_cast<const uint4*>(p.partials + rr * plane + off[j]));
                    }
                rv[j] = ld_global_nc_v4(p.residual + off[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < V; ++j) {
            if (!ok[j]) continue;
            uint4 sum = pv[j][0];
#pragma unroll
            for (int i = 1; i < NR; ++i)
                if (i < p.n_ranks) sum = bf16x8_add_tc(sum, pv[j][i]);
            st_global_v4(p.out + off[j], bf16x8_add_tc(rv[j], sum));
        }
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
    tc2_partial_kernel(const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_x, const Tc2Params p) {
    constexpr uint32_t kTmemCols = 2 * kTc2Tokens;   // two accumulators: 512 columns
    constexpr uint32_t kIdesc = idesc_bf16_f32(2 * kTcRows, kTc2Tokens);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int S = p.stages;
    uint8_t* a_ring = smem;
    uint8_t* b_ring = a_ring + static_cast<size_t>(S) * kTcATile;
    uint64_t* full = reinterpret_cast<uint64_t*>(b_ring + static_cast<size_t>(S) * kTc2BTile);
    uint64_t* empty = full + kTc2MaxStages;
    uint64_t* acc_full = empty + kTc2MaxStages;   // [2]
    uint64_t* acc_empty = acc_full + 2;           // [2], used in the leader
    uint64_t* mma_done = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    __shared__ int abort_flag;
    __shared__ int fold_mine;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();          // 0: leader, 1: peer
    const bool leader = rank == 0;
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int n_pairs = static_cast<int>(gridDim.x >> 1);
    const int nkb = (p.ks + kTcKBlock - 1) / kTcKBlock;
    const int my_units = p.units > pair ? (p.units - 1 - pair) / n_pairs + 1 : 0;
    // unit index -> (rank r, pair of H tiles hp, token tile mt); token tile fastest
    auto unit_of = [&](int lu, int& r, int& hp, int& mt) {
        const int u = pair + lu * n_pairs;
        mt = u % p.m_tiles;
        const int t = u / p.m_tiles;
        hp = t % p.h_pairs;
        r = t / p.h_pairs;
    };

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync_all();   // both CTAs' barriers exist before any cross-CTA arrival
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------------------------------------------------- producer --
        if (lane == 0) {
            tma_prefetch_desc(&tmap_w);
            tma_prefetch_desc(&tmap_x);
            const uint32_t tx_pair = 2 * kTc2Stage;   // both CTAs' bytes of a stage
            int lu = 0, kb = 0, r = 0, hp = 0, mt = 0;
            if (my_units > 0) unit_of(0, r, hp, mt);
            auto advance = [&]() {
                if (++kb == nkb) {
                    kb = 0;
                    if (++lu < my_units) unit_of(lu, r, hp, mt);
                }
            };
            const int row0 = static_cast<int>(rank) * kTcRows;
            const int tok0 = static_cast<int>(rank) * kTc2HalfTokens;
            int pre = 0;
            while (pre < S && lu < my_units) {
                if (leader) mbar_arrive_expect_tx(&full[pre], tx_pair);
                tma_load_3d_pair(a_ring + static_cast<size_t>(pre) * kTcATile, &tmap_w,
                                 pair_leader_addr(&full[pre]), kb * kTcKBlock,
                                 hp * 2 * kTcRows + row0, r);
                ++pre;
                advance();
            }
            pdl_wait();  // activations may be produced by the previous kernel
            {
                // the same first positions again, for their activation blocks
                int r0 = 0, hp0 = 0, mt0 = 0, lu0 = 0, kb0 = 0;
                unit_of(0, r0, hp0, mt0);
                for (int i = 0; i < pre; ++i) {
                    tma_load_3d_pair(b_ring + static_cast<size_t>(i) * kTc2BTile, &tmap_x,
                                     pair_leader_addr(&full[i]), kb0 * kTcKBlock, r0,
                                     mt0 * kTc2Tokens + tok0);
                    if (++kb0 == nkb) {
                        kb0 = 0;
                        if (++lu0 < my_units) unit_of(lu0, r0, hp0, mt0);
                    }
                }
            }
            int issued = pre;
            int s = pre % S;
            uint32_t phase = pre >= S ? 1u : 0u;
            while (lu < my_units) {
                if (!mbar_wait_bounded(&empty[s], phase ^ 1u)) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                if (*reinterpret_cast<volatile int*>(&abort_flag)) break;
                if (leader) mbar_arrive_expect_tx(&full[s], tx_pair);
                tma_load_3d_pair(a_ring + static_cast<size_t>(s) * kTcATile, &tmap_w,
                                 pair_leader_addr(&full[s]), kb * kTcKBlock,
                                 hp * 2 * kTcRows + row0, r);
                tma_load_3d_pair(b_ring + static_cast<size_t>(s) * kTc2BTile, &tmap_x,
                                 pair_leader_addr(&full[s]), kb * kTcKBlock, r,
                                 mt * kTc2Tokens + tok0);
                ++issued;
                advance();
                if (++s == S) {
                    s = 0;
                    phase ^= 1u;
                }
            }
            // The leader's barriers count both CTAs' copies: the leader waits
            // for the last stages to land before the pair may leave.
            if (leader) {
                const int first = issued > S ? issued - S : 0;
                for (int i = first; i < issued; ++i)
                    if (!mbar_wait_bounded(&full[i % S], static_cast<uint32_t>(i / S) & 1u)) break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issue (leader) --
        if (leader && lane == 0) {
            int i = 0;
            bool issued_any = false;
            for (int lu = 0; lu < my_units; ++lu) {
                const int b = lu & 1;
                const uint32_t aph = static_cast<uint32_t>(lu >> 1) & 1u;
                if (!mbar_wait_bounded(&acc_empty[b], aph ^ 1u)) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d = tmem_base + static_cast<uint32_t>(b * kTc2Tokens);
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb, ++i) {
                    const int s = i % S;
                    if (!mbar_wait_bounded(&full[s], static_cast<uint32_t>(i / S) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t ad = smem_desc_k128(a_ring + static_cast<size_t>(s) * kTcATile);
                    const uint64_t bd = smem_desc_k128(b_ring + static_cast<size_t>(s) * kTc2BTile);
#pragma unroll
                    for (int kk = 0; kk < kTcKBlock / 16; ++kk)
                        umma_bf16_pair(d, ad + 2ull * kk, bd + 2ull * kk, kIdesc, (kb != 0) || (kk != 0));
                    umma_commit_pair_mc(&empty[s], 0x3);   // frees the stage in both CTAs
                    issued_any = true;
                }
                if (!ok) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                umma_commit_pair_mc(&acc_full[b], 0x3);
            }
            // Every MMA issued has finished before the tensor memory is freed.
            if (issued_any) {
                umma_commit_pair_mc(mma_done, 0x1);
                if (!mbar_wait_bounded(mma_done, 0)) (void)mbar_wait_bounded(mma_done, 0);
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue --
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        pdl_wait();  // the partial buffer is read by the previous call's ring kernel
        const uint32_t leader_acc_empty[2] = {mapa_shared(&acc_empty[0], 0),
                                              mapa_shared(&acc_empty[1], 0)};
        for (int lu = 0; lu < my_units; ++lu) {
            const int b = lu & 1;
            const uint32_t aph = static_cast<uint32_t>(lu >> 1) & 1u;
            bool bad = !__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&acc_full[b], aph));
            if (bad) atomicExch(&abort_flag, 1);
            bad = bad || *reinterpret_cast<volatile int*>(&abort_flag) != 0;
            if (bar_sync_any(2, 128, bad)) break;
            tc_fence_after_sync();
            int r, hp, mt;
            unit_of(lu, r, hp, mt);
            const int h = hp * 2 * kTcRows + static_cast<int>(rank) * kTcRows + q * 32 + lane;
            const int m0 = mt * kTc2Tokens;
            const size_t plane = static_cast<size_t>(p.tokens) * p.hidden;
#pragma unroll 1
            for (int c0 = 0; c0 < kTc2Tokens; c0 += 32) {
                uint32_t v[32];
                tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(b * kTc2Tokens + c0),
                               v);
                if (h < p.hidden) {
                    uint16_t* dst = p.partials + static_cast<size_t>(r) * plane + h;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = m0 + c0 + j;
                        if (m < p.tokens)
                            dst[static_cast<size_t>(m) * p.hidden] = f32_to_bf16_rne(__uint_as_float(v[j]));
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_acc_empty[b]);
            if (p.fold) {
                // This CTA's 128 rows of the tile are stored: count them; the
                // CTA storing the N-th rank's folds those rows of the tile.
                unsigned int* cnt = p.counters + (hp * p.m_tiles + mt) * 2 + static_cast<int>(rank);
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (threadIdx.x == 64) {
                    __threadfence();   // this CTA's stores (ordered by the barrier) before the count
                    const unsigned int prev = atomicAdd(cnt, 1u);
                    fold_mine = prev == static_cast<unsigned int>(p.n_ranks - 1);
                    if (fold_mine) __threadfence();   // the other ranks' stores, counted, before the loads
                }
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (fold_mine) {
                    const int h0 = hp * 2 * kTcRows + static_cast<int>(rank) * kTcRows;
                    const int m1 = min(p.tokens, m0 + kTc2Tokens);
                    const int et = static_cast<int>(threadIdx.x) - 64;
                    if (p.n_ranks <= 4) tc2_fold_half<4, 4>(p, h0, m0, m1, et);
                    else tc2_fold_half<2, kMaxRanks>(p, h0, m0, m1, et);
                    if (threadIdx.x == 64) *cnt = 0u;   // zero for the next call
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    cluster_sync_all();   // the leader's MMAs are done and both epilogues have read
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

}  // namespace tpr
