// Partial kernel on CUDA cores with the k-ascending fp32 FMA chain (S1),
// optionally fused with the ring fold and the residual add (S2-S4).
//
// "Interconnects e clusters", 01 Conceito: each weight matrix is split
// between ranks and each rank computes a partial result over its slice; the
// slices are summed (all-reduce) before the residual stream continues.
//
// Work decomposition. A CTA owns BH output rows h0..h0+BH-1 for ALL N ranks
// and MT tokens m0..m0+MT-1, so every partial an output element needs is
// produced inside the CTA and the ring fold needs no second kernel.
// Consumer thread t = r*BH + j runs the MT fp32 accumulation chains of
// partial (rank r, row h0+j), one FMA per element in ascending k, so each
// partial is exactly the k-ascending fp32 sum rounded once to bf16.
//
// Memory path. One producer thread streams 64-column k-blocks with 3-D TMA
// bulk-tensor loads into a STAGES-deep shared-memory ring:
//   W box {64 k, BH rows, N ranks} of w_packed [N][H][Ks], 128-byte swizzled
//   x box {64 k, N ranks, MT tokens} of x viewed as [M][N][Ks]
// Each stage has a "full" mbarrier (TMA transaction bytes) and an "empty"
// mbarrier (one arrive per consumer warp). Weight loads for the first STAGES
// blocks are issued before griddepcontrol.wait, so with programmatic
// dependent launch they overlap the previous kernel's tail; activations,
// the residual and the outputs are touched only after it.
//
// Shared-memory banks: a consumer reads 16-byte chunk c of its own 128-byte
// row; with the 128-byte swizzle the physical chunk is c ^ (row & 7), so the
// eight lanes of each quarter-warp hit eight different chunks.
#pragma once

#include "tp_common.cuh"

namespace tpr {

constexpr int kMaxStages = 16;
constexpr int kKBlock = 64;  // bf16 columns per TMA box row (128 bytes)
constexpr int kMaxExactChains = 512;                 // N * BH per CTA
constexpr int kMaxExactThreads = kMaxExactChains + 32;  // + the producer warp

struct ExactParams {
    int n_ranks;     // N
    int bh;          // output rows per CTA
    int ks;          // K / N
    int hidden;      // H
    int hc;          // H / N
    int tokens;      // M
    int stages;      // pipeline depth, 2..kMaxStages
    int fused;       // 1: fold + residual in-kernel; 0: write partials
    uint32_t w_stage_bytes;  // stride of the W ring (multiple of 1024)
    uint32_t x_stage_bytes;  // stride of the x ring (multiple of 128)
    uint32_t w_box_bytes;    // 64 * bh * N * 2
    uint32_t x_box_bytes;    // 64 * N * MT * 2
    const uint16_t* residual;  // [M][H]
    uint16_t* out;             // [M][H]           (fused)
    uint16_t* partials;        // [N][M][H]        (not fused)
};

template <int MT>
__global__ void __launch_bounds__(kMaxExactThreads, 1)
    exact_partial_kernel(const __grid_constant__ CUtensorMap tmap_w,
                         const __grid_constant__ CUtensorMap tmap_x, const ExactParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // Align the dynamic shared-memory base to 1024 bytes (128-byte swizzle atom).
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int N = p.n_ranks, BH = p.bh, S = p.stages;
    uint8_t* w_ring = smem;
    uint8_t* x_ring = w_ring + static_cast<size_t>(S) * p.w_stage_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(x_ring + static_cast<size_t>(S) * p.x_stage_bytes);
    uint64_t* empty = full + kMaxStages;
    uint16_t* part = reinterpret_cast<uint16_t*>(empty + kMaxStages);  // [N][BH][MT]
    __shared__ int abort_flag;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int consumer_warps = (blockDim.x >> 5) - 1;
    const int n_consumers = consumer_warps * 32;
    const int T = N * BH;  // chains-owning consumer threads
    const int h0 = blockIdx.x * BH;
    const int m0 = blockIdx.y * MT;
    const int nkb = (p.ks + kKBlock - 1) / kKBlock;

    if (tid == 0) {
        abort_flag = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], consumer_warps);
        }
        fence_barrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == consumer_warps) {
        // ------------------------------------------------------- producer --
        if (lane == 0) {
            tma_prefetch_desc(&tmap_w);
            tma_prefetch_desc(&tmap_x);
            const uint32_t tx = p.w_box_bytes + p.x_box_bytes;
            const int pre = nkb < S ? nkb : S;
            for (int kb = 0; kb < pre; ++kb) {
                mbar_arrive_expect_tx(&full[kb], tx);
                tma_load_3d(w_ring + static_cast<size_t>(kb) * p.w_stage_bytes, &tmap_w, &full[kb],
                            kb * kKBlock, h0, 0);
            }
            pdl_wait();  // activations may be produced by the previous kernel
            for (int kb = 0; kb < pre; ++kb)
                tma_load_3d(x_ring + static_cast<size_t>(kb) * p.x_stage_bytes, &tmap_x, &full[kb],
                            kb * kKBlock, 0, m0);
            int issued = pre;
            int s = 0;
            uint32_t phase = 0;
            for (int kb = pre; kb < nkb; ++kb) {
                // stage kb % S, its (kb / S)-th reuse
                s = kb % S;
                phase = static_cast<uint32_t>(kb / S) & 1u;
                if (!mbar_wait_bounded(&empty[s], phase ^ 1u)) {
                    atomicExch(&abort_flag, 1);
                    break;
                }
                if (*reinterpret_cast<volatile int*>(&abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], tx);
                tma_load_3d(w_ring + static_cast<size_t>(s) * p.w_stage_bytes, &tmap_w, &full[s],
                            kb * kKBlock, h0, 0);
                tma_load_3d(x_ring + static_cast<size_t>(s) * p.x_stage_bytes, &tmap_x, &full[s],
                            kb * kKBlock, 0, m0);
                issued = kb + 1;
            }
            // Wait (bounded) for the last copies issued into every stage. A wait
            // that runs out has set the device error word; the launch's results
            // are then invalid and the context should be discarded.
            const int first = issued > S ? issued - S : 0;
            for (int kb = first; kb < issued; ++kb)
                if (!mbar_wait_bounded(&full[kb % S], static_cast<uint32_t>(kb / S) & 1u)) break;
        }
        return;
    }

    // ---------------------------------------------------------- consumers --
    const bool owner = tid < T;
    const int r = owner ? tid / BH : 0;
    const int row = tid;  // == r * BH + j: the thread's 128-byte row in a W box
    float acc[MT];
#pragma unroll
    for (int i = 0; i < MT; ++i) acc[i] = 0.0f;

    for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % S;
        const uint32_t phase = static_cast<uint32_t>(kb / S) & 1u;
        // Every lane waits (each needs the barrier's acquire); the warp then
        // agrees, so a wait that ran out on one lane stops the whole warp.
        const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], phase));
        if (!ok) {
            atomicExch(&abort_flag, 1);
            break;
        }
        if (owner) {
            // Plain shared-memory loads (ordered after the barrier wait by its
            // memory clobber) so the compiler can issue the block's loads
            // ahead of the FMA chain.
            const uint4* wrow = reinterpret_cast<const uint4*>(
                w_ring + static_cast<size_t>(s) * p.w_stage_bytes + row * 128);
            const uint4* xs = reinterpret_cast<const uint4*>(
                x_ring + static_cast<size_t>(s) * p.x_stage_bytes + r * 128);
            const int sw = row & 7;
            const int rem = p.ks - kb * kKBlock;
            const int nv = rem >= kKBlock ? 8 : rem >> 3;  // K/N % 8 == 0: whole 16-byte vectors
            uint4 wv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c < nv) wv[c] = wrow[c ^ sw];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const uint4* xm = xs + mt * N * 8;
                float a = acc[mt];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    if (c < nv) {
                        const uint4 xv = xm[c];
                        a = fma2_bf16(xv.x, wv[c].x, a);
                        a = fma2_bf16(xv.y, wv[c].y, a);
                        a = fma2_bf16(xv.z, wv[c].z, a);
                        a = fma2_bf16(xv.w, wv[c].w, a);
                    }
                }
                acc[mt] = a;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }

    // Every consumer thread reaches this barrier (no early return above).
    asm volatile("bar.sync 1, %0;" ::"r"(n_consumers) : "memory");
    if (*reinterpret_cast<volatile int*>(&abort_flag)) return;
    pdl_wait();  // the residual and the outputs belong to the stream's order

    const int j = tid - r * BH;
    if (!p.fused) {
        if (owner && h0 + j < p.hidden) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
                if (m0 + mt < p.tokens)
                    p.partials[(static_cast<size_t>(r) * p.tokens + m0 + mt) * p.hidden + h0 + j] =
                        f32_to_bf16_rne(acc[mt]);
        }
        return;
    }

    if (owner) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) part[(r * BH + j) * MT + mt] = f32_to_bf16_rne(acc[mt]);
    }
    asm volatile("bar.sync 1, %0;" ::"r"(n_consumers) : "memory");
    // Ring fold: chunk c = h / (H/N) starts at rank c and adds ranks c+1, ...,
    // c-1 (mod N) from the left; then the residual.
    for (int o = tid; o < BH * MT; o += n_consumers) {
        const int mt = o / BH, jj = o - mt * BH;
        const int h = h0 + jj, m = m0 + mt;
        if (h >= p.hidden || m >= p.tokens) continue;
        const int c = h / p.hc;
        uint16_t acc16 = part[(c * BH + jj) * MT + mt];
        for (int i = 1; i < N; ++i) {
            int rr = c + i;
            if (rr >= N) rr -= N;
            acc16 = bf16_add(acc16, part[(rr * BH + jj) * MT + mt]);
        }
        const size_t o_idx = static_cast<size_t>(m) * p.hidden + h;
        p.out[o_idx] = bf16_add(p.residual[o_idx], acc16);
    }
}

// ------------------------------------------------------------------ S2-S4 --
// Ring reduce-scatter fold over partials staged in memory, the all-gather
// (one result buffer stands for every rank's copy) and the residual add.
// Thread per 8 consecutive columns (16-byte vectors; H/N % 8 == 0 keeps a
// vector inside one chunk), grid-stride. The N partial vectors of a thread
// are all loaded before the first add (the rank loop is unrolled to the
// largest N), so their memory latencies overlap instead of adding up; the
// adds go two columns at a time (bf16x2).
__global__ void __launch_bounds__(256)
    ring_reduce_kernel(const uint16_t* __restrict__ partials, const uint16_t* __restrict__ residual,
                       uint16_t* __restrict__ out, int n_ranks, int64_t tokens, int hidden, int hc) {
    pdl_launch_dependents();
    pdl_wait();
    const int64_t hv = hidden >> 3;
    const int64_t total = tokens * hv;
    const size_t plane = static_cast<size_t>(tokens) * hidden;
    for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < total;
         v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = v / hv;
        const int h = static_cast<int>(v - m * hv) << 3;
        const int c = h / hc;
        const size_t off = static_cast<size_t>(m) * hidden + h;
        uint4 pv[kMaxRanks];
#pragma unroll
        for (int i = 0; i < kMaxRanks; ++i) {
            if (i < n_ranks) {
                int rr = c + i;   // ring order: the chunk's owner first
                if (rr >= n_ranks) rr -= n_ranks;
                pv[i] = ld_global_nc_v4(partials + static_cast<size_t>(rr) * plane + off);
            }
        }
        const uint4 rv = ld_global_nc_v4(residual + off);
        uint4 sum = pv[0];
#pragma unroll
        for (int i = 1; i < kMaxRanks; ++i) {
            if (i < n_ranks) {
                sum.x = bf16x2_add(sum.x, pv[i].x);
                sum.y = bf16x2_add(sum.y, pv[i].y);
                sum.z = bf16x2_add(sum.z, pv[i].z);
                sum.w = bf16x2_add(sum.w, pv[i].w);
            }
        }
        uint4 o;
        o.x = bf16x2_add(rv.x, sum.x);
        o.y = bf16x2_add(rv.y, sum.y);
        o.z = bf16x2_add(rv.z, sum.z);
        o.w = bf16x2_add(rv.w, sum.w);
        st_global_v4(out + off, o);
    }
}

// S2-S4 over k-split partials: rank r's partial is first assembled as
// bf16_rne(part_0 + part_1 + ... ) -- the fp32 sums of its K parts added in
// split order -- then folded in ring order as above. Few tokens take this
// path (it exists to fill the SMs when there are few units), so a thread
// takes one output element and loads all N * SPLITS parts before adding.
// Grid: x over H in blocks of 256 columns, y over tokens (grid-stride).
__global__ void __launch_bounds__(256)
    ring_reduce_splits_kernel(const float* __restrict__ parts, int splits,
                              const uint16_t* __restrict__ residual, uint16_t* __restrict__ out,
                              int n_ranks, int64_t tokens, int hidden, int hc) {
    pdl_launch_dependents();
    pdl_wait();
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= hidden) return;
    const int c = h / hc;
    const size_t plane = static_cast<size_t>(tokens) * hidden;
    for (int64_t m = blockIdx.y; m < tokens; m += gridDim.y) {
        const size_t off = static_cast<size_t>(m) * hidden + h;
        const uint16_t s = ring_fold_f32_parts<false>(parts, splits, n_ranks, plane, off, c);
        const uint16_t rv = residual[off];
        out[off] = bf16_add(rv, s);
    }
}

// --------------------------------------------------------------------- S0 --
// Linear weight [H][K] -> [N][H][K/N]: shard r is columns r*Ks .. r*Ks+Ks-1.
__global__ void __launch_bounds__(256)
    pack_weights_kernel(const uint16_t* __restrict__ w, uint16_t* __restrict__ wp, int hidden,
                        int64_t k, int64_t ks) {
    const int64_t kv = k >> 3;
    const int64_t total = static_cast<int64_t>(hidden) * kv;
    for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < total;
         v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t h = v / kv;
        const int64_t col = (v - h * kv) << 3;
        const int64_t r = col / ks;
        const int64_t kk = col - r * ks;
        const uint4 val = ld_global_nc_v4(w + h * k + col);
        st_global_v4(wp + (r * hidden + h) * ks + kk, val);
    }
}

}  // namespace tpr
