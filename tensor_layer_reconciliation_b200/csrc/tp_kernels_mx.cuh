// MXFP8 weight shards: quantisation (S0) and the decode reconciliation over
// them (S1-S4 in one kernel).
//
// Format (the NVL72 hosting post's MXFP8 weights, laid out per the OCP
// Microscaling v1.0 specification): each run of 32 consecutive weights
// along K inside one rank's slice shares an E8M0 scale X = 2^s, stored as
// the byte s + 127, with s = floor(log2 max|w|) - 8 clamped to [-127, 127]
// (-127 for an all-zero run); each weight is the FP8 E4M3 code nearest to
// w / X, ties to even, saturating at 448.
//   q      [N][H][K/N] E4M3 codes      (K/N a multiple of 32)
//   scales [N][H][K/N/32] E8M0 bytes
#pragma once

#include "tp_common.cuh"

namespace tpr {

constexpr int kMxBlock = 32;        // weights per shared scale
constexpr int kMxMaxTokens = 4;     // decode token counts the fused kernel takes (MT = tokens)
constexpr int kMxWarps = 4;         // output rows in flight per CTA (one per warp)

// Two f32 values -> two E4M3 codes, nearest even, saturating at +-448; the
// code of `lo` in bits 0-7 of the result.
__device__ __forceinline__ uint16_t e4m3x2_from_f32(float lo, float hi) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

// Two E4M3 codes (bits 0-7 and 8-15 of v) -> two exact f16 values as f16x2.
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint16_t v) {
    uint32_t d;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(v));
    return d;
}

__device__ __forceinline__ float f16_lo_to_f32(uint32_t v) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(v & 0xFFFF)));
}
__device__ __forceinline__ float f16_hi_to_f32(uint32_t v) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(v >> 16)));
}

// 2^(b - 127) for an E8M0 byte b (b = 255, NaN, is never stored).
__device__ __forceinline__ float e8m0_to_f32(uint32_t b) {
    return b == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(b << 23);
}

// 2^e as an f32, e in [-127, 127] (2^-127 is the f32 subnormal 0x00400000).
__device__ __forceinline__ float pow2_f32(int e) {
    return e8m0_to_f32(static_cast<uint32_t>(e + 127));
}

// floor(log2 |v|) of a nonzero finite bf16 pattern (v without its sign bit).
__device__ __forceinline__ int bf16_floor_log2(uint32_t mag) {
    const int e = static_cast<int>(mag >> 7);
    if (e != 0) return e - 127;
    // subnormal: m * 2^-133, m = mag in 1 .. 127
    return (31 - __clz(static_cast<int>(mag))) - 133;
}

// ------------------------------------------------------------------- S0 --
// One thread per 32-weight block: the block's largest magnitude fixes the
// scale; every weight is divided by it (a power of two: exact) and rounded.
__global__ void __launch_bounds__(256)
    pack_weights_mx_kernel(const uint16_t* __restrict__ w, uint8_t* __restrict__ q,
                           uint8_t* __restrict__ scales, int n_ranks, int hidden, int64_t k,
                           int64_t ks) {
    const int64_t nb = ks / kMxBlock;
    const int64_t total = static_cast<int64_t>(n_ranks) * hidden * nb;
    for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t b = t % nb;
        const int64_t row = t / nb;              // r * H + h
        const int64_t h = row % hidden;
        const int64_t r = row / hidden;
        const uint4* src = reinterpret_cast<const uint4*>(w + h * k + r * ks + b * kMxBlock);
        uint32_t words[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = src[i];
            words[4 * i] = v.x;
            words[4 * i + 1] = v.y;
            words[4 * i + 2] = v.z;
            words[4 * i + 3] = v.w;
        }
        uint32_t amax = 0;   // largest magnitude as a bf16 pattern (ordered like the value)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            amax = max(amax, words[i] & 0x7FFFu);
            amax = max(amax, (words[i] >> 16) & 0x7FFFu);
        }
        int s = amax == 0 ? -127 : bf16_floor_log2(amax) - 8;
        s = max(-127, min(127, s));
        scales[row * nb + b] = static_cast<uint8_t>(s + 127);
        // w / 2^s = w * 2^-s: a power of two, exact unless it drops below the
        // f32 range, where the E4M3 code is a signed zero either way.
        const float inv = pow2_f32(-s);
        uint32_t out[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t a = words[2 * i], c = words[2 * i + 1];
            const uint16_t lo = e4m3x2_from_f32(bf16_lo(a) * inv, bf16_hi(a) * inv);
            const uint16_t hi = e4m3x2_from_f32(bf16_lo(c) * inv, bf16_hi(c) * inv);
            out[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
        }
        uint4* dst = reinterpret_cast<uint4*>(q + row * ks + b * kMxBlock);
        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    }
}

// ---------------------------------------------------------------- S1-S4 --
// One warp per output row h (grid-stride), all N ranks in turn. Lane i
// takes the 32 consecutive codes of one scale block out of every 1024 (two
// 16-byte loads: a warp load is 1024 contiguous bytes), two such chunks in
// flight at a time. The codes become exact f32 values (E4M3 -> f16x2 ->
// f32), the bf16 activations f32 pairs, and the 32 products of a chunk are
// summed with packed f32x2 fused multiply-adds (two interleaved chains), the
// chunk's sum scaled by 2^s into the lane's accumulator; lanes meet by
// shuffles. The N partials of the row then fold in ring order from the
// chunk's owner and meet the residual: nothing is staged. Codes of the first
// chunks are loaded before griddepcontrol.wait. The summation order differs
// from the oracle's k-ascending chain, so a partial can round to the other
// bf16 neighbour where its exact value lies next to a rounding boundary.
constexpr int kMxLaneChunk = kMxBlock;                 // codes per lane per step
constexpr int kMxWarpStep = 32 * kMxLaneChunk;         // 1024 codes per warp step

struct MxParams {
    int n_ranks;
    int hidden;
    int hc;          // H / N
    int tokens;      // = MT, 1 .. kMxMaxTokens
    int64_t k;       // K
    int64_t ks;      // K / N
    const uint16_t* x;       // [M][K]
    const uint8_t* q;        // [N][H][Ks]
    const uint8_t* scales;   // [N][H][Ks/32]
    const uint16_t* residual;  // [M][H]
    uint16_t* out;             // [M][H]
};

// d (f32x2) += a (f32x2) * b (f32x2), each lane of the pair rounded once.
__device__ __forceinline__ void fma_f32x2(uint64_t& d, uint64_t a, uint64_t b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}

// Sum of the 32 products of one chunk: codes in q0, q1 (32 bytes), the
// activations' 32 bf16 at xp (64 bytes, 16-byte aligned).
__device__ __forceinline__ float mx_chunk_dot(const uint4& q0, const uint4& q1, const uint16_t* xp) {
    const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    const uint4* x4 = reinterpret_cast<const uint4*>(xp);
    uint64_t s0 = 0, s1 = 0;   // two chains of f32x2 sums
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 xv = __ldg(x4 + j);              // 8 activations: codes 8j .. 8j+7
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t c = qw[2 * j + i];            // 4 codes
            const uint32_t a = f16x2_from_e4m3x2(static_cast<uint16_t>(c & 0xFFFF));
            const uint32_t b = f16x2_from_e4m3x2(static_cast<uint16_t>(c >> 16));
            const uint64_t w01 = pack_f32x2(f16_lo_to_f32(a), f16_hi_to_f32(a));
            const uint64_t w23 = pack_f32x2(f16_lo_to_f32(b), f16_hi_to_f32(b));
            const uint32_t x01 = xw[2 * i], x23 = xw[2 * i + 1];
            fma_f32x2(s0, pack_f32x2(bf16_lo(x01), bf16_hi(x01)), w01);
            fma_f32x2(s1, pack_f32x2(bf16_lo(x23), bf16_hi(x23)), w23);
        }
    }
    const float a0 = __uint_as_float(static_cast<uint32_t>(s0));
    const float a1 = __uint_as_float(static_cast<uint32_t>(s0 >> 32));
    const float b0 = __uint_as_float(static_cast<uint32_t>(s1));
    const float b1 = __uint_as_float(static_cast<uint32_t>(s1 >> 32));
    return (a0 + a1) + (b0 + b1);
}

// One token: at most 56 registers, so 9 CTAs (36 warps) fit on an SM and a
// 5120-row call runs in one wave on 148 SMs.
template <int MT>
__global__ void __launch_bounds__(kMxWarps * 32, MT == 1 ? 9 : 4)
    mx_reconcile_kernel(const MxParams p) {
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ks = static_cast<int>(p.ks);
    const int nb = ks / kMxBlock;
    bool waited = false;
    for (int h = blockIdx.x * kMxWarps + warp; h < p.hidden; h += gridDim.x * kMxWarps) {
        float part[kMaxRanks][MT];
#pragma unroll
        for (int r = 0; r < kMaxRanks; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) part[r][m] = 0.0f;
#pragma unroll 1
        for (int r = 0; r < p.n_ranks; ++r) {
            const int64_t row = static_cast<int64_t>(r) * p.hidden + h;
            const uint8_t* qrow = p.q + row * ks;
            const uint8_t* srow = p.scales + row * nb;
            const uint16_t* xr = p.x + static_cast<int64_t>(r) * ks;
            float acc[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
            for (int k0 = lane * kMxLaneChunk; k0 < ks; k0 += 2 * kMxWarpStep) {
                const int k1 = k0 + kMxWarpStep;
                const bool has1 = k1 < ks;
                const uint4* qa = reinterpret_cast<const uint4*>(qrow + k0);
                const uint4 qa0 = ld_global_nc_v4(qa), qa1 = ld_global_nc_v4(qa + 1);
                const uint32_t sa = srow[k0 / kMxBlock];
                uint4 qb0 = make_uint4(0, 0, 0, 0), qb1 = qb0;
                uint32_t sbb = 0;
                if (has1) {
                    const uint4* qb = reinterpret_cast<const uint4*>(qrow + k1);
                    qb0 = ld_global_nc_v4(qb);
                    qb1 = ld_global_nc_v4(qb + 1);
                    sbb = srow[k1 / kMxBlock];
                }
                if (!waited) {
                    pdl_wait();   // activations and residual follow the stream's order
                    waited = true;
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint16_t* xm = xr + static_cast<int64_t>(m) * p.k;
                    acc[m] = fmaf(mx_chunk_dot(qa0, qa1, xm + k0), e8m0_to_f32(sa), acc[m]);
                    if (has1) acc[m] = fmaf(mx_chunk_dot(qb0, qb1, xm + k1), e8m0_to_f32(sbb), acc[m]);
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    acc[m] += __shfl_xor_sync(0xFFFFFFFFu, acc[m], off);
            }
#pragma unroll
            for (int rr = 0; rr < kMaxRanks; ++rr)
                if (rr == r)
#pragma unroll
                    for (int m = 0; m < MT; ++m) part[rr][m] = acc[m];
        }
        if (!waited) {
            pdl_wait();
            waited = true;
        }
        // S2-S4: lane m folds token m's partials in ring order, adds the residual.
        if (lane < MT) {
            const int c = h / p.hc;
            float pm[kMaxRanks];
#pragma unroll
            for (int rr = 0; rr < kMaxRanks; ++rr) {
                pm[rr] = part[rr][0];
#pragma unroll
                for (int m = 1; m < MT; ++m)
                    if (lane == m) pm[rr] = part[rr][m];
            }
            uint16_t s = 0;
#pragma unroll
            for (int i = 0; i < kMaxRanks; ++i) {
                if (i < p.n_ranks) {
                    int rr = c + i;
                    if (rr >= p.n_ranks) rr -= p.n_ranks;
                    float pv = pm[0];
#pragma unroll
                    for (int j = 1; j < kMaxRanks; ++j)
                        if (j == rr) pv = pm[j];
                    const uint16_t pb = f32_to_bf16_rne(pv);
                    s = i == 0 ? pb : bf16_add(s, pb);
                }
            }
            const size_t o = static_cast<size_t>(lane) * p.hidden + h;
            p.out[o] = bf16_add(p.residual[o], s);
        }
    }
    if (!waited) pdl_wait();
}

}  // namespace tpr
