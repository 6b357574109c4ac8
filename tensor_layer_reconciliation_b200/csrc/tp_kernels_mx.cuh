// Quantised weight shards: the element and scale conversions and the
// quantisation kernels (S0) of the two formats; the reconciliation over the
// shards runs on the tensor cores (tp_kernels_tc.cuh, quantised forms).
//
// MXFP8 (the NVL72 hosting post's MXFP8 weights, laid out per the OCP
// Microscaling v1.0 specification): each run of 32 consecutive weights
// along K inside one rank's slice shares an E8M0 scale X = 2^s, stored as
// the byte s + 127, with s = floor(log2 max|w|) - 8 clamped to [-127, 127]
// (-127 for an all-zero run); each weight is the FP8 E4M3 code nearest to
// w / X, ties to even, saturating at 448.
//   q      [N][H][K/N] E4M3 codes                     (K/N a multiple of 64)
//   scales [N][ceil(H/128)][ceil(K/N/128)][512] E8M0 bytes: one 512-byte chunk
//          holds the scales of a 128-row tile for four 32-weight runs (128
//          columns): row t of the tile, run j at byte 16 (t % 32) + 4 (t / 32)
//          + j -- the order in which the block-scaled MMA reads them from
//          tensor memory; rows past H and runs past K/N hold 0
//
// NVFP4 (the TP=4-vs-TP=8 post's NVFP4 weights, in NVIDIA's published
// layout): E2M1 elements, one E4M3 block scale per 16 weights along K inside a
// rank slice, and a second-level scale 2^g for the whole tensor, g the
// smallest integer with max|W| / 2^g <= 6 * 448 (0 for an all-zero tensor):
//   b = E4M3 nearest to max|block| / (6 * 2^g); q = E2M1 nearest to
//   w / (b * 2^g), ties to even, saturating at 6 (zeros where b is 0).
//   q      [N][H][K/N/2] bytes, two codes each, the earlier k in bits 0-3
//   scales [N][K/N/64][H][4] E4M3 bytes (the four block scales of each row
//          for one 64-column block), then 16 bytes: g (int32), max|W| bits
#pragma once

#include "tp_common.cuh"

namespace tpr {

constexpr int kMxBlock = 32;        // weights per shared scale
constexpr int kMxPair = 64;         // K/N is a multiple of this
constexpr int kMxChunk = 512;       // scale bytes of a 128-row tile x 128 columns
constexpr int kMxChunkCols = 128;   // columns a scale chunk covers

// Byte of the scale of run b (32 columns) of row h of rank r in the chunked
// scale array (h_tiles = ceil(H/128), kg = ceil(K/N/128)).
__host__ __device__ constexpr int64_t mx_scale_index(int64_t r, int64_t h, int64_t b, int64_t h_tiles,
                                                     int64_t kg) {
    return ((r * h_tiles + h / 128) * kg + b / 4) * kMxChunk + (h % 32) * 16 + ((h % 128) / 32) * 4 + b % 4;
}

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

// Two f32 values -> bf16x2, each rounded to nearest even; `lo` in bits 0-15.
__device__ __forceinline__ uint32_t bf16x2_from_f32(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
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
        scales[mx_scale_index(r, h, b, (hidden + 127) / 128, (ks + kMxChunkCols - 1) / kMxChunkCols)] =
            static_cast<uint8_t>(s + 127);
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

// ----------------------------------------------------------- S0, NVFP4 --

// Two f32 values -> two E2M1 codes, nearest even, saturating at +-6; the
// code of `lo` in bits 0-3 of the result.
__device__ __forceinline__ uint32_t e2m1x2_from_f32(float lo, float hi) {
    uint32_t d;
    asm("{\n\t.reg .b8 c;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c, %1, %2;\n\t"
        "cvt.u32.u8 %0, c;\n\t}"
        : "=r"(d)
        : "f"(hi), "f"(lo));
    return d;
}

// The largest magnitude of the Linear weight (as a bf16 pattern without its
// sign, which orders like the value) into *amax_bits (zero on entry).
__global__ void __launch_bounds__(256)
    nv_amax_kernel(const uint16_t* __restrict__ w, int64_t n_vec8, uint32_t* amax_bits) {
    uint32_t m = 0;
    for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < n_vec8;
         v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint4 q = ld_global_nc_v4(w + 8 * v);
        const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) m = max(m, max(wd[i] & 0x7FFFu, (wd[i] >> 16) & 0x7FFFu));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(amax_bits, m);
}

// One thread per 16-weight block: the block scale from the block maximum,
// then each weight divided by it (after the exact scaling by 2^-g) and
// rounded. The quotients are rounded to fp32 first; an fp32 rounding cannot
// carry a quotient of these few-bit operands onto or across an E4M3 or E2M1
// rounding boundary, so the codes are those of the exact quotients.
__global__ void __launch_bounds__(256)
    pack_weights_nv_kernel(const uint16_t* __restrict__ w, uint8_t* __restrict__ q,
                           uint8_t* __restrict__ scales, int* __restrict__ gexp,
                           const uint32_t* __restrict__ amax_bits, int n_ranks, int hidden, int64_t k,
                           int64_t ks) {
    const uint32_t amax_b = *amax_bits;
    // g: the smallest integer with amax <= 2688 * 2^g
    int g = 0;
    if (amax_b != 0) {
        const int e = bf16_floor_log2(amax_b);                       // 2^e <= amax < 2^(e+1)
        const float amax = bf16_bits_to_f32(amax_b);
        g = e - 11;
        if (amax > ldexpf(2688.0f, g)) g += 1;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *gexp = g;
    const int64_t nb = ks / 16, nkb = ks / 64;
    const int64_t total = static_cast<int64_t>(n_ranks) * hidden * nb;
    for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t b = t % nb;
        const int64_t row = t / nb;              // r * H + h
        const int64_t h = row % hidden;
        const int64_t r = row / hidden;
        const uint4* src = reinterpret_cast<const uint4*>(w + h * k + r * ks + b * 16);
        const uint4 v0 = src[0], v1 = src[1];
        const uint32_t wd[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t bmax = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) bmax = max(bmax, max(wd[i] & 0x7FFFu, (wd[i] >> 16) & 0x7FFFu));
        // block scale: E4M3 nearest to bmax / (6 * 2^g) (at most 448 by the choice of g)
        const float qs = __fdiv_rn(ldexpf(bf16_bits_to_f32(bmax), -g), 6.0f);
        const uint32_t bs = e4m3x2_from_f32(qs, 0.0f) & 0xFFu;
        scales[((r * nkb + (b >> 2)) * hidden + h) * 4 + (b & 3)] = static_cast<uint8_t>(bs);
        const float bval = f16_lo_to_f32(f16x2_from_e4m3x2(static_cast<uint16_t>(bs)));
        uint32_t out[2] = {0u, 0u};
        if (bval != 0.0f) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {   // word i: weights 2i, 2i+1 -> one byte of codes
                const float lo = __fdiv_rn(ldexpf(bf16_lo(wd[i]), -g), bval);
                const float hi = __fdiv_rn(ldexpf(bf16_hi(wd[i]), -g), bval);
                out[i >> 2] |= e2m1x2_from_f32(lo, hi) << (8 * (i & 3));
            }
        }
        *reinterpret_cast<uint2*>(q + row * (ks / 2) + b * 8) = make_uint2(out[0], out[1]);
    }
}

}  // namespace tpr
