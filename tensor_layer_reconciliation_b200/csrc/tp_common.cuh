// Device helpers shared by the reconciliation kernels (sm_100a).
//
// bf16 arithmetic used by the ring: an add is fp32 add then one
// round-to-nearest-even to bf16. With fp32's 24-bit significand at least
// 2*8+2 bits, the double rounding is innocuous (Figueroa, "When is double
// rounding innocuous?", 1995), so this is the correctly rounded bf16 sum.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tpr {

// Device-side error word: bit 0 = a bounded pipeline wait ran out.
constexpr uint32_t kErrWaitTimeout = 1u;
__device__ uint32_t g_device_error = 0;  // one translation unit

// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) {
    return __uint_as_float(b16 << 16);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// One bf16 add of the ring: bf16_rne(f32(a) + f32(b)).
__device__ __forceinline__ uint16_t bf16_add(uint16_t a, uint16_t b) {
    return f32_to_bf16_rne(__fadd_rn(bf16_bits_to_f32(a), bf16_bits_to_f32(b)));
}

// Two ring adds at once on packed bf16 pairs: add.rn.bf16x2 rounds the exact
// sum once to bf16, which equals bf16_add's fp32 add then rounding (fp32 holds
// more than 2 * 8 + 2 bits, so the double rounding is innocuous).
__device__ __forceinline__ uint32_t bf16x2_add(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier --

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before the async
// proxy's later reads of them (tcgen05.mma / tcgen05.cp operands, TMA stores).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

// Suspend-time hint for try_wait: a waiting thread sleeps until the phase
// completes or this many nanoseconds pass, instead of polling the barrier
// (polling threads compete with the bulk copies for the shared-memory path).
constexpr uint32_t kSuspendHintNs = 1000000u;  // 1 ms

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete. Gives up after
// kWaitLimitNs, sets the device error word and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_device_error, kErrWaitTimeout);
            return false;
        }
    }
    return true;
}

// Named barrier `id` over `nthreads` threads that also ORs a flag across
// them: every participant gets the same answer, so a decision taken on it
// (leaving a loop whose next iteration meets the barrier again) is uniform.
__device__ __forceinline__ bool bar_sync_any(int id, int nthreads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, p;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// ---------------------------------------------------------- ring fold --
constexpr int kMaxRanks = 8;     // tp_plan_create accepts 1 .. 8 ranks
constexpr int kMaxSplits = 8;    // k-splits of the tensor-core partials

// S2-S3 for one output element (token m, column h at offset `off` of an
// [M][H] plane) from partials staged in memory: starting at the owner c of
// the element's chunk, the ranks' partials are added in ring order, each add
// rounded to bf16. Every load is issued before the first add (loops unrolled
// to the largest counts), so one memory latency covers them all. kL2 loads
// through L2 only, for data written earlier by the same kernel.
template <bool kL2>
__device__ __forceinline__ uint16_t ring_fold_bf16(const uint16_t* partials, int n_ranks, size_t plane,
                                                   size_t off, int c) {
    uint16_t v[kMaxRanks];
#pragma unroll
    for (int i = 0; i < kMaxRanks; ++i) {
        if (i < n_ranks) {
            int rr = c + i;
            if (rr >= n_ranks) rr -= n_ranks;
            const uint16_t* a = partials + static_cast<size_t>(rr) * plane + off;
            v[i] = kL2 ? __ldcg(a) : *a;
        }
    }
    uint16_t s = v[0];
#pragma unroll
    for (int i = 1; i < kMaxRanks; ++i)
        if (i < n_ranks) s = bf16_add(s, v[i]);
    return s;
}

// As ring_fold_bf16 over k-split fp32 parts [SPLITS][N][M][H]: rank r's
// partial is bf16_rne(part_0 + part_1 + ...), the parts added in split
// (k-ascending) order in fp32, before the ring-order bf16 adds.
template <bool kL2>
__device__ __forceinline__ uint16_t ring_fold_f32_parts(const float* parts, int splits, int n_ranks,
                                                        size_t plane, size_t off, int c) {
    float a[kMaxRanks][kMaxSplits];
#pragma unroll
    for (int i = 0; i < kMaxRanks; ++i) {
        if (i < n_ranks) {
            int rr = c + i;
            if (rr >= n_ranks) rr -= n_ranks;
#pragma unroll
            for (int sp = 0; sp < kMaxSplits; ++sp)
                if (sp < splits) {
                    const float* q = parts + (static_cast<size_t>(sp) * n_ranks + rr) * plane + off;
                    a[i][sp] = kL2 ? __ldcg(q) : *q;
                }
        }
    }
    uint16_t s = 0;
#pragma unroll
    for (int i = 0; i < kMaxRanks; ++i) {
        if (i < n_ranks) {
            float f = a[i][0];
#pragma unroll
            for (int sp = 1; sp < kMaxSplits; ++sp)
                if (sp < splits) f = __fadd_rn(f, a[i][sp]);
            const uint16_t pr = f32_to_bf16_rne(f);
            s = i == 0 ? pr : bf16_add(s, pr);
        }
    }
    return s;
}

// --------------------------------------------------------------------- TMA --

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled bulk tensor load into this CTA's shared memory only.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// `bytes` (a multiple of 16) from the 16-byte aligned global address `src`
// into this CTA's shared memory at `dst` (16-byte aligned), counted on `bar`
// as transaction bytes (no tensor map: a contiguous run).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// `bytes` (a multiple of 16) from the 16-byte aligned global address into L2
// only: no shared memory, no completion to wait for. L2 is where global
// memory is kept coherent, so a line prefetched before another kernel writes
// it is updated in place by that write.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Counter handshake between the CTAs of one grid. red_release_add: this
// CTA's earlier writes (ordered before the calling thread by a barrier) are
// visible at gpu scope before the addition. ld_acquire_gpu: reads after it
// (and, through a barrier, the CTA's reads) see what the releases covered.
__device__ __forceinline__ void red_release_add(unsigned int* p, unsigned int v) {
    asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v)
                 : "memory");
}
__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// --------------------------------------------- programmatic dependent launch --

// Blocks until the grids this one depends on have completed and their memory
// operations are visible. A no-op when the launch had no such dependency.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Lets the next grid in the stream start its prologue early.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Two steps of an fp32 accumulation chain on a pair of bf16 values each:
// acc = fma(x.lo, w.lo, acc); acc = fma(x.hi, w.hi, acc). The mixed-precision
// FMA multiplies the bf16 operands exactly and rounds once to fp32, the same
// as fmaf on their fp32 widenings; the low half (the earlier k) goes first.
__device__ __forceinline__ float fma2_bf16(uint32_t x, uint32_t w, float acc) {
    asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\t"
        "mov.b32 {xl, xh}, %1;\n\t"
        "mov.b32 {wl, wh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, xl, wl, %0;\n\t"
        "fma.rn.f32.bf16 %0, xh, wh, %0;\n\t}"
        : "+f"(acc)
        : "r"(x), "r"(w));
    return acc;
}

// ------------------------------------------------------------ vector loads --

__device__ __forceinline__ uint4 ld_global_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_global_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

}  // namespace tpr
