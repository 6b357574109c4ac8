// Thin wrappers over the sm_100a tensor-core (tcgen05) and tensor-memory
// instructions the tensor-core partial kernel uses, plus the two descriptor
// encoders. Written from the PTX ISA description of tcgen05 (kind::f16,
// cta_group::1) and the layout of its shared-memory and instruction
// descriptors.
#pragma once

#include "tp_common.cuh"

namespace tpr {

// ------------------------------------------------------------- fences --

__device__ __forceinline__ void tc_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ------------------------------------------------------- tensor memory --

// Allocates ncols (a power of two >= 32) TMEM columns for this CTA; the
// base address is written to *slot (shared memory). Whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols)
                 : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes (lane = thread),
// followed by the wait for the load in the same statement, so no use of the
// registers can be scheduled before they hold the data.
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
          "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
          "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}

// Stores 16 consecutive 32-bit columns of this thread's lane (the warp's
// lane quarter in bits 31:16 of taddr). Asynchronous: tmem_st_wait() before
// the columns are read by an MMA.
__device__ __forceinline__ void tmem_st_16cols(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- mma --

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate; issued by
// one thread. accumulate = 0 overwrites D.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// As umma_bf16 with A read from tensor memory: 128 lanes (one row of A each)
// x 8 columns (16 bf16 of K, two a column, the lower k in the low half)
// from column a_tmem.
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Block-scaled MMA, kind::mxf8f6f4 with E4M3 A and B and E8M0 scales, one per
// 32 values of K (one K = 32 step): D[tmem] (+)= sum over k of
// (A[m][k] * SA[m]) * (B[n][k] * SB[n]). The scales are read from tensor
// memory: row m's from lane m of column sfa_tmem + m / 32, column n's from
// lane n of column sfb_tmem + n / 32, byte `sf_id` of the 32-bit cell (the
// layout tcgen05.cp .32x128b.warpx4 writes); the instruction descriptor
// carries the same byte index (idesc_mxf8_f32).
__device__ __forceinline__ void umma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Copies a 32-row x 16-byte shared-memory tile (descriptor `sdesc`) into 4
// columns of tensor memory from column taddr, once into each 32-lane
// quarter: lane 32q + r, column taddr + c <- bytes 16r + 4c .. 16r + 4c + 3.
// Asynchronous, in issue order with this thread's MMAs.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Arrives once on the mbarrier when every MMA this thread issued so far has
// completed (and their shared-memory reads are done).
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------- descriptors --

// Shared-memory matrix descriptor of a K-major operand tile stored as rows of
// 64 bf16 (128 bytes) with the 128-byte swizzle, 8-row atoms of 1024 bytes
// (the layout a TMA load with SWIZZLE_128B writes):
//   bits  0-13  start address >> 4
//   bits 16-29  leading-dimension byte offset >> 4 (unused for this layout: 1)
//   bits 32-45  stride-dimension byte offset >> 4 (1024 bytes between 8-row atoms)
//   bits 46-47  descriptor version, 1
//   bits 49-51  base offset, 0 (atoms are 1024-byte aligned)
//   bits 61-63  layout, 2 = 128-byte swizzle
// Stepping K by 16 elements inside the 128-byte row adds 32 bytes (2 units)
// to the start address.
__device__ __forceinline__ uint64_t smem_desc_k128(const void* tile) {
    const uint64_t addr = static_cast<uint64_t>(smem_u32(tile));
    uint64_t d = (addr >> 4) & 0x3FFFull;
    d |= 1ull << 16;                    // LBO (unused)
    d |= (1024ull >> 4) << 32;          // SBO
    d |= 1ull << 46;                    // version
    d |= 2ull << 61;                    // 128-byte swizzle
    return d;
}

// Descriptor of a 32-row x 16-byte shared-memory tile, rows 16 bytes apart
// (no swizzle: 8-row core matrices of 128 contiguous bytes, 128 bytes apart
// in the stride dimension; one core matrix wide, so the leading offset is
// not used), the source of tmem_cp_32x128b_x4.
__device__ __forceinline__ uint64_t smem_desc_rows16(const void* tile) {
    const uint64_t addr = static_cast<uint64_t>(smem_u32(tile));
    uint64_t d = (addr >> 4) & 0x3FFFull;
    d |= (128ull >> 4) << 16;           // LBO (unused)
    d |= (128ull >> 4) << 32;           // SBO
    d |= 1ull << 46;                    // version
    return d;                           // layout 0: no swizzle
}

// Instruction descriptor of tcgen05.mma kind::mxf8f6f4.block_scale with E4M3
// A and B (format 0), fp32 D, both K-major, E8M0 scales:
//   bits 4-5 B scale byte, bits 7-9 / 10-12 A / B format (0 = E4M3),
//   bits 17-22 N >> 3, bit 23 scale format (1 = E8M0), bits 24-28 M >> 4,
//   bits 29-30 A scale byte, bit 31 K size (0: K = 32).
__host__ __device__ constexpr uint32_t idesc_mxf8_f32(int m, int n, int sf_id) {
    return (static_cast<uint32_t>(sf_id) << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(m >> 4) << 24) | (static_cast<uint32_t>(sf_id) << 29);
}

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A and B, fp32 D,
// both operands K-major, no negation or sparsity:
//   bits 4-5 D format (1 = f32), bits 7-9 A format (1 = bf16),
//   bits 10-12 B format (1 = bf16), bit 15/16 A/B major (0 = K),
//   bits 17-22 N >> 3, bits 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(m >> 4) << 24);
}

// ------------------------------------------------- CTA pairs (2-SM MMA) --
// A cluster of two CTAs on two SMs runs one M = 256 MMA: each CTA holds 128
// rows of A and half the columns of B in its shared memory (at the same
// offsets), the instruction is issued by one thread of the even CTA (the
// leader), and each CTA's tensor memory receives its own 128 rows of D.

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of both CTAs: arrive (release) and wait (acquire).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                     "memory");
}

// Shared-memory address, in the cluster window, of the same variable in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

// Arrive (release at cluster scope) on an mbarrier given by its cluster address.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// ------------------------------------------ cluster fold (distributed smem) --
// The N CTAs of a cluster each hold one rank's partial tile in their shared
// memory; a CTA reads its peers' tiles through the cluster's shared window.

// Orders this thread's (and, after a CTA barrier, its CTA's) shared-memory
// writes before later operations seen at cluster scope.
__device__ __forceinline__ void fence_acq_rel_cluster() {
    asm volatile("fence.acq_rel.cluster;" ::: "memory");
}

// As mbar_try_wait, with acquire at cluster scope: the writes that peer CTAs
// made before their release-arrivals on this barrier are visible after it.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Bounded like mbar_wait_bounded: gives up after kWaitLimitNs, sets the
// device error word and returns false.
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_cluster(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_device_error, kErrWaitTimeout);
            return false;
        }
    }
    return true;
}

// 16 bytes of a CTA's shared memory, by their address in the cluster window.
__device__ __forceinline__ uint4 ld_dsmem_v4(uint32_t cluster_addr) {
    uint4 v;
    asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(cluster_addr)
                 : "memory");
    return v;
}

// The leader CTA's copy of a barrier of this CTA: its shared::cta address with
// the pair bit cleared (the form the paired TMA load and commit expect).
__device__ __forceinline__ uint32_t pair_leader_addr(const void* p) {
    return smem_u32(p) & 0xFEFFFFFFu;
}

// Tensor memory for both CTAs of the pair: the same warp of each CTA runs
// these, with the same shared-memory slot.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t base, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols)
                 : "memory");
}

// D[tmem of both CTAs] (+)= A * B^T over the pair; leader thread only.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// When the leader's MMAs so far complete, arrive once on the barrier at this
// offset in every CTA of `cta_mask` (bit i = cluster rank i).
__device__ __forceinline__ void umma_commit_pair_mc(const uint64_t* bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
        "[%0], %1;" ::"r"(smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

// 3-D tiled load into this CTA's shared memory whose completed bytes count on
// the leader CTA's barrier (`leader_bar` from pair_leader_addr); each CTA loads its own half.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t leader_bar,
                                                 int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

}  // namespace tpr
