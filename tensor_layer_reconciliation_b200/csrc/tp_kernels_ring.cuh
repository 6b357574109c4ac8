// The ring all-reduce run as a protocol between ranks that each hold their
// own buffers (S2-S4 as N tensor-parallel GPUs would run them).
//
// "Interconnects e clusters", 01 Conceito: the ring all-reduce puts
// 2(N-1)/N of the payload on each rank's link -- a reduce-scatter, then an
// all-gather, of H/N-wide chunks. NVL72 hosting post, All-reduce section:
// each peer reduces one slice of the input, then broadcasts it to the rest.
//
// Rank r owns, in its own memory: its partial P_r [M][H] (input), a
// reduce-scatter buffer work_r and an all-gather buffer gather_r ([M][H]
// each), its output out_r [M][H] and one step flag per CTA of the rank.
// Chunk c is columns c*H/N .. (c+1)*H/N-1 of every token. Rank r pulls from
// its ring predecessor p = r-1 (mod N):
//   reduce-scatter step s = 0 .. N-2, chunk c = r-1-s (mod N):
//       work_r[c] = bf16(src[c] + P_r[c]),  src = P_p (s = 0) or work_p (s > 0)
//     (after step N-2 rank r holds the full sum of chunk r+1 in work_r)
//   all-gather step s = 0 .. N-2, chunk c = r-s (mod N):
//       v = work_p[c] (s = 0) or gather_p[c] (s > 0);  gather_r[c] = v
//   out_r[c] = bf16(residual[c] + v) for every chunk, its own (r+1) included.
// This is the order the oracle's message-by-message ring reaches: chunk c is
// folded P_c, P_c+1, ..., P_c-1 from the left; every add rounds to bf16.
// A buffer slot is written once per call and never rewritten, so a reader
// needs only the writer's progress: step t of rank r waits until its
// predecessor's flag shows step t-1 done (the flag's value at entry plus t).
// Flags only grow (the base of a call is the CTA's own flag at entry, which
// every CTA of every rank shares after a complete call), so one zeroed flag
// block serves any number of calls. At the end a rank waits until its
// successor has finished reading its buffers, so a next call may reuse them.
//
// CTA g of every rank takes the same slice of each chunk (16-byte vectors
// g*V/G .. (g+1)*V/G-1 of the chunk's M*H/(8N) vectors), so it depends only
// on CTA g of its predecessor. Every wait is bounded (wait_limit_ns of
// %globaltimer); a wait that runs out sets bit 1 of the device error word and
// the CTA stops (its rank's later steps are not done).
//
// Launched for ranks first_rank .. first_rank + launch_ranks - 1: one GPU
// emulating the whole group launches all N ranks at once, cooperatively, so
// all their CTAs are resident together; one GPU per rank would launch its own
// rank, with the other ranks' buffers given as peer pointers (plain loads
// only, no bulk or tensor copies of peer memory).
#pragma once

#include "tp_common.cuh"

namespace tpr {

constexpr uint32_t kErrPeerTimeout = 2u;   // device error word bit 1
constexpr int kRingThreads = 256;

struct RingRanks {
    const uint16_t* partial[kMaxRanks];  // P_r [M][H]
    uint16_t* work[kMaxRanks];           // reduce-scatter buffer [M][H]
    uint16_t* gather[kMaxRanks];         // all-gather buffer [M][H]
    uint16_t* out[kMaxRanks];            // out_r [M][H]
    uint32_t* flags[kMaxRanks];          // [ctas_per_rank] step flags
};

struct RingParams {
    int n_ranks;
    int first_rank;
    int ctas_per_rank;      // G
    int hidden;             // H
    int hc;                 // H / N
    int64_t tokens;         // M
    const uint16_t* residual;   // [M][H]
    uint64_t wait_limit_ns;
};

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// 16 bytes another CTA (or another GPU) wrote during this kernel: through L2,
// never a stale L1 line.
__device__ __forceinline__ uint4 ld_cg_v4(const uint16_t* p) {
    return __ldcg(reinterpret_cast<const uint4*>(p));
}

// Waits until *flag has reached `target` (wrap-safe: the flags only grow),
// at most limit_ns. Thread 0 of the CTA only.
__device__ __forceinline__ bool ring_wait(const uint32_t* flag, uint32_t target, uint64_t limit_ns) {
    if (static_cast<int32_t>(ld_acquire_sys(flag) - target) >= 0) return true;
    const uint64_t t0 = globaltimer_ns();
    while (static_cast<int32_t>(ld_acquire_sys(flag) - target) < 0) {
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(&g_device_error, kErrPeerTimeout);
            return false;
        }
        __nanosleep(64);
    }
    return true;
}

__device__ __forceinline__ uint4 bf16x8_add(uint4 a, uint4 b) {
    return make_uint4(bf16x2_add(a.x, b.x), bf16x2_add(a.y, b.y), bf16x2_add(a.z, b.z),
                      bf16x2_add(a.w, b.w));
}

__global__ void __launch_bounds__(kRingThreads)
    ring_protocol_kernel(const RingRanks rk, const RingParams p) {
    __shared__ int go;
    const int N = p.n_ranks;
    const int r = p.first_rank + static_cast<int>(blockIdx.x) / p.ctas_per_rank;
    const int g = static_cast<int>(blockIdx.x) % p.ctas_per_rank;
    const int G = p.ctas_per_rank;
    const int pred = r == 0 ? N - 1 : r - 1;
    const int succ = r == N - 1 ? 0 : r + 1;
    const int64_t vrow = p.hc / 8;                   // vectors of a chunk per token
    const int64_t V = p.tokens * vrow;               // vectors of a chunk
    const int64_t v0 = V * g / G, v1 = V * (g + 1) / G;
    uint32_t* my_flag = rk.flags[r] + g;
    const uint32_t* pred_flag = rk.flags[pred] + g;
    const uint32_t* succ_flag = rk.flags[succ] + g;
    // element offset of vector v of chunk c
    auto offset = [&](int c, int64_t v) {
        const int64_t m = v / vrow;
        return static_cast<size_t>(m) * p.hidden + static_cast<size_t>(c) * p.hc +
               static_cast<size_t>(v - m * vrow) * 8;
    };
    const uint32_t base = *reinterpret_cast<volatile uint32_t*>(my_flag);
    // step t (0 .. 2N-3) of this rank is done: flag = base + t + 1
    auto publish = [&](uint32_t t) {
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) st_release_sys(my_flag, base + t + 1);
    };
    // the predecessor has done its step t - 1 (t = 0 needs nothing)
    auto await_pred = [&](uint32_t t) -> bool {
        if (threadIdx.x == 0) go = t == 0 || ring_wait(pred_flag, base + t, p.wait_limit_ns);
        __syncthreads();
        return go != 0;
    };
    if (N == 1) {   // no ring: out = residual + P_0
        for (int64_t v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
            const size_t o = offset(0, v);
            const uint4 res = ld_global_nc_v4(p.residual + o);
            st_global_v4(rk.out[r] + o, bf16x8_add(res, ld_global_nc_v4(rk.partial[r] + o)));
        }
        return;
    }
    // ------------------------------------------------------ reduce-scatter --
    for (int s = 0; s < N - 1; ++s) {
        if (!await_pred(static_cast<uint32_t>(s))) return;
        const int c = ((r - 1 - s) % N + N) % N;
        const uint16_t* src = s == 0 ? rk.partial[pred] : rk.work[pred];
        for (int64_t v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
            const size_t o = offset(c, v);
            const uint4 a = ld_cg_v4(src + o);               // the chunk so far (left operand)
            const uint4 b = ld_global_nc_v4(rk.partial[r] + o);
            st_global_v4(rk.work[r] + o, bf16x8_add(a, b));
        }
        publish(static_cast<uint32_t>(s));
    }
    // this rank's fully reduced chunk: its output
    {
        const int c = (r + 1) % N;
        for (int64_t v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
            const size_t o = offset(c, v);
            const uint4 res = ld_global_nc_v4(p.residual + o);
            st_global_v4(rk.out[r] + o, bf16x8_add(res, ld_cg_v4(rk.work[r] + o)));
        }
    }
    // ----------------------------------------------------------- all-gather --
    for (int s = 0; s < N - 1; ++s) {
        const uint32_t t = static_cast<uint32_t>(N - 1 + s);
        if (!await_pred(t)) return;
        const int c = ((r - s) % N + N) % N;
        const uint16_t* src = s == 0 ? rk.work[pred] : rk.gather[pred];
        for (int64_t v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
            const size_t o = offset(c, v);
            const uint4 val = ld_cg_v4(src + o);
            st_global_v4(rk.gather[r] + o, val);
            const uint4 res = ld_global_nc_v4(p.residual + o);
            st_global_v4(rk.out[r] + o, bf16x8_add(res, val));
        }
        publish(t);
    }
    // the successor has read everything it needs from this rank's buffers
    if (threadIdx.x == 0) (void)ring_wait(succ_flag, base + static_cast<uint32_t>(2 * N - 2), p.wait_limit_ns);
}

}  // namespace tpr
