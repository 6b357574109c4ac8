/*
 * tp_reconcile.h -- C ABI of the tensor-parallel reconciliation point on one
 * B200 (sm_100a).
 *
 * The operation ("Interconnects e clusters", section 01 Conceito; NVL72 hosting
 * post, All-reduce section): a row-parallel projection -- the attention
 * out-projection or the FFN down-projection -- has its weight split across N
 * tensor-parallel ranks along the input dimension K. Rank r owns the slice
 * W_r = W[:, r*K/N : (r+1)*K/N] and computes the partial hidden vector
 * P_r = x_r . W_r^T over its slice of the input x. The N partials are summed
 * by a ring all-reduce -- a reduce-scatter in which each rank reduces one of
 * N chunks of H/N hidden columns, then an all-gather of the reduced chunks --
 * and the sum is added to the residual stream. Here all N ranks live in one
 * GPU's memory: the ring is its summation order, carried out on the device.
 *
 * Arithmetic of the product (identical bit for bit to the oracle's reading of
 * the pages):
 *   P[r][m][h] = bf16_rne( sum_k x[m][r*Ks+k] * Wr[h][k] )   fp32 accumulate
 *   chunk c = h / (H/N) is folded P_c, P_c+1, ..., P_c-1 (indices mod N), each
 *   add being bf16_rne(f32(s) + f32(P)), then
 *   out[m][h] = bf16_rne( f32(residual[m][h]) + f32(s) ).
 * TP_VARIANT_EXACT accumulates each partial with fused multiply-adds in
 * ascending k; TP_VARIANT_TENSOR accumulates on the tensor cores in fp32 in
 * the hardware's order (see tp_plan_set_variant).
 *
 * Conventions for every function below:
 *  - Element type: bf16 only (dtype argument TP_BF16). Tensors are dense and
 *    row-major as stated per argument.
 *  - Device pointers: every tensor argument is a CUDA device pointer on the
 *    plan's device, 16-byte aligned; the caller allocates and owns it. The
 *    library never allocates device memory and never synchronises the stream
 *    on the compute path: calls are asynchronous on `stream` (a cudaStream_t
 *    passed as void*; NULL means the legacy default stream).
 *  - Errors: arguments are checked before anything is launched; a failed
 *    check returns its status and launches nothing. A CUDA launch error maps
 *    to TP_ERR_CUDA (tp_last_cuda_error gives the CUDA code).
 *  - Threads: a plan is immutable after its set-up calls; concurrent calls
 *    with one plan are safe as long as they use distinct output and
 *    workspace buffers.
 */
#ifndef TP_RECONCILE_H
#define TP_RECONCILE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TP_API __attribute__((visibility("default")))
#else
#define TP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tp_plan tp_plan; /* opaque, host side, owned by the caller */

typedef enum {
    TP_OK = 0,
    TP_ERR_INVALID = 1,     /* bad shape, null pointer, aliasing, tokens > max */
    TP_ERR_ALIGN = 2,       /* pointer not 16-byte aligned */
    TP_ERR_UNSUPPORTED = 3, /* shape or variant the library has no kernel for */
    TP_ERR_WORKSPACE = 4,   /* workspace missing or too small */
    TP_ERR_CUDA = 5         /* CUDA runtime error (see tp_last_cuda_error) */
} tp_status;

enum { TP_BF16 = 0 };

typedef enum {
    TP_VARIANT_AUTO = 0,    /* TENSOR (the fastest on B200 at every token count) */
    TP_VARIANT_EXACT = 1,   /* CUDA cores, fp32 FMA chain per partial, k ascending */
    TP_VARIANT_TENSOR = 2,  /* tcgen05 tensor cores, fp32 accumulate in TMEM; the
                               partials go through the workspace (folded by the
                               CTA completing a tile for 1-2 tokens, else by a
                               ring kernel) */
    TP_VARIANT_CLUSTER = 3  /* the TENSOR kernels, folding the ranks on chip where
                               the N ranks x K parts of a tile make at most 8 CTAs
                               (at most 4 parts) and the token tile is at most 128:
                               one cluster of those CTAs, partials exchanged
                               through distributed shared memory, no workspace.
                               One kernel per call, but its CTAs stay until the
                               whole cluster has folded: in a chain of calls
                               slower than TENSOR on B200 */
} tp_variant;

/* Creates a plan for one projection shape.
 *   n_ranks     N, 1..8 tensor-parallel ranks
 *   max_tokens  largest M any call will pass (>= 0)
 *   k           projection input width K; K % N == 0 and (K/N) % 8 == 0
 *   hidden      H; H % N == 0 and (H/N) % 8 == 0
 *   dtype       TP_BF16
 * Records the current CUDA device; every later call must run with that
 * device current. On success *out owns a plan to release with
 * tp_plan_destroy. Returns TP_ERR_INVALID on a bad shape or null out,
 * TP_ERR_UNSUPPORTED for another dtype, TP_ERR_CUDA if no device is usable. */
TP_API tp_status tp_plan_create(tp_plan** out, int n_ranks, int64_t max_tokens, int64_t k,
                         int64_t hidden, int dtype);

/* Chooses the partial kernel and, for EXACT, whether the partials are staged.
 *   variant  a tp_variant
 *   staged   EXACT: 0 keeps the partials on chip, one kernel doing partials,
 *            ring fold and residual add (no workspace); 1 writes all N
 *            partials to the workspace and a separate ring kernel
 *            (tp_ring_reduce's) folds them. TENSOR (and AUTO) ignore it:
 *            see tp_plan_launches and tp_plan_workspace_bytes for where
 *            their partials go.
 * Call before the plan is shared between threads. */
TP_API tp_status tp_plan_set_variant(tp_plan* plan, int variant, int staged);

/* Bytes of workspace tp_rowlinear_reconcile needs for `tokens` tokens with
 * the plan's current setting; 0 when the partials stay on chip (EXACT, not
 * staged; TENSOR folding across a cluster). Otherwise the tensor-core
 * variant writes its partials to the workspace, whether its own kernel
 * folds them (one or two tokens: the CTA holding a tile's last ticket; more
 * than 128 tokens on CTA pairs: the CTA storing a half tile's last rank) or
 * a ring kernel does: N*M*H*2 bytes (bf16), or splits*N*M*H*4 (fp32 sums of
 * K parts) when it splits K across CTAs to fill the SMs; one or two tokens
 * store each part with its call's tag in one 8-byte word (N*M*H*8, or
 * splits*N*M*H*8).
 * Layout: a counter block (256-byte rounded) of 32-bit words -- per 128-row
 * H tile a ticket count (zero between calls) and a fold count (one more each
 * call), then per 256-row x 256-token tile of max_tokens two rank counts
 * (zero between calls) -- then the partials. Rounded up to 256 in all.
 * Returns 0 for a null plan or tokens <= 0. A workspace a call left with a
 * device error flag set must be zeroed again before its next use. */
TP_API size_t tp_plan_workspace_bytes(const tp_plan* plan, int64_t tokens);

/* The partial kernel a call with `tokens` tokens runs under the plan's
 * current setting: TP_VARIANT_EXACT or TP_VARIANT_TENSOR (AUTO and CLUSTER
 * resolved; CLUSTER runs the tensor-core kernels).
 * Returns -1 for a null plan or tokens < 1. A query only; launches nothing. */
TP_API int tp_plan_kernel_variant(const tp_plan* plan, int64_t tokens);

/* Kernels one tp_rowlinear_reconcile call with `tokens` tokens launches under
 * the plan's current setting: 1 (EXACT not staged; TENSOR when its partial
 * kernel also folds: for 1 or 2 tokens, for more than 128 tokens on CTA
 * pairs, and with CLUSTER across a cluster of the N ranks x K parts of a
 * tile when they make at most 8 CTAs and the token tile is at most 128) or
 * 2 (a partial kernel, then a ring fold kernel: TENSOR at 3 to 128 tokens);
 * 0 for tokens = 0; -1 for a null plan or tokens < 0. */
TP_API int tp_plan_launches(const tp_plan* plan, int64_t tokens);

/* Bytes of the packed weight buffer tp_pack_weights writes: N*H*(K/N)*2,
 * the size of the Linear weight. Returns 0 for a null plan. */
TP_API size_t tp_plan_packed_bytes(const tp_plan* plan);

/* S0, once per weight. Packs a torch Linear weight into the sharded layout.
 *   w_hk      [H][K] bf16, the Linear weight (input)
 *   w_packed  [N][H][K/N] bf16 (output): shard r is columns r*K/N ..
 *             (r+1)*K/N-1 of w_hk, rank-major, K/N innermost, so each rank's
 *             slice W_r is one contiguous block as on its own GPU
 * ("Interconnects e clusters", 01 Conceito: each weight matrix is divided
 * between the ranks.) The buffers must not overlap. */
TP_API tp_status tp_pack_weights(const tp_plan* plan, const void* w_hk, void* w_packed, void* stream);

/* S1-S4: one reconciliation point.
 *   x          [M][K] bf16 activations (rank r reads columns r*K/N ..)
 *   w_packed   [N][H][K/N] bf16 from tp_pack_weights
 *   residual   [M][H] bf16
 *   out        [M][H] bf16 (output); must not overlap any input or the workspace
 *   tokens     M, 0 <= M <= max_tokens (M = 0 launches nothing)
 *   workspace  tp_plan_workspace_bytes(plan, M) bytes of device memory, or
 *              NULL when that is 0. Zero it before its first use: its fold
 *              counters (see tp_plan_workspace_bytes) must start at zero, and
 *              every call that sets no device error flag leaves them zero
 *              again, so one zeroed workspace serves any number of calls (of
 *              any plans with the same H, in stream order). After a call that
 *              set a device error flag, zero it again. The rest of its
 *              contents on entry are ignored.
 * Partials per the header comment, summed in ring order, then the residual
 * add ("Interconnects e clusters", 01 Conceito: the slices are summed before
 * the residual stream continues). */
TP_API tp_status tp_rowlinear_reconcile(const tp_plan* plan, const void* x, const void* w_packed,
                                 const void* residual, void* out, int64_t tokens,
                                 void* workspace, void* stream);

/* One reconciliation point exactly like tp_rowlinear_reconcile (same
 * arguments, same kernels, same result), for callers that cannot allocate
 * device memory: code that runs while a CUDA graph is being captured
 * (allocation is not an operation a capture can record), latency-critical
 * decode loops (cudaMalloc may synchronize the device), and hosts whose
 * device memory is budgeted up front by an embedding framework. Instead of a
 * caller-supplied workspace, the partials that this call stages (the
 * tensor-core variant, or a staged plan) go to a fixed scratch array inside
 * the library: 16 MiB, a file-scope device array that every GPU loading the
 * library holds until the process exits. Its device address is looked up
 * once per device when a plan is created on it, so this call does no set-up
 * of its own and allocates nothing.
 *  - Returns TP_ERR_WORKSPACE, launching nothing, when the call needs more
 *    scratch than that: staged partials above 16 MiB - 8 KiB (N*M*H*2
 *    bytes, or splits*N*M*H*4; e.g. N=8, M=64, H=4096 needs 4 MiB), or
 *    H > 131072 (the first 8 KiB hold the fold counters of every plan).
 *  - Every call, from every plan and thread on a device, shares the one
 *    array, which keeps the last call's partials; each call writes every
 *    partial it reads. The fold counters at its start are zero when the
 *    library is loaded; every call that sets no device error flag leaves the
 *    ticket counts at zero (and each tile's fold count one higher); after one
 *    that does, this entry point may give wrong results until
 *    tp_device_error_flags with reset != 0 clears the whole array. Calls whose kernels overlap
 *    on the GPU (different streams without ordering between them) race on
 *    the array and give wrong results: order them on one stream.
 * The pages describe no counterpart of this entry point. */
TP_API tp_status tp_rowlinear_reconcile_noalloc(const tp_plan* plan, const void* x,
                                                const void* w_packed, const void* residual,
                                                void* out, int64_t tokens, void* stream);

/* S1 only: the N partials, no ring, no residual.
 *   partials  [N][M][H] bf16 (output)
 * Same x, w_packed and tokens rules as tp_rowlinear_reconcile. */
TP_API tp_status tp_rowlinear_partials(const tp_plan* plan, const void* x, const void* w_packed,
                                void* partials, int64_t tokens, void* stream);

/* S2-S4 only: ring reduce-scatter fold in ring order, the all-gather (one
 * result buffer stands for every rank's copy) and the residual add.
 *   partials  [N][M][H] bf16
 *   residual  [M][H] bf16
 *   out       [M][H] bf16 (output, must not overlap the inputs)
 * (NVL72 hosting post, All-reduce section: each peer reduces one of N slices
 * of the input, then broadcasts it to the rest.) */
TP_API tp_status tp_ring_reduce(const tp_plan* plan, const void* partials, const void* residual,
                         void* out, int64_t tokens, void* stream);

/* S5: bytes each rank puts on its wire for `points` ring all-reduces of
 * tokens x hidden elements of elem_bytes each: 2(N-1)/N times the payload
 * ("Interconnects e clusters", 01 Conceito: 1.25 MiB per token at N=2 and
 * about 1.875 MiB at N=4 for H=5120 bf16 and 128 reconciliations per token).
 * Host only, exact (multiplies before the one division). Returns 0 for
 * n_ranks < 1 or a negative argument. */
TP_API uint64_t tp_ring_bytes(int n_ranks, int64_t tokens, int64_t hidden, int elem_bytes,
                       int64_t points);

/* ---------------------------------------------------------------------
 * The ring all-reduce as a protocol between ranks that each hold their own
 * buffers: S2-S4 as N tensor-parallel GPUs run them ("Interconnects e
 * clusters", 01 Conceito: a reduce-scatter and an all-gather of H/N-wide
 * chunks; NVL72 hosting post, All-reduce section: each peer reduces one slice,
 * then broadcasts it). Rank r pulls each chunk from its predecessor r-1 once
 * the predecessor's step flag shows it written: reduce-scatter steps s =
 * 0..N-2 fold chunk r-1-s into rank r's buffer (bf16 round-to-nearest-even
 * per add, the received sum on the left), all-gather steps pass the reduced
 * chunks on, and every rank adds the residual to every chunk. Every rank's
 * output equals tp_ring_reduce's on the same partials, bit for bit.
 * ------------------------------------------------------------------- */

/* Bytes of one rank's workspace for tp_ring_allreduce_ranks: its step flags
 * (one 32-bit flag per CTA of the rank, 256-byte rounded) first, then two
 * [M][H] bf16 buffers (reduce-scatter, all-gather), each 256-byte rounded.
 * 0 for a null plan or tokens outside 0..max_tokens. */
TP_API size_t tp_ring_rank_workspace_bytes(const tp_plan* plan, int64_t tokens);

/* Runs ranks first_rank .. first_rank + launch_ranks - 1 of the ring
 * protocol in one launch on the current stream.
 *   partials    [N] device pointers: rank r's partial [M][H] bf16
 *   residual    [M][H] bf16 (the residual every rank adds)
 *   outs        [N] device pointers: rank r's output [M][H] bf16
 *   workspaces  [N] device pointers of tp_ring_rank_workspace_bytes each,
 *               the flag block zeroed before the first call; every call
 *               that completes leaves the flags equal again, so the same
 *               workspaces serve any number of calls (after a call that set
 *               the error bit, zero the flag blocks again)
 *   wait_limit_ns  the bound of every wait on another rank's flag (0: 1 s);
 *               a wait that runs out sets bit 1 of the device error word
 *               (tp_device_error_flags) and that part of the rank stops
 * The arrays are host arrays. On one GPU (all ranks in memory of this
 * device) launch all N ranks at once: the launch is cooperative, so all their
 * CTAs are resident together. With one GPU per rank, each process launches
 * its own rank with the other ranks' buffers as peer pointers (peer memory is
 * read with plain loads only). Launching only some ranks of a group whose
 * other ranks never run makes their waits run out: a test of the bound.
 * Checks: pointers non-null and 16-byte aligned, outputs and workspaces
 * disjoint from each other and from the inputs, ranks within 0..N-1. */
TP_API tp_status tp_ring_allreduce_ranks(const tp_plan* plan, const void* const* partials,
                                         const void* residual, void* const* outs,
                                         void* const* workspaces, int first_rank, int launch_ranks,
                                         int64_t tokens, uint64_t wait_limit_ns, void* stream);

/* ---------------------------------------------------------------------
 * MXFP8 weight shards. The NVL72 hosting post stores the MoE GEMM's weights
 * as MXFP8; the format here is the OCP Microscaling v1.0 MXFP8 (E4M3)
 * applied to each rank's slice: every 32 consecutive weights along K share
 * one E8M0 scale X = 2^s (byte s + 127), s = floor(log2 max|w|) - 8 clamped
 * to [-127, 127] (-127 for an all-zero run), and each weight is the E4M3
 * code nearest to w / X, ties to even, saturating at +-448. The
 * reconciliation over such shards is S1-S4 over the dequantised weights
 * E4M3 * X, which are exact in bf16 for any run whose largest weight is at
 * least 2^-116. Requires (K/N) % 64 == 0.
 * ------------------------------------------------------------------- */

/* Sizes of the two shard buffers: q_bytes = H*K (one E4M3 code per weight,
 * [N][H][K/N]), scale_bytes = N * ceil(H/128) * ceil(K/N/128) * 512: the
 * E8M0 scales in 512-byte chunks [N][ceil(H/128)][ceil(K/N/128)], one per
 * rank, 128-row tile and 128 columns (four 32-weight runs) of a rank slice;
 * row t of the tile, run j of the four at byte 16 (t % 32) + 4 (t / 32) + j
 * of the chunk (the order in which the block-scaled MMA reads scales from
 * tensor memory); rows past H and runs past K/N hold 0. TP_ERR_UNSUPPORTED
 * when K/N is not a multiple of 64; TP_ERR_INVALID for null arguments. */
TP_API tp_status tp_plan_mxfp8_bytes(const tp_plan* plan, size_t* q_bytes, size_t* scale_bytes);

/* S0 for MXFP8: Linear weight [H][K] bf16 -> w_q codes and w_scales (device
 * buffers of tp_plan_mxfp8_bytes' sizes and layouts; all 16-byte aligned; no
 * overlap). Asynchronous on `stream`; the result is identical, bit for bit,
 * to the format's definition above. */
TP_API tp_status tp_pack_weights_mxfp8(const tp_plan* plan, const void* w_hk, void* w_q,
                                       void* w_scales, void* stream);

/* Bytes of workspace tp_rowlinear_reconcile_mxfp8 needs for `tokens` tokens
 * (0 when the call folds in clusters and stages nothing); the same layout
 * and zeroing rule as tp_rowlinear_reconcile's workspace. Whatever the
 * plan's variant, MXFP8 calls run on the tensor cores. 0 for a null plan or
 * tokens <= 0. */
TP_API size_t tp_plan_mxfp8_workspace_bytes(const tp_plan* plan, int64_t tokens);

/* S1-S4 over MXFP8 shards, on the tensor cores:
 *   x, residual, out, tokens as in tp_rowlinear_reconcile; w_q, w_scales
 *   from tp_pack_weights_mxfp8; workspace of
 *   tp_plan_mxfp8_workspace_bytes(plan, tokens) bytes (NULL when 0), zeroed
 *   before its first use.
 * More than 8 tokens: code tiles are widened to bf16 tiles in tensor memory
 * (E4M3 * 2^s, exact) and multiplied with the bf16 activations in fp32 on
 * the tensor cores. At most 8 tokens: the codes and scales go to the
 * block-scaled MMA (kind::mxf8f6f4) as stored, and each 32-value run of the
 * activations is split on chip into two E4M3 terms with E8M0 scales,
 * x = 2^e1 q1 + 2^e2 q2 with e1 = floor(log2 max|run|) - 7: exact for every
 * x of at least 2^(e1 - 6), within 2^(e1 - 14) below that (plus 2^-137 for
 * runs whose remainders fall below 2^-119). Either way the partials are
 * fp32 sums rounded once to bf16 and folded in ring order with the
 * residual, as for bf16 shards. TP_ERR_UNSUPPORTED when K/N is not a
 * multiple of 64. */
TP_API tp_status tp_rowlinear_reconcile_mxfp8(const tp_plan* plan, const void* x, const void* w_q,
                                              const void* w_scales, const void* residual,
                                              void* out, int64_t tokens, void* workspace,
                                              void* stream);

/* ---------------------------------------------------------------------
 * NVFP4 weight shards. The TP=4-vs-TP=8 post runs NVFP4 weights with
 * 16-bit activations; the format is NVIDIA's NVFP4 applied to each rank's
 * slice: FP4 E2M1 elements, one FP8 E4M3 block scale per 16 consecutive
 * weights along K, and a second-level scale 2^g for the whole weight, g the
 * smallest integer with max|W| / 2^g <= 6 * 448 (0 for an all-zero weight):
 *   block scale b = E4M3 nearest to max|block| / (6 * 2^g), ties to even;
 *   element     q = E2M1 nearest to w / (b * 2^g), ties to even, saturating
 *                   at +-6 (0 where b is 0).
 * (The second-level scale is a power of two so that every dequantised weight
 * q * b * 2^g is exact in bf16.) The reconciliation over such shards is
 * S1-S4 over the dequantised weights. Requires (K/N) % 64 == 0.
 * ------------------------------------------------------------------- */

/* Sizes of the two shard buffers: q_bytes = H*K/2 ([N][H][K/N/2], two E2M1
 * codes a byte, the earlier k in bits 0-3); scale_bytes = H*K/16 + 16: the
 * block scales laid out [N][K/N/64][H][4] (the four scales of each row for
 * one 64-column block, row after row), then 16 bytes holding g (int32) and
 * the weight's largest magnitude. TP_ERR_UNSUPPORTED when K/N is not a
 * multiple of 64; TP_ERR_INVALID for null arguments. */
TP_API tp_status tp_plan_nvfp4_bytes(const tp_plan* plan, size_t* q_bytes, size_t* scale_bytes);

/* S0 for NVFP4: Linear weight [H][K] bf16 -> w_q codes and w_scales (device
 * buffers of tp_plan_nvfp4_bytes' sizes; all 16-byte aligned; no overlap).
 * Two kernels (the weight's largest magnitude, then the blocks), async on
 * `stream`; identical, bit for bit, to the definition above. */
TP_API tp_status tp_pack_weights_nvfp4(const tp_plan* plan, const void* w_hk, void* w_q,
                                       void* w_scales, void* stream);

/* Workspace of tp_rowlinear_reconcile_nvfp4 (as for MXFP8). */
TP_API size_t tp_plan_nvfp4_workspace_bytes(const tp_plan* plan, int64_t tokens);

/* S1-S4 over NVFP4 shards on the tensor cores, as
 * tp_rowlinear_reconcile_mxfp8: code tiles widened to bf16 tiles in shared
 * memory (E2M1 * block scale * 2^g, exact), multiplied with the bf16
 * activations in fp32, partials rounded once to bf16 and folded in ring
 * order with the residual. */
TP_API tp_status tp_rowlinear_reconcile_nvfp4(const tp_plan* plan, const void* x, const void* w_q,
                                              const void* w_scales, const void* residual,
                                              void* out, int64_t tokens, void* workspace,
                                              void* stream);

/* All-reduce schemes of tp_allreduce_bytes. */
typedef enum {
    TP_ALLREDUCE_RING = 0,   /* reduce the slices, then broadcast them */
    TP_ALLREDUCE_NAIVE = 1,  /* every rank loads every peer's whole buffer */
    TP_ALLREDUCE_SWITCH = 2  /* the switch sums each slice (SHARP, multimem) */
} tp_allreduce_scheme;

/* Bytes one rank's NVLink port carries for the all-reduce of B = tokens *
 * hidden * elem_bytes * points bytes per rank, under the schemes of the NVL72
 * hosting post's All-reduce section:
 *   RING    2(N-1)/N * B   (= tp_ring_bytes; N ranks move 2(N-1)B in all)
 *   NAIVE   (N-1) * B      (N(N-1)B read in all)
 *   SWITCH  B              (the peers' N-1 copies of the rank's slice are
 *                           read by the switch, which returns one reduced
 *                           slice: N/(2(N-1)) of the ring's transfers)
 * Reading: the switch scheme counts, like the page, the transfers of the
 * reduction of one rank's slice on both sides of the switch. Host only,
 * exact (multiplies before the one division). Returns 0 for one rank, an
 * unknown scheme, n_ranks < 1 or a negative argument. The pages' kernels for
 * these schemes run across GPUs; this is their byte model only. */
TP_API uint64_t tp_allreduce_bytes(int scheme, int n_ranks, int64_t tokens, int64_t hidden,
                                   int elem_bytes, int64_t points);

/* Bytes one rank's NVLink port carries for the combine step of an MoE layer
 * (NVL72 hosting post, MoE dispatch/combine section): the combine first
 * accumulates, on each rank, the weighted contributions of the experts the
 * rank hosts for every token, then all-reduces the accumulated
 * [tokens][hidden] buffer of elem_bytes elements across the N ranks under
 * `scheme` (a tp_allreduce_scheme).
 *   local_accumulate 1  the post's combine: one all-reduce, tp_allreduce_bytes
 *                       of the buffer (points = 1), whatever top_k is;
 *                    0  for comparison: each of a token's top_k expert slots
 *                       all-reduced on its own, top_k times that.
 * Host only, exact. Returns 0 for top_k < 1, local_accumulate not 0 or 1,
 * and wherever tp_allreduce_bytes returns 0. A byte model only: the expert
 * GEMMs and the routing are not part of this library. */
TP_API uint64_t tp_moe_combine_bytes(int scheme, int n_ranks, int64_t tokens, int64_t hidden,
                                     int elem_bytes, int64_t top_k, int local_accumulate);

/* Releases a plan. NULL is allowed. */
TP_API void tp_plan_destroy(tp_plan* plan);

/* Static, NUL-terminated text for a status value. */
TP_API const char* tp_status_string(tp_status status);

/* The CUDA error code behind the calling thread's last TP_ERR_CUDA
 * (0 if none). */
TP_API int tp_last_cuda_error(void);

/* Reads, and with reset != 0 clears, the device-side error word of the
 * plan's device: bit 1 is set when a wait of tp_ring_allreduce_ranks on
 * another rank's flag ran out; bit 0 is set when a kernel's bounded wait on a
 * pipeline barrier ran out (the kernel then stops early, so its output is invalid;
 * copies or tensor-core operations it had in flight may not have finished
 * when it returned, so the context should be discarded, e.g. by
 * cudaDeviceReset, before results are trusted again). With reset != 0 and a
 * nonzero word it also zeroes the fold counters of the library's own
 * scratch array (tp_rowlinear_reconcile_noalloc); a caller's workspace must
 * be zeroed by the caller. Synchronises the device. */
TP_API tp_status tp_device_error_flags(const tp_plan* plan, uint32_t* flags, int reset);

#ifdef __cplusplus
}
#endif

#endif /* TP_RECONCILE_H */
