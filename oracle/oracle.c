/*
 * ORACLE for the tensor-parallel reconciliation point -- TEST INFRASTRUCTURE.
 *
 * A plain, slow, obviously correct CPU implementation of what the GPU path
 * computes. Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline leg load this library; the product path never does, and this
 * file shares no code, header or table with the CUDA library.
 *
 * What it computes ("Interconnects e clusters", section 01 Conceito, and the
 * all-reduce section of the NVL72 hosting post):
 *   1. Partials. Each of N ranks owns the K/N-wide slice r of the projection
 *      input; rank r's partial hidden vector is x_r . W_r (the weight matrix
 *      is split between ranks, each rank computes a partial result over its
 *      slice). Reading of an unstated step: the products are accumulated in
 *      fp32, k ascending, starting from +0, each product added to the running
 *      sum with one rounding (fused multiply-add, round-to-nearest-even; the
 *      product of two bf16 values is exact in fp32 unless it underflows, so
 *      this is also "round the product, then add" everywhere else), and the
 *      sum is rounded once to bf16 for the wire.
 *   2. Ring all-reduce. The partials are summed before the residual stream
 *      continues, by a ring all-reduce that puts 2(N-1)/N times the payload on
 *      each rank's wire: a reduce-scatter in which each rank reduces one of N
 *      slices, then a broadcast (all-gather) of the reduced slices. Simulated
 *      literally with N rank-local buffers: at reduce-scatter step s rank r
 *      sends chunk (r - s) mod N to rank (r + 1) mod N, which stores
 *      bf16_rne(f32(received) + f32(own)). Reading: chunks are H/N-wide column
 *      ranges of each token's hidden vector; chunk c is folded P_c, P_c+1, ...,
 *      P_c-1, left to right.
 *   3. Residual. out = bf16_rne(f32(residual) + f32(reduced)).
 *   4. MXFP8 weight shards (the "next" weight format): quantisation of the
 *      Linear weight to E4M3 codes with one E8M0 scale per 32 weights of a
 *      rank's slice, and back; a reconciliation over such shards is the
 *      point above over the dequantised weights (exact in bf16).
 *   5. NVFP4 weight shards: E2M1 codes with one E4M3 scale per 16 weights
 *      and a power-of-two second-level scale, and back (exact in bf16).
 *   6. Byte models: the ring's 2(N-1)/N per rank, the naive, ring and switch
 *      all-reduce schemes, and the MoE combine (local accumulation, then one
 *      all-reduce).
 *
 * Build: plain C11, -ffp-contract=off (no fused multiply-add other than the
 * explicit fmaf), no fast-math, so every float operation is one IEEE
 * round-to-nearest-even operation with subnormals kept.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARGS 1
#define ORC_ERR_ALLOC 2
#define ORC_ERR_RING 3

/* ---------------------------------------------------------------- bf16 -- */

/* bf16 bits -> float: the bf16 pattern is the top half of the float. */
float orc_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* float -> bf16, round to nearest, ties to even, on the bit pattern: add
 * 0x7FFF plus the bit that will become the last kept bit, keep the top half.
 * A carry out of the fraction bumps the exponent, which is the correct result
 * (up to overflow into infinity). NaN keeps its sign and becomes the quiet NaN
 * 0x7FC0. Subnormals are not flushed. */
uint16_t orc_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0u)
        return (uint16_t)(((u >> 16) & 0x8000u) | 0x7FC0u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* double -> bf16, correctly rounded (to nearest, ties to even) straight from
 * the double, by scaling to the bf16 quantum of |v| and rounding to an
 * integer: quantum 2^(e-8) for |v| in [2^(e-1), 2^e) (8 significant bits),
 * never finer than the subnormal quantum 2^-133. Used to classify partials
 * whose fp64 value lies near a bf16 rounding boundary. */
uint16_t orc_bf16_rne_f64(double v)
{
    if (isnan(v))
        return (uint16_t)((signbit(v) ? 0x8000u : 0u) | 0x7FC0u);
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0)
        return sign;
    int ex;
    (void)frexp(a, &ex);               /* a = f * 2^ex, f in [0.5, 1) */
    int q = ex - 8;
    if (q < -133)
        q = -133;
    double r = nearbyint(ldexp(a, -q)); /* default rounding mode: ties to even */
    double res = ldexp(r, q);
    if (res >= 0x1p128)
        return (uint16_t)(sign | 0x7F80u);
    float rf = (float)res;             /* exact: res has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &rf, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

/* ------------------------------------------------------------ partials -- */

typedef struct {
    int n_ranks;
    int64_t tokens, k, n_rows, row_begin, row_end;
    const uint16_t *x, *w_rows;
    uint16_t *p;
    double *p64, *pabs;
} partial_job;

static void partial_rows(const partial_job *j)
{
    const int64_t ks = j->k / j->n_ranks;
    for (int r = 0; r < j->n_ranks; ++r)
        for (int64_t m = 0; m < j->tokens; ++m)
            for (int64_t i = j->row_begin; i < j->row_end; ++i) {
                const uint16_t *xr = j->x + m * j->k + (int64_t)r * ks;
                const uint16_t *wr = j->w_rows + i * j->k + (int64_t)r * ks;
                float acc = 0.0f;
                double d = 0.0, a = 0.0;
                for (int64_t kk = 0; kk < ks; ++kk) {
                    acc = fmaf(orc_f32(xr[kk]), orc_f32(wr[kk]), acc);
                    double dp = (double)orc_f32(xr[kk]) * (double)orc_f32(wr[kk]);
                    d += dp;
                    a += fabs(dp);
                }
                int64_t o = ((int64_t)r * j->tokens + m) * j->n_rows + i;
                j->p[o] = orc_bf16_rne(acc);
                if (j->p64)
                    j->p64[o] = d;
                if (j->pabs)
                    j->pabs[o] = a;
            }
}

static void *partial_thread(void *arg)
{
    partial_rows((const partial_job *)arg);
    return NULL;
}

/* Partials of the selected output rows.
 *   x       [tokens][k]     bf16 activations (the full projection input)
 *   w_rows  [n_rows][k]     the selected rows h of the Linear weight W[H][K]
 *   p       [n_ranks][tokens][n_rows]  bf16 partials (out)
 *   p64     same shape, fp64 sum of the same products (out, may be NULL)
 *   pabs    same shape, fp64 sum of |products| (out, may be NULL)
 * Rows are split across n_threads threads; every element is computed by one
 * thread in the same order, so the result does not depend on n_threads. */
int orc_partials(int n_ranks, int64_t tokens, int64_t k, const uint16_t *x,
                 int64_t n_rows, const uint16_t *w_rows, uint16_t *p, double *p64,
                 double *pabs, int n_threads)
{
    if (n_ranks < 1 || tokens < 0 || k < 0 || n_rows < 0 || k % n_ranks != 0)
        return ORC_ERR_ARGS;
    if ((tokens && k && !x) || (n_rows && k && !w_rows) || (n_rows && tokens && !p))
        return ORC_ERR_ARGS;
    if (n_threads < 1)
        n_threads = 1;
    if (n_threads > n_rows)
        n_threads = n_rows > 0 ? (int)n_rows : 1;
    partial_job *jobs = calloc((size_t)n_threads, sizeof *jobs);
    pthread_t *th = calloc((size_t)n_threads, sizeof *th);
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return ORC_ERR_ALLOC;
    }
    for (int t = 0; t < n_threads; ++t) {
        partial_job *j = &jobs[t];
        j->n_ranks = n_ranks;
        j->tokens = tokens;
        j->k = k;
        j->n_rows = n_rows;
        j->row_begin = n_rows * t / n_threads;
        j->row_end = n_rows * (t + 1) / n_threads;
        j->x = x;
        j->w_rows = w_rows;
        j->p = p;
        j->p64 = p64;
        j->pabs = pabs;
    }
    int started = 0;
    for (int t = 1; t < n_threads; ++t) {
        if (pthread_create(&th[t], NULL, partial_thread, &jobs[t]) != 0)
            break;
        started = t;
    }
    partial_rows(&jobs[0]);
    for (int t = 1; t <= started; ++t)
        pthread_join(th[t], NULL);
    for (int t = started + 1; t < n_threads; ++t) /* threads that failed to start */
        partial_rows(&jobs[t]);
    free(jobs);
    free(th);
    return ORC_OK;
}

/* ---------------------------------------------------------------- ring -- */

/* Ring all-reduce of the partials, simulated message by message.
 *   hidden    H, the full hidden size (chunks are H/N wide)
 *   cols      [n_cols] the global column h of each stored column; the ring
 *             runs on whatever subset of columns is given, each column in
 *             the chunk h / (H/N) it belongs to
 *   p         [n_ranks][tokens][n_cols] bf16 partials
 *   reduced   [tokens][n_cols] bf16 all-reduced sum (out)
 *   bytes_sent [n_ranks] bytes each rank put on its wire (out, may be NULL);
 *             every message is a whole chunk of tokens * H/N bf16 values
 * Returns ORC_ERR_RING if the ranks do not end with identical buffers. */
int orc_ring(int n_ranks, int64_t tokens, int64_t hidden, int64_t n_cols,
             const int64_t *cols, const uint16_t *p, uint16_t *reduced,
             uint64_t *bytes_sent)
{
    if (n_ranks < 1 || tokens < 0 || hidden < 0 || n_cols < 0 || hidden % n_ranks != 0)
        return ORC_ERR_ARGS;
    const int N = n_ranks;
    const int64_t hc = hidden / N;
    const int64_t plane = tokens * n_cols;
    for (int64_t i = 0; i < n_cols; ++i)
        if (cols[i] < 0 || cols[i] >= hidden)
            return ORC_ERR_ARGS;
    if (bytes_sent)
        for (int r = 0; r < N; ++r)
            bytes_sent[r] = 0;
    if (plane == 0)
        return ORC_OK;

    uint16_t *buf = malloc((size_t)N * (size_t)plane * sizeof *buf);  /* buf[r] */
    uint16_t *msg = malloc((size_t)N * (size_t)plane * sizeof *msg);  /* in flight */
    int *chunk_of = malloc((size_t)n_cols * sizeof *chunk_of);
    if (!buf || !msg || !chunk_of) {
        free(buf);
        free(msg);
        free(chunk_of);
        return ORC_ERR_ALLOC;
    }
    memcpy(buf, p, (size_t)N * (size_t)plane * sizeof *buf);
    for (int64_t i = 0; i < n_cols; ++i)
        chunk_of[i] = (int)(cols[i] / hc);
    const uint64_t chunk_bytes = (uint64_t)tokens * (uint64_t)hc * 2u;

    /* Reduce-scatter: N-1 steps. All ranks send at once, then all receive. */
    for (int s = 0; s < N - 1; ++s) {
        for (int r = 0; r < N; ++r) {
            int c = ((r - s) % N + N) % N;
            for (int64_t m = 0; m < tokens; ++m)
                for (int64_t i = 0; i < n_cols; ++i)
                    if (chunk_of[i] == c)
                        msg[(int64_t)r * plane + m * n_cols + i] =
                            buf[(int64_t)r * plane + m * n_cols + i];
            if (bytes_sent)
                bytes_sent[r] += chunk_bytes;
        }
        for (int r = 0; r < N; ++r) {
            int src = (r - 1 + N) % N;
            int c = ((src - s) % N + N) % N;
            for (int64_t m = 0; m < tokens; ++m)
                for (int64_t i = 0; i < n_cols; ++i)
                    if (chunk_of[i] == c) {
                        int64_t o = m * n_cols + i;
                        float recv = orc_f32(msg[(int64_t)src * plane + o]);
                        float own = orc_f32(buf[(int64_t)r * plane + o]);
                        buf[(int64_t)r * plane + o] = orc_bf16_rne(recv + own);
                    }
        }
    }
    /* All-gather: rank r now holds the reduced chunk (r + 1) mod N; N-1 steps
     * pass the reduced chunks around the ring. */
    for (int s = 0; s < N - 1; ++s) {
        for (int r = 0; r < N; ++r) {
            int c = ((r + 1 - s) % N + N) % N;
            for (int64_t m = 0; m < tokens; ++m)
                for (int64_t i = 0; i < n_cols; ++i)
                    if (chunk_of[i] == c)
                        msg[(int64_t)r * plane + m * n_cols + i] =
                            buf[(int64_t)r * plane + m * n_cols + i];
            if (bytes_sent)
                bytes_sent[r] += chunk_bytes;
        }
        for (int r = 0; r < N; ++r) {
            int src = (r - 1 + N) % N;
            int c = ((src + 1 - s) % N + N) % N;
            for (int64_t m = 0; m < tokens; ++m)
                for (int64_t i = 0; i < n_cols; ++i)
                    if (chunk_of[i] == c) {
                        int64_t o = m * n_cols + i;
                        buf[(int64_t)r * plane + o] = msg[(int64_t)src * plane + o];
                    }
        }
    }
    int rc = ORC_OK;
    for (int r = 1; r < N; ++r)
        if (memcmp(buf, buf + (int64_t)r * plane, (size_t)plane * sizeof *buf) != 0)
            rc = ORC_ERR_RING;
    memcpy(reduced, buf, (size_t)plane * sizeof *buf);
    free(buf);
    free(msg);
    free(chunk_of);
    return rc;
}

/* ------------------------------------------------------------ residual -- */

void orc_residual(int64_t count, const uint16_t *residual, const uint16_t *reduced,
                  uint16_t *out)
{
    for (int64_t i = 0; i < count; ++i)
        out[i] = orc_bf16_rne(orc_f32(residual[i]) + orc_f32(reduced[i]));
}

/* ---------------------------------------------------------- whole point -- */

/* One reconciliation point on the selected output columns.
 *   x         [tokens][k]
 *   w_rows    [n_cols][k]   rows cols[i] of the Linear weight W[H][K]
 *   residual  [tokens][n_cols]  the residual at those columns
 *   out       [tokens][n_cols]
 *   partials  [n_ranks][tokens][n_cols] (out, may be NULL)
 *   p64, pabs same shape (out, may be NULL)
 *   bytes_sent [n_ranks] (out, may be NULL) */
int orc_reconcile(int n_ranks, int64_t tokens, int64_t k, int64_t hidden, const uint16_t *x,
                  int64_t n_cols, const int64_t *cols, const uint16_t *w_rows,
                  const uint16_t *residual, uint16_t *out, uint16_t *partials, double *p64,
                  double *pabs, uint64_t *bytes_sent, int n_threads)
{
    if (n_ranks < 1 || hidden % n_ranks != 0 || k % n_ranks != 0)
        return ORC_ERR_ARGS;
    const int64_t plane = tokens * n_cols;
    uint16_t *p = partials;
    uint16_t *red = malloc((size_t)(plane > 0 ? plane : 1) * sizeof *red);
    if (!p)
        p = malloc((size_t)(n_ranks * plane > 0 ? n_ranks * plane : 1) * sizeof *p);
    if (!p || !red) {
        if (!partials)
            free(p);
        free(red);
        return ORC_ERR_ALLOC;
    }
    int rc = orc_partials(n_ranks, tokens, k, x, n_cols, w_rows, p, p64, pabs, n_threads);
    if (rc == ORC_OK)
        rc = orc_ring(n_ranks, tokens, hidden, n_cols, cols, p, red, bytes_sent);
    if (rc == ORC_OK)
        orc_residual(plane, residual, red, out);
    if (!partials)
        free(p);
    free(red);
    return rc;
}

/* ----------------------------------------------------------- byte model -- */

/* Bytes one rank puts on its wire for a ring all-reduce of `points`
 * reconciliations of tokens x hidden values of elem_bytes each:
 * 2(N-1)/N times the payload (multiplied out before the one division). */
uint64_t orc_ring_bytes(int n_ranks, int64_t tokens, int64_t hidden, int elem_bytes,
                        int64_t points)
{
    if (n_ranks < 1 || tokens < 0 || hidden < 0 || elem_bytes < 0 || points < 0)
        return 0;
    uint64_t payload = (uint64_t)tokens * (uint64_t)hidden * (uint64_t)elem_bytes;
    return 2u * (uint64_t)(n_ranks - 1) * payload * (uint64_t)points / (uint64_t)n_ranks;
}

/*
 * Bytes one rank's NVLink port carries for the all-reduce of `payload` bytes
 * per rank, under three schemes of the all-reduce section of the NVL72
 * hosting post, counted message by message over slices of B/N bytes (B =
 * tokens * hidden * elem_bytes * points):
 *   0 ring (reduce the slices, then broadcast): rank r receives slice r from
 *     each of its N-1 peers and sends its reduced slice r to each of them;
 *     2(N-1) slice messages (the same count as the first page's
 *     reduce-scatter plus all-gather).
 *   1 naive: rank r loads every peer's whole buffer: N-1 buffers of N slices.
 *   2 switch reduction (SHARP): slice r is summed inside the switch, which
 *     reads it from the N-1 peers and hands rank r one reduced slice; counted
 *     for slice r: N-1 peer reads plus 1 slice from the switch.
 * One rank communicates nothing. Exact: slice messages are counted, then
 * multiplied by B before the one division by N.
 */
uint64_t orc_allreduce_bytes(int scheme, int n_ranks, int64_t tokens, int64_t hidden, int elem_bytes,
                             int64_t points)
{
    if (n_ranks < 1 || tokens < 0 || hidden < 0 || elem_bytes < 0 || points < 0)
        return 0;
    if (n_ranks == 1)
        return 0;
    uint64_t slices = 0;  /* slice messages counted at rank 0 */
    const int r = 0;
    if (scheme == 0) {
        for (int peer = 0; peer < n_ranks; ++peer)
            if (peer != r)
                slices += 1;  /* peer's slice r arrives for the reduction */
        for (int peer = 0; peer < n_ranks; ++peer)
            if (peer != r)
                slices += 1;  /* reduced slice r goes out to the peer */
    } else if (scheme == 1) {
        for (int peer = 0; peer < n_ranks; ++peer)
            if (peer != r)
                for (int c = 0; c < n_ranks; ++c)
                    slices += 1;  /* every slice of the peer's buffer */
    } else if (scheme == 2) {
        for (int peer = 0; peer < n_ranks; ++peer)
            if (peer != r)
                slices += 1;  /* the switch reads the peer's slice r */
        slices += 1;          /* the reduced slice r from the switch */
    } else {
        return 0;
    }
    const uint64_t b = (uint64_t)tokens * (uint64_t)hidden * (uint64_t)elem_bytes * (uint64_t)points;
    return slices * b / (uint64_t)n_ranks;
}

/*
 * Bytes one rank's NVLink port carries for the combine step of an MoE layer
 * (NVL72 hosting post, MoE dispatch/combine section): the combine kernel
 * first accumulates, on each rank, the weighted contributions of the experts
 * that rank hosts for every token, then all-reduces the accumulated
 * [tokens][hidden] buffer across the ranks. Counted buffer by buffer:
 *   local_accumulate = 1  every rank all-reduces one [tokens][hidden]
 *                         buffer, whatever top_k and the routing are;
 *   local_accumulate = 0  (for comparison) each of the top_k expert slots of
 *                         a token is all-reduced as its own [tokens][hidden]
 *                         buffer, the weighted sum taken afterwards.
 * Each buffer costs orc_allreduce_bytes under `scheme` (points = 1).
 * Returns 0 for top_k < 1 or the arguments orc_allreduce_bytes rejects.
 */
uint64_t orc_moe_combine_bytes(int scheme, int n_ranks, int64_t tokens, int64_t hidden,
                               int elem_bytes, int64_t top_k, int local_accumulate)
{
    if (top_k < 1 || (local_accumulate != 0 && local_accumulate != 1))
        return 0;
    const int64_t buffers = local_accumulate ? 1 : top_k;
    uint64_t total = 0;
    for (int64_t b = 0; b < buffers; ++b)
        total += orc_allreduce_bytes(scheme, n_ranks, tokens, hidden, elem_bytes, 1);
    return total;
}

/* -------------------------------------------------- MXFP8 weight shards -- */
/*
 * Micro-scaled FP8 weights (the NVL72 hosting post quantises the MoE GEMM's
 * weights to MXFP8; the format itself is the OCP Microscaling (MX) v1.0
 * specification's MXFP8 E4M3): every block of 32 consecutive weights along
 * K, inside one rank's slice, shares one E8M0 scale X = 2^s (byte s + 127),
 * and each weight is stored as the FP8 E4M3 value nearest to w / X.
 *   s = floor(log2(max |w| of the block)) - 8   (8 = E4M3's largest exponent),
 *       clamped to [-127, 127]; an all-zero block takes s = -127;
 *   w / X rounded to nearest, ties to even, on the E4M3 grid (3 fraction
 *       bits; normals 2^-6 .. 448, subnormals in steps of 2^-9), saturating
 *       at +-448 (the block maximum can exceed 448 before rounding).
 * Reading: the specification leaves the rounding and overflow of the
 * element conversion to the implementation; round-to-nearest-even with
 * saturation is used, as for the bf16 rounding of the rest of the path.
 */

/* E4M3 code of the exact value v (|v| < 2^10), rounded to nearest even,
 * saturating at 448. */
uint8_t orc_e4m3_rne(double v)
{
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs(v);
    if (a >= 448.0)
        return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {                 /* subnormal: multiples of 2^-9 */
        const double q = a * 512.0;           /* exact: a has few significant bits */
        double m = floor(q);
        const double rem = q - m;
        if (rem > 0.5 || (rem == 0.5 && fmod(m, 2.0) == 1.0))
            m += 1.0;
        return sign | (uint8_t)m;             /* m == 8 is the smallest normal, 0x08 */
    }
    int e;
    (void)frexp(a, &e);
    e -= 1;                                   /* a = f * 2^e, f in [1, 2) */
    const double q = (ldexp(a, -e) - 1.0) * 8.0;
    double m = floor(q);
    const double rem = q - m;
    if (rem > 0.5 || (rem == 0.5 && fmod(m, 2.0) == 1.0))
        m += 1.0;
    if (m == 8.0) {
        m = 0.0;
        e += 1;
    }
    return sign | (uint8_t)(((e + 7) << 3) | (int)m);
}

/* Value of an E4M3 code (never NaN here: the encoder does not produce 0x7F). */
double orc_e4m3_value(uint8_t c)
{
    const int ex = (c >> 3) & 0xF, m = c & 7;
    const double mag = ex == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, ex - 7);
    return (c & 0x80) ? -mag : mag;
}

/* Shared exponent of a block from its largest magnitude. */
static int mx_shared_exp(double amax)
{
    if (amax == 0.0)
        return -127;
    int e;
    (void)frexp(amax, &e);
    int s = (e - 1) - 8;
    if (s < -127)
        s = -127;
    if (s > 127)
        s = 127;
    return s;
}

/* Linear weight [hidden][k] (bf16) -> per-rank MXFP8 shards:
 *   q      [n_ranks][hidden][k/n_ranks] E4M3 codes
 *   scales [n_ranks][hidden][k/n_ranks/32] E8M0 bytes (s + 127)
 * k/n_ranks must be a multiple of 32 (blocks never straddle two ranks). */
int orc_mx_quantize(int n_ranks, int64_t hidden, int64_t k, const uint16_t *w_hk, uint8_t *q,
                    uint8_t *scales)
{
    if (n_ranks < 1 || hidden < 0 || k < 0 || k % n_ranks != 0 || (k / n_ranks) % 32 != 0)
        return ORC_ERR_ARGS;
    const int64_t ks = k / n_ranks, nb = ks / 32;
    for (int r = 0; r < n_ranks; ++r)
        for (int64_t h = 0; h < hidden; ++h)
            for (int64_t b = 0; b < nb; ++b) {
                const uint16_t *w = w_hk + h * k + (int64_t)r * ks + 32 * b;
                double amax = 0.0;
                for (int i = 0; i < 32; ++i) {
                    const double a = fabs((double)orc_f32(w[i]));
                    if (a > amax)
                        amax = a;
                }
                const int s = mx_shared_exp(amax);
                const int64_t row = (int64_t)r * hidden + h;
                scales[row * nb + b] = (uint8_t)(s + 127);
                for (int i = 0; i < 32; ++i)
                    q[row * ks + 32 * b + i] = orc_e4m3_rne(ldexp((double)orc_f32(w[i]), -s));
            }
    return ORC_OK;
}

/* Dequantised shards back in the Linear layout [hidden][k] as bf16: every
 * value E4M3 * 2^s has at most 4 significant bits, so it is exact in bf16
 * unless it leaves bf16's range (returns ORC_ERR_ARGS then, which only
 * blocks whose largest weight is below 2^-116 can cause). */
int orc_mx_dequant_bf16(int n_ranks, int64_t hidden, int64_t k, const uint8_t *q,
                        const uint8_t *scales, uint16_t *w_hk)
{
    if (n_ranks < 1 || hidden < 0 || k < 0 || k % n_ranks != 0 || (k / n_ranks) % 32 != 0)
        return ORC_ERR_ARGS;
    const int64_t ks = k / n_ranks, nb = ks / 32;
    for (int r = 0; r < n_ranks; ++r)
        for (int64_t h = 0; h < hidden; ++h)
            for (int64_t j = 0; j < ks; ++j) {
                const int64_t row = (int64_t)r * hidden + h;
                const int s = (int)scales[row * nb + j / 32] - 127;
                const double v = ldexp(orc_e4m3_value(q[row * ks + j]), s);
                const uint16_t b = orc_bf16_rne_f64(v);
                if ((double)orc_f32(b) != v)
                    return ORC_ERR_ARGS;
                w_hk[h * k + (int64_t)r * ks + j] = b;
            }
    return ORC_OK;
}

/* -------------------------------------------------- NVFP4 weight shards -- */
/*
 * 4-bit weights (the TP=4-vs-TP=8 post deploys NVFP4 weights with 16-bit
 * activations; the post itself garbles the element format, so the format is
 * NVIDIA's published NVFP4): each weight is an FP4 E2M1 value (sign, 2
 * exponent bits, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6),
 * every 16 consecutive weights along K inside one rank's slice share an FP8
 * E4M3 block scale, and one second-level scale serves the whole tensor.
 * Reading: the second-level scale is the power of two 2^g with g the
 * smallest integer such that amax(W) / 2^g <= 6 * 448 (every block scale then
 * fits E4M3; a power of two keeps every dequantised weight exact in bf16: at
 * most 2 x 4 significant bits); an all-zero tensor takes g = 0.
 *   block scale  b = E4M3 nearest to amax(block) / (6 * 2^g), ties to even
 *   element      q = E2M1 nearest to w / (b * 2^g), ties to even,
 *                    saturating at +-6; a block whose b is 0 stores zeros
 *   value        q * b * 2^g
 * Codes: sign in bit 3, magnitude index in bits 0-2. Two codes per byte,
 * the earlier k in the low nibble.
 */

/* E2M1 code (0..15) of the exact value v, nearest even, saturating at 6. */
uint8_t orc_e2m1_rne(double v)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    const uint8_t sign = signbit(v) ? 0x8 : 0x0;
    const double a = fabs(v);
    if (a >= 6.0)
        return sign | 7;
    int lo = 0;
    while (lo < 7 && mag[lo + 1] <= a)
        ++lo;                                 /* mag[lo] <= a < mag[lo + 1] */
    const double d_lo = a - mag[lo], d_hi = mag[lo + 1] - a;
    int m = lo;
    if (d_hi < d_lo || (d_hi == d_lo && (lo & 1)))
        m = lo + 1;                           /* nearer, or a tie to the even index */
    return sign | (uint8_t)m;
}

double orc_e2m1_value(uint8_t c)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    return (c & 0x8) ? -mag[c & 7] : mag[c & 7];
}

/* The second-level exponent g of a tensor whose largest magnitude is amax. */
int orc_nvfp4_global_exp(double amax)
{
    if (amax == 0.0)
        return 0;
    int g = -200;
    while (amax / ldexp(1.0, g) > 6.0 * 448.0)
        ++g;
    return g;
}

/* Linear weight [hidden][k] (bf16) -> per-rank NVFP4 shards:
 *   q      [n_ranks][hidden][k/n_ranks/2] bytes, two E2M1 codes each
 *   scales [n_ranks][hidden][k/n_ranks/16] E4M3 block scales
 *   *g     the second-level exponent
 * k/n_ranks must be a multiple of 16. */
int orc_nvfp4_quantize(int n_ranks, int64_t hidden, int64_t k, const uint16_t *w_hk, uint8_t *q,
                       uint8_t *scales, int *g_out)
{
    if (n_ranks < 1 || hidden < 0 || k < 0 || k % n_ranks != 0 || (k / n_ranks) % 16 != 0)
        return ORC_ERR_ARGS;
    double amax = 0.0;
    for (int64_t i = 0; i < hidden * k; ++i) {
        const double a = fabs((double)orc_f32(w_hk[i]));
        if (a > amax)
            amax = a;
    }
    const int g = orc_nvfp4_global_exp(amax);
    const double two_g = ldexp(1.0, g);
    const int64_t ks = k / n_ranks, nb = ks / 16;
    for (int r = 0; r < n_ranks; ++r)
        for (int64_t h = 0; h < hidden; ++h) {
            const int64_t row = (int64_t)r * hidden + h;
            for (int64_t b = 0; b < nb; ++b) {
                const uint16_t *w = w_hk + h * k + (int64_t)r * ks + 16 * b;
                double bmax = 0.0;
                for (int i = 0; i < 16; ++i) {
                    const double a = fabs((double)orc_f32(w[i]));
                    if (a > bmax)
                        bmax = a;
                }
                const uint8_t bs = orc_e4m3_rne(bmax / (6.0 * two_g));
                scales[row * nb + b] = bs;
                const double bval = orc_e4m3_value(bs);
                for (int i = 0; i < 16; ++i) {
                    const uint8_t c = bval == 0.0 ? 0 : orc_e2m1_rne((double)orc_f32(w[i]) / (bval * two_g));
                    const int64_t j = 16 * b + i;           /* index within the row */
                    uint8_t *dst = &q[row * (ks / 2) + j / 2];
                    if (j % 2 == 0)
                        *dst = c;
                    else
                        *dst = (uint8_t)(*dst | (c << 4));
                }
            }
        }
    *g_out = g;
    return ORC_OK;
}

/* Dequantised NVFP4 shards back in the Linear layout [hidden][k] as bf16
 * (exact; ORC_ERR_ARGS if a value leaves bf16's range). */
int orc_nvfp4_dequant_bf16(int n_ranks, int64_t hidden, int64_t k, const uint8_t *q,
                           const uint8_t *scales, int g, uint16_t *w_hk)
{
    if (n_ranks < 1 || hidden < 0 || k < 0 || k % n_ranks != 0 || (k / n_ranks) % 16 != 0)
        return ORC_ERR_ARGS;
    const int64_t ks = k / n_ranks, nb = ks / 16;
    for (int r = 0; r < n_ranks; ++r)
        for (int64_t h = 0; h < hidden; ++h) {
            const int64_t row = (int64_t)r * hidden + h;
            for (int64_t j = 0; j < ks; ++j) {
                const uint8_t byte = q[row * (ks / 2) + j / 2];
                const uint8_t c = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);
                const double v = ldexp(orc_e2m1_value(c) * orc_e4m3_value(scales[row * nb + j / 16]), g);
                const uint16_t b = orc_bf16_rne_f64(v);
                if ((double)orc_f32(b) != v)
                    return ORC_ERR_ARGS;
                w_hk[h * k + (int64_t)r * ks + j] = b;
            }
        }
    return ORC_OK;
}

/* ------------------------------------------------------- array helpers -- */

void orc_bf16_rne_array(int64_t count, const float *in, uint16_t *out)
{
    for (int64_t i = 0; i < count; ++i)
        out[i] = orc_bf16_rne(in[i]);
}

void orc_bf16_rne_f64_array(int64_t count, const double *in, uint16_t *out)
{
    for (int64_t i = 0; i < count; ++i)
        out[i] = orc_bf16_rne_f64(in[i]);
}
