/*
 * fp64 CPU oracle for Ulysses sequence-parallel self-attention.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark use this file.  It shares no code, header, table or
 * helper with the CUDA path, and it is deliberately plain and slow: loops in
 * the order of the definitions, fp64 arithmetic, no blocking or fusion.
 *
 * Sources of the definitions (web pages on the method):
 *  - fal.ai, "Generate video with WAN 2.2 across four GPUs", section
 *    "Splitting one generation across four GPUs": at every attention layer an
 *    all-to-all exchanges token shards for head groups, so that each GPU
 *    attends over all tokens for its share of the heads (10 of 40 at four
 *    GPUs); afterwards the outputs go back to the GPUs that own the tokens.
 *  - same page, section "Tuning cost and GPU count": the degree has to be a
 *    divisor of the head count.
 *  - LTX-2 "Multi-GPU Inference" README, Capabilities table: sequence
 *    parallelism gives the single-GPU result.  The
 *    oracle therefore computes the unsharded (single-GPU) attention for every
 *    degree P.
 *
 * Readings where the pages are silent (stated, not taken from the pages):
 *  - layout: rank r holds tokens r*Nl .. r*Nl+Nl-1 of the sequence as
 *    [B][Nl][H][D]; the P shards are stored one after another, [P][B][Nl][H][D];
 *    Nl = ceil(N/P); token slots >= N are padding.
 *  - head group j holds heads j*Hl .. j*Hl+Hl-1 (Hl = H/P); after the exchange
 *    group j's buffer is [B][Np][Hl][D] with Np = P*Nl, chunks in rank order,
 *    and the P group buffers are stored one after another.
 *  - attention is non-causal softmax(q k^T * scale) v over all N tokens with
 *    scale = 1/sqrt(D) unless given; no mask except the padding slots.
 *
 *  - FP8 attention (named for the FastVideo stack on "Pair two NVIDIA DGX
 *    Sparks" without a definition): the same attention on inputs stored as
 *    E4M3 bytes, each element scaled by a factor; Q and K carry one factor per
 *    block of consecutive tokens, V one per channel (the contraction of q.k
 *    runs over channels and that of p.v over tokens, so these factors come
 *    out of the sums).
 *  - the projection in front of attention (the step next to it in a DiT
 *    block, which the pages never describe): one linear layer from each
 *    token's hidden state to its q, k and v, with no rotary embedding or
 *    normalisation.
 *  - block-sparse attention (the sparse stage of video sparse attention, named
 *    on "Pair two NVIDIA DGX Sparks" with 64-token tiles and sparsity 0.8,
 *    its block selection not defined there): a query attends only the keys
 *    of the key cubes a block mask selects for its query cube; the mask is an
 *    input.  A query whose cube selects nothing gets O = 0 and lse = -inf.
 *
 * Element type: bf16, given as its 16-bit pattern, or E4M3 bytes with their
 * factors.  The oracle widens each value exactly to double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_f64(uint16_t x) {
    uint32_t u = (uint32_t)x << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* OCP 8-bit floating point E4M3 (sign, 4 exponent bits with bias 7, 3
 * mantissa bits; exponent 0 is subnormal, S.1111.111 is NaN, no infinity),
 * decoded exactly. */
static double e4m3_to_f64(uint8_t x) {
    int s = x >> 7, e = (x >> 3) & 15, m = x & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

double sp_oracle_e4m3_value(uint8_t x) { return e4m3_to_f64(x); }

/*
 * Pack (sequence-sharded -> head-sharded): the send-buffer reorder plus the
 * all-to-all of the page section "Splitting one generation across four GPUs".
 * Rank r's tokens for head group j land in group j's buffer at token index
 * r*Nl + n:
 *     xh[j][b][r*Nl + n][hh][c] = xs[r][b][n][j*Hl + hh][c]
 * xs: [P][B][Nl][H][D] words; xh: [P][B][P*Nl][Hl][D] words.
 * Returns 0, or -1 when P does not divide H (page section "Tuning cost and
 * GPU count").
 */
int sp_oracle_pack(const uint16_t *xs, uint16_t *xh, int64_t B, int64_t N,
                   int64_t H, int64_t D, int64_t P) {
    if (P < 1 || H % P != 0) return -1;
    int64_t Hl = H / P, Nl = (N + P - 1) / P, Np = P * Nl;
    for (int64_t j = 0; j < P; ++j)
        for (int64_t b = 0; b < B; ++b)
            for (int64_t r = 0; r < P; ++r)
                for (int64_t n = 0; n < Nl; ++n)
                    for (int64_t hh = 0; hh < Hl; ++hh)
                        for (int64_t c = 0; c < D; ++c) {
                            int64_t src = (((r * B + b) * Nl + n) * H + (j * Hl + hh)) * D + c;
                            int64_t dst = (((j * B + b) * Np + (r * Nl + n)) * Hl + hh) * D + c;
                            xh[dst] = xs[src];
                        }
    return 0;
}

/*
 * Unpack (head-sharded -> sequence-sharded): the outputs go back to the
 * token owners (same page section); the inverse of the pack:
 *     os[r][b][n][j*Hl + hh][c] = oh[j][b][r*Nl + n][hh][c]
 */
int sp_oracle_unpack(const uint16_t *oh, uint16_t *os, int64_t B, int64_t N,
                     int64_t H, int64_t D, int64_t P) {
    if (P < 1 || H % P != 0) return -1;
    int64_t Hl = H / P, Nl = (N + P - 1) / P, Np = P * Nl;
    for (int64_t r = 0; r < P; ++r)
        for (int64_t b = 0; b < B; ++b)
            for (int64_t n = 0; n < Nl; ++n)
                for (int64_t j = 0; j < P; ++j)
                    for (int64_t hh = 0; hh < Hl; ++hh)
                        for (int64_t c = 0; c < D; ++c) {
                            int64_t src = (((j * B + b) * Np + (r * Nl + n)) * Hl + hh) * D + c;
                            int64_t dst = (((r * B + b) * Nl + n) * H + (j * Hl + hh)) * D + c;
                            os[dst] = oh[src];
                        }
    return 0;
}

/*
 * Shard: the token sequence of one generation divided across the P ranks
 * (same page section), rank r holding tokens r*Nl .. r*Nl+Nl-1 of the
 * logical [B][N][H][D] tensor; slots past the last token are zero:
 *     xs[r][b][n][h][c] = x[b][r*Nl + n][h][c]   if r*Nl + n < N, else 0
 */
int sp_oracle_shard(const uint16_t *x, uint16_t *xs, int64_t B, int64_t N,
                    int64_t H, int64_t D, int64_t P) {
    if (P < 1) return -1;
    int64_t Nl = (N + P - 1) / P;
    for (int64_t r = 0; r < P; ++r)
        for (int64_t b = 0; b < B; ++b)
            for (int64_t n = 0; n < Nl; ++n)
                for (int64_t h = 0; h < H; ++h)
                    for (int64_t c = 0; c < D; ++c) {
                        int64_t t = r * Nl + n;
                        int64_t dst = (((r * B + b) * Nl + n) * H + h) * D + c;
                        xs[dst] = t < N ? x[((b * N + t) * H + h) * D + c] : 0;
                    }
    return 0;
}

/*
 * Unshard: the P shards back to the logical tensor, padding slots dropped:
 *     x[b][t][h][c] = xs[t / Nl][b][t % Nl][h][c]
 */
int sp_oracle_unshard(const uint16_t *xs, uint16_t *x, int64_t B, int64_t N,
                      int64_t H, int64_t D, int64_t P) {
    if (P < 1) return -1;
    int64_t Nl = (N + P - 1) / P;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t t = 0; t < N; ++t)
            for (int64_t h = 0; h < H; ++h)
                for (int64_t c = 0; c < D; ++c) {
                    int64_t r = t / Nl, n = t % Nl;
                    x[((b * N + t) * H + h) * D + c] = xs[(((r * B + b) * Nl + n) * H + h) * D + c];
                }
    return 0;
}

/*
 * Exchange pack on one rank (the send-buffer reorder in front of the
 * all-to-all of "Splitting one generation across four GPUs" when every rank
 * is its own GPU): rank r's shard xs_r [B][Nl][H][D] becomes P send chunks,
 * chunk j holding r's tokens for head group j:
 *     send[j][b][n][hh][c] = xs_r[b][n][j*Hl + hh][c]
 * After the all-to-all, rank j holds chunk j of every rank r in rank order,
 * [P][B][Nl][Hl][D]: the full sequence for its heads.
 */
int sp_oracle_exchange_pack(const uint16_t *xs_r, uint16_t *send, int64_t B, int64_t N,
                            int64_t H, int64_t D, int64_t P) {
    if (P < 1 || H % P != 0) return -1;
    int64_t Hl = H / P, Nl = (N + P - 1) / P;
    for (int64_t j = 0; j < P; ++j)
        for (int64_t b = 0; b < B; ++b)
            for (int64_t n = 0; n < Nl; ++n)
                for (int64_t hh = 0; hh < Hl; ++hh)
                    for (int64_t c = 0; c < D; ++c)
                        send[(((j * B + b) * Nl + n) * Hl + hh) * D + c] =
                            xs_r[((b * Nl + n) * H + (j * Hl + hh)) * D + c];
    return 0;
}

/*
 * Exchange unpack on one rank (outputs back to the token owners): the
 * P chunks received back from the head groups, recv[j][b][n][hh][c] (group
 * j's output for this rank's tokens), become the shard [B][Nl][H][D]:
 *     os_r[b][n][j*Hl + hh][c] = recv[j][b][n][hh][c]
 */
int sp_oracle_exchange_unpack(const uint16_t *recv, uint16_t *os_r, int64_t B, int64_t N,
                              int64_t H, int64_t D, int64_t P) {
    if (P < 1 || H % P != 0) return -1;
    int64_t Hl = H / P, Nl = (N + P - 1) / P;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t n = 0; n < Nl; ++n)
            for (int64_t j = 0; j < P; ++j)
                for (int64_t hh = 0; hh < Hl; ++hh)
                    for (int64_t c = 0; c < D; ++c)
                        os_r[((b * Nl + n) * H + (j * Hl + hh)) * D + c] =
                            recv[(((j * B + b) * Nl + n) * Hl + hh) * D + c];
    return 0;
}

/*
 * Attention for a list of query rows of the unsharded problem.
 *
 * For query row i of batch b and head h, with scores
 *     s_k = scale * sum_c q[b][i][h][c] * k[b][k][h][c]      (k = 0 .. N-1)
 * the two-pass exact softmax
 *     m = max_k s_k,  w_k = exp(s_k - m),  l = sum_k w_k
 * gives
 *     o[c] = (sum_k w_k * v[b][k][h][c]) / l,   lse = m + ln(l).
 * This is the plain definition softmax(q K^T scale) V of "attention over the
 * full sequence" for one head; the sequence-parallel result equals it for
 * every degree (LTX-2 README, Capabilities table).
 *
 * q, k, v: logical [B][N][H][D] bf16 words.  rows: nrows triples (b, h, i).
 * out_o: nrows x D doubles; out_lse: nrows doubles (may be NULL).
 */
typedef struct {
    const uint16_t *q, *k, *v;
    const uint8_t *q8, *k8, *v8;       /* e4m3 inputs instead of bf16, or NULL */
    /* Scale factors of the e4m3 inputs: dq and dk [B][H][nblk], one per block
     * of blk consecutive tokens; dv [B][H][D], one per channel. */
    const double *dq, *dk, *dv;
    int64_t blk, nblk;
    /* Block mask, or NULL for every key: key kk is attended by query i of
     * (b, h) iff mask[((b * H + h) * ncube + i / cube) * ncube + kk / cube]
     * is non-zero (cubes of `cube` consecutive tokens, ncube of them). */
    const uint8_t *mask;
    int64_t cube, ncube;
    int64_t B, N, H, D;
    double scale;
    int64_t nrows;
    const int64_t *rows;
    double *out_o, *out_lse;
    int64_t next;
    pthread_mutex_t lock;
    int failed;
} attn_job_t;

/* Element e of a logical [B][N][H][D] input: bf16 words, or e4m3 bytes
 * times the scale factor that applies to that element. */
static double elem(const uint16_t *x16, const uint8_t *x8, double scale, int64_t e) {
    if (x8) return e4m3_to_f64(x8[e]) * scale;
    return bf16_to_f64(x16[e]);
}

static void attention_one_row(const attn_job_t *J, int64_t r, double *s) {
    int64_t b = J->rows[3 * r], h = J->rows[3 * r + 1], i = J->rows[3 * r + 2];
    int64_t N = J->N, H = J->H, D = J->D, bh = b * H + h;
    int64_t qi = ((b * N + i) * H + h) * D;
    double sq = J->q8 ? J->dq[bh * J->nblk + i / J->blk] : 1.0;
    const uint8_t *sel = J->mask ? J->mask + (bh * J->ncube + i / J->cube) * J->ncube : NULL;
    double m = -INFINITY;
    for (int64_t kk = 0; kk < N; ++kk) {
        if (sel && !sel[kk / J->cube]) {
            s[kk] = -INFINITY;              /* key not in a selected cube */
            continue;
        }
        int64_t kr = ((b * N + kk) * H + h) * D;
        double sk = J->k8 ? J->dk[bh * J->nblk + kk / J->blk] : 1.0;
        double dot = 0.0;
        for (int64_t c = 0; c < D; ++c)
            dot += elem(J->q, J->q8, sq, qi + c) * elem(J->k, J->k8, sk, kr + c);
        s[kk] = J->scale * dot;
        if (s[kk] > m) m = s[kk];
    }
    double *o = J->out_o + r * D;
    for (int64_t c = 0; c < D; ++c) o[c] = 0.0;
    if (m == -INFINITY) {                   /* no key selected: O = 0, lse = -inf */
        if (J->out_lse) J->out_lse[r] = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int64_t kk = 0; kk < N; ++kk) {
        if (s[kk] == -INFINITY) continue;
        double w = exp(s[kk] - m);
        l += w;
        int64_t vr = ((b * N + kk) * H + h) * D;
        for (int64_t c = 0; c < D; ++c)
            o[c] += w * elem(J->v, J->v8, J->v8 ? J->dv[bh * D + c] : 1.0, vr + c);
    }
    for (int64_t c = 0; c < D; ++c) o[c] /= l;
    if (J->out_lse) J->out_lse[r] = m + log(l);
}

static void *attention_worker(void *arg) {
    attn_job_t *J = (attn_job_t *)arg;
    double *s = (double *)malloc(sizeof(double) * (size_t)(J->N > 0 ? J->N : 1));
    if (!s) {
        pthread_mutex_lock(&J->lock);
        J->failed = 1;
        pthread_mutex_unlock(&J->lock);
        return NULL;
    }
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t r = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (r >= J->nrows) break;
        attention_one_row(J, r, s);
    }
    free(s);
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments, -2 when out of host memory.
 * Rows are handed to up to nthreads threads in list order; callers that sort
 * the list by (b, h) let the threads share each head's K/V in cache. */
static int attention_rows_impl(attn_job_t *J, int nthreads);

int sp_oracle_attention_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             int64_t B, int64_t N, int64_t H, int64_t D, double scale,
                             int64_t nrows, const int64_t *rows, double *out_o,
                             double *out_lse, int nthreads) {
    attn_job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v;
    J.B = B; J.N = N; J.H = H; J.D = D;
    J.scale = scale;
    J.nrows = nrows; J.rows = rows;
    J.out_o = out_o; J.out_lse = out_lse;
    return attention_rows_impl(&J, nthreads);
}

/* The same attention on e4m3 inputs.  Element values are the exact e4m3
 * values times scale factors: q[b][t][h][c] and k[b][t][h][c] take
 * dq[b][h][t / blk] and dk[b][h][t / blk] (one factor per block of blk
 * tokens, nblk = ceil(N / blk) blocks), v[b][t][h][c] takes dv[b][h][c]. */
int sp_oracle_attention_rows_e4m3(const uint8_t *q8, const uint8_t *k8, const uint8_t *v8,
                                  const double *dq, const double *dk, const double *dv,
                                  int64_t blk,
                                  int64_t B, int64_t N, int64_t H, int64_t D, double scale,
                                  int64_t nrows, const int64_t *rows, double *out_o,
                                  double *out_lse, int nthreads) {
    attn_job_t J;
    memset(&J, 0, sizeof(J));
    if (blk < 1) return -1;
    J.q8 = q8; J.k8 = k8; J.v8 = v8;
    J.dq = dq; J.dk = dk; J.dv = dv;
    J.blk = blk; J.nblk = (N + blk - 1) / blk;
    J.B = B; J.N = N; J.H = H; J.D = D;
    J.scale = scale;
    J.nrows = nrows; J.rows = rows;
    J.out_o = out_o; J.out_lse = out_lse;
    return attention_rows_impl(&J, nthreads);
}

/* The same attention restricted by a block mask (the sparse stage of video
 * sparse attention): query i of (b, h) attends key kk only when the mask
 * selects kk's cube for i's cube, mask [B][H][ncube][ncube] bytes with
 * ncube = ceil(N / cube).  A query whose cube selects no key gets O = 0 and
 * lse = -inf. */
int sp_oracle_attention_rows_masked(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                    const uint8_t *mask, int64_t cube,
                                    int64_t B, int64_t N, int64_t H, int64_t D, double scale,
                                    int64_t nrows, const int64_t *rows, double *out_o,
                                    double *out_lse, int nthreads) {
    attn_job_t J;
    memset(&J, 0, sizeof(J));
    if (mask == NULL || cube < 1) return -1;
    J.q = q; J.k = k; J.v = v;
    J.mask = mask; J.cube = cube; J.ncube = (N + cube - 1) / cube;
    J.B = B; J.N = N; J.H = H; J.D = D;
    J.scale = scale;
    J.nrows = nrows; J.rows = rows;
    J.out_o = out_o; J.out_lse = out_lse;
    return attention_rows_impl(&J, nthreads);
}

/*
 * The projection in front of attention: a linear layer that maps each
 * token's hidden state to its q, k and v (the transformer block around the
 * attention; the pages describe no more of it, so no rotary embedding or
 * normalisation is applied).  For every requested row m:
 *     y[m][c] = sum_k x[m][k] * w[c][k]  (+ bias[c])     c = 0 .. nout-1
 * with the output features laid out as q (H*D), then k, then v, a feature's
 * weights in one row of w as a linear layer stores them.
 * x [M][K], w [nout][K], bias [nout] or NULL: bf16 words; rows: nrows row
 * indices; y: nrows x nout doubles.
 */
typedef struct {
    const uint16_t *x, *w, *bias;
    int64_t M, K, nout, nrows;
    const int64_t *rows;
    double *y;
    int64_t next;
    pthread_mutex_t lock;
} linear_job_t;

static void *linear_worker(void *arg) {
    linear_job_t *J = (linear_job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t r = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (r >= J->nrows) break;
        const uint16_t *xr = J->x + J->rows[r] * J->K;
        double *yr = J->y + r * J->nout;
        for (int64_t c = 0; c < J->nout; ++c) {
            const uint16_t *wc = J->w + c * J->K;
            double acc = 0.0;
            for (int64_t k = 0; k < J->K; ++k) acc += bf16_to_f64(xr[k]) * bf16_to_f64(wc[k]);
            yr[c] = acc + (J->bias ? bf16_to_f64(J->bias[c]) : 0.0);
        }
    }
    return NULL;
}

int sp_oracle_linear_rows(const uint16_t *x, const uint16_t *w, const uint16_t *bias,
                          int64_t M, int64_t K, int64_t nout, int64_t nrows,
                          const int64_t *rows, double *y, int nthreads) {
    if (M < 1 || K < 1 || nout < 1 || nrows < 0) return -1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= M) return -1;
    linear_job_t J;
    memset(&J, 0, sizeof(J));
    J.x = x; J.w = w; J.bias = bias;
    J.M = M; J.K = K; J.nout = nout; J.nrows = nrows; J.rows = rows; J.y = y;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 512) nthreads = 512;
    pthread_t th[512];
    int started = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&th[started], NULL, linear_worker, &J) != 0) break;
        ++started;
    }
    linear_worker(&J);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

static int attention_rows_impl(attn_job_t *JP, int nthreads) {
    attn_job_t J = *JP;
    int64_t B = J.B, N = J.N, H = J.H, D = J.D, nrows = J.nrows;
    const int64_t *rows = J.rows;
    double scale = J.scale;
    if (B < 1 || N < 1 || H < 1 || D < 1 || nrows < 0) return -1;
    for (int64_t r = 0; r < nrows; ++r) {
        if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 ||
            rows[3 * r + 1] >= H || rows[3 * r + 2] < 0 || rows[3 * r + 2] >= N)
            return -1;
    }
    if (!(scale > 0.0)) scale = 1.0 / sqrt((double)D);
    J.scale = scale;
    J.next = 0;
    J.failed = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 512) nthreads = 512;
    pthread_t th[512];
    int started = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&th[started], NULL, attention_worker, &J) != 0) break;
        ++started;
    }
    attention_worker(&J);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    pthread_mutex_destroy(&J.lock);
    return J.failed ? -2 : 0;
}
