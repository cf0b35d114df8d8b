/*
 * sta_oracle.c -- plain fp64 CPU reference for Sliding Tile Attention (STA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file; only tests/, the smoke check and the bench's CPU-baseline leg
 * use it.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (sources: "Fast Video Generation with Sliding Tile
 * Attention"; the podcast transcript at hotaipapers.com, segment on tiles and
 * on dense / empty / mixed blocks; the atlas.scime.ai summary, "Approach";
 * the dianyo.github.io ICML-2025 post, STA section "Observation & Proposed
 * Method"):
 *
 *   - The video latent is L_t x L_h x L_w tokens in raster order (t, h, w; w
 *     fastest).  It is cut into tiles: contiguous spatio-temporal cubes of
 *     T_t x T_h x T_w tokens.
 *   - Every query tile attends to the key tiles inside a 3D window of tiles
 *     centred on it; the window slides tile by tile, so all queries of one
 *     tile share one key set and every (query tile, key tile) block is either
 *     fully attended or fully skipped.
 *   - The window size is given per head, in tokens.
 *   - Attention inside the attended set is exact softmax attention.
 *
 * Readings of points the pages leave open (each one is listed in the design
 * notes with its justification):
 *   - window extent in tiles e_d = min(W_d / T_d, n_d) (a window larger than
 *     the volume covers the volume);
 *   - the window is shifted to stay inside the volume: start
 *     s_d = clamp(q_d - floor(e_d / 2), 0, n_d - e_d), so an even window puts
 *     its extra tile on the lower side;
 *   - LSE is the natural log of sum_j exp(scale * q . k_j) over attended keys;
 *   - scale is applied as the double value of the fp32 softmax scale;
 *   - inputs are bf16 values, widened exactly to double;
 *   - a latent axis that is not a multiple of the tile is padded at its high
 *     end to whole tiles: the tile grid has n_d = ceil(L_d / T_d) tiles, the
 *     windows are placed on that grid by the rule above, and a query attends
 *     the real tokens of its window's tiles (padding tokens are neither keys
 *     nor queries).  The pages fix only divisible latents; this is the plain
 *     extension that keeps every interior block dense and puts mixed blocks at
 *     the padded edge only.
 *
 * The oracle never builds a tile list and never permutes tokens: it evaluates
 * the token-level mask straight from token coordinates, in raster order.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t lat[3];  /* L_t, L_h, L_w in tokens */
    int32_t tile[3]; /* T_t, T_h, T_w in tokens */
} ora_geom;

/* Status codes of this file (not the library's). */
#define ORA_OK 0
#define ORA_BAD_ARG 1
#define ORA_NO_MEM 2

static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int geom_ok(const ora_geom* g)
{
    for (int d = 0; d < 3; ++d) {
        if (g->lat[d] <= 0 || g->tile[d] <= 0) return 0;
    }
    return 1;
}

/* Tiles along axis d: the latent padded up to whole tiles. */
static int32_t tiles_along(const ora_geom* g, int d)
{
    return (g->lat[d] + g->tile[d] - 1) / g->tile[d];
}

static int window_ok(const ora_geom* g, const int32_t* win)
{
    for (int d = 0; d < 3; ++d) {
        if (win[d] <= 0 || win[d] % g->tile[d] != 0) return 0;
    }
    return 1;
}

int64_t ora_num_tokens(const ora_geom* g)
{
    return (int64_t)g->lat[0] * g->lat[1] * g->lat[2];
}

static void unravel(const ora_geom* g, int64_t token, int32_t c[3])
{
    c[2] = (int32_t)(token % g->lat[2]);
    token /= g->lat[2];
    c[1] = (int32_t)(token % g->lat[1]);
    c[0] = (int32_t)(token / g->lat[1]);
}

/* Window start (in tiles) along one axis: centred on query tile q, extent e
 * tiles, shifted to stay inside [0, n). */
static int32_t window_start(int32_t q, int32_t e, int32_t n)
{
    int32_t s = q - e / 2;
    if (s < 0) s = 0;
    if (s > n - e) s = n - e;
    return s;
}

/* Token-level STA mask: may query token qi attend to key token kj under the
 * window `win` (tokens per axis)?  Returns 1 or 0; -1 on bad arguments. */
static int key_allowed(const ora_geom* g, const int32_t* win, int64_t qi, int64_t kj)
{
    int32_t qc[3], kc[3];
    unravel(g, qi, qc);
    unravel(g, kj, kc);
    for (int d = 0; d < 3; ++d) {
        int32_t n = tiles_along(g, d);
        int32_t e = win[d] / g->tile[d];
        if (e > n) e = n;
        int32_t s = window_start(qc[d] / g->tile[d], e, n);
        int32_t k_tile = kc[d] / g->tile[d];
        if (k_tile < s || k_tile >= s + e) return 0;
    }
    return 1;
}

int ora_key_allowed(const ora_geom* g, const int32_t* win, int64_t qi, int64_t kj)
{
    if (!geom_ok(g) || !window_ok(g, win)) return -1;
    int64_t n_tok = ora_num_tokens(g);
    if (qi < 0 || qi >= n_tok || kj < 0 || kj >= n_tok) return -1;
    return key_allowed(g, win, qi, kj);
}

/* Whole mask row of query token qi: out[j] = allowed(qi, j), j in [0, N). */
int ora_mask_row(const ora_geom* g, const int32_t* win, int64_t qi, uint8_t* out)
{
    if (!geom_ok(g) || !window_ok(g, win) || out == NULL) return ORA_BAD_ARG;
    int64_t n_tok = ora_num_tokens(g);
    if (qi < 0 || qi >= n_tok) return ORA_BAD_ARG;
    for (int64_t j = 0; j < n_tok; ++j) out[j] = (uint8_t)key_allowed(g, win, qi, j);
    return ORA_OK;
}

/* Position of raster token `token` in tile-major order: tiles in raster order
 * over the tile grid, tokens inside a tile in raster order over the tile's own
 * (t, h, w) offsets.  The pages only say a tile is a contiguous cube of tokens;
 * this fixed order is the reading every layout test uses.  With a padded
 * latent the tile-major layout holds every tile whole (padding rows included),
 * so positions range over n_tiles * tile volume. */
int64_t ora_tile_major_index(const ora_geom* g, int64_t token)
{
    if (!geom_ok(g)) return -1;
    if (token < 0 || token >= ora_num_tokens(g)) return -1;
    int32_t c[3];
    unravel(g, token, c);
    int64_t n_h = tiles_along(g, 1);
    int64_t n_w = tiles_along(g, 2);
    int64_t tile_id = ((int64_t)(c[0] / g->tile[0]) * n_h + c[1] / g->tile[1]) * n_w + c[2] / g->tile[2];
    int64_t local = ((int64_t)(c[0] % g->tile[0]) * g->tile[1] + c[1] % g->tile[1]) * g->tile[2] + c[2] % g->tile[2];
    return tile_id * ((int64_t)g->tile[0] * g->tile[1] * g->tile[2]) + local;
}

/* ------------------------------------------------------------------------ */
/* Attention                                                                  */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q, *k, *v; /* [B, H, N, d] raster order, bf16 bits */
    const ora_geom* g;
    int64_t heads;
    int32_t d;
    const int32_t* win; /* [H][3] tokens */
    double scale;
    const int64_t* rows; /* nrows pairs (bh, token) */
    int64_t nrows;
    double *out_o, *out_lse;
    int64_t next; /* shared row counter */
    pthread_mutex_t lock;
    int status;
} ora_job;

static int64_t job_take(ora_job* job)
{
    pthread_mutex_lock(&job->lock);
    int64_t r = job->next++;
    pthread_mutex_unlock(&job->lock);
    return r;
}

static void* attention_worker(void* arg)
{
    ora_job* job = (ora_job*)arg;
    const int64_t n_tok = ora_num_tokens(job->g);
    const int32_t d = job->d;
    double* score = (double*)malloc(sizeof(double) * (size_t)n_tok);
    uint8_t* allowed = (uint8_t*)malloc((size_t)n_tok);
    double* qrow = (double*)malloc(sizeof(double) * (size_t)d);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    if (!score || !allowed || !qrow || !acc) {
        pthread_mutex_lock(&job->lock);
        job->status = ORA_NO_MEM;
        pthread_mutex_unlock(&job->lock);
        free(score); free(allowed); free(qrow); free(acc);
        return NULL;
    }
    for (;;) {
        int64_t r = job_take(job);
        if (r >= job->nrows) break;
        int64_t bh = job->rows[2 * r];
        int64_t qi = job->rows[2 * r + 1];
        int64_t h = bh % job->heads;
        const int32_t* win = job->win + 3 * h;
        const uint16_t* qp = job->q + (bh * n_tok + qi) * d;
        const uint16_t* kbase = job->k + bh * n_tok * d;
        const uint16_t* vbase = job->v + bh * n_tok * d;
        for (int32_t c = 0; c < d; ++c) qrow[c] = bf16_bits_to_double(qp[c]);

        /* 1. token-level mask and scores s_j = scale * q . k_j */
        double m = -INFINITY;
        for (int64_t j = 0; j < n_tok; ++j) {
            allowed[j] = (uint8_t)key_allowed(job->g, win, qi, j);
            if (!allowed[j]) continue;
            const uint16_t* kp = kbase + j * d;
            double dot = 0.0;
            for (int32_t c = 0; c < d; ++c) dot += qrow[c] * bf16_bits_to_double(kp[c]);
            score[j] = job->scale * dot;
            if (score[j] > m) m = score[j];
        }
        /* 2. softmax: l = sum exp(s_j - m); O = sum exp(s_j - m) v_j / l */
        double l = 0.0;
        for (int32_t c = 0; c < d; ++c) acc[c] = 0.0;
        for (int64_t j = 0; j < n_tok; ++j) {
            if (!allowed[j]) continue;
            double w = exp(score[j] - m);
            l += w;
            const uint16_t* vp = vbase + j * d;
            for (int32_t c = 0; c < d; ++c) acc[c] += w * bf16_bits_to_double(vp[c]);
        }
        for (int32_t c = 0; c < d; ++c) job->out_o[r * d + c] = acc[c] / l;
        /* 3. LSE = m + ln l (natural log, scaled-score units) */
        job->out_lse[r] = m + log(l);
    }
    free(score); free(allowed); free(qrow); free(acc);
    return NULL;
}

/* STA attention for an explicit list of query rows.
 *   q, k, v     : bf16 bits, [batch, heads, N, d], raster token order
 *   win         : [heads][3] window in tokens, multiples of the tile
 *   softmax_scale: fp32 scale; used as (double)softmax_scale
 *   rows        : nrows pairs (bh = b * heads + h, raster query token)
 *   out_o       : nrows * d doubles; out_lse: nrows doubles
 *   nthreads    : worker threads (>= 1)
 * Returns ORA_OK, ORA_BAD_ARG or ORA_NO_MEM. */
int ora_sta_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const ora_geom* g, int64_t batch, int64_t heads, int32_t d,
                      const int32_t* win, float softmax_scale,
                      const int64_t* rows, int64_t nrows,
                      double* out_o, double* out_lse, int32_t nthreads)
{
    if (!q || !k || !v || !g || !win || !rows || !out_o || !out_lse) return ORA_BAD_ARG;
    if (batch <= 0 || heads <= 0 || d <= 0 || nrows < 0 || nthreads <= 0) return ORA_BAD_ARG;
    if (!geom_ok(g)) return ORA_BAD_ARG;
    for (int64_t h = 0; h < heads; ++h)
        if (!window_ok(g, win + 3 * h)) return ORA_BAD_ARG;
    int64_t n_tok = ora_num_tokens(g);
    for (int64_t r = 0; r < nrows; ++r) {
        if (rows[2 * r] < 0 || rows[2 * r] >= batch * heads) return ORA_BAD_ARG;
        if (rows[2 * r + 1] < 0 || rows[2 * r + 1] >= n_tok) return ORA_BAD_ARG;
    }
    ora_job job;
    job.q = q; job.k = k; job.v = v; job.g = g; job.heads = heads; job.d = d;
    job.win = win; job.scale = (double)softmax_scale; job.rows = rows; job.nrows = nrows;
    job.out_o = out_o; job.out_lse = out_lse; job.next = 0; job.status = ORA_OK;
    pthread_mutex_init(&job.lock, NULL);
    pthread_t* tid = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!tid) { pthread_mutex_destroy(&job.lock); return ORA_NO_MEM; }
    int started = 0;
    for (int32_t t = 0; t < nthreads; ++t) {
        if (pthread_create(&tid[t], NULL, attention_worker, &job) != 0) break;
        ++started;
    }
    if (started == 0) attention_worker(&job);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    free(tid);
    pthread_mutex_destroy(&job.lock);
    return job.status;
}

/* ------------------------------------------------------------------------ */
/* Gradients                                                                  */
/* ------------------------------------------------------------------------ */
/*
 * Fine-tuning a model with STA in place of full attention (page 1, the
 * fine-tuning segment; page 4, "Observation & Proposed Method", last
 * paragraph) needs the gradients of STA attention.  The pages give no backward
 * pass; the reading here is the exact gradient of the function above with the
 * window held fixed (the mask has no gradient).  For one query row i with
 * attended key set A_i, upstream gradient dO_i and the forward's probabilities
 * P_ij = exp(s_ij - LSE_i), s_ij = scale q_i . k_j (chain rule through O = P V
 * and through the row softmax):
 *
 *   dV_j  += P_ij dO_i                      for every i with j in A_i
 *   dP_ij  = dO_i . v_j
 *   D_i    = sum_{j in A_i} P_ij dP_ij
 *   dS_ij  = P_ij (dP_ij - D_i)             (gradient w.r.t. s_ij)
 *   dQ_i   = scale sum_{j in A_i} dS_ij k_j
 *   dK_j  += scale dS_ij q_i
 *
 * All in double; q, k, v, dO are bf16 values widened exactly.
 */

typedef struct {
    const uint16_t *q, *k, *v, *dout; /* [B, H, N, d] raster order, bf16 bits */
    const ora_geom* g;
    int64_t heads;
    int32_t d;
    const int32_t* win;
    double scale;
    const int64_t* items; /* nitems pairs (bh, token) */
    int64_t nitems;
    double* stat;         /* dq: unused; dkdv: [B*H*N][2] (LSE, D) of each needed query */
    const uint8_t* need;  /* dkdv: [B*H*N] 1 where a query's statistics are needed */
    double *out_a, *out_b;
    int64_t next;
    pthread_mutex_t lock;
    int status;
} ora_bjob;

static int64_t bjob_take(ora_bjob* job)
{
    pthread_mutex_lock(&job->lock);
    int64_t r = job->next++;
    pthread_mutex_unlock(&job->lock);
    return r;
}

static void bjob_fail(ora_bjob* job, int st)
{
    pthread_mutex_lock(&job->lock);
    job->status = st;
    pthread_mutex_unlock(&job->lock);
}

static double dot_bf16(const double* a, const uint16_t* b, int32_t d)
{
    double s = 0.0;
    for (int32_t c = 0; c < d; ++c) s += a[c] * bf16_bits_to_double(b[c]);
    return s;
}

/* One query row: its attended keys, scores s_j, LSE, dP_j and D.  `score` and
 * `dp` have room for N entries; `allowed` marks the attended keys. */
static void row_pass(const ora_bjob* job, int64_t bh, int64_t qi, const double* qrow, const double* dorow,
                     double* score, double* dp, uint8_t* allowed, double* lse, double* dsum)
{
    const int64_t n_tok = ora_num_tokens(job->g);
    const int32_t d = job->d;
    const int32_t* win = job->win + 3 * (bh % job->heads);
    const uint16_t* kbase = job->k + bh * n_tok * d;
    const uint16_t* vbase = job->v + bh * n_tok * d;
    double m = -INFINITY;
    for (int64_t j = 0; j < n_tok; ++j) {
        allowed[j] = (uint8_t)key_allowed(job->g, win, qi, j);
        if (!allowed[j]) continue;
        score[j] = job->scale * dot_bf16(qrow, kbase + j * d, d);
        dp[j] = dot_bf16(dorow, vbase + j * d, d);
        if (score[j] > m) m = score[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < n_tok; ++j)
        if (allowed[j]) l += exp(score[j] - m);
    *lse = m + log(l);
    double D = 0.0;
    for (int64_t j = 0; j < n_tok; ++j)
        if (allowed[j]) D += exp(score[j] - *lse) * dp[j];
    *dsum = D;
}

static void load_row(const uint16_t* base, int64_t bh, int64_t tok, int64_t n_tok, int32_t d, double* out)
{
    const uint16_t* p = base + (bh * n_tok + tok) * d;
    for (int32_t c = 0; c < d; ++c) out[c] = bf16_bits_to_double(p[c]);
}

/* dQ of listed query rows: out_a[r * d + c]. */
static void* dq_worker(void* arg)
{
    ora_bjob* job = (ora_bjob*)arg;
    const int64_t n_tok = ora_num_tokens(job->g);
    const int32_t d = job->d;
    double* score = (double*)malloc(sizeof(double) * (size_t)n_tok);
    double* dp = (double*)malloc(sizeof(double) * (size_t)n_tok);
    uint8_t* allowed = (uint8_t*)malloc((size_t)n_tok);
    double* qrow = (double*)malloc(sizeof(double) * (size_t)d);
    double* dorow = (double*)malloc(sizeof(double) * (size_t)d);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    if (!score || !dp || !allowed || !qrow || !dorow || !acc) {
        bjob_fail(job, ORA_NO_MEM);
        free(score); free(dp); free(allowed); free(qrow); free(dorow); free(acc);
        return NULL;
    }
    for (;;) {
        int64_t r = bjob_take(job);
        if (r >= job->nitems) break;
        int64_t bh = job->items[2 * r], qi = job->items[2 * r + 1];
        load_row(job->q, bh, qi, n_tok, d, qrow);
        load_row(job->dout, bh, qi, n_tok, d, dorow);
        double lse, D;
        row_pass(job, bh, qi, qrow, dorow, score, dp, allowed, &lse, &D);
        for (int32_t c = 0; c < d; ++c) acc[c] = 0.0;
        const uint16_t* kbase = job->k + bh * n_tok * d;
        for (int64_t j = 0; j < n_tok; ++j) {
            if (!allowed[j]) continue;
            double ds = exp(score[j] - lse) * (dp[j] - D);
            const uint16_t* kp = kbase + j * d;
            for (int32_t c = 0; c < d; ++c) acc[c] += ds * bf16_bits_to_double(kp[c]);
        }
        for (int32_t c = 0; c < d; ++c) job->out_a[r * d + c] = job->scale * acc[c];
    }
    free(score); free(dp); free(allowed); free(qrow); free(dorow); free(acc);
    return NULL;
}

/* LSE and D of every query whose `need` flag is set (items = all (bh, token)). */
static void* stat_worker(void* arg)
{
    ora_bjob* job = (ora_bjob*)arg;
    const int64_t n_tok = ora_num_tokens(job->g);
    const int32_t d = job->d;
    double* score = (double*)malloc(sizeof(double) * (size_t)n_tok);
    double* dp = (double*)malloc(sizeof(double) * (size_t)n_tok);
    uint8_t* allowed = (uint8_t*)malloc((size_t)n_tok);
    double* qrow = (double*)malloc(sizeof(double) * (size_t)d);
    double* dorow = (double*)malloc(sizeof(double) * (size_t)d);
    if (!score || !dp || !allowed || !qrow || !dorow) {
        bjob_fail(job, ORA_NO_MEM);
        free(score); free(dp); free(allowed); free(qrow); free(dorow);
        return NULL;
    }
    for (;;) {
        int64_t r = bjob_take(job);
        if (r >= job->nitems) break;
        if (!job->need[r]) continue;
        int64_t bh = r / n_tok, qi = r % n_tok;
        load_row(job->q, bh, qi, n_tok, d, qrow);
        load_row(job->dout, bh, qi, n_tok, d, dorow);
        row_pass(job, bh, qi, qrow, dorow, score, dp, allowed, &job->stat[2 * r], &job->stat[2 * r + 1]);
    }
    free(score); free(dp); free(allowed); free(qrow); free(dorow);
    return NULL;
}

/* dK and dV of listed key rows: out_a (dK), out_b (dV), [r * d + c].  Sums
 * over every query of the head that attends the key. */
static void* dkdv_worker(void* arg)
{
    ora_bjob* job = (ora_bjob*)arg;
    const int64_t n_tok = ora_num_tokens(job->g);
    const int32_t d = job->d;
    double* krow = (double*)malloc(sizeof(double) * (size_t)d);
    double* vrow = (double*)malloc(sizeof(double) * (size_t)d);
    double* qrow = (double*)malloc(sizeof(double) * (size_t)d);
    double* dorow = (double*)malloc(sizeof(double) * (size_t)d);
    double* ak = (double*)malloc(sizeof(double) * (size_t)d);
    double* av = (double*)malloc(sizeof(double) * (size_t)d);
    if (!krow || !vrow || !qrow || !dorow || !ak || !av) {
        bjob_fail(job, ORA_NO_MEM);
        free(krow); free(vrow); free(qrow); free(dorow); free(ak); free(av);
        return NULL;
    }
    for (;;) {
        int64_t r = bjob_take(job);
        if (r >= job->nitems) break;
        int64_t bh = job->items[2 * r], kj = job->items[2 * r + 1];
        const int32_t* win = job->win + 3 * (bh % job->heads);
        load_row(job->k, bh, kj, n_tok, d, krow);
        load_row(job->v, bh, kj, n_tok, d, vrow);
        for (int32_t c = 0; c < d; ++c) ak[c] = av[c] = 0.0;
        for (int64_t qi = 0; qi < n_tok; ++qi) {
            if (!key_allowed(job->g, win, qi, kj)) continue;
            load_row(job->q, bh, qi, n_tok, d, qrow);
            load_row(job->dout, bh, qi, n_tok, d, dorow);
            const double* st = &job->stat[2 * (bh * n_tok + qi)];
            double p = exp(job->scale * dot_bf16(krow, job->q + (bh * n_tok + qi) * d, d) - st[0]);
            double dpv = 0.0;
            for (int32_t c = 0; c < d; ++c) dpv += dorow[c] * vrow[c];
            double ds = p * (dpv - st[1]);
            for (int32_t c = 0; c < d; ++c) {
                ak[c] += ds * qrow[c];
                av[c] += p * dorow[c];
            }
        }
        for (int32_t c = 0; c < d; ++c) {
            job->out_a[r * d + c] = job->scale * ak[c];
            job->out_b[r * d + c] = av[c];
        }
    }
    free(krow); free(vrow); free(qrow); free(dorow); free(ak); free(av);
    return NULL;
}

static int run_bjob(ora_bjob* job, void* (*fn)(void*), int32_t nthreads)
{
    job->next = 0;
    pthread_t* tid = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!tid) return ORA_NO_MEM;
    int started = 0;
    for (int32_t t = 0; t < nthreads; ++t) {
        if (pthread_create(&tid[t], NULL, fn, job) != 0) break;
        ++started;
    }
    if (started == 0) fn(job);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    free(tid);
    return job->status;
}

static int bjob_init(ora_bjob* job, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     const uint16_t* dout, const ora_geom* g, int64_t batch, int64_t heads, int32_t d,
                     const int32_t* win, float softmax_scale, const int64_t* items, int64_t nitems)
{
    if (!q || !k || !v || !dout || !g || !win || (nitems > 0 && !items)) return ORA_BAD_ARG;
    if (batch <= 0 || heads <= 0 || d <= 0 || nitems < 0) return ORA_BAD_ARG;
    if (!geom_ok(g)) return ORA_BAD_ARG;
    for (int64_t h = 0; h < heads; ++h)
        if (!window_ok(g, win + 3 * h)) return ORA_BAD_ARG;
    int64_t n_tok = ora_num_tokens(g);
    for (int64_t r = 0; r < nitems; ++r) {
        if (items[2 * r] < 0 || items[2 * r] >= batch * heads) return ORA_BAD_ARG;
        if (items[2 * r + 1] < 0 || items[2 * r + 1] >= n_tok) return ORA_BAD_ARG;
    }
    memset(job, 0, sizeof *job);
    job->q = q; job->k = k; job->v = v; job->dout = dout; job->g = g; job->heads = heads; job->d = d;
    job->win = win; job->scale = (double)softmax_scale; job->items = items; job->nitems = nitems;
    job->status = ORA_OK;
    return ORA_OK;
}

/* dQ of an explicit list of query rows.
 *   q, k, v, dout : bf16 bits, [batch, heads, N, d], raster token order
 *   rows          : nrows pairs (bh, raster query token)
 *   out_dq        : nrows * d doubles
 * Returns ORA_OK, ORA_BAD_ARG or ORA_NO_MEM. */
int ora_sta_backward_dq(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                        const ora_geom* g, int64_t batch, int64_t heads, int32_t d,
                        const int32_t* win, float softmax_scale, const int64_t* rows, int64_t nrows,
                        double* out_dq, int32_t nthreads)
{
    ora_bjob job;
    int st = bjob_init(&job, q, k, v, dout, g, batch, heads, d, win, softmax_scale, rows, nrows);
    if (st != ORA_OK) return st;
    if (!out_dq || nthreads <= 0) return ORA_BAD_ARG;
    job.out_a = out_dq;
    pthread_mutex_init(&job.lock, NULL);
    st = run_bjob(&job, dq_worker, nthreads);
    pthread_mutex_destroy(&job.lock);
    return st;
}

/* dK and dV of an explicit list of key rows.
 *   keys          : nkeys pairs (bh, raster key token)
 *   out_dk, out_dv: nkeys * d doubles each
 * First the LSE and D of every query that attends one of the keys, then, per
 * key, the sums over those queries. */
int ora_sta_backward_dkdv(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                          const ora_geom* g, int64_t batch, int64_t heads, int32_t d,
                          const int32_t* win, float softmax_scale, const int64_t* keys, int64_t nkeys,
                          double* out_dk, double* out_dv, int32_t nthreads)
{
    ora_bjob job;
    int st = bjob_init(&job, q, k, v, dout, g, batch, heads, d, win, softmax_scale, keys, nkeys);
    if (st != ORA_OK) return st;
    if (!out_dk || !out_dv || nthreads <= 0) return ORA_BAD_ARG;
    const int64_t n_tok = ora_num_tokens(g);
    const int64_t total = batch * heads * n_tok;
    uint8_t* need = (uint8_t*)calloc((size_t)total, 1);
    double* stat = (double*)malloc(sizeof(double) * 2 * (size_t)total);
    if (!need || !stat) {
        free(need); free(stat);
        return ORA_NO_MEM;
    }
    for (int64_t r = 0; r < nkeys; ++r) {
        int64_t bh = keys[2 * r], kj = keys[2 * r + 1];
        const int32_t* w = win + 3 * (bh % heads);
        for (int64_t qi = 0; qi < n_tok; ++qi)
            if (key_allowed(g, w, qi, kj)) need[bh * n_tok + qi] = 1;
    }
    pthread_mutex_init(&job.lock, NULL);
    /* pass 1: query statistics */
    job.need = need;
    job.stat = stat;
    job.items = NULL;
    job.nitems = total;
    st = run_bjob(&job, stat_worker, nthreads);
    /* pass 2: per-key sums */
    if (st == ORA_OK) {
        job.items = keys;
        job.nitems = nkeys;
        job.out_a = out_dk;
        job.out_b = out_dv;
        st = run_bjob(&job, dkdv_worker, nthreads);
    }
    pthread_mutex_destroy(&job.lock);
    free(need);
    free(stat);
    return st;
}

/* ------------------------------------------------------------------------ */
/* Attention recall                                                           */
/* ------------------------------------------------------------------------ */
/*
 * "Attention recall" of a query row (page 1, the segment on the 3D locality
 * pattern; page 4, "Observation & Proposed Method"): the share of the row's
 * full-attention softmax mass that falls on the keys inside the local window.
 * Written out: with s_j = scale q . k_j over all N keys,
 *
 *   recall_i = sum_{j in A_i} exp(s_j) / sum_{j} exp(s_j)
 *
 * where A_i is the STA key set of row i (the token mask above).
 */
static void* recall_worker(void* arg)
{
    ora_bjob* job = (ora_bjob*)arg;
    const int64_t n_tok = ora_num_tokens(job->g);
    const int32_t d = job->d;
    double* score = (double*)malloc(sizeof(double) * (size_t)n_tok);
    double* qrow = (double*)malloc(sizeof(double) * (size_t)d);
    if (!score || !qrow) {
        bjob_fail(job, ORA_NO_MEM);
        free(score); free(qrow);
        return NULL;
    }
    for (;;) {
        int64_t r = bjob_take(job);
        if (r >= job->nitems) break;
        int64_t bh = job->items[2 * r], qi = job->items[2 * r + 1];
        const int32_t* win = job->win + 3 * (bh % job->heads);
        load_row(job->q, bh, qi, n_tok, d, qrow);
        const uint16_t* kbase = job->k + bh * n_tok * d;
        double m = -INFINITY;
        for (int64_t j = 0; j < n_tok; ++j) {
            score[j] = job->scale * dot_bf16(qrow, kbase + j * d, d);
            if (score[j] > m) m = score[j];
        }
        double all = 0.0, inside = 0.0;
        for (int64_t j = 0; j < n_tok; ++j) {
            double w = exp(score[j] - m);
            all += w;
            if (key_allowed(job->g, win, qi, j)) inside += w;
        }
        job->out_a[r] = inside / all;
    }
    free(score); free(qrow);
    return NULL;
}

/* Attention recall of an explicit list of query rows (bh, raster token):
 * out_recall[r] in (0, 1].  q and k as for ora_sta_attention. */
int ora_window_recall(const uint16_t* q, const uint16_t* k, const ora_geom* g, int64_t batch, int64_t heads,
                      int32_t d, const int32_t* win, float softmax_scale, const int64_t* rows, int64_t nrows,
                      double* out_recall, int32_t nthreads)
{
    ora_bjob job;
    /* v and dout are not used: pass q so the argument checks see non-null pointers */
    int st = bjob_init(&job, q, k, q, q, g, batch, heads, d, win, softmax_scale, rows, nrows);
    if (st != ORA_OK) return st;
    if (!out_recall || nthreads <= 0) return ORA_BAD_ARG;
    job.out_a = out_recall;
    pthread_mutex_init(&job.lock, NULL);
    st = run_bjob(&job, recall_worker, nthreads);
    pthread_mutex_destroy(&job.lock);
    return st;
}
