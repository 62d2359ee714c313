/*
 * gla_oracle.c -- fp64 CPU oracle for the key-gated GLA token mixer of GTR.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link
 * or call this file.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes (sources, by page and section):
 *   - "GTR: Gated Token Recurrence for Efficient Dense Prediction", ai.info
 *     paper summary, section "Methodology in Plain English": GTR uses the
 *     key-only variant of gated linear attention -- the state decays along
 *     the key dimension only, the value-side decay is fixed at one -- and
 *     each block runs exactly one directional scan (left-to-right,
 *     right-to-left, top-to-bottom or bottom-to-top) over the stride-16 patch
 *     grid, then puts tokens back in spatial order.
 *   - Same page, "Methodology in Plain English" (last paragraph) and "Future
 *     Directions": the inference operator starts from a zero state.
 *   - GTR project page, section "A Kernel That Makes Recurrence Fast": the
 *     chunkwise operator evaluates the exact recurrence -- the same state
 *     update in a different schedule: per-chunk summaries in parallel, a
 *     scan over chunk boundary states, then per-chunk outputs.
 *   - The recurrence itself is the gated linear attention recurrence of
 *     Yang et al., "Gated Linear Attention Transformers with
 *     Hardware-Efficient Training" (listed among the works GTR builds on):
 *         S_t = diag(exp(g_t)) S_{t-1} + k_t^T v_t,   S_0 = 0,
 *         o_t = (q_t / sqrt(d_k)) S_t
 *     with S_t a d_k x d_v matrix, g_t the per-key-dimension log-gate.
 *     The readout uses S_t *including* token t.
 *
 * Readings taken where the pages are silent:
 *   - tensor layout [B][N][heads][d], tokens in row-major spatial order;
 *   - R->L is the reversed row-major order, T->B is column-major order
 *     (t = col*H + row), B->T is the reversed column-major order;
 *   - the scale 1/sqrt(d_k) multiplies q.
 *
 * All arithmetic is double precision.  Inputs arrive as double arrays that
 * hold the exact fp16 / fp32 values given to the GPU; outputs stay double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Scan order -> row-major token index.  Directions: 0 L->R, 1 R->L,
 * 2 T->B, 3 B->T (ai.info summary, "Methodology in Plain English"; GTR
 * project page, "How GTR Works"). Returns -1 for a bad direction. */
int64_t gla_oracle_scan_index(int dir, int64_t t, int64_t H, int64_t W) {
    int64_t N = H * W;
    int64_t u;
    switch (dir) {
    case 0: return t;
    case 1: return N - 1 - t;
    case 2: return (t % H) * W + t / H;
    case 3: u = N - 1 - t; return (u % H) * W + u / H;
    default: return -1;
    }
}

typedef struct {
    const double *q, *k, *v, *g;
    double *out;
    int B, heads, H, W, dk, dv, dir, chunk;
    /* chunked form extras (may be NULL) */
    double *dS, *gamma, *S_enter;
    /* serial form extra: state after c*chunk tokens, [B][heads][nc+1][dk][dv] */
    double *states;
    /* serial form extras: the state before the first token (NULL: zero) and
     * the state after the last one, each [B][heads][dk][dv] */
    const double *S0;
    double *SN;
    const int *slices; /* optional list of (b*heads+h) slices to compute */
    int n_slices;
    int next;          /* work counter */
    pthread_mutex_t lock;
} job_t;

static int64_t tok_off(const job_t *j, int b, int64_t p, int h, int d) {
    return (((int64_t)b * ((int64_t)j->H * j->W) + p) * j->heads + h) * d;
}

/* The plain serial recurrence for one (b, h) slice. */
static void serial_slice(const job_t *j, int b, int h) {
    const int dk = j->dk, dv = j->dv;
    const int64_t N = (int64_t)j->H * j->W;
    const double scale = 1.0 / sqrt((double)dk);
    double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
    const int64_t slice = (int64_t)b * j->heads + h;
    if (j->S0) memcpy(S, j->S0 + slice * dk * dv, sizeof(double) * dk * dv);
    int64_t nc = j->chunk > 0 ? (N + j->chunk - 1) / j->chunk : 0;
    double *st = NULL;
    if (j->states) {
        st = j->states + ((int64_t)b * j->heads + h) * (nc + 1) * dk * dv;
        memset(st, 0, sizeof(double) * dk * dv); /* state after 0 tokens */
    }
    for (int64_t t = 0; t < N; ++t) {
        int64_t p = gla_oracle_scan_index(j->dir, t, j->H, j->W);
        const double *qt = j->q + tok_off(j, b, p, h, dk);
        const double *kt = j->k + tok_off(j, b, p, h, dk);
        const double *gt = j->g + tok_off(j, b, p, h, dk);
        const double *vt = j->v + tok_off(j, b, p, h, dv);
        double *ot = j->out + tok_off(j, b, p, h, dv);
        for (int i = 0; i < dk; ++i) {
            double a = exp(gt[i]);
            double *row = S + (int64_t)i * dv;
            for (int c = 0; c < dv; ++c) row[c] = a * row[c] + kt[i] * vt[c];
        }
        for (int c = 0; c < dv; ++c) ot[c] = 0.0;
        for (int i = 0; i < dk; ++i) {
            double qi = qt[i] * scale;
            const double *row = S + (int64_t)i * dv;
            for (int c = 0; c < dv; ++c) ot[c] += qi * row[c];
        }
        if (st && ((t + 1) % j->chunk == 0 || t + 1 == N)) {
            int64_t ci = (t + 1 + j->chunk - 1) / j->chunk;
            memcpy(st + ci * dk * dv, S, sizeof(double) * dk * dv);
        }
    }
    if (j->SN) memcpy(j->SN + slice * dk * dv, S, sizeof(double) * dk * dv);
    free(S);
}

/* The chunkwise form for one (b, h) slice, in the order the GTR project page
 * ("A Kernel That Makes Recurrence Fast") describes the schedule:
 *   (1) per-chunk summaries  gamma_c[i] = exp(sum of g over the chunk),
 *       dS_c[i][:] = sum_s exp(b_last[i] - b_s[i]) k_s[i] v_s[:]
 *       where b is the inclusive prefix sum of g inside the chunk;
 *   (2) the boundary scan  S_enter_0 = 0,
 *       S_enter_{c+1} = diag(gamma_c) S_enter_c + dS_c;
 *   (3) per-chunk outputs
 *       o_t = sum_i q~_t[i] exp(b_t[i]) S_enter_c[i][:]
 *           + sum_{s<=t in chunk} (sum_i q~_t[i] exp(b_t[i]-b_s[i]) k_s[i]) v_s.
 * Every decay factor is the exponential of a difference of prefix sums,
 * evaluated directly in double precision. */
static void chunked_slice(const job_t *j, int b, int h) {
    const int dk = j->dk, dv = j->dv, C = j->chunk;
    const int64_t N = (int64_t)j->H * j->W;
    const int64_t nc = (N + C - 1) / C;
    const double scale = 1.0 / sqrt((double)dk);
    const int64_t slice = (int64_t)b * j->heads + h;
    double *dS = j->dS ? j->dS + slice * nc * dk * dv
                       : (double *)malloc(sizeof(double) * nc * dk * dv);
    double *gam = j->gamma ? j->gamma + slice * nc * dk
                           : (double *)malloc(sizeof(double) * nc * dk);
    double *Se = j->S_enter ? j->S_enter + slice * nc * dk * dv
                            : (double *)malloc(sizeof(double) * nc * dk * dv);
    double *bsum = (double *)malloc(sizeof(double) * C * dk);
    int64_t *pos = (int64_t *)malloc(sizeof(int64_t) * C);

    /* (1) summaries, independent per chunk */
    for (int64_t c = 0; c < nc; ++c) {
        int64_t t0 = c * C;
        int len = (int)((N - t0) < C ? (N - t0) : C);
        for (int s = 0; s < len; ++s) {
            pos[s] = gla_oracle_scan_index(j->dir, t0 + s, j->H, j->W);
            const double *gs = j->g + tok_off(j, b, pos[s], h, dk);
            for (int i = 0; i < dk; ++i)
                bsum[s * dk + i] = (s ? bsum[(s - 1) * dk + i] : 0.0) + gs[i];
        }
        double *dSc = dS + c * dk * dv;
        memset(dSc, 0, sizeof(double) * dk * dv);
        for (int i = 0; i < dk; ++i) gam[c * dk + i] = exp(bsum[(len - 1) * dk + i]);
        for (int s = 0; s < len; ++s) {
            const double *ks = j->k + tok_off(j, b, pos[s], h, dk);
            const double *vs = j->v + tok_off(j, b, pos[s], h, dv);
            for (int i = 0; i < dk; ++i) {
                double w = exp(bsum[(len - 1) * dk + i] - bsum[s * dk + i]) * ks[i];
                for (int e = 0; e < dv; ++e) dSc[i * dv + e] += w * vs[e];
            }
        }
    }
    /* (2) boundary scan */
    memset(Se, 0, sizeof(double) * dk * dv);
    for (int64_t c = 0; c + 1 < nc; ++c) {
        const double *cur = Se + c * dk * dv;
        double *nxt = Se + (c + 1) * dk * dv;
        for (int i = 0; i < dk; ++i)
            for (int e = 0; e < dv; ++e)
                nxt[i * dv + e] = gam[c * dk + i] * cur[i * dv + e] + dS[c * dk * dv + i * dv + e];
    }
    /* (3) outputs, independent per chunk */
    for (int64_t c = 0; c < nc; ++c) {
        int64_t t0 = c * C;
        int len = (int)((N - t0) < C ? (N - t0) : C);
        for (int s = 0; s < len; ++s) {
            pos[s] = gla_oracle_scan_index(j->dir, t0 + s, j->H, j->W);
            const double *gs = j->g + tok_off(j, b, pos[s], h, dk);
            for (int i = 0; i < dk; ++i)
                bsum[s * dk + i] = (s ? bsum[(s - 1) * dk + i] : 0.0) + gs[i];
        }
        const double *Sc = Se + c * dk * dv;
        for (int t = 0; t < len; ++t) {
            const double *qt = j->q + tok_off(j, b, pos[t], h, dk);
            double *ot = j->out + tok_off(j, b, pos[t], h, dv);
            for (int e = 0; e < dv; ++e) ot[e] = 0.0;
            for (int i = 0; i < dk; ++i) {
                double w = qt[i] * scale * exp(bsum[t * dk + i]);
                for (int e = 0; e < dv; ++e) ot[e] += w * Sc[i * dv + e];
            }
            for (int s = 0; s <= t; ++s) {
                const double *ks = j->k + tok_off(j, b, pos[s], h, dk);
                const double *vs = j->v + tok_off(j, b, pos[s], h, dv);
                double a = 0.0;
                for (int i = 0; i < dk; ++i)
                    a += qt[i] * scale * exp(bsum[t * dk + i] - bsum[s * dk + i]) * ks[i];
                for (int e = 0; e < dv; ++e) ot[e] += a * vs[e];
            }
        }
    }
    if (!j->dS) free(dS);
    if (!j->gamma) free(gam);
    if (!j->S_enter) free(Se);
    free(bsum);
    free(pos);
}

typedef struct { job_t *job; int chunked; } worker_arg_t;

static void *worker(void *arg) {
    worker_arg_t *wa = (worker_arg_t *)arg;
    job_t *j = wa->job;
    int total = j->slices ? j->n_slices : j->B * j->heads;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        int idx = j->next++;
        pthread_mutex_unlock(&j->lock);
        if (idx >= total) break;
        int sl = j->slices ? j->slices[idx] : idx;
        int b = sl / j->heads, h = sl % j->heads;
        if (wa->chunked) chunked_slice(j, b, h);
        else serial_slice(j, b, h);
    }
    return NULL;
}

static int run(job_t *j, int chunked, int nthreads) {
    if (j->B < 0 || j->heads < 0 || j->H < 0 || j->W < 0 || j->dk <= 0 || j->dv <= 0) return 1;
    if (j->dir < 0 || j->dir > 3) return 1;
    if (chunked && j->chunk <= 0) return 1;
    if (j->slices) {
        for (int s = 0; s < j->n_slices; ++s)
            if (j->slices[s] < 0 || j->slices[s] >= j->B * j->heads) return 1;
    }
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    j->next = 0;
    pthread_mutex_init(&j->lock, NULL);
    pthread_t th[256];
    worker_arg_t wa = {j, chunked};
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &wa);
    worker(&wa);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&j->lock);
    return 0;
}

/* Serial recurrence over all slices (or the listed ones).  Arrays are
 * [B][H*W][heads][d].  If `states` is non-NULL it receives, per slice, the
 * state after 0, chunk, 2*chunk, ..., N tokens: [B][heads][nc+1][dk][dv]
 * (only written for the slices computed).  Returns 0 on success. */
int gla_oracle_serial(const double *q, const double *k, const double *v, const double *g,
                      int B, int heads, int H, int W, int dk, int dv, int dir,
                      double *out, int chunk, double *states,
                      const int *slices, int n_slices, int nthreads) {
    job_t j;
    memset(&j, 0, sizeof j);
    j.q = q; j.k = k; j.v = v; j.g = g; j.out = out;
    j.B = B; j.heads = heads; j.H = H; j.W = W; j.dk = dk; j.dv = dv; j.dir = dir;
    j.chunk = chunk; j.states = states; j.slices = slices; j.n_slices = n_slices;
    if (states && chunk <= 0) return 1;
    return run(&j, 0, nthreads);
}

/* Chunkwise form.  dS: [B][heads][nc][dk][dv], gamma: [B][heads][nc][dk],
 * S_enter: [B][heads][nc][dk][dv] (the state entering each chunk); each may
 * be NULL.  Returns 0 on success. */
int gla_oracle_chunked(const double *q, const double *k, const double *v, const double *g,
                       int B, int heads, int H, int W, int dk, int dv, int dir, int chunk,
                       double *out, double *dS, double *gamma, double *S_enter,
                       const int *slices, int n_slices, int nthreads) {
    job_t j;
    memset(&j, 0, sizeof j);
    j.q = q; j.k = k; j.v = v; j.g = g; j.out = out;
    j.B = B; j.heads = heads; j.H = H; j.W = W; j.dk = dk; j.dv = dv; j.dir = dir;
    j.chunk = chunk; j.dS = dS; j.gamma = gamma; j.S_enter = S_enter;
    j.slices = slices; j.n_slices = n_slices;
    return run(&j, 1, nthreads);
}

/* The serial recurrence from a given initial state, returning the final
 * state as well: the state carried across frames that the ai.info summary
 * names as the natural extension ("Future Directions").  S0 (may be NULL for
 * zero) and SN (may be NULL) are [B][heads][dk][dv]; everything else as
 * gla_oracle_serial.  Returns 0 on success. */
int gla_oracle_serial_state(const double *q, const double *k, const double *v, const double *g,
                            int B, int heads, int H, int W, int dk, int dv, int dir,
                            const double *S0, double *out, double *SN,
                            const int *slices, int n_slices, int nthreads) {
    job_t j;
    memset(&j, 0, sizeof j);
    j.q = q; j.k = k; j.v = v; j.g = g; j.out = out;
    j.B = B; j.heads = heads; j.H = H; j.W = W; j.dk = dk; j.dv = dv; j.dir = dir;
    j.S0 = S0; j.SN = SN; j.slices = slices; j.n_slices = n_slices;
    return run(&j, 0, nthreads);
}

/* The output gate on the RMS-normalised mixer output (ai.info summary,
 * "Methodology in Plain English": a data-dependent output gate applied to
 * the RMS-normalised output).  For every row of d_v values (one token of
 * one head) o, gate pre-activation r and the norm weight w:
 *     y[e] = o[e] / sqrt(mean_e'(o[e']^2) + eps) * w[e] * r[e] * sigmoid(r[e])
 * Root-mean-square normalisation as in Zhang and Sennrich (RMSNorm, on the
 * mlsanity reference list of GTR); the swish gate as in gated linear
 * attention (Yang et al., same list).  o, r, y: [rows][dv]; w: [dv]. */
void gla_oracle_output_gate(const double *o, const double *r, const double *w, double eps,
                            int64_t rows, int dv, double *y) {
    for (int64_t i = 0; i < rows; ++i) {
        const double *orow = o + i * dv, *rrow = r + i * dv;
        double ms = 0.0;
        for (int e = 0; e < dv; ++e) ms += orow[e] * orow[e];
        ms /= dv;
        const double inv = 1.0 / sqrt(ms + eps);
        for (int e = 0; e < dv; ++e) {
            const double sig = 1.0 / (1.0 + exp(-rrow[e]));
            y[i * dv + e] = orow[e] * inv * w[e] * rrow[e] * sig;
        }
    }
}

/* Spatial SwiGLU's gating with its 3x3 depthwise convolution (ai.info
 * summary, "Methodology in Plain English": a 3x3 depthwise convolution in the
 * value branch of a SwiGLU block, applied on the 2-D patch grid; GTR project
 * page, "Spatial SwiGLU").  a (gate branch) and bv (value branch) are
 * [B][H*W][C] in row-major spatial order, wc [C][3][3], bias [C] (may be
 * NULL); zero padding at the grid border:
 *     y[b][p][c] = silu(a[b][p][c]) * (bias[c] + sum_{dy,dx} wc[c][dy+1][dx+1] * bv[b][p + dy*W + dx][c])
 * with silu(x) = x * sigmoid(x).  y: [B][H*W][C]. */
void gla_oracle_sswiglu(const double *a, const double *bv, const double *wc, const double *bias,
                        int B, int H, int W, int C, double *y) {
    for (int b = 0; b < B; ++b)
        for (int r = 0; r < H; ++r)
            for (int col = 0; col < W; ++col)
                for (int c = 0; c < C; ++c) {
                    double acc = bias ? bias[c] : 0.0;
                    for (int dy = -1; dy <= 1; ++dy)
                        for (int dx = -1; dx <= 1; ++dx) {
                            const int rr = r + dy, cc = col + dx;
                            if (rr < 0 || rr >= H || cc < 0 || cc >= W) continue;
                            acc += wc[c * 9 + (dy + 1) * 3 + (dx + 1)] *
                                   bv[(((int64_t)b * H + rr) * W + cc) * C + c];
                        }
                    const int64_t o = (((int64_t)b * H + r) * W + col) * C + c;
                    const double x = a[o];
                    y[o] = x / (1.0 + exp(-x)) * acc;
                }
}
