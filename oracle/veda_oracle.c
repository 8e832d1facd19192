/*
 * ORACLE -- test infrastructure, not product code.
 *
 * A plain, slow, fp64 CPU statement of Veda-style learned block-sparse
 * attention, used only by tests/, by __graft_entry__.smoke() and by the
 * cpu_baseline leg of bench.py to check and time the CUDA library.  It shares
 * no code, header, table or helper with the CUDA path.
 *
 * What the method computes, and where the pages state it:
 *   - A lightweight predictor, distilled from a full-attention teacher,
 *     selects the blocks that a sparse kernel then computes
 *     (tao.media, "Affine launches MiniMax-H3 video studio ...", section
 *     "Training the Selector, Not the Generator").
 *   - The predictor's trainable parts are a query projection and a key
 *     projection per layer (same article, sections "Training the Selector,
 *     Not the Generator" and "How the SN120 Competition Works").
 *   - Kept blocks are a fixed count per (query tile, head): budgets 16/32/64
 *     (section "How the SN120 Competition Works"), or 32 reference + 32 video
 *     tiles chosen independently with text/VLM/audio keys always dense
 *     (veyrul.com, "Veda R2VA for MiniMax-H3", second paragraph).
 *
 * The pages give no formulas.  Where they are silent this oracle takes the
 * plainest reading (mean pooling over the valid tokens of a tile, a raw
 * dot-product score, the lowest key-tile index winning a tie, padded keys
 * excluded from the softmax); each function below states the one it uses.
 *
 * Arithmetic: every input element is converted exactly to double (fp32 and
 * bf16 both embed exactly); all sums, products and exponentials are fp64.
 * The loops are the definitions written out; the OpenMP pragmas only spread
 * independent output rows over host cores and change no arithmetic order.
 *
 * Parity pins for every function live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1

/* One element of an fp32 or bf16 array, converted exactly to double. */
static double elem(const void* base, int dtype, int64_t off)
{
    if (dtype == ORACLE_F32) return (double)((const float*)base)[off];
    uint32_t bits = ((uint32_t)((const uint16_t*)base)[off]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

/*
 * Tile pooling (the predictor's input, "Training the Selector ..." section).
 * Reading: arithmetic mean over the tokens that exist in the tile.  Tile i
 * covers tokens [i*T, min((i+1)*T, N)); its c_i valid tokens are averaged,
 * so a short last tile is divided by c_i, not by T.
 *
 * x: [B][N][H][d] addressed as x[b*sb + t*st + h*sh + e] (element strides)
 * out: [B][H][n][d], n = ceil(N / T)
 */
void oracle_pool(const void* x, int dtype, int64_t B, int64_t N, int64_t H, int64_t d,
                 int64_t sb, int64_t st, int64_t sh, int64_t T, double* out)
{
    int64_t n = (N + T - 1) / T;
#pragma omp parallel for collapse(3) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h)
            for (int64_t i = 0; i < n; ++i) {
                int64_t t0 = i * T;
                int64_t t1 = min64(N, t0 + T);
                int64_t c = t1 - t0;
                double* o = out + ((b * H + h) * n + i) * d;
                for (int64_t e = 0; e < d; ++e) o[e] = 0.0;
                for (int64_t t = t0; t < t1; ++t)
                    for (int64_t e = 0; e < d; ++e)
                        o[e] += elem(x, dtype, b * sb + t * st + h * sh + e);
                for (int64_t e = 0; e < d; ++e) o[e] = o[e] / (double)c;
            }
}

/*
 * Selector projection (the trained query / key projections, "How the SN120
 * Competition Works": one Q and one K projection per layer, stored in
 * (leading axis, in_features, out_features) order).  Reading: one [d][r]
 * matrix per head, applied to the pooled vector as a row vector:
 *     out[b][h][i][c] = sum_e pooled[b][h][i][e] * W[h][e][c]
 *
 * pooled: [B][H][n][d]; w: [H][d][r] (fp32 or bf16); out: [B][H][n][r]
 */
void oracle_project(const double* pooled, int64_t B, int64_t H, int64_t n, int64_t d,
                    const void* w, int wdtype, int64_t r, double* out)
{
#pragma omp parallel for collapse(3) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h)
            for (int64_t i = 0; i < n; ++i) {
                const double* p = pooled + ((b * H + h) * n + i) * d;
                double* o = out + ((b * H + h) * n + i) * r;
                for (int64_t c = 0; c < r; ++c) {
                    double acc = 0.0;
                    for (int64_t e = 0; e < d; ++e)
                        acc += p[e] * elem(w, wdtype, (h * d + e) * r + c);
                    o[c] = acc;
                }
            }
}

/* Score of key tile j for query tile i of head (b,h): raw dot product of the
 * projected pooled vectors, no scale and no bias (any positive scale leaves
 * the ranking unchanged). */
static double tile_score(const double* qhat, const double* khat, int64_t H, int64_t nq,
                         int64_t nk, int64_t r, int64_t b, int64_t h, int64_t i, int64_t j)
{
    const double* q = qhat + ((b * H + h) * nq + i) * r;
    const double* k = khat + ((b * H + h) * nk + j) * r;
    double acc = 0.0;
    for (int64_t c = 0; c < r; ++c) acc += q[c] * k[c];
    return acc;
}

/* Scores of whole rows: rows[] lists row ids (b*H + h)*nq + i; out: [nrows][nk]. */
void oracle_scores(const double* qhat, const double* khat, int64_t B, int64_t H, int64_t nq,
                   int64_t nk, int64_t r, const int64_t* rows, int64_t nrows, double* out)
{
    (void)B;
#pragma omp parallel for schedule(static)
    for (int64_t q = 0; q < nrows; ++q) {
        int64_t row = rows[q];
        int64_t i = row % nq;
        int64_t bh = row / nq;
        int64_t b = bh / H, h = bh % H;
        for (int64_t j = 0; j < nk; ++j)
            out[q * nk + j] = tile_score(qhat, khat, H, nq, nk, r, b, h, i, j);
    }
}

typedef struct {
    double s;
    int32_t j;
} scored_tile;

/* Rank order of the selection: higher score first; equal scores -> lower
 * key-tile index first (the lowest index wins a tie). */
static int by_score_desc_then_index(const void* pa, const void* pb)
{
    const scored_tile* a = (const scored_tile*)pa;
    const scored_tile* b = (const scored_tile*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int int32_ascending(const void* pa, const void* pb)
{
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/*
 * Fixed-budget selection: for every (b, h, query tile i), score all nk key
 * tiles, order them by (score descending, index ascending), keep the first k
 * and emit those k indices in ascending order.
 *
 * idx: [B][H][nq][k].  kth / next (nullable): per row, the k-th and (k+1)-th
 * scores in rank order (next = NAN when k == nk); they bound the tie band.
 */
void oracle_select(const double* qhat, const double* khat, int64_t B, int64_t H, int64_t nq,
                   int64_t nk, int64_t r, int64_t k, int32_t* idx, double* kth, double* next)
{
#pragma omp parallel
    {
        scored_tile* row = (scored_tile*)malloc(sizeof(scored_tile) * (size_t)nk);
#pragma omp for collapse(3) schedule(static)
        for (int64_t b = 0; b < B; ++b)
            for (int64_t h = 0; h < H; ++h)
                for (int64_t i = 0; i < nq; ++i) {
                    for (int64_t j = 0; j < nk; ++j) {
                        row[j].s = tile_score(qhat, khat, H, nq, nk, r, b, h, i, j);
                        row[j].j = (int32_t)j;
                    }
                    qsort(row, (size_t)nk, sizeof(scored_tile), by_score_desc_then_index);
                    int64_t rid = (b * H + h) * nq + i;
                    int32_t* dst = idx + rid * k;
                    for (int64_t m = 0; m < k; ++m) dst[m] = row[m].j;
                    qsort(dst, (size_t)k, sizeof(int32_t), int32_ascending);
                    if (kth) kth[rid] = row[k - 1].s;
                    if (next) next[rid] = (k < nk) ? row[k].s : NAN;
                }
        free(row);
    }
}

/* A key/value segment: [B][n][H][d] with element strides (d contiguous). */
typedef struct {
    const void* k;
    const void* v;
    int64_t n;
    int64_t sb, st, sh;
} oracle_segment;

/* One problem as the oracle sees it. */
typedef struct {
    const void* q;
    int64_t qsb, qst, qsh;
    int dtype;
    int64_t B, H, d, T;
    oracle_segment video, ref, dense;   /* ref.n == 0 / dense.n == 0: absent */
    double scale;                       /* softmax scale applied to q.k */
    int64_t nq_tok;                     /* query tokens: the video's own, or the rows of
                                           non-video (dense) queries */
} oracle_problem;

/*
 * Block-sparse attention restricted to the kept tiles.
 *
 * For query token t of query tile i (valid tokens only), the key set is
 *     every valid token of each kept video tile   (idx_v row of (b,h,i))
 *   + every valid token of each kept reference tile (idx_r row, if present)
 *   + every dense (text / VLM / audio) token.
 * Then, in fp64, with a plain two-pass softmax over that explicit set:
 *     l_u = scale * (q_t . k_u);  m = max_u l_u;  Z = sum_u exp(l_u - m)
 *     out_t = sum_u exp(l_u - m) v_u / Z;  lse_t = m + ln Z.
 * Padded key slots beyond a segment's end are not keys at all (excluded),
 * the reading of the zero-padded last tile.
 *
 * The queries are the video tokens (nq_tok = video.n), or, for dense-query
 * rows, the tokens of a non-video segment (text, VLM, audio or reference
 * tokens of a joint-attention layer) attending to every tile: the caller then
 * lists every tile of every segment (veyrul.com, "Veda R2VA for MiniMax-H3",
 * second paragraph: text, VLM and audio attention stay dense).
 *
 * units: n_units triples (b, h, i).  out: [n_units][T][d]; lse: [n_units][T]
 * (rows of tokens past the last query token are set to NAN).
 */
void oracle_attend(const oracle_problem* p, const int32_t* idx_v, int64_t k_v,
                   const int32_t* idx_r, int64_t k_r, const int64_t* units, int64_t n_units,
                   double* out, double* lse)
{
    const int64_t T = p->T, d = p->d, H = p->H;
    const int64_t nq = (p->nq_tok + T - 1) / T;
    const int64_t max_keys = k_v * T + (p->ref.n > 0 ? k_r * T : 0) + p->dense.n;

#pragma omp parallel
    {
        /* the explicit key list of one query tile: (segment, token) pairs */
        const oracle_segment** kseg =
            (const oracle_segment**)malloc(sizeof(oracle_segment*) * (size_t)(max_keys + 1));
        int64_t* ktok = (int64_t*)malloc(sizeof(int64_t) * (size_t)(max_keys + 1));
        double* logit = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1));
        double* qrow = (double*)malloc(sizeof(double) * (size_t)d);

#pragma omp for schedule(dynamic, 1)
        for (int64_t u = 0; u < n_units; ++u) {
            const int64_t b = units[3 * u], h = units[3 * u + 1], i = units[3 * u + 2];
            const int64_t rid = (b * H + h) * nq + i;

            int64_t nk = 0;
            for (int64_t m = 0; m < k_v; ++m) {
                int64_t j = idx_v[rid * k_v + m];
                for (int64_t t = j * T; t < min64(p->video.n, (j + 1) * T); ++t) {
                    kseg[nk] = &p->video;
                    ktok[nk++] = t;
                }
            }
            if (p->ref.n > 0) {
                for (int64_t m = 0; m < k_r; ++m) {
                    int64_t j = idx_r[rid * k_r + m];
                    for (int64_t t = j * T; t < min64(p->ref.n, (j + 1) * T); ++t) {
                        kseg[nk] = &p->ref;
                        ktok[nk++] = t;
                    }
                }
            }
            for (int64_t t = 0; t < p->dense.n; ++t) {
                kseg[nk] = &p->dense;
                ktok[nk++] = t;
            }

            for (int64_t tt = 0; tt < T; ++tt) {
                const int64_t t = i * T + tt;
                double* o = out + (u * T + tt) * d;
                if (t >= p->nq_tok) {
                    for (int64_t e = 0; e < d; ++e) o[e] = NAN;
                    if (lse) lse[u * T + tt] = NAN;
                    continue;
                }
                for (int64_t e = 0; e < d; ++e)
                    qrow[e] = elem(p->q, p->dtype, b * p->qsb + t * p->qst + h * p->qsh + e);

                /* pass 1: logits and their maximum */
                double mx = -INFINITY;
                for (int64_t a = 0; a < nk; ++a) {
                    const oracle_segment* s = kseg[a];
                    const int64_t base = b * s->sb + ktok[a] * s->st + h * s->sh;
                    double dot = 0.0;
                    for (int64_t e = 0; e < d; ++e) dot += qrow[e] * elem(s->k, p->dtype, base + e);
                    logit[a] = p->scale * dot;
                    if (logit[a] > mx) mx = logit[a];
                }
                /* pass 2: normaliser and weighted sum of values */
                double z = 0.0;
                for (int64_t e = 0; e < d; ++e) o[e] = 0.0;
                for (int64_t a = 0; a < nk; ++a) {
                    const oracle_segment* s = kseg[a];
                    const int64_t base = b * s->sb + ktok[a] * s->st + h * s->sh;
                    const double w = exp(logit[a] - mx);
                    z += w;
                    for (int64_t e = 0; e < d; ++e) o[e] += w * elem(s->v, p->dtype, base + e);
                }
                for (int64_t e = 0; e < d; ++e) o[e] = o[e] / z;
                if (lse) lse[u * T + tt] = mx + log(z);
            }
        }
        free(kseg);
        free(ktok);
        free(logit);
        free(qrow);
    }
}
