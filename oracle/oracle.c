/*
 * Lightning-indexer oracle: plain, slow, fp64 CPU definitions of every step of
 * the indexer path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark load this library.  The CUDA library never
 * includes, links or calls it, and it includes nothing from the CUDA side.
 *
 * Every function states the passage it follows.  The pages never print the
 * lightning-indexer formula itself; the definition used throughout is
 *
 *     I[t,s] = sum_j w[t,j] * ReLU(q[t,j,:] . k[s,:])
 *
 * In the pages each visible position receives one such score and top-k
 * follows (IndexCache explainer, Symbol Map); the indexer scans the whole
 * cache and keeps the 2048 best tokens (Multi-layer Indexer abstract); and
 * the score is a low-rank bilinear form of query and key, of the same kind
 * as an attention logit (Multi-layer Indexer podcast page, deep dive).
 *
 * Arithmetic: every score is accumulated in double.  The one place where the
 * oracle works in fp32 is the query quantiser, whose output is an integer code
 * and therefore must be decided in the precision the kernel uses (fp32 IEEE
 * division, round-to-nearest-even into e4m3).  Build with -ffp-contract=off so
 * that no multiply-add is fused behind the reader's back.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_E4M3 2
#define ORC_F64 3

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

/* e4m3 ("fn" variant): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent field 0 holds subnormals m * 2^-9; the pattern S.1111.111 is
 * NaN and there is no infinity, so the largest finite magnitude is
 * 1.75 * 2^8 = 448. */
double orc_e4m3_decode(uint8_t b)
{
    int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* Round an fp32 value to the nearest e4m3 value, ties to even mantissa, and
 * clamp finite values beyond 448 to +-448 (saturation to the largest finite).  Written
 * from the format definition above: find the binade, divide by the grid step
 * of that binade (a power of two, so exact), round with nearbyint (the default
 * rounding mode is round-to-nearest-even), then re-assemble the fields. */
uint8_t orc_e4m3_encode(float xf)
{
    double x = (double)xf, a, step, n;
    uint8_t s;
    int E;
    if (isnan(x)) return 0x7F;
    s = signbit(x) ? 0x80 : 0x00;
    a = fabs(x);
    if (a >= 448.0) return s | 0x7E;
    if (a == 0.0) return s;
    frexp(a, &E);
    E -= 1;                 /* a in [2^E, 2^(E+1)) */
    if (E < -6) E = -6;     /* below the smallest normal the grid is fixed at 2^-9 */
    step = ldexp(1.0, E - 3);
    n = nearbyint(a / step);
    if (n >= 16.0) {        /* rounded up into the next binade */
        E += 1;
        n = 8.0;
    }
    if (ldexp(n, E - 3) > 448.0) return s | 0x7E;
    if (n < 8.0) return s | (uint8_t)n; /* subnormal: exponent field 0 */
    return s | (uint8_t)(((E + 7) << 3) | ((int)n - 8));
}

/* bfloat16 is the upper half of an fp32 bit pattern. */
float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static double load_elem(const void* p, int dtype, size_t i)
{
    switch (dtype) {
    case ORC_F32: return (double)((const float*)p)[i];
    case ORC_BF16: return (double)orc_bf16_to_f32(((const uint16_t*)p)[i]);
    case ORC_E4M3: return orc_e4m3_decode(((const uint8_t*)p)[i]);
    default: return ((const double*)p)[i];
    }
}

/* ------------------------------------------------------------------------ */
/* Query quantisation                                                        */
/* ------------------------------------------------------------------------ */

/* FP8 scoring needs the query in e4m3 as well as the keys.  Per (row, head):
 *   sq = absmax(q[r,j,:]) / 448   (1 when the head is all zero),
 *   q8 = e4m3(q / sq)             (fp32 division, nearest-even, saturating),
 *   w_eff = w[r,j] * sq           (fp32 product).
 * The pages fix no query precision; this per-(row, head) absmax recipe is the
 * same per-token absmax rule the FP8 key cache uses. */
void orc_quantize_query(const uint16_t* q, const float* w, int R, int H, int d,
                        uint8_t* q8, float* sq, float* w_eff)
{
    for (int r = 0; r < R; ++r) {
        for (int j = 0; j < H; ++j) {
            size_t base = ((size_t)r * H + j) * (size_t)d;
            float amax = 0.0f, s;
            for (int e = 0; e < d; ++e) {
                float v = fabsf(orc_bf16_to_f32(q[base + e]));
                if (v > amax) amax = v;
            }
            s = amax > 0.0f ? amax / 448.0f : 1.0f;
            for (int e = 0; e < d; ++e) q8[base + e] = orc_e4m3_encode(orc_bf16_to_f32(q[base + e]) / s);
            sq[(size_t)r * H + j] = s;
            if (w) w_eff[(size_t)r * H + j] = w[(size_t)r * H + j] * s;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Indexer score                                                             */
/* ------------------------------------------------------------------------ */

typedef struct {
    int R, H, d, L;
    int q_dtype;
    const void* q;         /* [R, H, d] */
    const float* q_scale;  /* [R, H] or NULL: query value = q * q_scale */
    const float* w;        /* [R, H] */
    int k_dtype;
    const void* k;         /* rows of d elements */
    const float* k_scale;  /* one per key row, or NULL: key value = k * k_scale */
    long long k_batch_rows;/* rows between the caches of consecutive rows; 0 = one shared cache */
    const int* len;        /* [R] visible length per row, or NULL (= L); ignored when causal */
    int causal;            /* 1: row t sees positions s <= t + causal_offset */
    int causal_offset;
} orc_score_args;

/* Number of cache positions row r may see.  Decode: the whole cache of that
 * request, i.e. its first len[r] positions (Multi-layer Indexer abstract:
 * the scan covers the entire cache).  Causal prefill: query token t sees the
 * prefix up to and including its own position (IndexCache explainer, Why This
 * Exists: in prefill the indexer runs over the prefix; inclusive is this
 * oracle's reading). */
static int visible_len(const orc_score_args* a, int r)
{
    long long n;
    if (a->causal) n = (long long)r + 1 + a->causal_offset;
    else n = a->len ? a->len[r] : a->L;
    if (n < 0) n = 0;
    if (n > a->L) n = a->L;
    return (int)n;
}

typedef struct {
    const orc_score_args* a;
    const int* rows;
    int n_rows;
    double* out;
    double* mag;
    long long first, last; /* flattened (row slot, position) range */
} score_job;

static void* score_worker(void* p)
{
    score_job* J = (score_job*)p;
    const orc_score_args* a = J->a;
    int H = a->H, d = a->d, L = a->L;
    double* qrow = (double*)malloc(sizeof(double) * (size_t)H * d);
    double* krow = (double*)malloc(sizeof(double) * (size_t)d);
    int cur = -1;
    for (long long f = J->first; f < J->last; ++f) {
        int slot = (int)(f / L), s = (int)(f % L);
        int r = J->rows ? J->rows[slot] : slot;
        size_t o = (size_t)slot * L + s;
        long long krow0;
        double I = 0.0, M = 0.0;
        if (s >= visible_len(a, r)) {
            J->out[o] = -INFINITY;
            if (J->mag) J->mag[o] = 0.0;
            continue;
        }
        if (r != cur) { /* decode this row's query once */
            for (int j = 0; j < H; ++j) {
                double sc = a->q_scale ? (double)a->q_scale[(size_t)r * H + j] : 1.0;
                for (int e = 0; e < d; ++e)
                    qrow[(size_t)j * d + e] = load_elem(a->q, a->q_dtype, ((size_t)r * H + j) * d + e) * sc;
            }
            cur = r;
        }
        krow0 = (long long)r * a->k_batch_rows + s;
        for (int e = 0; e < d; ++e) {
            double sc = a->k_scale ? (double)a->k_scale[krow0] : 1.0;
            krow[e] = load_elem(a->k, a->k_dtype, (size_t)krow0 * d + e) * sc;
        }
        for (int j = 0; j < H; ++j) {
            double x = 0.0, wj = (double)a->w[(size_t)r * H + j];
            for (int e = 0; e < d; ++e) x += qrow[(size_t)j * d + e] * krow[e];
            I += wj * (x > 0.0 ? x : 0.0);
            M += fabs(wj) * fabs(x);
        }
        J->out[o] = I;
        if (J->mag) J->mag[o] = M;
    }
    free(qrow);
    free(krow);
    return NULL;
}

/* Score rows ``rows[0..n_rows)`` (all R rows when rows == NULL) against every
 * cache position.  out[slot, s] = I for visible positions and -inf beyond.
 * mag (optional) receives sum_j |w_j| * |q_j . k_s|, the scale against which a
 * rounding error in the sum is measured. */
int orc_index_score(const orc_score_args* a, const int* rows, int n_rows, double* out, double* mag,
                    int nthreads)
{
    long long total;
    pthread_t* th;
    score_job* jobs;
    if (!rows) n_rows = a->R;
    total = (long long)n_rows * a->L;
    if (nthreads < 1) nthreads = 1;
    th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    jobs = (score_job*)malloc(sizeof(score_job) * nthreads);
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].a = a;
        jobs[t].rows = rows;
        jobs[t].n_rows = n_rows;
        jobs[t].out = out;
        jobs[t].mag = mag;
        jobs[t].first = total * t / nthreads;
        jobs[t].last = total * (t + 1) / nthreads;
        pthread_create(&th[t], NULL, score_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Top-k selection                                                           */
/* ------------------------------------------------------------------------ */

typedef struct {
    double v;
    int i;
} vi_pair;

/* Selection order: larger score first; equal scores go to the lower position
 * (the deterministic lowest-index tie-break); NaN ranks below every number.
 * -0.0 and +0.0 compare equal, as numbers do. */
static int cmp_rank(const void* pa, const void* pb)
{
    const vi_pair* a = (const vi_pair*)pa;
    const vi_pair* b = (const vi_pair*)pb;
    int na = isnan(a->v), nb = isnan(b->v);
    if (na != nb) return na ? 1 : -1;
    if (!na) {
        if (a->v > b->v) return -1;
        if (a->v < b->v) return 1;
    }
    return a->i < b->i ? -1 : (a->i > b->i ? 1 : 0);
}

static int cmp_pos(const void* pa, const void* pb)
{
    int a = ((const vi_pair*)pa)->i, b = ((const vi_pair*)pb)->i;
    return a < b ? -1 : (a > b ? 1 : 0);
}

/* Keep the k highest-scoring of the n values (IndexCache explainer, Symbol
 * Map: the selected set T_t holds k token positions; Multi-layer Indexer
 * abstract: the 2048 best-scoring tokens are kept).  Full sort by rank,
 * take min(k, n), report them in ascending position order, pad with -1.
 * ``pos`` (optional) maps slot i to the reported position. */
static void topk_one(const double* v, int n, const int* pos, int k, int* idx, double* vals)
{
    int m = n < k ? n : k;
    vi_pair* p = (vi_pair*)malloc(sizeof(vi_pair) * (size_t)(n > 0 ? n : 1));
    for (int i = 0; i < n; ++i) {
        p[i].v = v[i];
        p[i].i = pos ? pos[i] : i;
    }
    qsort(p, (size_t)n, sizeof(vi_pair), cmp_rank);
    qsort(p, (size_t)m, sizeof(vi_pair), cmp_pos);
    for (int i = 0; i < k; ++i) {
        idx[i] = i < m ? p[i].i : -1;
        if (vals) vals[i] = i < m ? p[i].v : -INFINITY;
    }
    free(p);
}

/* Row r holds len[r] valid scores (all max_len when len == NULL; r + 1 +
 * causal_offset, clipped to [0, max_len], when causal is set). */
int orc_topk(const double* scores, long long ld, const int* len, int rows, int max_len, int causal,
             int causal_offset, int k, int* idx, double* vals)
{
    for (int r = 0; r < rows; ++r) {
        long long n = causal ? (long long)r + 1 + causal_offset : (len ? len[r] : max_len);
        if (n < 0) n = 0;
        if (n > max_len) n = max_len;
        topk_one(scores + (size_t)r * ld, (int)n, NULL, k, idx + (size_t)r * k, vals ? vals + (size_t)r * k : NULL);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* LatentIndex: decoder absorption and explicit key reconstruction           */
/* ------------------------------------------------------------------------ */

/* LatentIndex abstract and Figure 1: layer l's keys are defined by a decoder
 * applied to the shared latent cache, k^(l)_j[s] = W_dec[l,j] c[s]  (W_dec[l,j]
 * is d x dc, one per head j).  Absorbing the decoder into the query gives
 *     q~[b,j,:] = W_dec[l,j]^T q[b,j,:],   q~ . c[s] = q . k^(l)_j[s],
 * so the shared cache is scored directly, without rebuilding historical keys.
 * wdec is [H, d, dc] row-major, q is [B, H, d], qt receives [B, H, dc]. */
void orc_absorb(const uint16_t* q, const uint16_t* wdec, int B, int H, int d, int dc, double* qt)
{
    for (int b = 0; b < B; ++b)
        for (int j = 0; j < H; ++j)
            for (int c = 0; c < dc; ++c) {
                double acc = 0.0;
                for (int e = 0; e < d; ++e)
                    acc += (double)orc_bf16_to_f32(q[((size_t)b * H + j) * d + e]) *
                           (double)orc_bf16_to_f32(wdec[((size_t)j * d + e) * dc + c]);
                qt[((size_t)b * H + j) * dc + c] = acc;
            }
}

/* The non-absorbed route, kept only to check the identity above: rebuild the
 * per-head keys of one latent row, k[j,e] = sum_c W_dec[j,e,c] * c[c]. */
void orc_decode_keys(const uint16_t* wdec, const uint16_t* crow, int H, int d, int dc, double* kj)
{
    for (int j = 0; j < H; ++j)
        for (int e = 0; e < d; ++e) {
            double acc = 0.0;
            for (int c = 0; c < dc; ++c)
                acc += (double)orc_bf16_to_f32(wdec[((size_t)j * d + e) * dc + c]) * (double)orc_bf16_to_f32(crow[c]);
            kj[(size_t)j * d + e] = acc;
        }
}

/* Score of request b's query against latent row s through rebuilt per-head
 * keys: sum_j w[b,j] * ReLU(q[b,j,:] . k_j[s]).  Rows listed in ``pos``. */
void orc_latent_score_rebuilt(const uint16_t* q, const float* w, const uint16_t* wdec, const uint16_t* c,
                              long long c_batch_rows, int b, int H, int d, int dc, const int* pos, int n,
                              double* out)
{
    double* kj = (double*)malloc(sizeof(double) * (size_t)H * d);
    for (int i = 0; i < n; ++i) {
        const uint16_t* crow = c + ((size_t)b * c_batch_rows + pos[i]) * dc;
        double I = 0.0;
        orc_decode_keys(wdec, crow, H, d, dc, kj);
        for (int j = 0; j < H; ++j) {
            double x = 0.0;
            for (int e = 0; e < d; ++e)
                x += (double)orc_bf16_to_f32(q[((size_t)b * H + j) * d + e]) * kj[(size_t)j * d + e];
            I += (double)w[(size_t)b * H + j] * (x > 0.0 ? x : 0.0);
        }
        out[i] = I;
    }
    free(kj);
}

/* ------------------------------------------------------------------------ */
/* Hierarchical selection: followers refine the anchor's candidates          */
/* ------------------------------------------------------------------------ */

/* LatentIndex abstract: the anchor proposes a shared candidate set and each
 * follower refines it on its own.  Reading: a follower re-scores only
 * the candidate latent rows (cand[b, i] >= 0; negative entries are padding)
 * with its own absorbed query and keeps its k best by (score desc, cache
 * position asc); it never adds a position outside the candidates.  Output:
 * cache positions in ascending order, padded with -1.
 * qt: [F, B, H, dc] in qt_dtype; w: [F, B, H]; c: bf16 rows of dc;
 * cand: [B, C]; out: [F, B, k]; cand_scores (optional): [F, B, C]. */
typedef struct {
    int f0, f1; /* (follower, request) pairs [f0, f1) flattened as f * B + b */
    int qt_dtype;
    const void* qt;
    const float* w;
    const uint16_t* c;
    long long c_batch_rows;
    const int* cand;
    int F, B, H, dc, C, k;
    int* out;
    double* cand_scores;
} hs_job;

static void* hs_worker(void* p)
{
    hs_job* J = (hs_job*)p;
    double* v = (double*)malloc(sizeof(double) * (size_t)J->C);
    int* pos = (int*)malloc(sizeof(int) * (size_t)J->C);
    for (int fb = J->f0; fb < J->f1; ++fb) {
        int f = fb / J->B, b = fb % J->B, n = 0;
        for (int i = 0; i < J->C; ++i) {
            int s = J->cand[(size_t)b * J->C + i];
            double I = 0.0;
            if (s < 0) {
                if (J->cand_scores) J->cand_scores[(size_t)fb * J->C + i] = -INFINITY;
                continue;
            }
            for (int j = 0; j < J->H; ++j) {
                double x = 0.0;
                size_t qo = (((size_t)f * J->B + b) * J->H + j) * J->dc;
                for (int e = 0; e < J->dc; ++e)
                    x += load_elem(J->qt, J->qt_dtype, qo + e) *
                         (double)orc_bf16_to_f32(J->c[((size_t)b * J->c_batch_rows + s) * J->dc + e]);
                I += (double)J->w[((size_t)f * J->B + b) * J->H + j] * (x > 0.0 ? x : 0.0);
            }
            if (J->cand_scores) J->cand_scores[(size_t)fb * J->C + i] = I;
            v[n] = I;
            pos[n] = s;
            ++n;
        }
        topk_one(v, n, pos, J->k, J->out + (size_t)fb * J->k, NULL);
    }
    free(v);
    free(pos);
    return NULL;
}

int orc_hs_refine(int qt_dtype, const void* qt, const float* w, const uint16_t* c, long long c_batch_rows,
                  const int* cand, int F, int B, int H, int dc, int C, int k, int* out, double* cand_scores,
                  int nthreads)
{
    int total = F * B;
    pthread_t* th;
    hs_job* jobs;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > total) nthreads = total > 0 ? total : 1;
    th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    jobs = (hs_job*)malloc(sizeof(hs_job) * nthreads);
    for (int t = 0; t < nthreads; ++t) {
        hs_job J = {total * t / nthreads, total * (t + 1) / nthreads, qt_dtype, qt, w, c, c_batch_rows, cand,
                    F, B, H, dc, C, k, out, cand_scores};
        jobs[t] = J;
        pthread_create(&th[t], NULL, hs_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}
