/*
 * Oracle for the APB-V / Spava per-host approximate attention (prefill).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously correct
 * CPU statement of what the GPU library computes.  It is used by the test
 * suite, by the smoke check and by the CPU-baseline leg of the benchmark; no
 * product code path may call it.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * Arithmetic: every input is a bf16 bit pattern widened exactly to double;
 * everything after that is IEEE double (fp64), two-pass exact softmax, no
 * blocking, no online rescaling, no fusion.
 *
 * Sources (the method is given in prose only):
 *   [APB-V-IT] "Riepilogo Tecnico: APB-V" (gist.science/it/paper/2601.21444),
 *       section "Metodologia: APB-V", 1. "Design del Framework":
 *         - "Suddivisione del Contesto e Disposizione ZigZag": anchor block,
 *           query block, context blocks; physical host h holds the virtual
 *           hosts h and 2H-1-h;
 *         - "Meccanismo di Attenzione Approssimata" / "Blocco Ancora": a fixed
 *           initial segment of embeddings;
 *         - "Blocchi di Passaggio": for each host, the most essential KV pairs
 *           of the preceding hosts, found by query-to-context attention
 *           scores, aggregated into passing blocks;
 *         - "Computazione": attention over anchor, local context, the
 *           aggregated passing blocks and the query.
 *       section 2. "Ottimizzazioni a Livello di Sistema", "Forward Fuso di
 *       Contesto e Query": query partial results are merged through the
 *       log-sum-exp outputs, i.e. the query block itself is attended exactly.
 *       section "Limitazioni": with one host the method is standard attention.
 *   [Spava-abs] "Spava: Accelerating Long-Video Understanding via
 *       Sequence-Parallelism-aware Approximate Attention", abstract.
 *
 * Readings where the text is silent (each is stated where it is used):
 *   R1  H counts physical hosts = virtual-host PAIRS; there are 2H chunks.
 *   R2  local_pair_full=1: the later virtual host of a pair sees its partner's
 *       chunk in full (same physical host, so nothing crosses hosts) and takes
 *       no passing block from it.  local_pair_full=0: every virtual host is its
 *       own host and takes the passing blocks of all earlier chunks.
 *   R3  chunk u selects its passing block once, from the query block's scores
 *       against chunk u; every later chunk aggregates those blocks.
 *   R4  score of key j of chunk u for KV head g = sum over the query rows i and
 *       the query heads h of group g of softmax_{j in chunk u}(scale q_{h,i}.k_{g,j});
 *       no causal mask (the query block follows all context).
 *   R5  anchor = tokens [0, a); its own rows are causal over the anchor.
 *   R6  query block = the last q tokens; its rows attend [0, t] exactly.
 *   R7  top-l per KV head per producing chunk, l_eff = min(l, n_u).
 *   R8  ties: lower token index wins; indices emitted ascending, padded -1.
 *   R9  query head h uses KV head floor(h / (Hq/Hkv)).
 *   R10 inputs are post-rotary; kept keys keep their position.
 *   R11 scale = 1/sqrt(d) unless given; lse in natural log.
 *   R14 the last chunk produces no passing block (no successor).
 *   Selection variants (ablations of R4, off by default): score_norm 1 takes
 *   each query row's weights against its whole key set [0, t] instead of the
 *   chunk alone; score_pool w ranks keys by w-key window sums of the scores.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t H;          /* virtual-host pairs; 2H chunks */
    int32_t Hq, Hkv, d; /* query heads, KV heads, head dim */
    int64_t N, a, q;    /* tokens, anchor length, query-block length */
    const int64_t *off; /* [2H+1] chunk offsets: off[0]=a, off[2H]=N-q */
    int32_t l;          /* passing-block size per KV head per chunk */
    double scale;       /* <= 0 means 1/sqrt(d) */
    int32_t local_pair_full;
    int32_t score_norm; /* 0: softmax over the chunk (R4); 1: over the row's whole key set [0, t] */
    int32_t score_pool; /* 0 or 1: none; odd w >= 3: rank by sums over w-key windows */
} oracle_cfg;

enum { ORACLE_OK = 0, ORACLE_EINVAL = -1, ORACLE_ENOMEM = -2 };

static double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double cfg_scale(const oracle_cfg *c) {
    return c->scale > 0.0 ? c->scale : 1.0 / sqrt((double)c->d);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sequence split, [APB-V-IT] "Suddivisione del Contesto": [anchor | 2H context
 * chunks | query block], chunks contiguous and non-empty. */
int oracle_validate(const oracle_cfg *c) {
    if (!c || !c->off) return ORACLE_EINVAL;
    if (c->H < 1 || c->Hq < 1 || c->Hkv < 1 || c->d < 1) return ORACLE_EINVAL;
    if (c->Hq % c->Hkv) return ORACLE_EINVAL;
    if (c->a < 0 || c->q < 1 || c->l < 0) return ORACLE_EINVAL;
    if (c->score_norm < 0 || c->score_norm > 1) return ORACLE_EINVAL;
    if (c->score_pool < 0 || (c->score_pool > 1 && c->score_pool % 2 == 0)) return ORACLE_EINVAL;
    int nc = 2 * c->H;
    if (c->off[0] != c->a || c->off[nc] != c->N - c->q) return ORACLE_EINVAL;
    for (int v = 0; v < nc; ++v)
        if (c->off[v + 1] <= c->off[v]) return ORACLE_EINVAL;
    return ORACLE_OK;
}

/* Visual load balancing ([APB-V-IT] "Bilanciamento del Carico Visivo": the
 * video frames are spread evenly over the virtual hosts, so that no host's
 * share of the vision encoder is a bottleneck).  Reading: every virtual host
 * takes whole, consecutive frames; the frames are dealt out to the 2H hosts in
 * turn, frame f counting toward host f mod 2H, so the hosts' frame counts
 * differ by at most one and the larger counts go to the lower hosts; host v's
 * frames then follow those of hosts 0..v-1.  The chunk offsets are the token
 * positions where the hosts' runs start: off[0] = a (after the anchor),
 * off[v+1] = off[v] + the tokens of host v's frames.  n_frames >= 2H and every
 * frame has at least one token. */
int oracle_plan_chunks(int32_t H, const int64_t *frame_tokens, int64_t n_frames, int64_t a,
                       int64_t *off) {
    if (H < 1 || !frame_tokens || !off || a < 0) return ORACLE_EINVAL;
    const int nc = 2 * H;
    if (n_frames < nc) return ORACLE_EINVAL;
    int64_t *count = (int64_t *)calloc((size_t)nc, sizeof(int64_t));
    if (!count) return ORACLE_ENOMEM;
    for (int64_t f = 0; f < n_frames; ++f) count[f % nc] += 1; /* deal the frames */
    int64_t f = 0;
    off[0] = a;
    for (int v = 0; v < nc; ++v) {
        int64_t tok = 0;
        for (int64_t i = 0; i < count[v]; ++i, ++f) {
            if (frame_tokens[f] < 1) { free(count); return ORACLE_EINVAL; }
            tok += frame_tokens[f];
        }
        off[v + 1] = off[v] + tok;
    }
    free(count);
    return ORACLE_OK;
}

/* Physical host of virtual host v under the ZigZag layout: host h holds the
 * virtual hosts h and 2H-1-h ([APB-V-IT] "Disposizione ZigZag"). */
int oracle_pair(int H, int v) { return v < H ? v : 2 * H - 1 - v; }

static double dot_bf16(const uint16_t *x, const uint16_t *y, int d) {
    double s = 0.0;
    for (int c = 0; c < d; ++c) s += bf16_to_double(x[c]) * bf16_to_double(y[c]);
    return s;
}

/* Query-to-context scores of chunk u for KV head g ([APB-V-IT] "Blocchi di
 * Passaggio"; reading R4):
 *   S[j] = sum_{h in g} sum_{i in query block} exp(x_{h,i,j} - m_{h,i}) / l_{h,i},
 *   x_{h,i,j} = scale * q_{h,i} . k_{g,j},  m, l the max and the sum of exp
 *   over j in chunk u only (score_norm 0), or over every key the row attends,
 *   [0, t] with t = N - q + i (score_norm 1: the row's own attention weights,
 *   the variant normalised by the query pass's log-sum-exp).
 * S has n_u = off[u+1]-off[u] entries, S[j - off[u]].
 * Step 1 computes (m, l) per query row; step 2 sums the probabilities per key
 * in a fixed (h, i) order, so the result does not depend on the thread count. */
int oracle_chunk_scores(const oracle_cfg *c, const uint16_t *Q, const uint16_t *K,
                        int u, int g, double *S) {
    if (oracle_validate(c) != ORACLE_OK) return ORACLE_EINVAL;
    if (u < 0 || u >= 2 * c->H || g < 0 || g >= c->Hkv) return ORACLE_EINVAL;
    const int G = c->Hq / c->Hkv, d = c->d;
    const int64_t j0 = c->off[u], n = c->off[u + 1] - c->off[u];
    const int64_t nrow = (int64_t)G * c->q;
    const double sc = cfg_scale(c);
    double *m = (double *)malloc(sizeof(double) * nrow);
    double *ls = (double *)malloc(sizeof(double) * nrow);
    if (!m || !ls) { free(m); free(ls); return ORACLE_ENOMEM; }

    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrow; ++r) {
        const int h = g * G + (int)(r / c->q);
        const int64_t t = c->N - c->q + r % c->q;
        const uint16_t *qv = Q + ((size_t)t * c->Hq + h) * d;
        /* normaliser's key range: the chunk, or everything the row attends */
        const int64_t k0 = c->score_norm ? 0 : j0, k1 = c->score_norm ? t + 1 : j0 + n;
        double mx = -INFINITY;
        for (int64_t j = k0; j < k1; ++j) {
            double x = sc * dot_bf16(qv, K + ((size_t)j * c->Hkv + g) * d, d);
            if (x > mx) mx = x;
        }
        double sum = 0.0;
        for (int64_t j = k0; j < k1; ++j) {
            double x = sc * dot_bf16(qv, K + ((size_t)j * c->Hkv + g) * d, d);
            sum += exp(x - mx);
        }
        m[r] = mx;
        ls[r] = sum;
    }

    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t j = 0; j < n; ++j) {
        const uint16_t *kv = K + ((size_t)(j0 + j) * c->Hkv + g) * d;
        double s = 0.0;
        for (int64_t r = 0; r < nrow; ++r) {
            const int h = g * G + (int)(r / c->q);
            const int64_t t = c->N - c->q + r % c->q;
            double x = sc * dot_bf16(Q + ((size_t)t * c->Hq + h) * d, kv, d);
            s += exp(x - m[r]) / ls[r];
        }
        S[j] = s;
    }
    free(m);
    free(ls);
    return ORACLE_OK;
}

/* Pooled-score variant of the selection (the pages name SnapKV's scoring only
 * by title; the reading here: a window mean of w keys centred on each key,
 * zero outside the chunk).  The mean divides every window by the same w, so
 * ranking by it is ranking by the window SUM, which is what these return:
 * out[j] = sum of S[j'] for j' in [j - w/2, j + w/2] clipped to [0, n), added
 * in ascending j'.  w <= 1 copies S. */
int oracle_pool_sums(const double *S, int64_t n, int32_t w, double *out) {
    if (n < 0 || w < 0) return ORACLE_EINVAL;
    const int64_t h = w > 1 ? w / 2 : 0;
    for (int64_t j = 0; j < n; ++j) {
        double s = 0.0;
        for (int64_t k = (j - h < 0 ? 0 : j - h); k <= j + h && k < n; ++k) s += S[k];
        out[j] = s;
    }
    return ORACLE_OK;
}

/* The same sums in float arithmetic, in the same order: the selection decision
 * taken in the precision of the GPU's fp32 scores. */
int oracle_pool_sums_f32(const float *S, int64_t n, int32_t w, float *out) {
    if (n < 0 || w < 0) return ORACLE_EINVAL;
    const int64_t h = w > 1 ? w / 2 : 0;
    for (int64_t j = 0; j < n; ++j) {
        float s = 0.0f;
        for (int64_t k = (j - h < 0 ? 0 : j - h); k <= j + h && k < n; ++k) s += S[k];
        out[j] = s;
    }
    return ORACLE_OK;
}

typedef struct { double s; int64_t j; } scored;

/* Rank order of the selection: larger score first, then lower index (R8). */
static int by_score_then_index(const void *pa, const void *pb) {
    const scored *a = (const scored *)pa, *b = (const scored *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j < b->j) ? -1 : (a->j > b->j);
}

static int by_index(const void *pa, const void *pb) {
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* Passing-block selection ([APB-V-IT] "Blocchi di Passaggio": the most
 * essential KV pairs; reading R7/R8): sort the n scores by (score desc, index
 * asc), keep the first min(l, n), emit their absolute positions base+j in
 * ascending order, pad the rest of the l slots with -1. */
int oracle_select_top_l(const double *S, int64_t n, int64_t base, int32_t l, int32_t *idx) {
    if (n < 0 || l < 0) return ORACLE_EINVAL;
    scored *v = (scored *)malloc(sizeof(scored) * (n > 0 ? n : 1));
    if (!v) return ORACLE_ENOMEM;
    for (int64_t j = 0; j < n; ++j) { v[j].s = S[j]; v[j].j = j; }
    qsort(v, (size_t)n, sizeof(scored), by_score_then_index);
    int64_t keep = n < l ? n : l;
    for (int64_t r = 0; r < keep; ++r) idx[r] = (int32_t)(base + v[r].j);
    qsort(idx, (size_t)keep, sizeof(int32_t), by_index);
    for (int64_t r = keep; r < l; ++r) idx[r] = -1;
    free(v);
    return ORACLE_OK;
}

/* Key set of row t for KV head g ([APB-V-IT] "Computazione", R2, R5, R6):
 *   anchor row  (t < a):       [0, t]
 *   query row   (t >= N-q):    [0, t]
 *   context row (t in chunk v): anchor [0, a)
 *        + passing blocks P_u[g] of the earlier chunks u < v
 *          (local_pair_full=1: only those on another physical host)
 *        + the partner chunk 2H-1-v in full when v >= H and local_pair_full=1
 *        + the own chunk causally, [off[v], t].
 * idx is [2H-1][Hkv][l] absolute positions padded with -1.  Keys are written
 * ascending; returns their count, or a negative error. keys needs room for
 * t+1 entries. */
int64_t oracle_key_set(const oracle_cfg *c, const int32_t *idx, int64_t t, int g, int64_t *keys) {
    if (oracle_validate(c) != ORACLE_OK || t < 0 || t >= c->N) return ORACLE_EINVAL;
    const int H = c->H, nc = 2 * H;
    int64_t n = 0;
    if (t < c->a || t >= c->N - c->q) {
        for (int64_t j = 0; j <= t; ++j) keys[n++] = j;
        return n;
    }
    int v = 0;
    while (!(t >= c->off[v] && t < c->off[v + 1])) ++v;
    char *take = (char *)calloc((size_t)(t + 1), 1);
    if (!take) return ORACLE_ENOMEM;
    for (int64_t j = 0; j < c->a; ++j) take[j] = 1;
    for (int u = 0; u < v; ++u) {
        if (c->local_pair_full && oracle_pair(H, u) == oracle_pair(H, v)) continue;
        const int32_t *p = idx + ((size_t)u * c->Hkv + g) * c->l;
        for (int r = 0; r < c->l; ++r)
            if (p[r] >= 0) take[p[r]] = 1;
    }
    if (c->local_pair_full && v >= H) {
        const int p = nc - 1 - v;
        for (int64_t j = c->off[p]; j < c->off[p + 1]; ++j) take[j] = 1;
    }
    for (int64_t j = c->off[v]; j <= t; ++j) take[j] = 1;
    for (int64_t j = 0; j <= t; ++j)
        if (take[j]) keys[n++] = j;
    free(take);
    return n;
}

/* Number of (row, key) pairs per query head that the key sets above attend,
 * by row class (out[0] anchor rows, out[1] context rows, out[2] query rows),
 * counted from the same definition without listing the keys: an anchor or
 * query row t attends t+1 keys; a row at position r (0-based) of chunk v
 * attends a + the passing-block sizes min(l, n_u) of the earlier chunks it
 * takes + the partner chunk's n_p (v >= H, local_pair_full) + r + 1. */
int oracle_attended_pairs(const oracle_cfg *c, int64_t *out) {
    if (oracle_validate(c) != ORACLE_OK || !out) return ORACLE_EINVAL;
    const int H = c->H, nc = 2 * H;
    out[0] = c->a * (c->a + 1) / 2;
    out[1] = 0;
    for (int v = 0; v < nc; ++v) {
        const int64_t n_v = c->off[v + 1] - c->off[v];
        int64_t fixed = c->a;
        for (int u = 0; u < v; ++u) {
            if (c->local_pair_full && oracle_pair(H, u) == oracle_pair(H, v)) continue;
            const int64_t n_u = c->off[u + 1] - c->off[u];
            fixed += n_u < c->l ? n_u : c->l;
        }
        if (c->local_pair_full && v >= H) fixed += c->off[nc - v] - c->off[nc - 1 - v];
        out[1] += n_v * fixed + n_v * (n_v + 1) / 2;
    }
    const int64_t q0 = c->N - c->q; /* rows q0 .. N-1 attend t+1 keys each */
    out[2] = (c->N * (c->N + 1) - q0 * (q0 + 1)) / 2;
    return ORACLE_OK;
}

/* Exact softmax attention of row t, head h over the given keys ([APB-V-IT]
 * "Computazione"): two passes in double.  o[d] = sum_j p_j v_j, lse = ln sum_j
 * exp(x_j). xbuf needs nk entries. */
static void attend_row(const oracle_cfg *c, const uint16_t *Q, const uint16_t *K,
                       const uint16_t *V, int64_t t, int h, const int64_t *keys, int64_t nk,
                       double *xbuf, double *o, double *lse) {
    const int G = c->Hq / c->Hkv, g = h / G, d = c->d;
    const double sc = cfg_scale(c);
    const uint16_t *qv = Q + ((size_t)t * c->Hq + h) * d;
    double mx = -INFINITY;
    for (int64_t r = 0; r < nk; ++r) {
        xbuf[r] = sc * dot_bf16(qv, K + ((size_t)keys[r] * c->Hkv + g) * d, d);
        if (xbuf[r] > mx) mx = xbuf[r];
    }
    double sum = 0.0;
    for (int c2 = 0; c2 < d; ++c2) o[c2] = 0.0;
    for (int64_t r = 0; r < nk; ++r) {
        double p = exp(xbuf[r] - mx);
        sum += p;
        const uint16_t *vv = V + ((size_t)keys[r] * c->Hkv + g) * d;
        for (int c2 = 0; c2 < d; ++c2) o[c2] += p * bf16_to_double(vv[c2]);
    }
    for (int c2 = 0; c2 < d; ++c2) o[c2] /= sum;
    *lse = mx + log(sum);
}

/* Outputs of the approximate attention for the given rows and query heads.
 * O is [nrows][nheads][d], lse is [nrows][nheads]. */
int oracle_prefill_rows(const oracle_cfg *c, const uint16_t *Q, const uint16_t *K,
                        const uint16_t *V, const int32_t *idx, const int64_t *rows,
                        int64_t nrows, const int32_t *heads, int32_t nheads, double *O,
                        double *lse) {
    if (oracle_validate(c) != ORACLE_OK) return ORACLE_EINVAL;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= c->N) return ORACLE_EINVAL;
    for (int32_t k = 0; k < nheads; ++k)
        if (heads[k] < 0 || heads[k] >= c->Hq) return ORACLE_EINVAL;
    const int G = c->Hq / c->Hkv;
    int err = ORACLE_OK;
    #pragma omp parallel
    {
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)c->N);
        double *xbuf = (double *)malloc(sizeof(double) * (size_t)c->N);
        if (!keys || !xbuf) {
            #pragma omp atomic write
            err = ORACLE_ENOMEM;
        } else {
            #pragma omp for schedule(dynamic, 1)
            for (int64_t w = 0; w < nrows * nheads; ++w) {
                const int64_t r = w / nheads;
                const int k = (int)(w % nheads);
                const int h = heads[k];
                int64_t nk = oracle_key_set(c, idx, rows[r], h / G, keys);
                if (nk < 0) {
                    #pragma omp atomic write
                    err = (int)nk;
                    continue;
                }
                attend_row(c, Q, K, V, rows[r], h, keys, nk, xbuf,
                           O + ((size_t)r * nheads + k) * c->d, lse + (size_t)r * nheads + k);
            }
        }
        free(keys);
        free(xbuf);
    }
    return err;
}
