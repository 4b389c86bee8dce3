/*
 * Oracle for the single-device Megatron-style tensor-parallel transformer layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or helper with the CUDA
 * library; it is written from the definitions below, in plain fp64 loops, with
 * no blocking, fusion or reordering beyond what each definition states.
 * Parallelism (OpenMP) is over independent output elements only, so it never
 * changes the order of any sum.
 *
 * Sources (page title, section):
 *  [TSC]  "Tensor parallel scaling curves", section "What tensor parallelism
 *         actually splits": Q/K/V projections split by columns so that each
 *         shard owns whole attention heads -- shard s owns the contiguous
 *         block of query heads [s*n_q/t, (s+1)*n_q/t); each shard computes
 *         attention for its own heads with no exchange; the output
 *         projection is split by rows and yields a partial sum; gate and up
 *         are split by columns, down by rows; the row-split partials are
 *         summed (all-reduce), two such sums per layer, 2L per forward pass.
 *  [TPF]  "Tensor Parallelism Fundamentals", section "Mechanics of Matrix
 *         Slicing": column-parallel then row-parallel, the partial output is
 *         fed straight into the row-parallel layer, then summed.  Section
 *         "Memory Overhead and Communication Bottlenecks": weight footprint
 *         divided by t, and the per-GPU KV formula
 *         2*num_layers*num_kv_heads*head_dim*seq_length*bytes*batch / t.
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes of the repository):
 *  - pre-RMSNorm a = x*gamma/sqrt(mean(x^2)+eps) before QKV and before
 *    gate/up, and residual adds after O and after down, both switchable by
 *    flags (ORC_NORM, ORC_RESIDUAL); the pages name neither;
 *  - SwiGLU act = silu(g)*u with silu(z) = z/(1+exp(-z));
 *  - softmax scale 1/sqrt(head_dim), no mask in decode, causal mask inside a
 *    prefill chunk;
 *  - GQA: query head h reads kv head floor(h/g), g = n_q_heads/n_kv_heads;
 *  - decode: the cache holds S tokens, the new token's k/v is position S,
 *    attention spans S+1 keys; the new k/v enter the softmax unrounded;
 *  - weights use the nn.Linear orientation W[out][in]; "column split" in the
 *    pages' x@W notation therefore splits `out`, "row split" splits `in`;
 *  - rotary position embedding (ORC_ROPE, off unless flagged): not on the
 *    pages; the textbook rotation of RoFormer (Su et al., "RoFormer:
 *    Enhanced Transformer with Rotary Position Embedding", 2021) in the
 *    pairing the Llama family uses, element e with element e + d/2;
 *  - a prefill chunk may start at position P0 of a cache already holding P0
 *    tokens ("chunked prefill"): its token i sits at position P0 + i and
 *    attends the P0 cached keys (bf16) and the chunk's keys 0..i (unrounded).
 *
 * Data formats: weights are either raw bf16 bit patterns (uint16) or fp32,
 * widened exactly to double.  The KV cache is raw bf16 in the unsharded
 * layout [B][n_kv][S_cap][head_dim].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_NORM 1u
#define ORC_RESIDUAL 2u
#define ORC_ROPE 8u

typedef struct {
    int32_t hidden, n_q_heads, n_kv_heads, head_dim, ffn;
    double eps;
    uint32_t flags;
    double rope_base; /* the base of the rotary frequencies (ORC_ROPE) */
} orc_dims;

/* Unsharded layer weights in nn.Linear orientation.  wtype: 0 = bf16 bits,
 * 1 = fp32.  gamma_* are fp32 [hidden] (NULL means all ones). */
typedef struct {
    const void *wq;   /* [n_q_heads*head_dim][hidden] */
    const void *wk;   /* [n_kv_heads*head_dim][hidden] */
    const void *wv;   /* [n_kv_heads*head_dim][hidden] */
    const void *wo;   /* [hidden][n_q_heads*head_dim] */
    const void *wg;   /* [ffn][hidden] */
    const void *wu;   /* [ffn][hidden] */
    const void *wd;   /* [hidden][ffn] */
    const float *gamma_attn;
    const float *gamma_mlp;
    int32_t wtype;
} orc_weights;

static int g_threads = 1;

void orc_set_threads(int n) {
    g_threads = n < 1 ? 1 : n;
#ifdef _OPENMP
    omp_set_num_threads(g_threads);
#endif
}

int orc_get_threads(void) { return g_threads; }

double orc_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double wval(const void *w, int32_t wtype, size_t i) {
    if (wtype == 0) return orc_bf16_to_double(((const uint16_t *)w)[i]);
    return (double)((const float *)w)[i];
}

/* y[r] = sum_{c} W[row0 + r][col0 + c] * x[c], for r < rows, c < cols.
 * W has row stride ld.  Sum in ascending c. */
static void linear_block(const void *w, int32_t wtype, size_t ld, long row0, long rows, long col0,
                         long cols, const double *x, double *y) {
    long r;
#pragma omp parallel for schedule(static) if (rows >= 64)
    for (r = 0; r < rows; ++r) {
        size_t base = (size_t)(row0 + r) * ld + (size_t)col0;
        double acc = 0.0;
        for (long c = 0; c < cols; ++c) acc += wval(w, wtype, base + (size_t)c) * x[c];
        y[r] = acc;
    }
}

/* RMSNorm: out = x * gamma / sqrt(mean(x^2) + eps). */
void orc_rmsnorm(const double *x, const float *gamma, long n, double eps, double *out) {
    double ss = 0.0;
    for (long i = 0; i < n; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss / (double)n + eps);
    for (long i = 0; i < n; ++i) out[i] = x[i] * inv * (gamma ? (double)gamma[i] : 1.0);
}

double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* Rotary position embedding of one head vector v[d] at position pos: for
 * e < d/2 the pair (v[e], v[e + d/2]) is turned by the angle
 * pos * base^(-2e/d) (RoFormer's frequencies theta_e = base^(-2e/d)). */
void orc_rope(double *v, long d, long pos, double base) {
    const long half = d / 2;
    for (long e = 0; e < half; ++e) {
        const double ang = (double)pos * pow(base, -2.0 * (double)e / (double)d);
        const double c = cos(ang), s = sin(ang);
        const double a = v[e], b = v[e + half];
        v[e] = a * c - b * s;
        v[e + half] = b * c + a * s;
    }
}

/* Softmax-weighted sum for one query head over nkeys keys.
 * keys(j) / vals(j) are fetched through the callbacks' arrays: the first
 * n_cached keys come from a bf16 cache row block, the optional extra key is
 * given in fp64.  scale multiplies the logits. */
static void attend_one(const double *q, long d, const uint16_t *kc, const uint16_t *vc, long n_cached,
                       const double *k_extra, const double *v_extra, double scale, double *out) {
    long nk = n_cached + (k_extra ? 1 : 0);
    double *logit = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    double mx = -INFINITY;
    for (long j = 0; j < nk; ++j) {
        double s = 0.0;
        if (j < n_cached) {
            for (long e = 0; e < d; ++e) s += q[e] * orc_bf16_to_double(kc[(size_t)j * d + e]);
        } else {
            for (long e = 0; e < d; ++e) s += q[e] * k_extra[e];
        }
        logit[j] = s * scale;
        if (logit[j] > mx) mx = logit[j];
    }
    double den = 0.0;
    for (long j = 0; j < nk; ++j) {
        logit[j] = exp(logit[j] - mx);
        den += logit[j];
    }
    for (long e = 0; e < d; ++e) out[e] = 0.0;
    for (long j = 0; j < nk; ++j) {
        double p = logit[j] / den;
        if (j < n_cached) {
            for (long e = 0; e < d; ++e) out[e] += p * orc_bf16_to_double(vc[(size_t)j * d + e]);
        } else {
            for (long e = 0; e < d; ++e) out[e] += p * v_extra[e];
        }
    }
    free(logit);
}

/* Intermediates of one decode layer (any pointer may be NULL).  Shapes are
 * per batch row b, concatenated over b:
 *   q [B][nq*d], k_new/v_new [B][nkv*d], attn [B][nq*d], h [B][H],
 *   act [B][F]. */
typedef struct {
    double *q, *k_new, *v_new, *attn, *h, *act;
} orc_trace;

/* One unsharded decode layer for B independent sequences.
 * x [B][H] fp64; kc/vc raw bf16 [B][n_kv][S_cap][d] holding S cached tokens;
 * y [B][H] fp64.  Definition (per sequence):
 *   a   = RMSNorm(x; gamma_attn)                      (if ORC_NORM, else x)
 *   q,k,v = Wq a, Wk a, Wv a                          [TSC]
 *   q_h, k_j rotated to position S                    (if ORC_ROPE)
 *   o_h = sum_{j<=S} softmax_j(q_h . K_j / sqrt(d)) V_j, kv head floor(h/g),
 *         K_S = k, V_S = v (the new token)            [TSC] local attention
 *   h   = x + Wo o                                    (residual if flagged)
 *   m   = RMSNorm(h; gamma_mlp)                       (if ORC_NORM, else h)
 *   y   = h + Wd (silu(Wg m) * (Wu m))                (residual if flagged)
 */
int orc_decode_layer(const orc_dims *dm, const orc_weights *w, long B, const double *x,
                     const uint16_t *kc, const uint16_t *vc, long S_cap, long S, double *y,
                     const orc_trace *tr) {
    const long H = dm->hidden, nq = dm->n_q_heads, nkv = dm->n_kv_heads, d = dm->head_dim,
               F = dm->ffn;
    if (H <= 0 || nq <= 0 || nkv <= 0 || d <= 0 || F <= 0 || nq % nkv != 0) return 1;
    if (S < 0 || S > S_cap) return 1;
    const long g = nq / nkv;
    const double scale = 1.0 / sqrt((double)d);
    double *a = malloc(sizeof(double) * (size_t)H);
    double *q = malloc(sizeof(double) * (size_t)(nq * d));
    double *k = malloc(sizeof(double) * (size_t)(nkv * d));
    double *v = malloc(sizeof(double) * (size_t)(nkv * d));
    double *o = malloc(sizeof(double) * (size_t)(nq * d));
    double *hh = malloc(sizeof(double) * (size_t)H);
    double *m = malloc(sizeof(double) * (size_t)H);
    double *gg = malloc(sizeof(double) * (size_t)F);
    double *uu = malloc(sizeof(double) * (size_t)F);
    double *act = malloc(sizeof(double) * (size_t)F);
    double *dn = malloc(sizeof(double) * (size_t)H);
    for (long b = 0; b < B; ++b) {
        const double *xb = x + (size_t)b * H;
        if (dm->flags & ORC_NORM) orc_rmsnorm(xb, w->gamma_attn, H, dm->eps, a);
        else memcpy(a, xb, sizeof(double) * (size_t)H);
        linear_block(w->wq, w->wtype, (size_t)H, 0, nq * d, 0, H, a, q);
        linear_block(w->wk, w->wtype, (size_t)H, 0, nkv * d, 0, H, a, k);
        linear_block(w->wv, w->wtype, (size_t)H, 0, nkv * d, 0, H, a, v);
        if (dm->flags & ORC_ROPE) {
            for (long hq = 0; hq < nq; ++hq) orc_rope(q + hq * d, d, S, dm->rope_base);
            for (long j = 0; j < nkv; ++j) orc_rope(k + j * d, d, S, dm->rope_base);
        }
        long h;
#pragma omp parallel for schedule(static)
        for (h = 0; h < nq; ++h) {
            long j = h / g;
            size_t cache_off = (((size_t)b * nkv + j) * (size_t)S_cap) * d;
            attend_one(q + h * d, d, kc + cache_off, vc + cache_off, S, k + j * d, v + j * d, scale,
                       o + h * d);
        }
        linear_block(w->wo, w->wtype, (size_t)(nq * d), 0, H, 0, nq * d, o, hh);
        if (dm->flags & ORC_RESIDUAL)
            for (long i = 0; i < H; ++i) hh[i] = xb[i] + hh[i];
        if (dm->flags & ORC_NORM) orc_rmsnorm(hh, w->gamma_mlp, H, dm->eps, m);
        else memcpy(m, hh, sizeof(double) * (size_t)H);
        linear_block(w->wg, w->wtype, (size_t)H, 0, F, 0, H, m, gg);
        linear_block(w->wu, w->wtype, (size_t)H, 0, F, 0, H, m, uu);
        for (long i = 0; i < F; ++i) act[i] = orc_silu(gg[i]) * uu[i];
        linear_block(w->wd, w->wtype, (size_t)F, 0, H, 0, F, act, dn);
        double *yb = y + (size_t)b * H;
        for (long i = 0; i < H; ++i) yb[i] = (dm->flags & ORC_RESIDUAL) ? hh[i] + dn[i] : dn[i];
        if (tr) {
            if (tr->q) memcpy(tr->q + (size_t)b * nq * d, q, sizeof(double) * (size_t)(nq * d));
            if (tr->k_new) memcpy(tr->k_new + (size_t)b * nkv * d, k, sizeof(double) * (size_t)(nkv * d));
            if (tr->v_new) memcpy(tr->v_new + (size_t)b * nkv * d, v, sizeof(double) * (size_t)(nkv * d));
            if (tr->attn) memcpy(tr->attn + (size_t)b * nq * d, o, sizeof(double) * (size_t)(nq * d));
            if (tr->h) memcpy(tr->h + (size_t)b * H, hh, sizeof(double) * (size_t)H);
            if (tr->act) memcpy(tr->act + (size_t)b * F, act, sizeof(double) * (size_t)F);
        }
    }
    free(a); free(q); free(k); free(v); free(o); free(hh); free(m);
    free(gg); free(uu); free(act); free(dn);
    return 0;
}

/* One unsharded prefill layer over a chunk of T tokens of one sequence
 * whose cache already holds P0 tokens: token i sits at position P0 + i and
 * attends the P0 cached keys and the chunk's keys 0..i (causal).  The
 * layer's outputs are produced for the `nrows` token rows listed in `rows`
 * (each in [0, T)); the keys and values of every chunk token up to the
 * largest listed row are computed, since those rows attend to them.
 *   x [T][H]; kc/vc raw bf16 [n_kv][S_cap][d] with P0 cached tokens (may be
 *   NULL when P0 = 0); y [nrows][H] (row r of y is token rows[r]);
 *   k_out/v_out [R][n_kv*d], R = max(rows) + 1: the new keys (rotated when
 *   ORC_ROPE) and values, which are what cache slots P0..P0+R-1 hold
 *   afterwards (before rounding);
 *   trace (optional): q/attn [nrows][nq*d], h [nrows][H], act [nrows][F].
 * Per token the steps are those of orc_decode_layer with the cache's keys
 * followed by the chunk's own keys 0..i ("Tensor parallel scaling curves",
 * "Prefill vs decode: different curves"). */
int orc_prefill_chunk(const orc_dims *dm, const orc_weights *w, long T, const double *x, long P0,
                      const uint16_t *kc, const uint16_t *vc, long S_cap, long nrows, const long *rows,
                      double *y, double *k_out, double *v_out, const orc_trace *tr) {
    const long H = dm->hidden, nq = dm->n_q_heads, nkv = dm->n_kv_heads, d = dm->head_dim,
               F = dm->ffn;
    if (H <= 0 || nq <= 0 || nkv <= 0 || d <= 0 || F <= 0 || nq % nkv != 0 || T < 0 || nrows < 0)
        return 1;
    if (P0 < 0 || (P0 > 0 && (!kc || !vc || S_cap < P0))) return 1;
    long R = 0;
    for (long r = 0; r < nrows; ++r) {
        if (rows[r] < 0 || rows[r] >= T) return 1;
        if (rows[r] + 1 > R) R = rows[r] + 1;
    }
    const long g = nq / nkv;
    const double scale = 1.0 / sqrt((double)d);
    double *a = malloc(sizeof(double) * (size_t)H);
    double *q = malloc(sizeof(double) * (size_t)(nq * d));
    double *K = malloc(sizeof(double) * (size_t)(R * nkv * d + 1));
    double *V = malloc(sizeof(double) * (size_t)(R * nkv * d + 1));
    double *o = malloc(sizeof(double) * (size_t)(nq * d));
    double *hh = malloc(sizeof(double) * (size_t)H);
    double *m = malloc(sizeof(double) * (size_t)H);
    double *gg = malloc(sizeof(double) * (size_t)F);
    double *uu = malloc(sizeof(double) * (size_t)F);
    double *act = malloc(sizeof(double) * (size_t)F);
    double *dn = malloc(sizeof(double) * (size_t)H);
    /* keys and values of tokens 0..R-1 */
    for (long p = 0; p < R; ++p) {
        const double *xp = x + (size_t)p * H;
        if (dm->flags & ORC_NORM) orc_rmsnorm(xp, w->gamma_attn, H, dm->eps, a);
        else memcpy(a, xp, sizeof(double) * (size_t)H);
        linear_block(w->wk, w->wtype, (size_t)H, 0, nkv * d, 0, H, a, K + (size_t)p * nkv * d);
        linear_block(w->wv, w->wtype, (size_t)H, 0, nkv * d, 0, H, a, V + (size_t)p * nkv * d);
        if (dm->flags & ORC_ROPE)
            for (long j = 0; j < nkv; ++j) orc_rope(K + (size_t)p * nkv * d + (size_t)j * d, d, P0 + p, dm->rope_base);
    }
    for (long r = 0; r < nrows; ++r) {
        const long i = rows[r];
        const double *xi = x + (size_t)i * H;
        if (dm->flags & ORC_NORM) orc_rmsnorm(xi, w->gamma_attn, H, dm->eps, a);
        else memcpy(a, xi, sizeof(double) * (size_t)H);
        linear_block(w->wq, w->wtype, (size_t)H, 0, nq * d, 0, H, a, q);
        if (dm->flags & ORC_ROPE)
            for (long hq = 0; hq < nq; ++hq) orc_rope(q + (size_t)hq * d, d, P0 + i, dm->rope_base);
        long h;
#pragma omp parallel for schedule(static)
        for (h = 0; h < nq; ++h) {
            const long j = h / g;
            const double *qh = q + (size_t)h * d;
            double *out = o + (size_t)h * d;
            /* keys 0..P0-1 from the cache, then the chunk's keys 0..i */
            const long nk = P0 + i + 1;
            double *logit = malloc(sizeof(double) * (size_t)nk);
            double mx = -INFINITY;
            for (long p = 0; p < nk; ++p) {
                double s = 0.0;
                if (p < P0) {
                    const uint16_t *kp = kc + ((size_t)j * S_cap + (size_t)p) * d;
                    for (long e = 0; e < d; ++e) s += qh[e] * orc_bf16_to_double(kp[e]);
                } else {
                    const double *kp = K + (size_t)(p - P0) * nkv * d + (size_t)j * d;
                    for (long e = 0; e < d; ++e) s += qh[e] * kp[e];
                }
                logit[p] = s * scale;
                if (logit[p] > mx) mx = logit[p];
            }
            double den = 0.0;
            for (long p = 0; p < nk; ++p) {
                logit[p] = exp(logit[p] - mx);
                den += logit[p];
            }
            for (long e = 0; e < d; ++e) out[e] = 0.0;
            for (long p = 0; p < nk; ++p) {
                const double pr = logit[p] / den;
                if (p < P0) {
                    const uint16_t *vp = vc + ((size_t)j * S_cap + (size_t)p) * d;
                    for (long e = 0; e < d; ++e) out[e] += pr * orc_bf16_to_double(vp[e]);
                } else {
                    const double *vp = V + (size_t)(p - P0) * nkv * d + (size_t)j * d;
                    for (long e = 0; e < d; ++e) out[e] += pr * vp[e];
                }
            }
            free(logit);
        }
        linear_block(w->wo, w->wtype, (size_t)(nq * d), 0, H, 0, nq * d, o, hh);
        if (dm->flags & ORC_RESIDUAL)
            for (long c = 0; c < H; ++c) hh[c] = xi[c] + hh[c];
        if (dm->flags & ORC_NORM) orc_rmsnorm(hh, w->gamma_mlp, H, dm->eps, m);
        else memcpy(m, hh, sizeof(double) * (size_t)H);
        linear_block(w->wg, w->wtype, (size_t)H, 0, F, 0, H, m, gg);
        linear_block(w->wu, w->wtype, (size_t)H, 0, F, 0, H, m, uu);
        for (long c = 0; c < F; ++c) act[c] = orc_silu(gg[c]) * uu[c];
        linear_block(w->wd, w->wtype, (size_t)F, 0, H, 0, F, act, dn);
        double *yr = y + (size_t)r * H;
        for (long c = 0; c < H; ++c) yr[c] = (dm->flags & ORC_RESIDUAL) ? hh[c] + dn[c] : dn[c];
        if (tr) {
            if (tr->q) memcpy(tr->q + (size_t)r * nq * d, q, sizeof(double) * (size_t)(nq * d));
            if (tr->attn) memcpy(tr->attn + (size_t)r * nq * d, o, sizeof(double) * (size_t)(nq * d));
            if (tr->h) memcpy(tr->h + (size_t)r * H, hh, sizeof(double) * (size_t)H);
            if (tr->act) memcpy(tr->act + (size_t)r * F, act, sizeof(double) * (size_t)F);
        }
    }
    if (k_out) memcpy(k_out, K, sizeof(double) * (size_t)(R * nkv * d));
    if (v_out) memcpy(v_out, V, sizeof(double) * (size_t)(R * nkv * d));
    free(a); free(q); free(K); free(V); free(o); free(hh); free(m);
    free(gg); free(uu); free(act); free(dn);
    return 0;
}

/* A chunk at position 0 of an empty cache, outputs at the listed rows. */
int orc_prefill_rows(const orc_dims *dm, const orc_weights *w, long T, const double *x, long nrows,
                     const long *rows, double *y, double *k_out, double *v_out, const orc_trace *tr) {
    return orc_prefill_chunk(dm, w, T, x, 0, NULL, NULL, 0, nrows, rows, y, k_out, v_out, tr);
}

/* The whole chunk: every row 0..T-1.  x [T][H]; y [T][H]; k_out/v_out
 * [T][n_kv*d]. */
int orc_prefill_layer(const orc_dims *dm, const orc_weights *w, long T, const double *x, double *y,
                      double *k_out, double *v_out, const orc_trace *tr) {
    if (T < 0) return 1;
    long *rows = malloc(sizeof(long) * (size_t)(T > 0 ? T : 1));
    for (long i = 0; i < T; ++i) rows[i] = i;
    int rc = orc_prefill_rows(dm, w, T, x, T, rows, y, k_out, v_out, tr);
    free(rows);
    return rc;
}

/* ---------------------------------------------------------------------------
 * Sharded forms.  These follow the pages' own decomposition literally and are
 * used only to check, on exact (integer-valued) data, that the sum of the
 * row-split partials equals the unsharded product [TSC], [TPF].
 * ------------------------------------------------------------------------- */

/* MLP pair: column-split gate/up (shard s owns ffn columns
 * [s*F/t, (s+1)*F/t)), row-split down; partial_s = Wd[:, cols_s] act_s;
 * y = partial_0 + partial_1 + ... (ascending s).  x [B][H] is fed to gate/up
 * directly (no norm, no residual).  y_partials (optional) [t][B][H]. */
int orc_mlp_sharded(const orc_dims *dm, const orc_weights *w, int32_t t, long B, const double *x,
                    double *y, double *y_partials) {
    const long H = dm->hidden, F = dm->ffn;
    if (t <= 0 || F % t != 0) return 2;
    const long Fs = F / t;
    double *gg = malloc(sizeof(double) * (size_t)Fs);
    double *uu = malloc(sizeof(double) * (size_t)Fs);
    double *act = malloc(sizeof(double) * (size_t)Fs);
    double *part = malloc(sizeof(double) * (size_t)H);
    for (long b = 0; b < B; ++b) {
        const double *xb = x + (size_t)b * H;
        double *yb = y + (size_t)b * H;
        for (long i = 0; i < H; ++i) yb[i] = 0.0;
        for (int32_t s = 0; s < t; ++s) {
            linear_block(w->wg, w->wtype, (size_t)H, (long)s * Fs, Fs, 0, H, xb, gg);
            linear_block(w->wu, w->wtype, (size_t)H, (long)s * Fs, Fs, 0, H, xb, uu);
            for (long c = 0; c < Fs; ++c) act[c] = orc_silu(gg[c]) * uu[c];
            linear_block(w->wd, w->wtype, (size_t)F, 0, H, (long)s * Fs, Fs, act, part);
            for (long i = 0; i < H; ++i) yb[i] += part[i];
            if (y_partials)
                memcpy(y_partials + ((size_t)s * B + b) * H, part, sizeof(double) * (size_t)H);
        }
    }
    free(gg); free(uu); free(act); free(part);
    return 0;
}

/* Attention block, sharded: shard s owns query heads
 * [s*nq/t, (s+1)*nq/t) and kv heads [s*nkv/t, (s+1)*nkv/t) (whole heads, the
 * ownership rule of [TSC]); it computes q/k/v from its own rows of Wq/Wk/Wv,
 * attends over its own heads, and multiplies by its own column block of Wo,
 * giving a full-size partial; h = x + sum_s partial_s (residual if flagged).
 * Input a (already normalised, or raw) [B][H]; caches as in
 * orc_decode_layer. */
int orc_attn_sharded(const orc_dims *dm, const orc_weights *w, int32_t t, long B, const double *x,
                     const double *a_in, const uint16_t *kc, const uint16_t *vc, long S_cap, long S,
                     double *h_out, double *partials) {
    const long H = dm->hidden, nq = dm->n_q_heads, nkv = dm->n_kv_heads, d = dm->head_dim;
    if (t <= 0 || nq % t != 0 || nkv % t != 0 || nq % nkv != 0) return 2;
    const long nqs = nq / t, nkvs = nkv / t, g = nq / nkv;
    const double scale = 1.0 / sqrt((double)d);
    double *q = malloc(sizeof(double) * (size_t)(nqs * d));
    double *k = malloc(sizeof(double) * (size_t)(nkvs * d));
    double *v = malloc(sizeof(double) * (size_t)(nkvs * d));
    double *o = malloc(sizeof(double) * (size_t)(nqs * d));
    double *part = malloc(sizeof(double) * (size_t)H);
    for (long b = 0; b < B; ++b) {
        const double *ab = a_in + (size_t)b * H;
        double *hb = h_out + (size_t)b * H;
        for (long i = 0; i < H; ++i) hb[i] = 0.0;
        for (int32_t s = 0; s < t; ++s) {
            linear_block(w->wq, w->wtype, (size_t)H, (long)s * nqs * d, nqs * d, 0, H, ab, q);
            linear_block(w->wk, w->wtype, (size_t)H, (long)s * nkvs * d, nkvs * d, 0, H, ab, k);
            linear_block(w->wv, w->wtype, (size_t)H, (long)s * nkvs * d, nkvs * d, 0, H, ab, v);
            for (long hl = 0; hl < nqs; ++hl) {
                long hg = (long)s * nqs + hl;          /* global query head */
                long jg = hg / g;                      /* its kv head (global) */
                long jl = jg - (long)s * nkvs;         /* local index within shard */
                size_t off = (((size_t)b * nkv + jg) * (size_t)S_cap) * d;
                attend_one(q + hl * d, d, kc + off, vc + off, S, k + jl * d, v + jl * d, scale,
                           o + hl * d);
            }
            linear_block(w->wo, w->wtype, (size_t)(nq * d), 0, H, (long)s * nqs * d, nqs * d, o, part);
            for (long i = 0; i < H; ++i) hb[i] += part[i];
            if (partials) memcpy(partials + ((size_t)s * B + b) * H, part, sizeof(double) * (size_t)H);
        }
        if (dm->flags & ORC_RESIDUAL)
            for (long i = 0; i < H; ++i) hb[i] = x[(size_t)b * H + i] + hb[i];
    }
    free(q); free(k); free(v); free(o); free(part);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Shard maps and footprints, derived from the ownership rule and formulas.
 * ------------------------------------------------------------------------- */

/* Returns 0, or 2 if t does not divide the head/ffn counts or t is not one of
 * 1, 2, 4, 8 ("Tensor Parallelism" docs: the size is 1, 2, 4 or 8). */
int orc_plan_maps(const orc_dims *dm, int32_t t, int32_t *q_shard, int32_t *q_local,
                  int32_t *kv_shard, int32_t *ffn_shard) {
    if (!(t == 1 || t == 2 || t == 4 || t == 8)) return 2;
    if (dm->n_q_heads % t || dm->n_kv_heads % t || dm->ffn % t) return 2;
    int32_t hpg = dm->n_q_heads / t; /* query heads per shard */
    for (int32_t rank = 0; rank < t; ++rank) {
        for (int32_t h = rank * hpg; h < (rank + 1) * hpg; ++h) {
            if (q_shard) q_shard[h] = rank;
            if (q_local) q_local[h] = h - rank * hpg;
        }
        int32_t kpg = dm->n_kv_heads / t;
        for (int32_t j = rank * kpg; j < (rank + 1) * kpg; ++j)
            if (kv_shard) kv_shard[j] = rank;
        int32_t fpg = dm->ffn / t;
        for (int32_t c = rank * fpg; c < (rank + 1) * fpg; ++c)
            if (ffn_shard) ffn_shard[c] = rank;
    }
    return 0;
}

/* KV bytes per GPU: 2 * layers * kv_heads * head_dim * seq * bytes * batch / t
 * ("Tensor Parallelism Fundamentals", "Memory Overhead and Communication
 * Bottlenecks").  Exact integer arithmetic; returns -1 if t does not divide. */
long long orc_kv_bytes_per_shard(long long layers, long long kv_heads, long long head_dim,
                                 long long seq, long long bytes, long long batch, long long t) {
    long long total = 2LL * layers * kv_heads * head_dim * seq * bytes * batch;
    if (t <= 0 || total % t) return -1;
    return total / t;
}

/* Parameters of one layer held by one shard: its slices of Wq, Wk, Wv (rows),
 * Wo (columns), Wg, Wu (rows) and Wd (columns). */
long long orc_layer_params_per_shard(const orc_dims *dm, int32_t t) {
    long long H = dm->hidden, nq = dm->n_q_heads, nkv = dm->n_kv_heads, d = dm->head_dim,
              F = dm->ffn;
    long long qkv = (nq / t + 2 * (nkv / t)) * d * H;
    long long o = H * (nq / t) * d;
    long long gu = 2 * (F / t) * H;
    long long dn = H * (F / t);
    return qkv + o + gu + dn;
}

/* Sum reductions per forward pass: one after each row-split projection, two
 * per layer ([TSC], "What tensor parallelism actually splits"). */
long long orc_reductions_per_pass(long long layers) { return 2 * layers; }

/* ---------------------------------------------------------------------------
 * Planner extras.
 *  [TPD]  "Tensor Parallelism" docs, section "Auto": the smallest power of two
 *         that fits comfortably, preferring 1; where the target's memory cannot
 *         be seen, the largest power of two the node's GPU count allows.
 *  [TSC]  "Tensor parallel scaling curves", section "The scaling math":
 *         T(N) = T_compute/N + T_memory/N + 2L * T_allreduce(N), where
 *         T_allreduce(N) is a per-call latency plus a bandwidth part; section
 *         "What tensor parallelism actually splits": a ring all-reduce on N
 *         GPUs moves about 2 (N-1)/N times the message.
 * Readings: "fits comfortably" = per-GPU weights + KV <= budget * (1 -
 * headroom), the headroom given by the caller; t also has to divide the
 * query heads, kv heads and ffn; at N = 1 there is no all-reduce; the two
 * terms T_compute/N and T_memory/N are added as printed.
 * ------------------------------------------------------------------------- */

static int orc_t_divides(const orc_dims *dm, int t) {
    return dm->n_q_heads % t == 0 && dm->n_kv_heads % t == 0 && dm->ffn % t == 0;
}

/* Per-GPU bytes of weights of `layers` layers plus the KV cache for `batch`
 * sequences of `seq` tokens, at shard degree t (-1 if t does not divide). */
long long orc_footprint_per_gpu(const orc_dims *dm, long long layers, int t, long long batch, long long seq,
                                long long bytes_per_elem) {
    if (t <= 0 || !orc_t_divides(dm, t)) return -1;
    long long w = layers * orc_layer_params_per_shard(dm, t) * bytes_per_elem;
    long long kv = orc_kv_bytes_per_shard(layers, dm->n_kv_heads, dm->head_dim, seq, bytes_per_elem, batch, t);
    if (kv < 0) return -1;
    return w + kv;
}

/* [TPD] Auto: smallest t in 1, 2, 4, 8 (t <= max_t) that fits; with
 * budget_bytes <= 0 the largest such t.  0 when none qualifies. */
int orc_auto_t(const orc_dims *dm, long long layers, long long budget_bytes, double headroom, long long batch,
               long long seq, long long bytes_per_elem, int max_t) {
    int best = 0;
    for (int t = 1; t <= 8 && t <= max_t; t *= 2) {
        if (!orc_t_divides(dm, t)) continue;
        if (budget_bytes <= 0) {
            best = t;  /* blind: keep the largest */
            continue;
        }
        long long need = orc_footprint_per_gpu(dm, layers, t, batch, seq, bytes_per_elem);
        if (need >= 0 && (double)need <= (double)budget_bytes * (1.0 - headroom)) return t;
    }
    return budget_bytes <= 0 ? best : 0;
}

/* [TSC] one all-reduce on n GPUs: latency + 2 (n-1)/n * message / bandwidth;
 * none at n = 1. */
double orc_allreduce_time(int n, double message_bytes, double latency_s, double link_bytes_per_s) {
    if (n <= 1) return 0.0;
    return latency_s + 2.0 * (double)(n - 1) / (double)n * message_bytes / link_bytes_per_s;
}

/* [TSC] per-token time at degree n from the single-GPU time (compute plus
 * memory) and the per-call all-reduce time. */
double orc_tp_time(double t_single, int n, long long layers, double t_allreduce) {
    return t_single / (double)n + 2.0 * (double)layers * t_allreduce;
}
