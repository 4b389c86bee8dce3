// Host-side shard planner: validation, shard maps, packed layout, footprints
// and workspace layout.  No GPU is needed for anything in this file except
// num_sms_current().
//
// Ownership rule ("Tensor parallel scaling curves", section "What tensor
// parallelism actually splits"): shard s owns the query heads
// [s*n_q/t, (s+1)*n_q/t), the kv heads [s*n_kv/t, (s+1)*n_kv/t) and the ffn
// columns [s*F/t, (s+1)*F/t).  Footprints: "Tensor Parallelism Fundamentals",
// section "Memory Overhead and Communication Bottlenecks".

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>

#include "tpl_internal.h"

namespace {

int64_t align_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

int validate(const tpl_dims *d, int32_t t) {
    if (!d) return TPL_EINVAL;
    if (d->hidden <= 0 || d->n_q_heads <= 0 || d->n_kv_heads <= 0 || d->head_dim <= 0 ||
        d->ffn <= 0 || d->n_layers <= 0)
        return TPL_EINVAL;
    if (!(d->rms_eps >= 0.0f)) return TPL_EINVAL;
    if (d->flags & ~(TPL_NORM | TPL_RESIDUAL | TPL_FP32_WEIGHTS | TPL_ROPE)) return TPL_EINVAL;
    if ((d->flags & TPL_ROPE) && !(d->rope_base > 1.0f)) return TPL_EINVAL;
    if (!(t == 1 || t == 2 || t == 4 || t == 8)) return TPL_EINDIVISIBLE;
    if (d->n_q_heads % t || d->n_kv_heads % t || d->ffn % t) return TPL_EINDIVISIBLE;
    if (d->n_q_heads % d->n_kv_heads) return TPL_EINDIVISIBLE;
    if (d->head_dim != 128) return TPL_EUNSUPPORTED;
    if (d->n_q_heads / d->n_kv_heads > 16) return TPL_EUNSUPPORTED;
    if (d->hidden % 8 || (d->ffn / t) % 8) return TPL_EUNSUPPORTED;
    return TPL_OK;
}

}  // namespace

namespace tpl {

int gemv_geom(int N, int nseg, int Kseg, int B, int xbytes, int num_sms, GemvGeom *g, int xparts) {
    if (N <= 0 || nseg <= 0 || Kseg <= 0 || B <= 0 || num_sms <= 0) return TPL_EINVAL;
    std::memset(g, 0, sizeof(*g));
    g->N = N;
    g->nseg = nseg;
    g->Kseg = Kseg;
    g->nb = (Kseg + 127) / 128;
    int ksplit = 1, blocks = 0;
    for (;; ksplit *= 2) {
        if (ksplit > 64) return TPL_EUNSUPPORTED;
        if (ksplit <= nseg) {
            blocks = g->nb;  // per segment, nseg/ksplit whole segments
            int64_t bytes = (int64_t)xparts * B * ((int64_t)(nseg / ksplit) * blocks * 128 * xbytes + 64);
            if (bytes <= (int64_t)kXSmemMax) break;
        } else {
            int per = ksplit / nseg;
            if (per > g->nb) return TPL_EUNSUPPORTED;
            blocks = (g->nb + per - 1) / per;
            int64_t bytes = (int64_t)xparts * B * ((int64_t)blocks * 128 * xbytes + 64);
            if (bytes <= (int64_t)kXSmemMax) break;
        }
    }
    g->ksplit = ksplit;
    g->segs_per_cta = ksplit <= nseg ? nseg / ksplit : 1;
    g->pieces = ksplit <= nseg ? 1 : ksplit / nseg;
    g->cta_blocks = blocks;
    const int m = g->segs_per_cta;
    int wk = kGemvWarps;
    while (wk > m && blocks / (wk / m) < 2) wk /= 2;
    if (wk < m) wk = m;
    g->wk = wk;
    g->wr = kGemvWarps / wk;
    g->ng = (N + 7) / 8;
    int rb = std::max(1, num_sms / ksplit);
    rb = std::min(rb, g->ng);
    rb = std::min(rb, kMaxRowBlocks);
    g->rb = rb;
    int rg_cta = (g->ng + rb - 1) / rb;
    int rg_warp = (rg_cta + g->wr - 1) / g->wr;
    // Rounds of row groups per warp: one round when the partial sums fit,
    // else a multiple of 4 (the kernel's register ring holds 4 blocks and a
    // round must hold a multiple of that).
    int rgc_cap = (int)(kPartSmemMax / ((size_t)kGemvWarps * 8 * B * 4));
    g->rgc = rg_warp <= rgc_cap ? std::max(1, rg_warp) : std::max(4, rgc_cap / 4 * 4);
    g->x_stride = m * blocks * 128 * xbytes + 64;
    size_t part = (size_t)kGemvWarps * g->rgc * 8 * B * 4;
    g->smem = (size_t)xparts * B * g->x_stride + part + 128;
    g->gp_floats = ksplit > 1 ? (size_t)nseg * g->pieces * N * B : 0;
    return TPL_OK;
}

void attn_geom(int B, int nkv, int64_t keys, AttnGeom *a) {
    a->pairs = B * nkv;
    if (keys <= 0) {  // nothing in the cache: the splits are empty
        a->nsplit = kAttnWarps;
        a->kps = 16;
        return;
    }
    int64_t ns = (kAttnTargetWarps + a->pairs - 1) / a->pairs;
    ns = std::max<int64_t>(ns, 1);
    ns = std::min<int64_t>(ns, (keys + kAttnMinKeys - 1) / kAttnMinKeys);
    ns = std::min<int64_t>(ns, (int64_t)kAttnMaxCtasPerPair * kAttnWarps);
    ns = std::max<int64_t>(ns, 1);
    // whole CTAs of kAttnWarps splits, the keys spread over all of them
    ns = (ns + kAttnWarps - 1) / kAttnWarps * kAttnWarps;
    int64_t kps = (keys + ns - 1) / ns;
    kps = (kps + 15) / 16 * 16;
    ns = (keys + kps - 1) / kps;
    ns = (ns + kAttnWarps - 1) / kAttnWarps * kAttnWarps;
    a->nsplit = (int)ns;
    a->kps = (int)kps;
}

void attn_geom_staged(int B, int nkv, int64_t keys, int sms, AttnGeom *a) {
    a->pairs = B * nkv;
    int64_t cpp = std::max(1, sms / std::max(1, a->pairs));
    const int64_t by_keys = (keys + kAttnStgWarps * 64 - 1) / (kAttnStgWarps * 64);
    cpp = std::min(cpp, std::max<int64_t>(1, by_keys));
    cpp = std::min<int64_t>(cpp, kAttnMaxCtasPerPair);
    a->nsplit = (int)cpp * kAttnStgWarps;
    int64_t kps = keys > 0 ? (keys + a->nsplit - 1) / a->nsplit : 16;
    a->kps = (int)((kps + 15) / 16 * 16);
}

void attn_geom_tma(int B, int nkv, int64_t keys, int sms, AttnGeom *a) {
    a->pairs = B * nkv;
    a->nb = (int)((keys + kAttnTmaKeys - 1) / kAttnTmaKeys);
    const int64_t U = (int64_t)a->pairs * a->nb;
    int64_t grid = std::min<int64_t>(std::min(sms, kAttnTmaMaxCtas), U);
    a->grid = (int)std::max<int64_t>(grid, 1);
    a->cpp_max = std::min(a->grid, (a->grid + a->pairs - 1) / a->pairs + 1);
    a->nsplit = 0;
    a->kps = kAttnTmaKeys;
}

int ws_layout(const tpl_plan *p, int B, int64_t S, WsLayout *w) {
    if (B <= 0 || S < 0) return TPL_EINVAL;
    const tpl_dims &d = p->d;
    const int64_t H = d.hidden, nqd = (int64_t)d.n_q_heads * d.head_dim, F = d.ffn;
    const int es = p->esize;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = (size_t)align_up((int64_t)(off + bytes), 256);
        return o;
    };
    w->tickets = take(sizeof(uint32_t) * kTicketSlots);
    w->q = take((size_t)B * nqd * 4);
    w->o = take((size_t)B * nqd * es);
    w->h = take((size_t)B * H * 4);
    w->act = take((size_t)B * F * es);
    w->ybuf0 = take((size_t)B * H * es);
    w->ybuf1 = take((size_t)B * H * es);
    w->P = take((size_t)p->t * B * H * 4);
    w->knew = take((size_t)B * d.n_kv_heads * d.head_dim * 4);
    w->vnew = take((size_t)B * d.n_kv_heads * d.head_dim * 4);
    AttnGeom ag, ag1;  // splits over S keys (new key apart) or S + 1 keys
    attn_geom(B, d.n_kv_heads, S, &ag);
    attn_geom(B, d.n_kv_heads, S + 1, &ag1);
    AttnGeom sg, sg1;  // the staged kernel's splits, for the largest SM count
    attn_geom_staged(B, d.n_kv_heads, S, kAttnSmsBound, &sg);
    attn_geom_staged(B, d.n_kv_heads, S + 1, kAttnSmsBound, &sg1);
    AttnGeom tg;  // the TMA-streamed kernel's CTAs per pair, for the largest grid
    attn_geom_tma(B, d.n_kv_heads, S + 1, kAttnTmaMaxCtas, &tg);
    const size_t cpp = std::max((size_t)std::max(std::max(ag.nsplit, ag1.nsplit), std::max(sg.nsplit, sg1.nsplit)) /
                                    kAttnWarps,
                                (size_t)tg.cpp_max);
    w->part_o = take((size_t)ag.pairs * cpp * p->g * d.head_dim * 4);
    w->part_ml = take((size_t)ag.pairs * cpp * p->g * 2 * 4);
    // cross-CTA partials: the largest over the four matrix-vector steps
    size_t gp = 0;
    GemvGeom gg;
    const int xb = p->f32 ? 4 : 2;
    const int sms = 148;  // only the split-K factor matters here, not the SM count
    if (gemv_geom(p->t * p->qkv_rows_s, 1, (int)H, B, xb, sms, &gg, p->f32 ? 1 : 2) == TPL_OK)
        gp = std::max(gp, gg.gp_floats);
    if (gemv_geom((int)H, p->t, p->nq_s * d.head_dim, B, xb, sms, &gg) == TPL_OK) gp = std::max(gp, gg.gp_floats);
    if (gemv_geom(p->t * 2 * p->F_s, 1, (int)H, B, xb, sms, &gg, p->f32 ? 1 : 2) == TPL_OK)
        gp = std::max(gp, gg.gp_floats);
    if (gemv_geom((int)H, p->t, p->F_s, B, xb, sms, &gg) == TPL_OK) gp = std::max(gp, gg.gp_floats);
    w->gp = take(gp * 4 + 4);
    w->xs = take((size_t)gt_nx(B, true) * H * 2);  // [NX][hidden] bf16
    w->gpart = take((size_t)kGemvTcMaxCtas * 2 * p->t * 128 * gt_stride(B) * 4);
    w->total = off;
    return TPL_OK;
}

int prefill_ws_layout(const tpl_plan *p, int64_t T, PrefillWs *w) {
    if (T <= 0) return TPL_EINVAL;
    const tpl_dims &d = p->d;
    const int64_t H = d.hidden, nqd = (int64_t)d.n_q_heads * d.head_dim, nkvd = (int64_t)d.n_kv_heads * d.head_dim;
    size_t off = 0;
    auto take = [&](int64_t bytes) {
        size_t o = off;
        off = (size_t)align_up((int64_t)off + bytes, 256);
        return o;
    };
    w->a_hi = take(T * H * 2);
    w->a_lo = take(T * H * 2);
    w->q = take(T * nqd * 4);
    w->klo = take(T * nkvd * 2);
    w->vlo = take(T * nkvd * 2);
    w->o = take(T * nqd * 2);
    w->o_lo = take(T * nqd * 2);
    w->h = take(T * H * 4);
    w->act = take(T * (int64_t)d.ffn * 2);
    w->P = take((int64_t)p->t * T * H * 4);
    w->total = off;
    return TPL_OK;
}

int num_sms_current() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

}  // namespace tpl

extern "C" {

int tpl_plan_create(const tpl_dims *dims, int32_t t, tpl_plan **out) {
    if (!out) return TPL_EINVAL;
    *out = nullptr;
    int rc = validate(dims, t);
    if (rc != TPL_OK) return rc;
    tpl_plan *p = new (std::nothrow) tpl_plan;
    if (!p) return TPL_ENOMEM;
    p->d = *dims;
    p->t = t;
    p->nq_s = dims->n_q_heads / t;
    p->nkv_s = dims->n_kv_heads / t;
    p->F_s = dims->ffn / t;
    p->g = dims->n_q_heads / dims->n_kv_heads;
    p->qkv_rows_s = (p->nq_s + 2 * p->nkv_s) * dims->head_dim;
    p->f32 = (dims->flags & TPL_FP32_WEIGHTS) != 0;
    p->esize = p->f32 ? 4 : 2;
    p->gemv_mode = p->f32 ? 1 : 4;
    p->attn_prefill_mode = 0;
    p->prefill_split = TPL_SPLIT_DEFAULT;
    p->prefill_tail = 1;
    p->attn_decode_mode = 0;
    p->rope = (dims->flags & TPL_ROPE) != 0;
    for (int e = 0; e < 64; ++e)
        p->rope_theta[e] = p->rope ? std::pow((double)dims->rope_base, -2.0 * e / dims->head_dim) : 0.0;
    const int64_t H = dims->hidden, es = p->esize;
    // rows padded with zeros to whole 128-column blocks
    p->ld_h = (int)align_up(H, 128);
    p->ld_o = (int)align_up((int64_t)p->nq_s * dims->head_dim, 128);
    p->ld_f = (int)align_up(p->F_s, 128);
    p->blk_qkv = align_up((int64_t)p->qkv_rows_s * p->ld_h * es, 256);
    p->blk_o = align_up(H * p->ld_o * es, 256);
    p->blk_gu = align_up((int64_t)2 * p->F_s * p->ld_h * es, 256);
    p->blk_d = align_up(H * p->ld_f * es, 256);
    int64_t off = 0;
    p->off_qkv = off;
    off += t * p->blk_qkv;
    p->off_o = off;
    off += t * p->blk_o;
    p->off_gu = off;
    off += t * p->blk_gu;
    p->off_d = off;
    off += t * p->blk_d;
    p->off_g1 = off;
    off += align_up(H * 4, 256);
    p->off_g2 = off;
    off += align_up(H * 4, 256);
    p->packed_bytes = off;
    p->reductions.store(0);
    *out = p;
    return TPL_OK;
}

void tpl_plan_destroy(tpl_plan *plan) { delete plan; }

int tpl_plan_set_option(tpl_plan *p, int32_t option, int32_t value) {
    if (!p) return TPL_EINVAL;
    if (option == TPL_OPT_GEMV_MODE) {
        if (value != 0 && value != 2 && value != 3 && value != 4) return TPL_EINVAL;
        if (p->f32) return value == 0 ? TPL_OK : TPL_EINVAL;
        p->gemv_mode = value;
        return TPL_OK;
    }
    if (option == TPL_OPT_DECODE_ATTN) {
        if (value != 0 && value != 1 && value != 2) return TPL_EINVAL;
        p->attn_decode_mode = value;
        return TPL_OK;
    }
    if (option == TPL_OPT_PREFILL_ATTN) {
        if (value != 0 && value != 1) return TPL_EINVAL;
        p->attn_prefill_mode = value;
        return TPL_OK;
    }
    if (option == TPL_OPT_PREFILL_SPLIT) {
        if (value < 0 || value > (TPL_SPLIT_QKV | TPL_SPLIT_O | TPL_SPLIT_GU)) return TPL_EINVAL;
        p->prefill_split = value;
        return TPL_OK;
    }
    if (option == TPL_OPT_PREFILL_TAIL) {
        if (value != 0 && value != 1) return TPL_EINVAL;
        p->prefill_tail = value;
        return TPL_OK;
    }
    return TPL_EINVAL;
}

int tpl_plan_info_get(const tpl_plan *p, tpl_plan_info *out) {
    if (!p || !out) return TPL_EINVAL;
    const tpl_dims &d = p->d;
    const int64_t H = d.hidden, hd = d.head_dim;
    out->t = p->t;
    out->q_heads_per_shard = p->nq_s;
    out->kv_heads_per_shard = p->nkv_s;
    out->ffn_per_shard = p->F_s;
    out->group_size = p->g;
    out->qkv_rows_per_shard = p->qkv_rows_s;
    out->elem_bytes = p->esize;
    out->layer_params_per_shard = (int64_t)p->qkv_rows_s * H + H * p->nq_s * hd +
                                  2 * (int64_t)p->F_s * H + H * p->F_s;
    out->layer_weight_bytes_per_shard = out->layer_params_per_shard * p->esize;
    out->packed_layer_bytes = p->packed_bytes;
    out->reductions_per_step = 2 * (int64_t)d.n_layers;
    return TPL_OK;
}

int tpl_plan_maps(const tpl_plan *p, int32_t *q_shard, int32_t *q_local, int32_t *kv_shard,
                  int32_t *ffn_shard, int64_t *packed_offsets) {
    if (!p) return TPL_EINVAL;
    const tpl_dims &d = p->d;
    for (int h = 0; h < d.n_q_heads; ++h) {
        if (q_shard) q_shard[h] = h / p->nq_s;
        if (q_local) q_local[h] = h % p->nq_s;
    }
    if (kv_shard)
        for (int j = 0; j < d.n_kv_heads; ++j) kv_shard[j] = j / p->nkv_s;
    if (ffn_shard)
        for (int c = 0; c < d.ffn; ++c) ffn_shard[c] = c / p->F_s;
    if (packed_offsets) {
        for (int s = 0; s < p->t; ++s) {
            packed_offsets[s] = p->off_qkv + s * p->blk_qkv;
            packed_offsets[p->t + s] = p->off_o + s * p->blk_o;
            packed_offsets[2 * p->t + s] = p->off_gu + s * p->blk_gu;
            packed_offsets[3 * p->t + s] = p->off_d + s * p->blk_d;
        }
        packed_offsets[4 * p->t] = p->off_g1;
        packed_offsets[4 * p->t + 1] = p->off_g2;
    }
    return TPL_OK;
}

int64_t tpl_kv_bytes(const tpl_dims *d, int32_t t, int64_t batch, int64_t seq, int32_t bytes_per_elem) {
    if (!d || t <= 0 || batch < 0 || seq < 0 || bytes_per_elem <= 0) return -1;
    int64_t total = 2 * (int64_t)d->n_layers * d->n_kv_heads * d->head_dim * seq * bytes_per_elem * batch;
    if (total % t) return -1;
    return total / t;
}

int64_t tpl_footprint_bytes(const tpl_dims *d, int32_t t, int64_t batch, int64_t seq, int32_t bytes_per_elem) {
    if (!d || t <= 0 || d->n_layers < 0 || d->hidden <= 0 || d->head_dim <= 0 || d->n_q_heads <= 0 ||
        d->n_kv_heads <= 0 || d->ffn <= 0)
        return -1;
    if (d->n_q_heads % t || d->n_kv_heads % t || d->ffn % t) return -1;
    int64_t kv = tpl_kv_bytes(d, t, batch, seq, bytes_per_elem);
    if (kv < 0) return -1;
    const int64_t H = d->hidden, hd = d->head_dim;
    const int64_t per_shard = (d->n_q_heads / t + 2 * (d->n_kv_heads / t)) * hd * H  // Wq, Wk, Wv rows
                              + H * (d->n_q_heads / t) * hd                          // Wo columns
                              + 3 * (int64_t)(d->ffn / t) * H;                       // Wg, Wu rows, Wd columns
    return (int64_t)d->n_layers * per_shard * bytes_per_elem + kv;
}

int tpl_auto_t(const tpl_dims *d, int64_t budget_bytes, double headroom, int64_t batch, int64_t seq,
               int32_t bytes_per_elem, int32_t max_t, int32_t *t_out) {
    if (!d || !t_out || !(headroom >= 0.0 && headroom < 1.0) || batch < 0 || seq < 0 || bytes_per_elem <= 0 ||
        max_t < 1)
        return TPL_EINVAL;
    *t_out = 0;
    int32_t blind = 0;
    for (int32_t t = 1; t <= 8 && t <= max_t; t *= 2) {
        int64_t need = tpl_footprint_bytes(d, t, batch, seq, bytes_per_elem);
        if (need < 0) continue;  // t does not divide the heads or ffn
        if (budget_bytes <= 0) {
            blind = t;
            continue;
        }
        if ((double)need <= (double)budget_bytes * (1.0 - headroom)) {
            *t_out = t;
            return TPL_OK;
        }
    }
    if (budget_bytes <= 0 && blind > 0) {
        *t_out = blind;
        return TPL_OK;
    }
    return TPL_ENOFIT;
}

int tpl_tp_estimate_get(double t_compute, double t_memory, int32_t n, int32_t layers, double message_bytes,
                        double latency_s, double link_bytes_per_s, tpl_tp_estimate *out) {
    if (!out || n < 1 || layers < 0 || !(t_compute >= 0) || !(t_memory >= 0) || !(message_bytes >= 0) ||
        !(latency_s >= 0) || !(link_bytes_per_s > 0))
        return TPL_EINVAL;
    out->t_compute = t_compute;
    out->t_memory = t_memory;
    out->t_allreduce = n == 1 ? 0.0 : latency_s + 2.0 * (n - 1) / n * message_bytes / link_bytes_per_s;
    out->t_comm = 2.0 * layers * out->t_allreduce;
    out->t_total = t_compute / n + t_memory / n + out->t_comm;
    const double t1 = t_compute + t_memory;
    out->speedup = out->t_total > 0 ? t1 / out->t_total : 1.0;
    out->comm_share = out->t_total > 0 ? out->t_comm / out->t_total : 0.0;
    return TPL_OK;
}

int tpl_decode_times(const tpl_dims *d, int64_t batch, int64_t seq, int32_t bytes_per_elem, double flops_per_s,
                     double hbm_bytes_per_s, double *t_compute, double *t_memory) {
    if (!d || !t_compute || !t_memory || !(flops_per_s > 0) || !(hbm_bytes_per_s > 0)) return TPL_EINVAL;
    const int64_t bytes = tpl_footprint_bytes(d, 1, batch, seq, bytes_per_elem);
    const int64_t kv = tpl_kv_bytes(d, 1, batch, seq, bytes_per_elem);
    if (bytes < 0 || kv < 0) return TPL_EINVAL;
    const double params = (double)(bytes - kv) / bytes_per_elem;
    *t_compute = 2.0 * params * (double)batch / flops_per_s;
    *t_memory = (double)bytes / hbm_bytes_per_s;
    return TPL_OK;
}

int64_t tpl_kv_layer_bytes(const tpl_plan *p, int32_t batch_cap, int64_t seq_cap) {
    if (!p || batch_cap < 0 || seq_cap < 0) return -1;
    return (int64_t)batch_cap * p->d.n_kv_heads * seq_cap * p->d.head_dim * 2;
}

int tpl_workspace_size(const tpl_plan *p, int32_t batch, int64_t seq, size_t *out) {
    if (!p || !out || batch <= 0 || seq < 0) return TPL_EINVAL;
    tpl::WsLayout w;
    int rc = tpl::ws_layout(p, batch, seq, &w);
    if (rc != TPL_OK) return rc;
    *out = w.total;
    return TPL_OK;
}

int tpl_prefill_workspace_size(const tpl_plan *p, int32_t T, size_t *out) {
    if (!p || !out || T <= 0) return TPL_EINVAL;
    tpl::PrefillWs w;
    int rc = tpl::prefill_ws_layout(p, T, &w);
    if (rc != TPL_OK) return rc;
    *out = w.total;
    return TPL_OK;
}

int tpl_prefill_intermediates(const tpl_plan *p, int32_t T, size_t *offsets) {
    if (!p || !offsets || T <= 0) return TPL_EINVAL;
    tpl::PrefillWs w;
    int rc = tpl::prefill_ws_layout(p, T, &w);
    if (rc != TPL_OK) return rc;
    offsets[0] = w.q;
    offsets[1] = w.o;
    offsets[2] = w.h;
    offsets[3] = w.act;
    offsets[4] = w.o_lo;
    return TPL_OK;
}

int64_t tpl_reduction_count(const tpl_plan *p) { return p ? (int64_t)p->reductions.load() : -1; }

void tpl_reset_counters(tpl_plan *p) {
    if (p) p->reductions.store(0);
}

const char *tpl_status_string(int s) {
    switch (s) {
        case TPL_OK: return "ok";
        case TPL_EINVAL: return "invalid argument";
        case TPL_EINDIVISIBLE: return "shard degree must be 1, 2, 4 or 8 and divide the head and ffn counts";
        case TPL_EWORKSPACE: return "workspace too small";
        case TPL_ENOMEM: return "capacity too small";
        case TPL_ECUDA: return "CUDA error";
        case TPL_EDEVICE: return "device-side inconsistency recorded";
        case TPL_EUNSUPPORTED: return "unsupported dimensions";
        case TPL_ENOFIT: return "no admissible shard degree fits the memory budget";
        default: return "unknown status";
    }
}

}  // extern "C"
