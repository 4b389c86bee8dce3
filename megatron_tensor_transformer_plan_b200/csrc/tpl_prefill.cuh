// Prefill of one layer over a chunk of T tokens ("Tensor parallel scaling
// curves", sections "What tensor parallelism actually splits" and "Prefill vs
// decode: different curves"): the decode layer's splits with many tokens, so
// every projection is a matrix product on the tensor cores.
//
//   norm_split   a = RMSNorm(x) as bf16 hi + lo                 (HBM bound)
//   gemm QKV     column-parallel, fused scatter to q / cache / k,v remainders
//   attention    causal, each shard's own heads, mma.sync with hi + lo operands; writes
//                its output as bf16 hi + lo
//   gemm O       row-parallel on o as bf16 hi + lo, t TMEM accumulators summed
//                in shard order, + x
//   norm_split   m = RMSNorm(h) as bf16 hi + lo
//   gemm GU      column-parallel, SwiGLU in the epilogue
//   gemm down    row-parallel, t accumulators summed in shard order + h
//
// This file is part of the library's single translation unit: it is included
// by tpl_device.cu after the launch helpers it uses.
#pragma once

#include <cuda.h>

#include "tpl_attn_prefill.cuh"
#include "tpl_attn_tc.cuh"
#include "tpl_gemm.cuh"
#include "tpl_norm.cuh"
#include "tpl_tma.h"

namespace tpl {

namespace {

// ---- GEMM launches ---------------------------------------------------------

bool g_gemm_attr[64][4];  // per device: dynamic shared memory attribute set, per instantiation

template <bool SA, bool RS>
int gemm_go(int slot, GemmArgs &a, int shard_units, bool halves, cudaStream_t st) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TPL_ECUDA;
    if (!g_gemm_attr[dev][slot]) {
        if (cudaFuncSetAttribute(gemm_tc_kernel<SA, RS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmSmem<SA>::BYTES) != cudaSuccess)
            return TPL_ECUDA;
        g_gemm_attr[dev][slot] = true;
    }
    const int sms = num_sms_current();
    if (sms <= 0) return TPL_ECUDA;
    a.m_tiles = (a.M + kGemmMTile - 1) / kGemmMTile;
    a.n_tiles = (a.N + kGemmNTile - 1) / kGemmNTile;
    const int64_t tiles = (int64_t)a.m_tiles * a.n_tiles * shard_units;
    if (2 * tiles > 0x7fffffff) return TPL_EUNSUPPORTED;
    // A last wave that fills at most half the SMs runs as half tiles, two
    // units per tile: it then ends in about half a tile's time.
    const int64_t rem = tiles % sms;
    const int64_t split = (halves && rem > 0 && 2 * rem <= sms) ? rem : 0;
    a.full_units = (int)(tiles - split);
    a.units = (int)(tiles + split);
    const int grid = (int)std::min<int64_t>(a.units, sms);
    return cuda_rc(launch_pdl(gemm_tc_kernel<SA, RS>, grid, kGemmThreads, (size_t)GemmSmem<SA>::BYTES, st, a));
}

// Column-parallel projection: A = bf16 hi (+ lo, when a_lo is not NULL)
// [T][K] activations, W the shards' stacked rows [N][ld] (2-D).
int gemm_column(GemmArgs &a, const tpl_plan *p, const void *a_hi, const void *a_lo, int64_t K, const void *W,
                int64_t N, int64_t ld, cudaStream_t st) {
    int rc = make_map(&a.tm_a, a_hi, K, a.M, K * 2, kGemmKTile, kGemmMTile);
    if (rc == TPL_OK && a_lo) rc = make_map(&a.tm_a2, a_lo, K, a.M, K * 2, kGemmKTile, kGemmMTile);
    if (rc == TPL_OK) rc = make_map(&a.tm_w, W, ld, N, ld * 2, kGemmKTile, kGemmNTile);
    if (rc == TPL_OK) rc = make_map(&a.tm_wh, W, ld, N, ld * 2, kGemmKTile, kGemmHalfN);
    if (rc != TPL_OK) return rc;
    a.N = (int)N;
    a.k_blocks = (int)(ld / kGemmKTile);
    a.nseg = 1;
    a.a_col_stride = 0;
    a.w3d = 0;
    const bool halves = p->prefill_tail != 0;
    return a_lo ? gemm_go<true, false>(0, a, 1, halves, st) : gemm_go<false, false>(1, a, 1, halves, st);
}

// Row-parallel projection: A [T][t*Ks] bf16 (shard s owns columns
// [s*Ks, (s+1)*Ks)), optionally with its bf16 remainder A_lo, W the shards'
// blocks [t][N][ld] (3-D).  Fused: one accumulation segment per shard, summed
// in ascending shard order in the epilogue (GEPI_ROW).  Separate: one unit
// per (tile, shard) writing the shard's partial (GEPI_PARTIAL).
int gemm_row(GemmArgs &a, const tpl_plan *p, const void *A, const void *A_lo, int64_t Ks, const void *W, int64_t ld,
             int64_t blk, bool fused, cudaStream_t st) {
    const int t = p->t;
    const int64_t H = p->d.hidden;
    int rc = make_map(&a.tm_a, A, (uint64_t)t * Ks, a.M, (uint64_t)t * Ks * 2, kGemmKTile, kGemmMTile);
    if (rc == TPL_OK && A_lo)
        rc = make_map(&a.tm_a2, A_lo, (uint64_t)t * Ks, a.M, (uint64_t)t * Ks * 2, kGemmKTile, kGemmMTile);
    if (rc == TPL_OK) rc = make_map(&a.tm_w, W, ld, H, ld * 2, kGemmKTile, kGemmNTile, t, blk);
    if (rc == TPL_OK) rc = make_map(&a.tm_wh, W, ld, H, ld * 2, kGemmKTile, kGemmHalfN, t, blk);
    if (rc != TPL_OK) return rc;
    a.N = (int)H;
    a.k_blocks = (int)(ld / kGemmKTile);
    a.a_col_stride = (int)Ks;
    a.w3d = 1;
    const bool halves = p->prefill_tail != 0;
    if (!fused) {
        a.nseg = 1;
        a.epi = GEPI_PARTIAL;
        return A_lo ? gemm_go<true, false>(0, a, t, halves, st) : gemm_go<false, false>(1, a, t, halves, st);
    }
    a.nseg = t;
    a.epi = GEPI_ROW;
    return A_lo ? gemm_go<true, true>(2, a, 1, halves, st) : gemm_go<false, true>(3, a, 1, halves, st);
}

GemmArgs gemm_args(int M) {
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.M = M;
    return a;
}

int run_norm_split(const tpl_plan *p, const void *x, int x_f32, const float *gamma, int T, __nv_bfloat16 *hi,
                   __nv_bfloat16 *lo, cudaStream_t st) {
    const int norm = (p->d.flags & TPL_NORM) ? 1 : 0;
    return cuda_rc(launch_pdl(norm_split_kernel, T, 256, 0, st, x, x_f32, gamma, p->d.rms_eps, norm, p->d.hidden, hi,
                              lo, T));
}

bool g_ap_attr[64];
bool g_at_attr[64];

// Tensor-core attention: 128 rows per CTA = (128 / g) tokens x the g heads of
// a kv head, so g must be a power of two.
int run_attn_prefill_tc(const tpl_plan *p, const tpl_kv *kv, const float *q, const __nv_bfloat16 *klo,
                        const __nv_bfloat16 *vlo, int T, int p0, __nv_bfloat16 *o_hi, __nv_bfloat16 *o_lo,
                        cudaStream_t st, int dev) {
    if (!g_at_attr[dev]) {
        if (cudaFuncSetAttribute(attn_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAtSmem) !=
            cudaSuccess)
            return TPL_ECUDA;
        g_at_attr[dev] = true;
    }
    AttnTcArgs a;
    std::memset(&a, 0, sizeof(a));
    const int nkv = p->d.n_kv_heads;
    const uint64_t head_blocks = (uint64_t)p->t * kv->batch_cap * p->nkv_s;
    // cache planes: [head blocks][keys < p0 + T][128]; keys past the chunk read as 0
    const uint64_t keys = (uint64_t)p0 + (uint64_t)T;
    int rc = make_map(&a.tm_khi, kv->k, 128, keys, 256, 64, kAtKeys, head_blocks, (uint64_t)kv->seq_cap * 256);
    if (rc == TPL_OK)
        rc = make_map(&a.tm_vhi, kv->v, 128, keys, 256, 64, kAtKeys, head_blocks, (uint64_t)kv->seq_cap * 256);
    // remainder planes: [T][nkv][128]
    if (rc == TPL_OK) rc = make_map(&a.tm_klo, klo, 128, nkv, 256, 64, 1, (uint64_t)T, (uint64_t)nkv * 256, kAtKeys);
    if (rc == TPL_OK) rc = make_map(&a.tm_vlo, vlo, 128, nkv, 256, 64, 1, (uint64_t)T, (uint64_t)nkv * 256, kAtKeys);
    if (rc != TPL_OK) return rc;
    a.q32 = q;
    a.o_hi = o_hi;
    a.o_lo = o_lo;
    a.T = T;
    a.p0 = p0;
    a.nq = p->d.n_q_heads;
    a.nkv = nkv;
    a.nkv_s = p->nkv_s;
    a.g = p->g;
    a.tb = 128 / p->g;
    a.batch_cap = kv->batch_cap;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)p->d.head_dim);
    const int64_t grid = (int64_t)((T + a.tb - 1) / a.tb) * nkv;
    if (grid > 0x7fffffff) return TPL_EUNSUPPORTED;
    return cuda_rc(launch_pdl(attn_prefill_tc_kernel, (int)grid, kAtThreads, kAtSmem, st, a));
}

int run_attn_prefill(const tpl_plan *p, const tpl_kv *kv, const float *q, const __nv_bfloat16 *klo,
                     const __nv_bfloat16 *vlo, int T, int p0, __nv_bfloat16 *o_hi, __nv_bfloat16 *o_lo,
                     cudaStream_t st) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TPL_ECUDA;
    if ((p->g & (p->g - 1)) == 0 && p->attn_prefill_mode == 0)
        return run_attn_prefill_tc(p, kv, q, klo, vlo, T, p0, o_hi, o_lo, st, dev);
    if (!g_ap_attr[dev]) {
        if (cudaFuncSetAttribute(attn_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kApSmem) !=
            cudaSuccess)
            return TPL_ECUDA;
        g_ap_attr[dev] = true;
    }
    AttnPrefillArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q32 = q;
    a.khi = static_cast<const __nv_bfloat16 *>(kv->k);
    a.vhi = static_cast<const __nv_bfloat16 *>(kv->v);
    a.klo = klo;
    a.vlo = vlo;
    a.seq_cap = kv->seq_cap;
    a.batch_cap = kv->batch_cap;
    a.T = T;
    a.p0 = p0;
    a.nq = p->d.n_q_heads;
    a.nkv = p->d.n_kv_heads;
    a.nkv_s = p->nkv_s;
    a.g = p->g;
    int gc = 1;
    while (p->g / gc > kApMaxWarps || p->g % gc) ++gc;
    a.gc = gc;
    a.wpc = p->g / gc;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)p->d.head_dim);
    a.o_hi = o_hi;
    a.o_lo = o_lo;
    const int64_t grid = (int64_t)((T + 15) / 16) * a.nkv * gc;
    if (grid > 0x7fffffff) return TPL_EUNSUPPORTED;
    return cuda_rc(launch_pdl(attn_prefill_kernel, (int)grid, a.wpc * 32, kApSmem, st, a));
}

int prefill_layer(tpl_plan *p, const char *packed, const tpl_kv *kv, const void *x, int T, int p0, void *y,
                  float *y32, char *ws, const PrefillWs &L, int mode, cudaStream_t st) {
    const bool resid = (p->d.flags & TPL_RESIDUAL) != 0;
    const int64_t H = p->d.hidden, hd = p->d.head_dim;
    auto *a_hi = reinterpret_cast<__nv_bfloat16 *>(ws + L.a_hi);
    auto *a_lo = reinterpret_cast<__nv_bfloat16 *>(ws + L.a_lo);
    auto *q = reinterpret_cast<float *>(ws + L.q);
    auto *klo = reinterpret_cast<__nv_bfloat16 *>(ws + L.klo);
    auto *vlo = reinterpret_cast<__nv_bfloat16 *>(ws + L.vlo);
    auto *o = reinterpret_cast<__nv_bfloat16 *>(ws + L.o);
    auto *o_lo = reinterpret_cast<__nv_bfloat16 *>(ws + L.o_lo);
    auto *h = reinterpret_cast<float *>(ws + L.h);
    void *act = ws + L.act;
    auto *P = reinterpret_cast<float *>(ws + L.P);
    const bool fused = mode == TPL_REDUCE_FUSED;

    int rc = run_norm_split(p, x, 0, reinterpret_cast<const float *>(packed + p->off_g1), T, a_hi, a_lo, st);
    if (rc != TPL_OK) return rc;
    {  // QKV
        GemmArgs a = gemm_args(T);
        a.epi = GEPI_QKV;
        a.q32 = q;
        a.klo = klo;
        a.vlo = vlo;
        a.kc = static_cast<__nv_bfloat16 *>(kv->k);
        a.vc = static_cast<__nv_bfloat16 *>(kv->v);
        a.rps = p->qkv_rows_s;
        a.nq = p->d.n_q_heads;
        a.nq_s = p->nq_s;
        a.nkv_s = p->nkv_s;
        a.hd = (int)hd;
        a.batch_cap = kv->batch_cap;
        a.seq_cap = kv->seq_cap;
        a.pos0 = p0;
        a.rope = p->rope ? 1 : 0;
        std::memcpy(a.theta, p->rope_theta, sizeof(a.theta));
        rc = gemm_column(a, p, a_hi, (p->prefill_split & TPL_SPLIT_QKV) ? a_lo : nullptr, H, packed + p->off_qkv,
                         (int64_t)p->t * p->qkv_rows_s, p->ld_h, st);
        if (rc != TPL_OK) return rc;
    }
    rc = run_attn_prefill(p, kv, q, klo, vlo, T, p0, o, o_lo, st);
    if (rc != TPL_OK) return rc;
    {  // O: h = x + sum_s o_s Wo[s]^T
        GemmArgs a = gemm_args(T);
        if (fused) {
            a.resid = resid ? x : nullptr;
            a.resid_f32 = 0;
            a.out32 = h;
        } else {
            a.out32 = P;
        }
        rc = gemm_row(a, p, o, (p->prefill_split & TPL_SPLIT_O) ? o_lo : nullptr, (int64_t)p->nq_s * hd,
                      packed + p->off_o, p->ld_o, p->blk_o, fused, st);
        if (rc != TPL_OK) return rc;
        if (fused) p->reductions.fetch_add(1);
        else if ((rc = run_reduce(p, st, P, resid ? x : nullptr, 0, T, h, nullptr)) != TPL_OK) return rc;
    }
    rc = run_norm_split(p, h, 1, reinterpret_cast<const float *>(packed + p->off_g2), T, a_hi, a_lo, st);
    if (rc != TPL_OK) return rc;
    {  // gate/up + SwiGLU
        GemmArgs a = gemm_args(T);
        a.epi = GEPI_GU;
        a.out_act = act;
        a.act_f32 = 0;
        rc = gemm_column(a, p, a_hi, (p->prefill_split & TPL_SPLIT_GU) ? a_lo : nullptr, H, packed + p->off_gu,
                         (int64_t)p->t * 2 * p->F_s, p->ld_h, st);
        if (rc != TPL_OK) return rc;
    }
    {  // down: y = h + sum_s act_s Wd[s]^T
        GemmArgs a = gemm_args(T);
        if (fused) {
            a.resid = resid ? h : nullptr;
            a.resid_f32 = 1;
            a.out32 = y32;
            a.out_act = y;
            a.act_f32 = 0;
        } else {
            a.out32 = P;
        }
        rc = gemm_row(a, p, act, nullptr, p->F_s, packed + p->off_d, p->ld_f, p->blk_d, fused, st);
        if (rc != TPL_OK) return rc;
        if (fused) p->reductions.fetch_add(1);
        else if ((rc = run_reduce(p, st, P, resid ? h : nullptr, 1, T, y32, y)) != TPL_OK) return rc;
    }
    return TPL_OK;
}

}  // namespace
}  // namespace tpl
