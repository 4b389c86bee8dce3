// Prefill of one layer over a chunk of T tokens ("Tensor parallel scaling
// curves", sections "What tensor parallelism actually splits" and "Prefill vs
// decode: different curves"): the decode layer's splits with many tokens, so
// every projection is a matrix product on the tensor cores.
//
//   norm_split   a = RMSNorm(x) as bf16 hi + lo                 (HBM bound)
//   gemm QKV     column-parallel, fused scatter to q / cache / k,v remainders
//   attention    causal, owned heads, mma.sync with hi + lo operands; writes
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

namespace tpl {

// a = x * gamma / sqrt(mean(x^2) + eps) (or a = x without TPL_NORM), split
// into bf16 hi = rn(a) and lo = rn(a - hi).  One CTA per token row.
__global__ void __launch_bounds__(256) norm_split_kernel(const void *x, int x_f32, const float *gamma, float eps,
                                                         int norm, int H, __nv_bfloat16 *hi, __nv_bfloat16 *lo) {
    __shared__ float s_red[8];
    pdl_wait();
    pdl_trigger();
    const int64_t row = blockIdx.x;
    const int n8 = H / 8;
    float ss = 0.f;
    for (int c = threadIdx.x; c < n8; c += blockDim.x) {
        float v[8];
        if (x_f32) {
            const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(x) + row * H + 8 * c);
            const float4 u0 = p[0], u1 = p[1];
            v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w; v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
        } else {
            const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(x) + row * H + 8 * c);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            for (int e = 0; e < 4; ++e) {
                v[2 * e] = bf16lo(w[e]);
                v[2 * e + 1] = bf16hi(w[e]);
            }
        }
        for (int e = 0; e < 8; ++e) ss += v[e] * v[e];
    }
    float inv = 1.f;
    if (norm) {
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
        __syncthreads();
        float tot = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += s_red[w];
        inv = 1.0f / sqrtf(tot / (float)H + eps);
    }
    for (int c = threadIdx.x; c < n8; c += blockDim.x) {
        float v[8];
        if (x_f32) {
            const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(x) + row * H + 8 * c);
            const float4 u0 = p[0], u1 = p[1];
            v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w; v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
        } else {
            const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(x) + row * H + 8 * c);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            for (int e = 0; e < 4; ++e) {
                v[2 * e] = bf16lo(w[e]);
                v[2 * e + 1] = bf16hi(w[e]);
            }
        }
        uint32_t h4[4], l4[4];
        for (int e = 0; e < 4; ++e) {
            float a0 = v[2 * e], a1 = v[2 * e + 1];
            if (norm) {
                a0 = a0 * inv * gamma[8 * c + 2 * e];
                a1 = a1 * inv * gamma[8 * c + 2 * e + 1];
            }
            h4[e] = pack_bf16x2(a0, a1);
            l4[e] = pack_bf16x2(a0 - bf16lo(h4[e]), a1 - bf16hi(h4[e]));
        }
        *reinterpret_cast<uint4 *>(hi + row * H + 8 * c) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
        *reinterpret_cast<uint4 *>(lo + row * H + 8 * c) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
    }
}

namespace {

// ---- tensor maps (driver entry point fetched through the runtime) ---------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::atomic<EncodeTiledFn> g_encode{nullptr};

EncodeTiledFn encode_fn() {
    EncodeTiledFn f = g_encode.load();
    if (f) return f;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
        return nullptr;
    f = reinterpret_cast<EncodeTiledFn>(p);
    g_encode.store(f);
    return f;
}

// bf16 matrix [rows][cols] with `row_bytes` between rows (and, for 3-D,
// `planes` of them `plane_bytes` apart); boxes of box_cols x box_rows with the
// 128-byte swizzle the MMA descriptors expect; out-of-range elements read 0.
int make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t row_bytes, uint32_t box_cols,
             uint32_t box_rows, uint64_t planes = 0, uint64_t plane_bytes = 0, uint32_t box_planes = 1) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return TPL_ECUDA;
    if (((uintptr_t)base & 15u) || (row_bytes & 15u) || (plane_bytes & 15u)) return TPL_EINVAL;
    const cuuint64_t gdim[3] = {cols, rows, planes};
    const cuuint64_t gstr[2] = {row_bytes, plane_bytes};
    const cuuint32_t box[3] = {box_cols, box_rows, box_planes};
    const cuuint32_t es[3] = {1, 1, 1};
    const cuuint32_t rank = planes ? 3 : 2;
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), gdim, gstr, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? TPL_OK : TPL_EINVAL;
}

// ---- GEMM launches ---------------------------------------------------------

bool g_gemm_attr[64][4];  // per device: dynamic shared memory attribute set, per instantiation

template <bool SA, bool RS>
int gemm_go(int slot, GemmArgs &a, int shard_units, cudaStream_t st) {
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
    const int64_t units = (int64_t)a.m_tiles * a.n_tiles * shard_units;
    if (units > 0x7fffffff) return TPL_EUNSUPPORTED;
    a.units = (int)units;
    const int grid = (int)std::min<int64_t>(units, sms);
    return cuda_rc(launch_pdl(gemm_tc_kernel<SA, RS>, grid, kGemmThreads, (size_t)GemmSmem<SA>::BYTES, st, a));
}

// Column-parallel projection: A = bf16 hi + lo [T][K] activations, W the
// shards' stacked rows [N][ld] (2-D).
int gemm_column(GemmArgs &a, const void *a_hi, const void *a_lo, int64_t K, const void *W, int64_t N, int64_t ld,
                cudaStream_t st) {
    int rc = make_map(&a.tm_a, a_hi, K, a.M, K * 2, kGemmKTile, kGemmMTile);
    if (rc == TPL_OK) rc = make_map(&a.tm_a2, a_lo, K, a.M, K * 2, kGemmKTile, kGemmMTile);
    if (rc == TPL_OK) rc = make_map(&a.tm_w, W, ld, N, ld * 2, kGemmKTile, kGemmNTile);
    if (rc != TPL_OK) return rc;
    a.N = (int)N;
    a.k_blocks = (int)(ld / kGemmKTile);
    a.nseg = 1;
    a.a_col_stride = 0;
    a.w3d = 0;
    return gemm_go<true, false>(0, a, 1, st);
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
    if (rc != TPL_OK) return rc;
    a.N = (int)H;
    a.k_blocks = (int)(ld / kGemmKTile);
    a.a_col_stride = (int)Ks;
    a.w3d = 1;
    if (!fused) {
        a.nseg = 1;
        a.epi = GEPI_PARTIAL;
        return A_lo ? gemm_go<true, false>(0, a, t, st) : gemm_go<false, false>(1, a, t, st);
    }
    a.nseg = t;
    a.epi = GEPI_ROW;
    return A_lo ? gemm_go<true, true>(2, a, 1, st) : gemm_go<false, true>(3, a, 1, st);
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
                              lo));
}

bool g_ap_attr[64];
bool g_at_attr[64];

// Tensor-core attention: 128 rows per CTA = (128 / g) tokens x the g heads of
// a kv head, so g must be a power of two.
int run_attn_prefill_tc(const tpl_plan *p, const tpl_kv *kv, const float *q, const __nv_bfloat16 *klo,
                        const __nv_bfloat16 *vlo, int T, __nv_bfloat16 *o_hi, __nv_bfloat16 *o_lo, cudaStream_t st,
                        int dev) {
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
    // cache planes: [head blocks][keys < T][128]; keys past the chunk read as 0
    int rc = make_map(&a.tm_khi, kv->k, 128, (uint64_t)T, 256, 64, kAtKeys, head_blocks, (uint64_t)kv->seq_cap * 256);
    if (rc == TPL_OK)
        rc = make_map(&a.tm_vhi, kv->v, 128, (uint64_t)T, 256, 64, kAtKeys, head_blocks, (uint64_t)kv->seq_cap * 256);
    // remainder planes: [T][nkv][128]
    if (rc == TPL_OK) rc = make_map(&a.tm_klo, klo, 128, nkv, 256, 64, 1, (uint64_t)T, (uint64_t)nkv * 256, kAtKeys);
    if (rc == TPL_OK) rc = make_map(&a.tm_vlo, vlo, 128, nkv, 256, 64, 1, (uint64_t)T, (uint64_t)nkv * 256, kAtKeys);
    if (rc != TPL_OK) return rc;
    a.q32 = q;
    a.o_hi = o_hi;
    a.o_lo = o_lo;
    a.T = T;
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
                     const __nv_bfloat16 *vlo, int T, __nv_bfloat16 *o_hi, __nv_bfloat16 *o_lo, cudaStream_t st) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TPL_ECUDA;
    if ((p->g & (p->g - 1)) == 0 && p->attn_prefill_mode == 0)
        return run_attn_prefill_tc(p, kv, q, klo, vlo, T, o_hi, o_lo, st, dev);
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

int prefill_layer(tpl_plan *p, const char *packed, const tpl_kv *kv, const void *x, int T, void *y, float *y32,
                  char *ws, const PrefillWs &L, int mode, cudaStream_t st) {
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
        rc = gemm_column(a, a_hi, a_lo, H, packed + p->off_qkv, (int64_t)p->t * p->qkv_rows_s, p->ld_h, st);
        if (rc != TPL_OK) return rc;
    }
    rc = run_attn_prefill(p, kv, q, klo, vlo, T, o, o_lo, st);
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
        rc = gemm_row(a, p, o, o_lo, (int64_t)p->nq_s * hd, packed + p->off_o, p->ld_o, p->blk_o, fused, st);
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
        rc = gemm_column(a, a_hi, a_lo, H, packed + p->off_gu, (int64_t)p->t * 2 * p->F_s, p->ld_h, st);
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
