// Causal GQA attention of a prefill chunk on the 5th-generation tensor cores
// ("Tensor parallel scaling curves", "Prefill vs decode: different curves";
// each shard attends over its own heads, "What tensor parallelism actually splits"):
// the chunk's token i sits at position p0 + i and attends keys 0..p0 + i of
// the cache (slots below p0 were written by earlier chunks; their low parts
// are zero, read as the fill value of the remainder planes' negative
// coordinates).
//
// One CTA per (kv head j, block of 128/g tokens): its 128 rows are the block's
// tokens x the g query heads that share kv head j (row = token * g + head), so
// every K/V tile is used by all 128 rows of one MMA.  192 threads:
//   warp 0     TMA producer: K and V tiles of 64 keys (bf16 high parts from
//              the cache, low parts from the remainder planes the QKV
//              projection wrote), 3-stage ring, no multicast;
//   warp 1     TMEM owner and MMA issuer (one thread);
//   warps 2-5  softmax, one thread per row (its TMEM lane): they first load
//              q, split it into bf16 hi + lo and store both into TMEM.
// Tensor memory (512 columns): Q hi | Q lo | O (fp32, 128) | S0 | S1 (fp32,
// 64 each).  S = Q K^T is q_hi.k_hi + q_hi.k_lo + q_lo.k_hi (A from TMEM,
// B = the K tile, K-major); the softmax thread reads its S row, applies the
// causal mask and writes P as bf16 hi + lo over the same columns; then
// O += P_hi.v_hi + P_hi.v_lo + P_lo.v_hi (A = P from TMEM, B = the V tile,
// MN-major).  S of the next tile is computed while the softmax works.
// Online softmax with a lazily raised maximum: the running max moves (and O
// and the running sum are rescaled) only when a tile's max exceeds it by more
// than 8 in log2 units, so P stays below 2^8; the final division by the
// running sum makes the result independent of which maximum was used.
//
// Every wait is bounded (2 s); on a timeout the roles stop, the error word is
// set, copies in flight are waited for (bounded) and TMEM is released.
#pragma once

#include <cuda.h>

#include "tpl_common.cuh"
#include "tpl_gemm.cuh"

namespace tpl {

constexpr int kAtKeys = 64;      // keys per K/V tile
constexpr int kAtStages = 3;
constexpr int kAtThreads = 192;
constexpr int kAtTileBytes = kAtKeys * 128 * 2;  // one plane of one tile: 16 KB
constexpr int kAtStageBytes = 4 * kAtTileBytes;  // K hi, K lo, V hi, V lo
constexpr size_t kAtSmem = (size_t)kAtStages * kAtStageBytes + 1024 + 256;
// TMEM columns
constexpr uint32_t kAtQhi = 0, kAtQlo = 64, kAtO = 128, kAtS = 256;

struct AttnTcArgs {
    CUtensorMap tm_khi, tm_vhi;  // cache [heads of all shards][p0 + T (extent)][128] bf16, box {64, 64, 1}
    CUtensorMap tm_klo, tm_vlo;  // remainders [T][nkv][128] bf16, box {64, 1, 64}
    const float *q32;            // [T][nq][128]
    __nv_bfloat16 *o_hi, *o_lo;  // [T][nq*128]
    int T, nq, nkv, nkv_s, g, tb;  // tb = tokens per CTA = 128 / g
    int batch_cap;
    int p0;                      // position of the chunk's first token
    float scale_log2;
};

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// MMA with A read from tensor memory.
__device__ __forceinline__ void umma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(
            tmem_d),
        "r"(tmem_a), "l"(db), "r"(idesc), "r"(acc));
}

// 128-byte-swizzle descriptor with an explicit leading byte offset (the
// distance between 64-element chunks of an MN-major operand).
__device__ __forceinline__ uint64_t umma_desc_lbo(unsigned saddr, unsigned lbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__global__ void __launch_bounds__(kAtThreads, 1) attn_prefill_tc_kernel(const __grid_constant__ AttnTcArgs a) {
    extern __shared__ __align__(1024) unsigned char asm_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(((uintptr_t)asm_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *kfull = reinterpret_cast<uint64_t *>(sm + kAtStages * kAtStageBytes);
    uint64_t *vfull = kfull + kAtStages;
    uint64_t *kvempty = vfull + kAtStages;
    uint64_t *s_full = kvempty + kAtStages;  // [2]
    uint64_t *p_full = s_full + 2;          // [2]
    uint64_t *pv_done = p_full + 2;         // [2]
    uint64_t *q_ready = pv_done + 2;
    uint64_t *fin = q_ready + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + 1);
    volatile int *s_fail = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_issued = const_cast<int *>(s_fail) + 1;
    int *s_consumed = const_cast<int *>(s_fail) + 2;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntile = (a.T + a.tb - 1) / a.tb;
    const int rt = ntile - 1 - (int)(blockIdx.x / a.nkv);  // longest rows first
    const int j = (int)(blockIdx.x % a.nkv);
    const int t0 = rt * a.tb;
    const int t_last = min(a.T - 1, t0 + a.tb - 1);
    const int nkt = (a.p0 + t_last) / kAtKeys + 1;
    const int s_sh = j / a.nkv_s, jl = j % a.nkv_s;
    const int head_block = (s_sh * a.batch_cap) * a.nkv_s + jl;  // batch row 0

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAtStages; ++s) {
            mbar_init(&kfull[s], 1);
            mbar_init(&vfull[s], 1);
            mbar_init(&kvempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 4);
            mbar_init(&pv_done[b], 1);
        }
        mbar_init(q_ready, 4);
        mbar_init(fin, 1);
        *s_fail = 0;
        *s_issued = 0;
        *s_consumed = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            for (; it < nkt; ++it) {
                const int s = it % kAtStages;
                const unsigned ph = (unsigned)(it / kAtStages) & 1u;
                if (*s_fail || !mbar_wait(&kvempty[s], ph ^ 1u)) {
                    *s_fail = 1;
                    break;
                }
                unsigned char *st = sm + s * kAtStageBytes;
                const int key0 = it * kAtKeys;
                mbar_expect_tx(&kfull[s], 2 * kAtTileBytes);
                for (int h = 0; h < 2; ++h) {
                    tma_load_3d(st + h * (kAtTileBytes / 2), &a.tm_khi, 64 * h, key0, head_block, &kfull[s]);
                    tma_load_3d(st + kAtTileBytes + h * (kAtTileBytes / 2), &a.tm_klo, 64 * h, j, key0 - a.p0,
                                &kfull[s]);
                }
                mbar_expect_tx(&vfull[s], 2 * kAtTileBytes);
                for (int h = 0; h < 2; ++h) {
                    tma_load_3d(st + 2 * kAtTileBytes + h * (kAtTileBytes / 2), &a.tm_vhi, 64 * h, key0, head_block,
                                &vfull[s]);
                    tma_load_3d(st + 3 * kAtTileBytes + h * (kAtTileBytes / 2), &a.tm_vlo, 64 * h, j, key0 - a.p0,
                                &vfull[s]);
                }
            }
            *s_issued = it;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t IDESC_S = umma_idesc(128, kAtKeys);
            constexpr uint32_t IDESC_PV = umma_idesc(128, 128) | (1u << 16);  // B (V) MN-major
            bool ok = mbar_wait(q_ready, 0);
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            int consumed = 0;
            // S_i = Q K_i^T into buffer i & 1
            auto issue_s = [&](int i) -> bool {
                const int s = i % kAtStages;
                if (*s_fail || !mbar_wait(&kfull[s], (unsigned)(i / kAtStages) & 1u)) return false;
                if (i >= 2 && !mbar_wait(&pv_done[i & 1], (unsigned)((i - 2) >> 1) & 1u)) return false;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const unsigned kb = smem_u32(sm + s * kAtStageBytes);
                const uint32_t d = tmem + kAtS + (uint32_t)((i & 1) * kAtKeys);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const unsigned off = (unsigned)((kk >> 2) * (kAtTileBytes / 2) + 32 * (kk & 3));
                    const uint64_t dkh = umma_desc(kb + off);
                    const uint64_t dkl = umma_desc(kb + kAtTileBytes + off);
                    umma_ts(d, tmem + kAtQhi + 8 * kk, dkh, IDESC_S, kk > 0 ? 1u : 0u);
                    umma_ts(d, tmem + kAtQhi + 8 * kk, dkl, IDESC_S, 1u);
                    umma_ts(d, tmem + kAtQlo + 8 * kk, dkh, IDESC_S, 1u);
                }
                umma_commit(&s_full[i & 1]);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int i = 0; ok && i < nkt; ++i) {
                if (i + 1 < nkt && !issue_s(i + 1)) {
                    ok = false;
                    break;
                }
                const int s = i % kAtStages;
                if (*s_fail || !mbar_wait(&p_full[i & 1], (unsigned)(i >> 1) & 1u) ||
                    !mbar_wait(&vfull[s], (unsigned)(i / kAtStages) & 1u)) {
                    ok = false;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const unsigned vb = smem_u32(sm + s * kAtStageBytes + 2 * kAtTileBytes);
                const uint32_t pcol = tmem + kAtS + (uint32_t)((i & 1) * kAtKeys);
#pragma unroll
                for (int ks = 0; ks < kAtKeys / 16; ++ks) {
                    // 16 keys = two 8-row groups of both 64-column chunks of V
                    const uint64_t dvh = umma_desc_lbo(vb + 2048 * ks, kAtTileBytes / 2);
                    const uint64_t dvl = umma_desc_lbo(vb + kAtTileBytes + 2048 * ks, kAtTileBytes / 2);
                    umma_ts(tmem + kAtO, pcol + 8 * ks, dvh, IDESC_PV, (i > 0 || ks > 0) ? 1u : 0u);
                    umma_ts(tmem + kAtO, pcol + 8 * ks, dvl, IDESC_PV, 1u);
                    umma_ts(tmem + kAtO, pcol + 32 + 8 * ks, dvh, IDESC_PV, 1u);
                }
                umma_commit(&pv_done[i & 1]);
                umma_commit(&kvempty[s]);
                consumed = i + 1;
            }
            if (!ok) *s_fail = 1;
            *s_consumed = consumed;
            umma_commit(fin);
            if (!mbar_wait(fin, 0)) *s_fail = 1;
        }
    } else {
        // ---- softmax warps: thread = row (TMEM lane 32*(warp%4) + lane) ----
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const int tok = t0 + r / a.g;
        const int head = j * a.g + r % a.g;
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        // q row -> bf16 hi + lo in TMEM
        {
            const float *qp = a.q32 + ((int64_t)tok * a.nq + head) * 128;
            const bool live = tok < a.T;
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // 32 dims per chunk -> 16 columns each
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float2 v = make_float2(0.f, 0.f);
                    if (live) v = *reinterpret_cast<const float2 *>(qp + 32 * c + 2 * e);
                    hi[e] = pack_bf16x2(v.x, v.y);
                    lo[e] = pack_bf16x2(v.x - bf16lo(hi[e]), v.y - bf16hi(hi[e]));
                }
                tmem_st16(tmem + lane_off + kAtQhi + 16 * c, hi);
                tmem_st16(tmem + lane_off + kAtQlo + 16 * c, lo);
            }
            tmem_st_wait();
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(q_ready);
        }
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int i = 0; i < nkt; ++i) {
            const int b = i & 1;
            // warp-uniform decision before the warp-collective TMEM loads
            const bool got = __all_sync(0xffffffffu, !*s_fail && mbar_wait(&s_full[b], (unsigned)(i >> 1) & 1u));
            if (!got) {
                *s_fail = 1;
                ok = false;
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t sadr = tmem + lane_off + kAtS + (uint32_t)(b * kAtKeys);
            float x[64];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v[16];
                tmem_ld16(sadr + 16 * c, v);
#pragma unroll
                for (int e = 0; e < 16; ++e) x[16 * c + e] = v[e];
            }
            const int key0 = i * kAtKeys;
            float mx = -INFINITY;
#pragma unroll
            for (int e = 0; e < 64; ++e) {
                x[e] = (key0 + e <= a.p0 + tok) ? x[e] * a.scale_log2 : -INFINITY;
                mx = fmaxf(mx, x[e]);
            }
            // raise the running max only when this tile exceeds it by > 8
            const bool need = mx > m + 8.0f;
            if (__any_sync(0xffffffffu, need)) {
                const float mn = fmaxf(m, mx);
                const float f = (m == -INFINITY) ? 0.f : exp2f(m - mn);
                if (i > 0) {
                    // O holds tiles 0..i-1: wait for the last PV, rescale in TMEM
                    if (!mbar_wait(&pv_done[(i - 1) & 1], (unsigned)((i - 1) >> 1) & 1u)) {
                        *s_fail = 1;
                        ok = false;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    if (__any_sync(0xffffffffu, !ok)) {
                        ok = false;
                        break;
                    }
#pragma unroll 1
                    for (int c = 0; c < 8; ++c) {
                        float v[16];
                        uint32_t w[16];
                        tmem_ld16(tmem + lane_off + kAtO + 16 * c, v);
#pragma unroll
                        for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(v[e] * f);
                        tmem_st16(tmem + lane_off + kAtO + 16 * c, w);
                    }
                    tmem_st_wait();
                }
                l *= f;
                m = mn;
            }
            uint32_t ph[32], pl[32];
            float sum = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float p0 = exp2f(x[2 * e] - m), p1 = exp2f(x[2 * e + 1] - m);
                sum += p0 + p1;
                ph[e] = pack_bf16x2(p0, p1);
                pl[e] = pack_bf16x2(p0 - bf16lo(ph[e]), p1 - bf16hi(ph[e]));
            }
            l += sum;
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = ph[e];
            tmem_st16(sadr, w);
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = ph[16 + e];
            tmem_st16(sadr + 16, w);
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = pl[e];
            tmem_st16(sadr + 32, w);
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = pl[16 + e];
            tmem_st16(sadr + 48, w);
            tmem_st_wait();
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[b]);
        }
        if (ok) {
            const int last = nkt - 1;
            if (!mbar_wait(&pv_done[last & 1], (unsigned)(last >> 1) & 1u)) {
                *s_fail = 1;
                ok = false;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        }
        if (__all_sync(0xffffffffu, ok)) {
            const float inv = 1.0f / l;
            const int64_t base = (int64_t)tok * a.nq * 128 + (int64_t)head * 128;
#pragma unroll 1
            for (int c = 0; c < 8; ++c) {
                float v[16];
                tmem_ld16(tmem + lane_off + kAtO + 16 * c, v);
                if (tok < a.T) {
                    uint32_t hw[8], lw[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float v0 = v[2 * e] * inv, v1 = v[2 * e + 1] * inv;
                        hw[e] = pack_bf16x2(v0, v1);
                        lw[e] = pack_bf16x2(v0 - bf16lo(hw[e]), v1 - bf16hi(hw[e]));
                    }
                    uint4 *dh = reinterpret_cast<uint4 *>(a.o_hi + base + 16 * c);
                    uint4 *dl = reinterpret_cast<uint4 *>(a.o_lo + base + 16 * c);
                    dh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    dh[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
                    dl[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                    dl[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (*s_fail && threadIdx.x == 0) {
        record_error(8u);
        for (int it = *s_consumed; it < *s_issued; ++it) {
            mbar_wait(&kfull[it % kAtStages], (unsigned)(it / kAtStages) & 1u);
            mbar_wait(&vfull[it % kAtStages], (unsigned)(it / kAtStages) & 1u);
        }
    }
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

}  // namespace tpl
